"""Seeded synthetic inputs: determinism, rounding and the configuration recipe."""
import numpy as np
import torch

from workloads import WORKLOADS, U_LOW_RHO_095, bf16_bits, generate, round_bf16, weight_shapes


def test_round_bf16_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0],
                                 dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(round_bf16(x), ref)
    bits = bf16_bits(ref)
    np.testing.assert_array_equal(
        torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy(), ref)


def test_generation_is_deterministic_and_rounded():
    wl = WORKLOADS[1].replace(batch=1, seq=8)
    a, b = generate(wl), generate(wl)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    for k in ("e", "wq", "w1", "w_router"):
        np.testing.assert_array_equal(round_bf16(a[k]), a[k])
    assert a["h0"] is a["e"]                       # "h0 = e": the same tensor


def test_recipe_ranges():
    for wl in WORKLOADS:
        shapes = weight_shapes(wl)
        assert shapes["w_router"] == (wl.n_experts, wl.dim)
        assert wl.top_k <= wl.n_experts
    w3 = WORKLOADS[3].replace(batch=1, seq=4, dim=8192, n_heads=1, n_kv_heads=1, head_dim=8,
                              n_experts=1, top_k=1, expert_hidden=1, n_shared=0)  # many u draws
    A = generate(w3)["A"]
    assert A.max() <= 0.95 + 1e-7 and A.min() >= np.exp(-1.0) - 1e-7
    assert abs(np.exp(-np.exp(U_LOW_RHO_095)) - 0.95) < 1e-12
    w1 = WORKLOADS[1].replace(batch=1, seq=4)
    g = generate(w1)
    assert g["B"].shape == (w1.dim,) and abs(g["B"].mean() - 1.0) < 0.02
    g0 = generate(WORKLOADS[0])
    assert g0["B"].shape == (128, 128) and g0["e"].dtype == np.float32


def test_act_head_recipe():
    from workloads import ACT_THRESHOLD, act_head
    wl = WORKLOADS[1]
    a, b = act_head(wl), act_head(wl)
    np.testing.assert_array_equal(a["w_halt"], b["w_halt"])                 # reproducible
    assert a["w_halt"].dtype == np.float32 and a["w_halt"].shape == (wl.dim,)
    assert a["b_halt"] == -1.0 and a["threshold"] == ACT_THRESHOLD == 0.99
    assert abs(a["w_halt"].std() * np.sqrt(wl.dim) - 0.5) < 0.05              # N(0, 0.25 / dim)
    assert not np.array_equal(act_head(wl, seed=wl.seed + 1)["w_halt"], a["w_halt"])
    # a stream of its own: not a replay of generate()'s first draws
    e = generate(wl.replace(batch=1, seq=1))["e"].ravel()
    assert not np.allclose(a["w_halt"] / a["w_halt"].std(), e / e.std())
