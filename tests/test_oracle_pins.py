"""Pins of the fp64 oracle against facts fixed outside it.

Each test ties one oracle function to something independent of its own code:
a closed form, a hand-computed fixture from the pages' equation, a library
routine that computes a special case (PyTorch CPU in float64), an algebraic
identity, or brute force on tiny inputs. A dropped term, a sign error, a
transposed operand or a wrong head/expert index in the oracle fails at least
one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as tF

import oracle as O
from workloads import WORKLOADS, Workload, generate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TD = torch.float64


def _t(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64))


def small_gqa(**kw) -> Workload:
    base = dict(name="pin-gqa", dtype="f32", batch=2, seq=12, dim=32, attn="gqa", n_heads=4,
                n_kv_heads=2, head_dim=8, n_experts=4, top_k=2, expert_hidden=16,
                b_kind="diag", loops=(3,), seed=7)
    base.update(kw)
    return Workload(**base)


def small_mla(**kw) -> Workload:
    base = dict(name="pin-mla", dtype="f32", batch=2, seq=10, dim=32, attn="mla", n_heads=4,
                q_lora_rank=24, kv_lora_rank=16, qk_nope_dim=8, qk_rope_dim=4, v_head_dim=8,
                n_experts=4, top_k=2, expert_hidden=16, b_kind="diag", loops=(2,), seed=11)
    base.update(kw)
    return Workload(**base)


# ----------------------------------------------------------------------------- norms / rope

def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 7, 33)) * 3.0
    g = rng.standard_normal(33)
    ref = tF.rms_norm(_t(x), (33,), weight=_t(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-13)


def test_rope_is_complex_rotation():
    # Pair (i, i + r/2) as the complex number z = x_i + j x_{i+r/2}; RoPE multiplies it by
    # exp(j * pos * base^(-2i/r)).
    rng = np.random.default_rng(1)
    Bn, S, H, r, base = 2, 9, 3, 8, 1.0e4
    x = rng.standard_normal((Bn, S, H, r))
    got = O.apply_rope(x, base)
    z = x[..., : r // 2] + 1j * x[..., r // 2:]
    ang = np.arange(S)[:, None] * base ** (-np.arange(r // 2) * 2.0 / r)[None, :]
    zr = z * np.exp(1j * ang)[None, :, None, :]
    np.testing.assert_allclose(got[..., : r // 2], zr.real, atol=1e-13)
    np.testing.assert_allclose(got[..., r // 2:], zr.imag, atol=1e-13)


def test_rope_position_zero_and_relative():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 1, 16))
    k = rng.standard_normal((1, 1, 1, 16))
    S = 40
    qs = O.apply_rope(np.repeat(q, S, axis=1), 1e4)[0, :, 0]
    ks = O.apply_rope(np.repeat(k, S, axis=1), 1e4)[0, :, 0]
    np.testing.assert_allclose(qs[0], q[0, 0, 0], atol=0)          # position 0: identity
    dots = qs @ ks.T                                              # <R_m q, R_n k>
    for off in (0, 3, 17):
        diag = np.array([dots[m, m - off] for m in range(off, S)])
        np.testing.assert_allclose(diag, diag[0], atol=1e-12)     # depends on m - n only


# ----------------------------------------------------------------------------- attention

def test_attention_hand_example():
    # q, k scalar (dh = 1), scale 1, v in R^2. Row 0 sees key 0 only; row 1 keys {0, 1} with
    # scores {0, 1}; row 2 keys {0, 1, 2} with scores {0, 2, 2}.
    q = np.array([[1.0], [1.0], [2.0]])
    k = np.array([[0.0], [1.0], [1.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, 2.0]])
    e1, e2 = math.e, math.e ** 2
    want = np.array([[1.0, 0.0],
                     [1.0 / (1.0 + e1), e1 / (1.0 + e1)],
                     [(1.0 + 2.0 * e2) / (1.0 + 2.0 * e2), 3.0 * e2 / (1.0 + 2.0 * e2)]])
    np.testing.assert_allclose(O.causal_attention(q, k, v, 1.0), want, rtol=1e-14)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 1), (8, 2)])
def test_gqa_attention_matches_sdpa(hq, hkv):
    rng = np.random.default_rng(hq * 10 + hkv)
    Bn, S, dq, dv = 2, 23, 12, 10
    q = rng.standard_normal((Bn, S, hq, dq))
    k = rng.standard_normal((Bn, S, hkv, dq))
    v = rng.standard_normal((Bn, S, hkv, dv))
    scale = 1.0 / math.sqrt(dq)
    got = O.gqa_attention(q, k, v, scale)
    ref = tF.scaled_dot_product_attention(_t(q).transpose(1, 2), _t(k).transpose(1, 2),
                                          _t(v).transpose(1, 2), is_causal=True, scale=scale,
                                          enable_gqa=True).transpose(1, 2).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(3)
    Bn, S, hq, hkv, dh = 1, 15, 8, 2, 6
    q = rng.standard_normal((Bn, S, hq, dh))
    k = rng.standard_normal((Bn, S, hkv, dh))
    v = rng.standard_normal((Bn, S, hkv, dh))
    rep = hq // hkv
    mha = O.gqa_attention(q, np.repeat(k, rep, axis=2), np.repeat(v, rep, axis=2), 0.3)
    np.testing.assert_array_equal(O.gqa_attention(q, k, v, 0.3), mha)


def test_attention_query_subset_and_blocking():
    rng = np.random.default_rng(4)
    S = 2500                                       # spans several query blocks
    q, k, v = rng.standard_normal((S, 4)), rng.standard_normal((S, 4)), rng.standard_normal((S, 3))
    full = O.causal_attention(q, k, v, 0.5)
    pos = np.array([0, 1, 1023, 1024, 2499])
    np.testing.assert_allclose(O.causal_attention(q[pos], k, v, 0.5, q_pos=pos), full[pos],
                               rtol=1e-13, atol=1e-13)
    # brute force for one late row
    s = (q[2000] @ k[:2001].T) * 0.5
    p = np.exp(s - s.max())
    np.testing.assert_allclose(full[2000], (p / p.sum()) @ v[:2001], rtol=1e-12)


# ----------------------------------------------------------------------------- MLA

def _mla_torch(xn, W, cfg):
    """MLA written with PyTorch library calls: rms_norm, complex RoPE and SDPA."""
    H, nope, rope, vd = cfg.n_heads, cfg.qk_nope_dim, cfg.qk_rope_dim, cfg.v_head_dim
    x = _t(xn)
    Bn, S, _ = x.shape

    def rot(t):                                       # t [B, S, h, r]
        r = t.shape[-1]
        z = torch.complex(t[..., : r // 2], t[..., r // 2:])
        ang = torch.arange(S, dtype=TD)[:, None] * cfg.rope_base ** (
            -torch.arange(r // 2, dtype=TD) * 2.0 / r)[None, :]
        z = z * torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    c_q = tF.rms_norm(x @ _t(W["w_dq"]).T, (cfg.q_lora_rank,), weight=_t(W["q_norm"]), eps=cfg.norm_eps)
    c_kv = tF.rms_norm(x @ _t(W["w_dkv"]).T, (cfg.kv_lora_rank,), weight=_t(W["kv_norm"]), eps=cfg.norm_eps)
    kr = rot((x @ _t(W["w_kr"]).T).reshape(Bn, S, 1, rope))
    heads = []
    for h in range(H):
        wuq = _t(W["w_uq"]).reshape(H, nope + rope, -1)[h]
        qh = c_q @ wuq.T
        qh = torch.cat([qh[..., :nope], rot(qh[..., nope:].reshape(Bn, S, 1, rope))[:, :, 0]], -1)
        kh = torch.cat([c_kv @ _t(W["w_uk"]).reshape(H, nope, -1)[h].T, kr[:, :, 0]], -1)
        vh = c_kv @ _t(W["w_uv"]).reshape(H, vd, -1)[h].T
        heads.append(tF.scaled_dot_product_attention(qh, kh, vh, is_causal=True,
                                                     scale=1.0 / math.sqrt(nope + rope)))
    return torch.cat(heads, dim=-1).numpy()


def test_mla_explicit_matches_torch_composition():
    cfg = small_mla()
    W = generate(cfg)
    xn = O.rmsnorm(W["e"] * 1.7, W["norm1"], cfg.norm_eps)
    np.testing.assert_allclose(O.mla_attention_explicit(xn, W, cfg), _mla_torch(xn, W, cfg),
                               rtol=1e-11, atol=1e-12)


def test_mla_absorbed_equals_explicit():
    cfg = small_mla()
    W = generate(cfg)
    xn = O.rmsnorm(W["e"], W["norm1"], cfg.norm_eps)
    np.testing.assert_allclose(O.mla_attention_absorbed(xn, W, cfg),
                               O.mla_attention_explicit(xn, W, cfg), rtol=1e-11, atol=1e-12)


def _gqa_torch(x, W, cfg, t):
    """The GQA attention sublayer written with PyTorch library calls: rms_norm, F.linear for
    the projections (the loop's LoRA delta on Q and O), RoPE as a complex rotation of the
    pairs (i, i + dh/2) of q and k only, SDPA with grouped KV heads, the O projection."""
    hq, hkv, dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    xt = _t(x)
    Bn, S, d = xt.shape
    xn = tF.rms_norm(xt, (d,), weight=_t(W["norm1"]), eps=cfg.norm_eps)
    li = min(t, cfg.n_lora - 1) if cfg.n_lora else None
    q = tF.linear(xn, _t(W["wq"]))
    if li is not None:
        q = q + tF.linear(tF.linear(xn, _t(W["lq_a"][li])), _t(W["lq_b"][li]))
    k = tF.linear(xn, _t(W["wk"]))
    v = tF.linear(xn, _t(W["wv"]))
    # [B, S, H*dh] -> [B, H, S, dh]: head h owns columns h*dh .. h*dh + dh - 1
    q = q.view(Bn, S, hq, dh).transpose(1, 2)
    k = k.view(Bn, S, hkv, dh).transpose(1, 2)
    v = v.view(Bn, S, hkv, dh).transpose(1, 2)

    def rot(u):
        z = torch.complex(u[..., : dh // 2], u[..., dh // 2:])
        ang = torch.arange(S, dtype=TD)[:, None] * cfg.rope_base ** (
            -torch.arange(dh // 2, dtype=TD) * 2.0 / dh)[None, :]
        z = z * torch.polar(torch.ones_like(ang), ang)
        return torch.cat([z.real, z.imag], dim=-1)

    o = tF.scaled_dot_product_attention(rot(q), rot(k), v, is_causal=True, scale=1.0 / math.sqrt(dh),
                                        enable_gqa=True)
    o = o.transpose(1, 2).reshape(Bn, S, hq * dh)
    a = tF.linear(o, _t(W["wo"]))
    if li is not None:
        a = a + tF.linear(tF.linear(o, _t(W["lo_a"][li])), _t(W["lo_b"][li]))
    return a.numpy()


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (4, 1)])
@pytest.mark.parametrize("lora", [False, True])
def test_gqa_sublayer_matches_torch_composition(hq, hkv, lora):
    kw = dict(lora_rank=3, n_lora=2) if lora else {}
    cfg = small_gqa(n_heads=hq, n_kv_heads=hkv, head_dim=8, dim=32, seq=13, **kw)
    W = generate(cfg)
    x = W["e"] * 1.3 + 0.2
    for t in ((0, 1, 3) if lora else (0,)):
        np.testing.assert_allclose(O.attention_sublayer(x, W, cfg, t), _gqa_torch(x, W, cfg, t),
                                   rtol=1e-11, atol=1e-12)


def _planted_gqa_qkv(kind):
    """A copy of the oracle's Q/K/V step with one plausible mistake planted."""
    def qkv(xn, W, cfg, t):
        Bn, S, _ = xn.shape
        hq, hkv, dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
        q = xn @ np.asarray(W["wq"], np.float64).T
        if cfg.n_lora:
            li = min(t, cfg.n_lora - 1)
            delta = (xn @ np.asarray(W["lq_a"][li], np.float64).T) @ np.asarray(W["lq_b"][li], np.float64).T
            q = q + (0.0 if kind == "lora_dropped" else delta)
        wk, wv = ("wv", "wk") if kind == "k_v_swapped" else ("wk", "wv")
        k = xn @ np.asarray(W[wk], np.float64).T
        v = xn @ np.asarray(W[wv], np.float64).T
        if kind == "dim_major_heads":
            q = q.reshape(Bn, S, dh, hq).swapaxes(2, 3)
            k = k.reshape(Bn, S, dh, hkv).swapaxes(2, 3)
            v = v.reshape(Bn, S, dh, hkv).swapaxes(2, 3)
        else:
            q, k, v = q.reshape(Bn, S, hq, dh), k.reshape(Bn, S, hkv, dh), v.reshape(Bn, S, hkv, dh)
        q = O.apply_rope(q, cfg.rope_base)
        k = k if kind == "rope_on_q_only" else O.apply_rope(k, cfg.rope_base)
        if kind == "rope_on_v":
            v = O.apply_rope(v, cfg.rope_base)
        return q, k, v
    return qkv


@pytest.mark.parametrize("kind", ["dim_major_heads", "rope_on_v", "rope_on_q_only", "k_v_swapped",
                                  "lora_dropped"])
def test_gqa_pin_catches_planted_mistakes(kind, monkeypatch):
    cfg = small_gqa(n_heads=8, n_kv_heads=2, head_dim=8, dim=32, seq=13, lora_rank=3, n_lora=2)
    W = generate(cfg)
    x = W["e"] * 1.3 + 0.2
    ref = _gqa_torch(x, W, cfg, 1)
    np.testing.assert_allclose(O.attention_sublayer(x, W, cfg, 1), ref, rtol=1e-11, atol=1e-12)
    monkeypatch.setattr(O.rdt_oracle, "gqa_qkv", _planted_gqa_qkv(kind))
    assert np.max(np.abs(O.attention_sublayer(x, W, cfg, 1) - ref)) > 1e-6


def test_mla_page_example_dims_absorbed_equals_explicit():
    g = json.load(open(os.path.join(GOLDEN, "mythos_config_examples.json")))
    m = g["passo5_mla"]
    cfg = small_mla(dim=64, n_heads=2, seq=5, batch=1, q_lora_rank=m["q_lora_rank"],
                    kv_lora_rank=m["kv_lora_rank"], qk_rope_dim=m["qk_rope_head_dim"],
                    qk_nope_dim=m["qk_nope_head_dim"], v_head_dim=m["v_head_dim"])
    W = generate(cfg)
    xn = O.rmsnorm(W["e"], W["norm1"], cfg.norm_eps)
    np.testing.assert_allclose(O.mla_attention_absorbed(xn, W, cfg),
                               O.mla_attention_explicit(xn, W, cfg), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- router / MoE

def test_router_matches_brute_force_sort():
    rng = np.random.default_rng(5)
    N, E, k = 200, 9, 3
    logits = np.round(rng.standard_normal((N, E)), 1)      # many exact ties
    bias = np.round(rng.standard_normal(E) * 0.1, 1)
    r = O.router_topk(logits, bias, k)
    for n in range(N):
        score = [(logits[n, e] + bias[e], e) for e in range(E)]
        ranked = sorted(score, key=lambda p: (-p[0], p[1]))
        assert list(r.idx[n]) == [e for _, e in ranked[:k]]
        assert math.isclose(r.gap[n], ranked[k - 1][0] - ranked[k][0], abs_tol=1e-15)
        sel = logits[n, [e for _, e in ranked[:k]]]
        full = np.exp(logits[n] - logits[n].max())
        full /= full.sum()
        ren = full[[e for _, e in ranked[:k]]]
        np.testing.assert_allclose(r.w[n], ren / ren.sum(), rtol=1e-13)
    np.testing.assert_allclose(r.w.sum(axis=1), 1.0, rtol=1e-14)


def test_moe_top_k_equal_E_is_dense_softmax_mixture():
    rng = np.random.default_rng(6)
    N, d, E, hid = 11, 8, 5, 6
    yn = rng.standard_normal((N, d))
    w1, w3 = rng.standard_normal((E, hid, d)), rng.standard_normal((E, hid, d))
    w2 = rng.standard_normal((E, d, hid))
    wr = rng.standard_normal((E, d))
    r = O.router_topk(yn @ wr.T, None, E)
    f = O.moe_combine(yn, r.idx, r.w, w1, w3, w2)
    p = torch.softmax(_t(yn) @ _t(wr).T, dim=-1)
    ref = torch.zeros(N, d, dtype=TD)
    for e in range(E):
        u = tF.silu(_t(yn) @ _t(w1[e]).T) * (_t(yn) @ _t(w3[e]).T)
        ref += p[:, e:e + 1] * (u @ _t(w2[e]).T)
    np.testing.assert_allclose(f, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_moe_single_expert_and_shared_is_plain_swiglu():
    rng = np.random.default_rng(7)
    N, d, hid = 9, 8, 12
    yn = rng.standard_normal((N, d))
    w1, w3, w2 = (rng.standard_normal((1, hid, d)), rng.standard_normal((1, hid, d)),
                  rng.standard_normal((1, d, hid)))
    r = O.router_topk(rng.standard_normal((N, 1)), None, 1)
    np.testing.assert_array_equal(r.w, 1.0)
    ref = ((tF.silu(_t(yn) @ _t(w1[0]).T) * (_t(yn) @ _t(w3[0]).T)) @ _t(w2[0]).T).numpy()
    np.testing.assert_allclose(O.moe_combine(yn, r.idx, r.w, w1, w3, w2), ref, rtol=1e-12)
    # a shared expert with the same weights contributes the same amount again (weight 1)
    f2 = O.moe_combine(yn, r.idx, r.w, w1, w3, w2, w1, w3, w2)
    np.testing.assert_allclose(f2, 2.0 * ref, rtol=1e-12)


def test_moe_token_permutation_equivariance():
    cfg = small_gqa()
    W = generate(cfg)
    y = W["e"].reshape(-1, cfg.dim)[None] * 2.0
    perm = np.random.default_rng(8).permutation(y.shape[1])
    f, r, _ = O.moe_sublayer(y, W, cfg)
    fp, rp, _ = O.moe_sublayer(y[:, perm], W, cfg)
    np.testing.assert_allclose(fp, f[:, perm], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(rp.idx, r.idx[perm])


def test_follow_mode_adopts_only_near_ties():
    cfg = small_gqa(n_experts=6, top_k=2)
    W = generate(cfg)
    y = W["e"] * 1.3
    f, r, st = O.moe_sublayer(y, W, cfg, follow_idx=None)
    f2, r2, st2 = O.moe_sublayer(y, W, cfg, follow_idx=r.idx)
    np.testing.assert_array_equal(f2, f)
    assert st2 == {"near_ties": 0, "mismatch": 0}
    other = r.idx.copy()
    n_far = int(np.argmax(r.gap))
    other[n_far] = [e for e in range(cfg.n_experts) if e not in r.idx[n_far]][:2]
    _, r3, st3 = O.moe_sublayer(y, W, cfg, follow_idx=other)
    assert st3["mismatch"] == 1
    np.testing.assert_array_equal(r3.idx, r.idx)                # far from a tie: keeps its own


# ----------------------------------------------------------------------------- the loop

def _zero_block_cfg(dim=2):
    return Workload(name="pin-zero", dtype="f32", batch=1, seq=1, dim=dim, attn="gqa", n_heads=1,
                    n_kv_heads=1, head_dim=dim, n_experts=1, top_k=1, expert_hidden=1,
                    b_kind="diag", loops=(3,), seed=0)


def test_update_equation_hand_fixture():
    g = json.load(open(os.path.join(GOLDEN, "update_equation_zero_block.json")))
    cfg = _zero_block_cfg()
    W = generate(cfg, zero_block=True)
    W["A"] = np.array(g["A"])
    W["B"] = np.array(g["B"])
    e = np.array(g["e"]).reshape(1, 1, 2)
    h0 = np.array(g["h0"]).reshape(1, 1, 2)
    tr = O.LoopTrace()
    O.loop_forward(h0, e, 3, W, cfg, trace=tr)
    for t, want in enumerate(g["expected"]):
        np.testing.assert_array_equal(tr.h[t + 1].reshape(2), want)


@pytest.mark.parametrize("T", [1, 2, 5, 16])
def test_zero_block_closed_form(T):
    # h_T = A^T h0 + (1 - A^T) / (1 - A) * B e   (geometric series of the update equation)
    cfg = WORKLOADS[1].replace(batch=2, seq=6, dim=64, n_heads=4, n_kv_heads=2, head_dim=16,
                               n_experts=4, top_k=2, expert_hidden=8)
    W = generate(cfg, zero_block=True, h0_independent=True)
    A = W["A"].astype(np.float64)
    Be = W["B"].astype(np.float64) * W["e"].astype(np.float64)
    got = O.loop_forward(W["h0"], W["e"], T, W, cfg)
    want = A ** T * W["h0"] + (1.0 - A ** T) / (1.0 - A) * Be
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_dense_B_closed_form_and_diag_embedding():
    cfg = WORKLOADS[0].replace(seq=5)
    W = generate(cfg, zero_block=True)
    T = 4
    got = O.loop_forward(W["h0"], W["e"], T, W, cfg)
    A = W["A"].astype(np.float64)
    Be = W["e"].astype(np.float64) @ W["B"].astype(np.float64).T
    want = A ** T * W["h0"] + (1.0 - A ** T) / (1.0 - A) * Be
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    b = np.random.default_rng(9).standard_normal(cfg.dim)
    np.testing.assert_allclose(O.input_injection(W["e"], np.diag(b)), O.input_injection(W["e"], b),
                               rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("wl_index", [0, 2])
def test_superposition_identity(wl_index):
    # Unrolling the update equation: h_T = A^T h0 + sum_k A^k Be + sum_s A^(T-1-s) Delta_s
    cfg = small_gqa() if wl_index == 0 else small_mla()
    W = generate(cfg, h0_independent=True)
    T = 5
    tr = O.LoopTrace()
    got = O.loop_forward(W["h0"], W["e"], T, W, cfg, trace=tr)
    A = W["A"].astype(np.float64)
    Be = O.input_injection(W["e"], W["B"])
    want = A ** T * W["h0"] + sum(A ** k for k in range(T)) * Be
    for s, dl in enumerate(tr.delta):
        want = want + A ** (T - 1 - s) * dl
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-11)
    for t in range(T):
        np.testing.assert_allclose(tr.delta[t], tr.attn[t] + tr.moe[t], rtol=0, atol=0)


def test_T1_is_one_block_and_x_includes_e():
    cfg = small_gqa()
    W = generate(cfg, h0_independent=True)
    h0, e = W["h0"].astype(np.float64), W["e"].astype(np.float64)
    got = O.loop_forward(h0, e, 1, W, cfg)
    x0 = h0 + e
    a = O.attention_sublayer(x0, W, cfg, 0)
    f, _, _ = O.moe_sublayer(x0 + a, W, cfg)
    np.testing.assert_allclose(got, W["A"] * h0 + W["B"] * e + a + f, rtol=1e-13, atol=1e-13)
    cfg0 = cfg.replace(inject_e=False)
    a0 = O.attention_sublayer(h0, W, cfg0, 0)
    f0, _, _ = O.moe_sublayer(h0 + a0, W, cfg0)
    np.testing.assert_allclose(O.loop_forward(h0, e, 1, W, cfg0),
                               W["A"] * h0 + W["B"] * e + a0 + f0, rtol=1e-13, atol=1e-13)


def test_stability_bound_long_run():
    # rho(A) < 1 ([GS] Passo 6) and |Delta| bounded give a bounded state:
    # |h_t| <= A^t |h0| + (|Be| + M)(1 - A^t)/(1 - A), M = max_s |Delta_s|.
    cfg = WORKLOADS[0]
    W = generate(cfg)
    assert O.spectral_radius(W["A"]) < 1.0
    T = 64
    tr = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], T, W, cfg, trace=tr)
    A = W["A"].astype(np.float64)
    Be = np.abs(O.input_injection(W["e"], W["B"]))
    M = max(np.max(np.abs(d)) for d in tr.delta)
    for t in range(T + 1):
        bound = A ** t * np.abs(W["h0"]) + (Be + M) * (1.0 - A ** t) / (1.0 - A)
        assert np.all(np.abs(tr.h[t]) <= bound * (1 + 1e-12) + 1e-12)
    # uniform in t: the state never leaves |h0| + (|Be| + M) / (1 - A)
    cap = np.abs(W["h0"]) + (Be + M) / (1.0 - A)
    assert all(np.all(np.abs(h) <= cap * (1 + 1e-12)) for h in tr.h)


def test_spectral_radius_rule():
    assert O.spectral_radius(np.array([0.2, -0.97, 0.5])) == pytest.approx(0.97)
    assert O.spectral_radius(np.array([0.2, 1.0])) >= 1.0        # the page's assert would fire


def test_causality_and_batch_independence():
    cfg = small_gqa(seq=16)
    W = generate(cfg)
    h = O.loop_forward(W["h0"], W["e"], 3, W, cfg)
    e2, h02 = W["e"].copy(), W["h0"].copy()
    e2[0, 9:] += 1.0
    h02[0, 9:] -= 2.0
    e2[1] *= -1.0                                               # the other sequence changes too
    h2 = O.loop_forward(h02, e2, 3, W, cfg)
    np.testing.assert_array_equal(h2[0, :9], h[0, :9])


def test_lora_zero_up_is_base_and_merged_equals_unmerged():
    cfg = small_gqa(lora_rank=3, n_lora=4)
    base = cfg.replace(lora_rank=0, n_lora=0)
    Wz = generate(cfg, lora_b_zero=True)
    np.testing.assert_array_equal(O.loop_forward(Wz["h0"], Wz["e"], 3, Wz, cfg),
                                  O.loop_forward(Wz["h0"], Wz["e"], 3, Wz, base))
    W = generate(cfg)
    x = W["e"] * 1.5
    for t in (0, 2, 6):                                         # t >= L uses the last adapter
        li = min(t, cfg.n_lora - 1)
        Wm = dict(W)
        Wm["wq"] = W["wq"].astype(np.float64) + W["lq_b"][li].astype(np.float64) @ W["lq_a"][li]
        Wm["wo"] = W["wo"].astype(np.float64) + W["lo_b"][li].astype(np.float64) @ W["lo_a"][li]
        np.testing.assert_allclose(O.attention_sublayer(x, W, cfg, t),
                                   O.attention_sublayer(x, Wm, base, t), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("which", ["gqa", "mla"])
def test_loop_step_rows_matches_full_loop(which):
    cfg = small_gqa(seq=14) if which == "gqa" else small_mla(seq=14)
    W = generate(cfg)
    tr = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], 3, W, cfg, trace=tr)
    rows = [(0, 0), (1, 13), (0, 7), (1, 5)]
    hn, r, st = O.loop_step_rows(tr.h[2], W["e"], W, cfg, 2, rows)
    for i, (b, s) in enumerate(rows):
        np.testing.assert_allclose(hn[i], tr.h[3][b, s], rtol=1e-12, atol=1e-12)


def test_page_config_example_runs_and_stays_bounded():
    g = json.load(open(os.path.join(GOLDEN, "mythos_config_examples.json")))["passo2"]
    cfg = Workload(name="passo2", dtype="f32", batch=1, seq=8, dim=g["dim"], attn="gqa",
                   n_heads=g["n_heads"], n_kv_heads=g["n_kv_heads"], head_dim=g["dim"] // g["n_heads"],
                   n_experts=g["n_experts"], top_k=g["n_experts_per_tok"], n_shared=g["n_shared_experts"],
                   expert_hidden=g["expert_dim"], lora_rank=g["lora_rank"], n_lora=g["max_loop_iters"],
                   loops=(g["max_loop_iters"],), seed=3)
    W = generate(cfg)
    tr = O.LoopTrace()
    h = O.loop_forward(W["h0"], W["e"], g["max_loop_iters"] + 2, W, cfg, trace=tr)  # N + k loops
    assert h.shape == (1, 8, g["dim"]) and np.all(np.isfinite(h))
    assert all(r.idx.shape == (8, g["n_experts_per_tok"]) for r in tr.routing)
