"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances: hidden states after T loops within max-abs 3e-2 and relative Frobenius 1e-2;
router indices identical wherever the oracle's k-th/(k+1)-th score gap exceeds 1e-3 (the
oracle adopts the GPU's choice only on near-ties and counts every other difference).
"""
import numpy as np
import pytest

import oracle as O
from workloads import WORKLOADS, generate, prefix, round_bf16

from rdt_testlib import (MAX_ABS, REL_FRO, act, assert_close, errors, handle, oracle_follow,
                         run_loop, torch_mod)

pytestmark = pytest.mark.gpu

C0, C1, C2, C3, C4 = WORKLOADS

# Reduced-size variants: same widths, heads and experts, fewer tokens; sequence lengths
# that leave ragged GEMM row tiles (not multiples of 128) and ragged attention blocks.
SMALL = {
    "tiny-f32": C0,
    "gqa-s200": C1.replace(batch=2, seq=200),
    "mla-s136": C2.replace(batch=2, seq=136),
    "widemoe-s192": C3.replace(batch=1, seq=192),
    "long-lora-s320": C4.replace(seq=320),
}


def _loops(name):
    return 4 if name == "tiny-f32" else 3


@pytest.mark.parametrize("name", list(SMALL))
def test_loop_matches_oracle_small(name):
    wl = SMALL[name]
    inputs = generate(wl)
    T = _loops(name)
    got, idx, w, _, diag = run_loop(wl, inputs, T)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    want, mism, ties, _ = oracle_follow(wl, inputs, T, idx)
    assert mism == 0, f"{mism} routing differences outside near-ties"
    assert_close(got, want, what=name)


@pytest.mark.parametrize("name", ["gqa-s200", "tiny-f32", "long-lora-s320"])
def test_block_input_without_e_matches_oracle(name):
    """inject_e = 0: the block input is h alone (x = h) while B.e still enters the update.
    RMSNorm1 reads no e; the O projection's epilogue takes B.e from the hoist (a diagonal B
    is not applied to e there) or, for the dense B of the fp32 configuration, from the
    once-per-call product."""
    wl = SMALL[name].replace(inject_e=False)
    inputs = generate(wl)
    T = _loops(name)
    got, idx, _, _, diag = run_loop(wl, inputs, T)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    want, mism, _, _ = oracle_follow(wl, inputs, T, idx)
    assert mism == 0, f"{mism} routing differences outside near-ties"
    assert_close(got, want, what=f"{name} without e in the block input")


@pytest.mark.parametrize("tiles", [1, 2])
@pytest.mark.parametrize("name", ["gqa-s200", "mla-s136", "widemoe-s192", "long-lora-s320"])
def test_gemm_tile_modes_match_oracle(name, tiles):
    """The projection and expert GEMMs forced onto single-CTA 128-row tiles (1) or CTA-pair
    256-row tiles (2): both must match the oracle; the ragged sizes leave partial pair tiles
    in the dense GEMMs and in every expert group."""
    wl = SMALL[name]
    inputs = generate(wl)
    got, idx, _, _, diag = run_loop(wl, inputs, 2, gemm_tiles=tiles)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    want, mism, _, _ = oracle_follow(wl, inputs, 2, idx)
    assert mism == 0, f"{mism} routing differences outside near-ties"
    assert_close(got, want, what=f"{name} tiles={tiles}")


@pytest.mark.parametrize("tiles", [0, 1, 2])
def test_all_tokens_on_two_experts(tiles):
    """A router bias of +8 on experts 0 and 1 sends every token there: two groups at full
    capacity (several row tiles, ragged last one), fourteen empty groups; the oracle applies
    the same bias in its selection (the gap to the third expert is ~8: no near-ties)."""
    wl = C1.replace(batch=2, seq=200)
    inputs = generate(wl)
    inputs["router_bias"] = np.zeros(wl.n_experts, dtype=np.float32)
    inputs["router_bias"][:2] = 8.0
    got, idx, _, _, diag = run_loop(wl, inputs, 2, gemm_tiles=tiles)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    assert set(np.unique(idx)) == {0, 1}
    want, mism, ties, _ = oracle_follow(wl, inputs, 2, idx)
    assert mism == 0 and ties == 0
    assert_close(got, want, what=f"two experts, tiles={tiles}")


@pytest.mark.parametrize("E,k", [(8, 8), (16, 12)])
def test_top_k_up_to_all_experts(E, k):
    """k = E: every token goes to every expert (each group holds all tokens; the fused
    router); k = 12 > 8: the tensor-core router with its 16-wide top-k epilogue."""
    wl = C1.replace(batch=1, seq=192, n_experts=E, top_k=k)
    inputs = generate(wl)
    got, idx, w, _, diag = run_loop(wl, inputs, 2)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    assert all(len(set(r)) == k for r in idx.reshape(-1, k))          # k distinct experts per token
    np.testing.assert_allclose(w.reshape(-1, k).sum(axis=1), 1.0, atol=1e-5)
    want, mism, _, _ = oracle_follow(wl, inputs, 2, idx)
    assert mism == 0
    assert_close(got, want, what=f"E={E} k={k}")


def test_zero_block_is_closed_form():
    # every block weight zero: h_T = A^T h0 + (1 - A^T)/(1 - A) B e exactly (fp32 state)
    wl = C1.replace(batch=2, seq=64)
    inputs = generate(wl, zero_block=True, h0_independent=True)
    for T in (1, 2, 7, 16):
        got, *_ = run_loop(wl, inputs, T, trace=False)
        A = inputs["A"].astype(np.float64)
        Be = inputs["B"].astype(np.float64) * inputs["e"]
        want = A ** T * inputs["h0"] + (1 - A ** T) / (1 - A) * Be
        ma, _ = errors(got, want)
        assert ma < 2e-4 * max(1.0, np.max(np.abs(want))), (T, ma)


def test_dense_B_and_h0_independent():
    wl = C2.replace(batch=1, seq=96, b_kind="dense")
    inputs = generate(wl, h0_independent=True)
    got, idx, *_ = run_loop(wl, inputs, 3)
    want, mism, _, _ = oracle_follow(wl, inputs, 3, idx)
    assert mism == 0
    assert_close(got, want, what="mla dense B")


def test_lora_depth_extrapolation_uses_last_adapter():
    wl = C4.replace(seq=128, n_lora=2)
    inputs = generate(wl)
    got, idx, *_ = run_loop(wl, inputs, 4)            # loops 2, 3 reuse adapter 1
    want, mism, _, _ = oracle_follow(wl, inputs, 4, idx)
    assert mism == 0
    assert_close(got, want, what="lora T > n_lora")


def test_attention_sublayer():
    torch = torch_mod()
    for wl in (C0, C1.replace(batch=2, seq=200), C2.replace(batch=2, seq=136), C4.replace(seq=192)):
        inputs = generate(wl)
        x = inputs["e"].astype(np.float32) * 1.5 + 0.25
        if wl.dtype == "bf16":
            x = round_bf16(x)                    # x is passed in the configuration's type
        with handle(wl, inputs) as h:
            a = h.attn_forward(act(wl, x), loop=1)
            torch.cuda.synchronize()
            got = a.cpu().numpy()
        want = O.attention_sublayer(x, inputs, wl, 1)
        assert_close(got, want, max_abs=2e-2, rel_fro=1e-2, what=f"attn {wl.name}")


def test_moe_sublayer_and_router_exactness():
    torch = torch_mod()
    for wl in (C0, C1.replace(batch=2, seq=200), C3.replace(batch=1, seq=192)):
        inputs = generate(wl)
        y = inputs["e"].astype(np.float32) * 3.0
        N = wl.batch * wl.seq
        idx = torch.empty((N, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((N, wl.top_k), dtype=torch.float32, device="cuda")
        with handle(wl, inputs) as h:
            f = h.moe_forward(torch.from_numpy(y).cuda(), idx=idx, w=w)
            torch.cuda.synchronize()
            got, gi, gw = f.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
            counts = h.diagnostics()["expert_counts"]
        fo, r, st = O.moe_sublayer(y, inputs, wl, follow_idx=gi)
        assert st["mismatch"] == 0
        np.testing.assert_array_equal(np.bincount(gi.ravel(), minlength=wl.n_experts),
                                      counts[:wl.n_experts])
        np.testing.assert_allclose(gw, r.w, atol=1e-5)
        np.testing.assert_allclose(gw.sum(axis=1), 1.0, atol=1e-5)
        assert_close(got, fo, max_abs=2e-2, rel_fro=1e-2, what=f"moe {wl.name}")


def test_moe_token_permutation_equivariance():
    """Routing and the expert rows are per token: permuting the tokens permutes the MoE
    output (only the fp32 order of the k reductions into a row may differ)."""
    torch = torch_mod()
    wl = C1.replace(batch=1, seq=256)
    inputs = generate(wl)
    y = inputs["e"].astype(np.float32) * 3.0
    perm = np.random.default_rng(7).permutation(wl.seq)
    with handle(wl, inputs) as h:
        f1 = h.moe_forward(torch.from_numpy(y).cuda()).cpu().numpy()
        f2 = h.moe_forward(torch.from_numpy(np.ascontiguousarray(y[:, perm])).cuda()).cpu().numpy()
    ma, _ = errors(f2, f1[:, perm])
    assert ma < 1e-4, ma


def test_T1_equals_sublayer_composition():
    torch = torch_mod()
    wl = C1.replace(batch=1, seq=256)
    inputs = generate(wl)
    with handle(wl, inputs) as h:
        e = act(wl, inputs["e"])
        hT = h.loop_forward(e, e, 1)
        x0 = e + e                          # exact in bf16: the block input h0 + e
        a = h.attn_forward(x0, loop=0)
        f = h.moe_forward(x0.float() + a)
        A = torch.from_numpy(inputs["A"]).cuda()
        B = torch.from_numpy(inputs["B"]).cuda()
        comp = A * e.float() + B * e.float() + a + f
        torch.cuda.synchronize()
    ma, rf = errors(hT.cpu().numpy(), comp.cpu().numpy())
    assert ma < 1e-2 and rf < 1e-3, (ma, rf)


def test_causality_and_batch_independence():
    torch = torch_mod()
    wl = C1.replace(batch=2, seq=256)
    inputs = generate(wl)
    with handle(wl, inputs) as h:
        e = act(wl, inputs["e"])
        out1 = h.loop_forward(e, e, 2).clone()
        e2 = e.clone()
        e2[0, 100:] = e2[0, 100:] * -1.0
        e2[1] = e2[1] * 0.5
        out2 = h.loop_forward(e2, e2, 2)
        torch.cuda.synchronize()
    d = (out1[0, :100] - out2[0, :100]).abs().max().item()
    assert d < 2e-3, d      # leakage would show as O(0.1); atomics only reorder sums


def test_host_entry_matches_device_entry():
    # deterministic mode: the host entry runs the same kernels on the same data, so the two
    # results agree bit for bit (in the default mode the fp32 atomics' order moves the last
    # bits, ~1e-3 after three loops)
    torch = torch_mod()
    wl = C1.replace(batch=1, seq=128)
    inputs = generate(wl)
    with handle(wl, inputs, deterministic=True) as h:
        e = act(wl, inputs["e"])
        dev = h.loop_forward(e, e, 3).cpu()
        eh = e.cpu().pin_memory()
        out = torch.empty(dev.shape, dtype=torch.float32).pin_memory()
        h.loop_forward_host(eh, eh, 3, out)
    assert np.array_equal(out.numpy(), dev.numpy())


def sampled_rows(wl, seed, per_batch_min=8, total_min=32):
    """(batch, position) pairs covering every 128-row query tile of every sequence (one
    random row per tile band, plus each sequence's last row), topped up with random rows
    until there are at least total_min."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(wl.batch):
        for t0 in range(0, wl.seq, 128):
            rows.add((b, int(t0 + rng.integers(0, min(128, wl.seq - t0)))))
        rows.add((b, wl.seq - 1))
        while sum(1 for bb, _ in rows if bb == b) < per_batch_min:
            rows.add((b, int(rng.integers(0, wl.seq))))
    while len(rows) < total_min:
        rows.add((int(rng.integers(wl.batch)), int(rng.integers(0, wl.seq))))
    return sorted(rows)


@pytest.mark.parametrize("wi", [1, 2, 3, 4])
def test_full_size_prefix_and_sampled_rows(wi):
    """The configuration at its full size in the benchmark's launch configuration: the first
    64 positions of every sequence through all loops against the oracle (causality makes
    them independent of later positions); and at the first and the last loop, rows from
    every 128-row query tile of every sequence, each computed by the oracle's single-step
    evaluation from the GPU's own state before that loop."""
    wl = WORKLOADS[wi]
    T = max(wl.loops)
    inputs = generate(wl)
    got, idx, _, traj, diag = run_loop(wl, inputs, T, traj=True)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    H = traj.reshape(T + 1, wl.batch, wl.seq, wl.dim)
    P = 64
    pin = prefix(inputs, P)
    pwl = wl.replace(seq=P)
    pidx = idx.reshape(T, wl.batch, wl.seq, wl.top_k)[:, :, :P]
    # every loop from the GPU's own state: routing identical outside near-ties (one loop of
    # rounding between the two), the next state within the bounds
    prows = [(b, s) for b in range(wl.batch) for s in range(P)]
    for t in range(T):
        fidx = pidx[t].reshape(-1, wl.top_k)
        want1, _, st = O.loop_step_rows(H[t][:, :P], pin["e"], pin, pwl, t, prows, follow_idx=fidx)
        assert st["mismatch"] == 0, f"loop {t}: {st['mismatch']} routing differences outside near-ties"
        assert_close(H[t + 1][:, :P].reshape(-1, wl.dim), want1, what=f"{wl.name} prefix, loop {t} from the GPU's state")
    # all T loops from h0: over many loops the two trajectories drift apart (within the
    # bounds), enough to move logits by more than the near-tie gap, so the oracle adopts the
    # GPU's routing everywhere here and the states are compared
    want = O.loop_forward(pin["h0"], pin["e"], T, pin, pwl,
                          follow=[pidx[t].reshape(-1, wl.top_k) for t in range(T)], tie_band=np.inf)
    assert_close(got[:, :P], want, what=f"{wl.name} prefix")
    rows = sampled_rows(wl, wi)
    for t in (0, T - 1):
        fidx = np.stack([idx[t].reshape(wl.batch, wl.seq, -1)[b, s] for b, s in rows])
        hn, r, st = O.loop_step_rows(H[t], inputs["e"], inputs, wl, t, rows, follow_idx=fidx)
        assert st["mismatch"] == 0
        gt = np.stack([H[t + 1][b, s] for b, s in rows])
        assert_close(gt, hn, what=f"{wl.name} loop {t}, {len(rows)} sampled rows")
    np.testing.assert_array_equal(H[T], got)


def test_invalid_arguments_return_errors():
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    wl = C1.replace(batch=1, seq=64)
    inputs = generate(wl)
    with handle(wl, inputs, max_loops=4) as h:
        e = act(wl, inputs["e"])
        with pytest.raises(R.RdtError) as ex:
            h.loop_forward(e, e, 0)
        assert ex.value.status == 1
        with pytest.raises(R.RdtError) as ex:
            h.loop_forward(e, e, 5)
        assert ex.value.status == 1
        bad = torch.empty(e.numel() * 2 + 8, dtype=torch.uint8, device="cuda")[1:]
        with pytest.raises(R.RdtError) as ex:
            h.attn_forward(bad, 0)
        assert ex.value.status == 3
    unstable = dict(inputs)
    unstable["A"] = inputs["A"].copy()
    unstable["A"][3] = 1.0
    with pytest.raises(R.RdtError) as ex:
        handle(wl, unstable)
    assert ex.value.status == 4


def test_graph_replay_matches_eager_and_oracle():
    """Same pointers and T: call 1 runs eagerly, call 2 captures a CUDA graph, later calls
    replay it; every output must match the eager one and the oracle."""
    torch = torch_mod()
    wl = C1.replace(batch=2, seq=200)
    inputs = generate(wl)
    T = 3
    _, idx, *_ = run_loop(wl, inputs, T)
    want, mism, _, _ = oracle_follow(wl, inputs, T, idx)
    assert mism == 0
    with handle(wl, inputs, max_loops=T) as h:
        e = act(wl, inputs["e"])
        out = torch.empty(e.shape, dtype=torch.float32, device="cuda")
        outs, counts = [], []
        for _ in range(4):
            n0 = h.launch_count()
            h.loop_forward(e, e, T, out=out)
            torch.cuda.synchronize()
            counts.append(h.launch_count() - n0)
            outs.append(out.cpu().numpy().copy())
    assert len(set(counts)) == 1 and counts[0] > 0
    # the expert sums are reduced with atomics, so bits may differ between runs; bf16
    # rounding of the next loop's inputs can turn such ulp differences into ~1e-4 ones
    for o in outs[1:]:
        assert errors(o, outs[0])[0] < 2e-3
    for o in outs:
        assert_close(o, want, what="graph replay")
