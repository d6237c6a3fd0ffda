"""Depth attention (a token's attention over its own earlier loop states) through the C ABI,
against the fp64 oracle.

Reduced size, all positions: h_T within the loop's bounds (max-abs 3e-2, relative Frobenius
1e-2) with router indices identical outside near-ties. Full size (batch 4 x 512, 8 loops):
every loop from the GPU's own states on the first 64 positions (depth attention over the
GPU's block inputs of loops 0 .. t, then the sequence attention, the experts and the update
equation), routing identical outside near-ties; then all loops from h0 with the GPU's
routing. A zero output projection of the depth attention gives the plain loop; the
deterministic mode repeats bit for bit.
"""
import numpy as np
import pytest

import oracle as O
from workloads import DEPTH_WORKLOAD, generate, prefix

from rdt_testlib import act, assert_close, errors, oracle_follow, run_loop, torch_mod

pytestmark = pytest.mark.gpu

WL = DEPTH_WORKLOAD


def test_depth_attention_loop_matches_oracle_small():
    wl = WL.replace(batch=2, seq=200)
    inputs = generate(wl)
    T = 4
    got, idx, _, _, diag = run_loop(wl, inputs, T)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    want, mism, _, _ = oracle_follow(wl, inputs, T, idx)
    assert mism == 0
    assert_close(got, want, what="depth attention, 200 positions")


def _step_from_states(H, inputs, wl, t, T, P, fidx):
    """h_{t+1} of the first P positions from the given states h_0 .. h_t (one loop)."""
    W = inputs
    e = inputs["e"][:, :P].astype(np.float64)
    kv = O.DepthKV()
    d = None
    for s in range(t + 1):
        d = O.depth_attention_sublayer(H[s][:, :P] + e, W, wl, s, T, kv)
    x = H[t][:, :P] + e + d
    a = O.attention_sublayer(x, W, wl, t)
    y = x + a
    f, r, st = O.moe_sublayer(y, W, wl, fidx)
    Be = O.input_injection(e, W["B"])
    return W["A"].astype(np.float64) * H[t][:, :P] + Be + d + a + f, st


def test_depth_attention_full_size():
    wl = WL
    T = max(wl.loops)
    inputs = generate(wl)
    got, idx, _, traj, diag = run_loop(wl, inputs, T, traj=True)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    H = traj.reshape(T + 1, wl.batch, wl.seq, wl.dim).astype(np.float64)
    P = 64
    pidx = idx.reshape(T, wl.batch, wl.seq, wl.top_k)[:, :, :P]
    pwl = wl.replace(seq=P)
    for t in range(T):
        want1, st = _step_from_states(H, inputs, pwl, t, T, P, pidx[t].reshape(-1, wl.top_k))
        assert st["mismatch"] == 0, f"loop {t}: {st['mismatch']} routing differences outside near-ties"
        assert_close(H[t + 1][:, :P], want1, what=f"depth attention, loop {t} from the GPU's states")
    pin = prefix(inputs, P)
    want = O.loop_forward(pin["h0"], pin["e"], T, pin, pwl,
                          follow=[pidx[t].reshape(-1, wl.top_k) for t in range(T)], tie_band=np.inf)
    assert_close(got[:, :P], want, what="depth attention prefix, all loops")


def test_zero_depth_output_gives_the_plain_loop():
    wl = WL.replace(batch=2, seq=136)
    inputs = generate(wl)
    inputs["wo_d"] = np.zeros_like(inputs["wo_d"])
    got, *_ = run_loop(wl, inputs, 3, trace=False)
    plain, *_ = run_loop(wl.replace(da_heads=0, da_kv_heads=0), inputs, 3, trace=False)
    assert errors(got, plain)[0] < 2e-3          # the same sums up to atomics order


def test_depth_attention_deterministic_repeats_bit_for_bit():
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    wl = WL.replace(batch=2, seq=136)
    inputs = generate(wl)
    w = R.device_weights(inputs, True)
    with R.RDT(R.make_config(wl, max_loops=4, deterministic=True), w) as h:
        e = act(wl, inputs["e"])
        out = torch.empty(e.shape, dtype=torch.float32, device="cuda")
        outs = []
        for _ in range(4):
            h.loop_forward(e, e, 4, out=out)
            torch.cuda.synchronize()
            outs.append(out.cpu().numpy().copy())
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])
