"""GPU parity of the ACT halting loop (rdt_set_act / rdt_loop_forward_act) through the C ABI.

Against the fp64 oracle: the output within max-abs 3e-2 and relative Frobenius 1e-2 (the
plain loop's bounds; the output is a convex combination of states); halting loops identical
wherever the oracle's summed probability is more than 2e-2 from the threshold (nearer, the
oracle adopts the GPU's decision, as it does for routing near-ties); router indices
identical outside near-ties.

Against the GPU's own recorded states, recomputed in fp64: every halting decision follows
the rule within 1e-4 of the threshold, halted states stay bit-identical, halted tokens are
routed nowhere, and the output is the weighted sum of the states within 1e-3.
"""
import math

import numpy as np
import pytest

import oracle as O
from workloads import WORKLOADS, act_head, generate

from rdt_testlib import act, assert_close, errors, handle, torch_mod

pytestmark = pytest.mark.gpu

C0, C1, C2, C3, C4 = WORKLOADS

SMALL = {
    "tiny-f32": (C0, 4),
    "gqa-s200": (C1.replace(batch=2, seq=200), 6),
    "mla-s136": (C2.replace(batch=2, seq=136), 4),
    "widemoe-s192": (C3.replace(batch=1, seq=192), 3),
    "long-lora-s320": (C4.replace(seq=320), 3),
}


def run_act(wl, inputs, T, head, traj=True, h=None):
    """Run rdt_loop_forward_act with routing and state traces; returns
    (out [B,S,d], n_loops [B,S], idx [T,N,k], traj [T+1,N,d] or None, diagnostics)."""
    torch = torch_mod()
    own = h is None
    if own:
        h = handle(wl, inputs, max_loops=T)
    N = wl.batch * wl.seq
    idx = torch.full((T, N, wl.top_k), -2, dtype=torch.int32, device="cuda")
    wts = torch.zeros((T, N, wl.top_k), dtype=torch.float32, device="cuda")
    tr = torch.zeros((T + 1, N, wl.dim), dtype=torch.float32, device="cuda") if traj else None
    h.set_trace(idx, wts, tr)
    w = torch.from_numpy(np.ascontiguousarray(head["w_halt"], dtype=np.float32)).cuda()
    h.set_act(w, head["b_halt"], head["threshold"])
    e = act(wl, inputs["e"])
    h0 = e if inputs["h0"] is inputs["e"] else act(wl, inputs["h0"])
    out, nl = h.loop_forward_act(h0, e, T)
    torch.cuda.synchronize()
    diag = h.diagnostics()
    h.set_trace(None, None, None)
    res = (out.cpu().numpy(), nl.cpu().numpy().reshape(wl.batch, wl.seq), idx.cpu().numpy(),
           None if tr is None else tr.cpu().numpy(), diag)
    if own:
        h.close()
    return res


def oracle_act(wl, inputs, T, head, idx, n_loops, trace=None):
    N = wl.batch * wl.seq
    follow = [idx[t].reshape(N, wl.top_k) for t in range(T)]
    return O.loop_forward_act(inputs["h0"], inputs["e"], T, inputs, wl, head["w_halt"], head["b_halt"],
                              head["threshold"], follow=follow, follow_loops=n_loops, trace=trace)


def running_sums(states, head, n_loops, T):
    """c + p_t of every position still running at loop t (NaN once halted), from the states
    h_1 .. h_T of one implementation, in fp64."""
    N = n_loops.size
    nl = n_loops.reshape(N)
    w = np.asarray(head["w_halt"], dtype=np.float64)
    c = np.zeros(N)
    out = np.full((T, N), np.nan)
    for t in range(T):
        run = nl > t
        h = np.asarray(states[t + 1], dtype=np.float64).reshape(N, -1)
        reach = c + 1.0 / (1.0 + np.exp(-(h @ w + head["b_halt"])))
        out[t, run] = reach[run]
        c = np.where(run, reach, c)
    return out


def check_self_consistent(wl, head, T, out, nl, idx, traj, band=1e-4):
    """The GPU's decisions, frozen states, routing and output, from its own states in fp64."""
    N, d = wl.batch * wl.seq, wl.dim
    H = traj.reshape(T + 1, N, d).astype(np.float64)
    nl = nl.reshape(N)
    assert nl.min() >= 1 and nl.max() <= T
    w = np.asarray(head["w_halt"], dtype=np.float64)
    thr = head["threshold"]
    c = np.zeros(N)
    want = np.zeros((N, d))
    for t in range(T):
        run = nl > t
        here = nl == t + 1
        frozen = ~run
        np.testing.assert_array_equal(H[t + 1][frozen], H[t][frozen])
        routed = idx[t].reshape(N, -1)
        assert np.all(routed[frozen] == -1) and np.all(routed[run] >= 0)
        p = 1.0 / (1.0 + np.exp(-(H[t + 1] @ w + head["b_halt"])))
        reach = c + p
        if t < T - 1:
            assert np.all(reach[run & ~here] < thr + band), "a token ran on past the threshold"
            assert np.all(reach[here] >= thr - band), "a token halted below the threshold"
        wgt = np.where(here, 1.0 - c, np.where(run, p, 0.0))
        want += wgt[:, None] * H[t + 1]
        c = np.where(run, reach, c)
    assert errors(out.reshape(N, d), want)[0] < 1e-3


@pytest.mark.parametrize("name", list(SMALL))
def test_act_matches_oracle_small(name):
    wl, T = SMALL[name]
    inputs = generate(wl)
    head = act_head(wl)
    out, nl, idx, traj, diag = run_act(wl, inputs, T, head)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    assert len(np.unique(nl)) >= 2, "the head must halt tokens at different loops"
    check_self_consistent(wl, head, T, out, nl, idx, traj)
    tr = O.LoopTrace()
    r = oracle_act(wl, inputs, T, head, idx, nl, trace=tr)
    assert r.stats["mismatch"] == 0, f"{r.stats['mismatch']} routing differences outside near-ties"
    assert r.stats["halt_mismatch"] == 0, f"{r.stats['halt_mismatch']} halting differences outside the band"
    np.testing.assert_array_equal(r.n_loops, nl)
    assert_close(out, r.out, what=f"{name} ACT")
    # Evidence for the follow band: how far the GPU's running sums c + p_t (from its fp32
    # states) are from the oracle's (fp64 states), and how many decisions the oracle adopted.
    gpu = running_sums(traj, head, nl, T)
    ora = running_sums(tr.h, head, nl, T)
    diff = np.nanmax(np.abs(gpu - ora))
    n = wl.batch * wl.seq
    print(f"ACT band {name}: max|sum_p gpu - oracle| = {diff:.3e} over {np.count_nonzero(~np.isnan(gpu))} "
          f"running (token, loop) pairs; {r.stats['near_halts']} of {n} decisions adopted in the "
          f"{O.NEAR_HALT:g} band")
    assert diff < O.NEAR_HALT / 2, "the band must cover the measured difference with margin"
    assert r.stats["near_halts"] <= max(2, n // 100)


def test_act_certain_halt_is_one_loop():
    wl = C1.replace(batch=2, seq=200)
    inputs = generate(wl)
    head = {"w_halt": np.zeros(wl.dim, dtype=np.float32), "b_halt": 60.0, "threshold": 0.99}
    with handle(wl, inputs, max_loops=5) as h:
        out, nl, idx, _, diag = run_act(wl, inputs, 5, head, traj=False, h=h)
        e = act(wl, inputs["e"])
        one = h.loop_forward(e, e, 1).cpu().numpy()
    assert np.all(nl == 1)
    assert errors(out, one)[0] < 1e-4            # one loop, weight exactly 1
    N = wl.batch * wl.seq
    want = O.loop_forward(inputs["h0"], inputs["e"], 1, inputs, wl, follow=[idx[0].reshape(N, -1)])
    assert_close(out, want, what="certain halt")


@pytest.mark.parametrize("T,loops", [(6, 4), (2, 2)])
def test_act_constant_probability(T, loops):
    """w = 0, p = 0.3: every token halts at loop min(4, T), weights 0.3 per loop and the
    remainder at the halting loop."""
    wl = C1.replace(batch=2, seq=200)
    inputs = generate(wl)
    head = {"w_halt": np.zeros(wl.dim, dtype=np.float32), "b_halt": math.log(0.3 / 0.7), "threshold": 0.99}
    out, nl, idx, traj, diag = run_act(wl, inputs, T, head)
    assert np.all(nl == loops)
    check_self_consistent(wl, head, T, out, nl, idx, traj)
    r = oracle_act(wl, inputs, T, head, idx, nl)
    assert r.stats["mismatch"] == 0
    assert_close(out, r.out, what="constant p")


def test_act_threshold_one_runs_every_loop():
    wl = C3.replace(batch=1, seq=192)
    inputs = generate(wl)
    head = {"w_halt": np.zeros(wl.dim, dtype=np.float32), "b_halt": -4.0, "threshold": 1.0}
    T = 4
    out, nl, idx, traj, diag = run_act(wl, inputs, T, head)
    assert np.all(nl == T)
    check_self_consistent(wl, head, T, out, nl, idx, traj)
    r = oracle_act(wl, inputs, T, head, idx, nl)
    assert r.stats["mismatch"] == 0
    assert_close(out, r.out, what="threshold 1")


def test_act_graph_replay_and_plain_loop_unaffected():
    """Same pointers and T: the ACT loop runs eagerly, is captured, then replayed; a plain
    loop on the same handle before and after gives the same result."""
    torch = torch_mod()
    wl = C1.replace(batch=2, seq=200)
    inputs = generate(wl)
    head = act_head(wl)
    T = 5
    with handle(wl, inputs, max_loops=T) as h:
        e = act(wl, inputs["e"])
        plain0 = h.loop_forward(e, e, T).cpu().numpy()
        h.set_act(torch.from_numpy(head["w_halt"]).cuda(), head["b_halt"], head["threshold"])
        out = torch.empty(e.shape, dtype=torch.float32, device="cuda")
        nl = torch.empty(e.shape[:-1], dtype=torch.int32, device="cuda")
        outs, loops, counts = [], [], []
        for _ in range(4):
            n0 = h.launch_count()
            h.loop_forward_act(e, e, T, out=out, n_loops=nl)
            torch.cuda.synchronize()
            counts.append(h.launch_count() - n0)
            outs.append(out.cpu().numpy().copy())
            loops.append(nl.cpu().numpy().copy())
        plain1 = h.loop_forward(e, e, T).cpu().numpy()
        diag = h.diagnostics()
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    assert len(set(counts)) == 1 and counts[0] > 0
    for o, l in zip(outs[1:], loops[1:]):
        assert np.mean(l == loops[0]) >= 0.99       # atomics may move a near-threshold token
        same = (l == loops[0])
        assert errors(o[same], outs[0][same])[0] < 2e-3
    assert errors(plain1, plain0)[0] < 2e-3


def test_act_full_size_self_consistent_and_sampled_rows():
    """The GQA configuration at full size (batch 4 x 512, 8 loops): decisions, frozen states,
    routing and output from the GPU's own states, and one loop at sampled running rows
    against the oracle's single-step evaluation from the GPU's h_t."""
    wl = C1
    T = 8
    inputs = generate(wl)
    head = act_head(wl)
    out, nl, idx, traj, diag = run_act(wl, inputs, T, head)
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    assert len(np.unique(nl)) >= 4
    check_self_consistent(wl, head, T, out, nl, idx, traj)
    t = 3
    run_rows = np.argwhere(nl > t)
    rng = np.random.default_rng(8)
    pick = run_rows[rng.choice(len(run_rows), size=4, replace=False)]
    rows = [(int(b), int(s)) for b, s in pick]
    H = traj.reshape(T + 1, wl.batch, wl.seq, wl.dim)
    fidx = np.stack([idx[t].reshape(wl.batch, wl.seq, -1)[b, s] for b, s in rows])
    hn, _, st = O.loop_step_rows(H[t], inputs["e"], inputs, wl, t, rows, follow_idx=fidx)
    assert st["mismatch"] == 0
    assert_close(np.stack([H[t + 1][b, s] for b, s in rows]), hn, what="ACT sampled rows")


def test_act_invalid_arguments():
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    wl = C1.replace(batch=1, seq=64)
    inputs = generate(wl)
    with handle(wl, inputs, max_loops=4) as h:
        e = act(wl, inputs["e"])
        with pytest.raises(R.RdtError) as ex:
            h.loop_forward_act(e, e, 2)                 # no head set
        assert ex.value.status == 1
        w = torch.zeros(wl.dim, dtype=torch.float32, device="cuda")
        for b, thr in ((0.0, 0.0), (0.0, 1.5), (float("nan"), 0.99)):
            with pytest.raises(R.RdtError) as ex:
                h.set_act(w, b, thr)
            assert ex.value.status == 1
        h.set_act(w, 0.0, 0.99)
        with pytest.raises(R.RdtError) as ex:
            h.loop_forward_act(e, e, 5)                 # T > max_loops
        assert ex.value.status == 1
