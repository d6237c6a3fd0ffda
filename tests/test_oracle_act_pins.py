"""Pins of the oracle's ACT halting loop against facts fixed outside it: a hand-computed
fixture, closed forms for a constant halting probability, the plain loop for positions
whose prefix never halts, and a library sigmoid. A head applied to the old state instead
of the new one, a dropped remainder, halted positions that keep updating, or a scaled
expert term each fail one of them."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from workloads import Workload, generate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_gqa(**kw) -> Workload:
    base = dict(name="pin-act", dtype="f32", batch=2, seq=12, dim=32, attn="gqa", n_heads=4,
                n_kv_heads=2, head_dim=8, n_experts=4, top_k=2, expert_hidden=16,
                b_kind="diag", loops=(3,), seed=11)
    base.update(kw)
    return Workload(**base)


def _logit(p):
    return math.log(p / (1.0 - p))


def test_halting_probability_is_torch_sigmoid():
    rng = np.random.default_rng(5)
    h = rng.standard_normal((3, 7, 16)) * 4.0
    w = rng.standard_normal(16) * 0.3
    got = O.halting_probability(h, w, -0.7)
    want = torch.sigmoid(torch.from_numpy(h) @ torch.from_numpy(w) - 0.7).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)


@pytest.mark.parametrize("case", range(4))
def test_act_hand_fixture(case):
    g = json.load(open(os.path.join(GOLDEN, "act_halting_zero_block.json")))
    c = g["cases"][case]
    cfg = Workload(name="pin-zero", dtype="f32", batch=1, seq=1, dim=2, attn="gqa", n_heads=1,
                   n_kv_heads=1, head_dim=2, n_experts=1, top_k=1, expert_hidden=1,
                   b_kind="diag", loops=(3,), seed=0)
    W = generate(cfg, zero_block=True)
    W["A"] = np.array(g["A"])
    W["B"] = np.array(g["B"])
    e = np.array(g["e"]).reshape(1, 1, 2)
    h0 = np.array(g["h0"]).reshape(1, 1, 2)
    ln3 = math.log(3.0)
    w = np.array(g["w_halt_over_ln3"]) * ln3
    r = O.loop_forward_act(h0, e, c["T"], W, cfg, w, g["b_halt_over_ln3"] * ln3, c["threshold"])
    assert int(r.n_loops[0, 0]) == c["n_loops"]
    np.testing.assert_allclose(r.weights[:, 0, 0], c["weights"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(r.out.reshape(2), c["out"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("T,want_loops,want_w", [(6, 4, [0.3, 0.3, 0.3, 0.1, 0, 0]),
                                                 (3, 3, [0.3, 0.3, 0.4]),
                                                 (1, 1, [1.0])])
def test_act_constant_probability_closed_form(T, want_loops, want_w):
    """w = 0, p = 0.3 everywhere: every position halts at loop min(4, T) (0.9 < 0.99 <= 1.2)
    with the remainder, and until then all states are the plain loop's."""
    cfg = small_gqa()
    W = generate(cfg)
    r = O.loop_forward_act(W["h0"], W["e"], T, W, cfg, np.zeros(cfg.dim), _logit(0.3), 0.99)
    assert np.all(r.n_loops == want_loops)
    np.testing.assert_allclose(r.weights[:, 0, 0], want_w, rtol=0, atol=1e-12)
    tr = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], want_loops, W, cfg, trace=tr)
    want = sum(want_w[t] * tr.h[t + 1] for t in range(want_loops))
    np.testing.assert_allclose(r.out, want, rtol=1e-12, atol=1e-12)


def test_act_certain_halt_is_one_plain_loop():
    cfg = small_gqa()
    W = generate(cfg)
    r = O.loop_forward_act(W["h0"], W["e"], 5, W, cfg, np.zeros(cfg.dim), 60.0, 0.99)
    assert np.all(r.n_loops == 1)
    np.testing.assert_allclose(r.out, O.loop_forward(W["h0"], W["e"], 1, W, cfg), rtol=1e-13, atol=1e-13)


def _mixed():
    """A head that halts positions at several different loops."""
    cfg = small_gqa(seq=16)
    W = generate(cfg)
    rng = np.random.default_rng(3)
    w = rng.standard_normal(cfg.dim) * 1.5 / math.sqrt(cfg.dim)
    tr = O.LoopTrace()
    r = O.loop_forward_act(W["h0"], W["e"], 5, W, cfg, w, -0.5, 0.99, trace=tr)
    return cfg, W, w, r, tr


def test_act_mixed_weights_and_frozen_states():
    cfg, W, w, r, tr = _mixed()
    assert len(np.unique(r.n_loops)) >= 3, np.bincount(r.n_loops.ravel())
    np.testing.assert_allclose(r.weights.sum(axis=0), 1.0, rtol=0, atol=1e-12)
    assert np.all(r.weights >= 0)
    for b in range(cfg.batch):
        for s in range(cfg.seq):
            n = int(r.n_loops[b, s])
            for t in range(n + 1, 6):                 # states after the halting loop stay put
                np.testing.assert_array_equal(tr.h[t][b, s], tr.h[n][b, s])
            want = sum(r.weights[t, b, s] * tr.h[t + 1][b, s] for t in range(n))
            np.testing.assert_allclose(r.out[b, s], want, rtol=1e-12, atol=1e-12)


def test_act_running_prefix_follows_plain_loop_and_halted_keys_are_frozen():
    """A position whose whole prefix is still running at loop t has the plain loop's state
    (causal attention sees only running, unchanged positions); a position after a halted
    one departs from the plain loop (its keys are the frozen state)."""
    cfg, W, w, r, tr = _mixed()
    plain = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], 5, W, cfg, trace=plain)
    departed = 0
    for b in range(cfg.batch):
        for t in range(5):
            for s in range(cfg.seq):
                prefix_running = np.all(r.n_loops[b, : s + 1] > t)
                if prefix_running:
                    np.testing.assert_allclose(tr.h[t + 1][b, s], plain.h[t + 1][b, s], rtol=1e-12, atol=1e-12)
                elif r.n_loops[b, s] > t:
                    departed += int(not np.allclose(tr.h[t + 1][b, s], plain.h[t + 1][b, s], rtol=1e-9, atol=1e-9))
    assert departed > 0


def test_act_follow_adopts_only_near_halts():
    cfg, W, w, r, _ = _mixed()
    same = O.loop_forward_act(W["h0"], W["e"], 5, W, cfg, w, -0.5, 0.99, follow_loops=r.n_loops)
    assert same.stats["halt_mismatch"] == 0 and same.stats["near_halts"] == 0
    np.testing.assert_array_equal(same.out, r.out)
    never = np.full_like(r.n_loops, 5)               # another run that never halts early
    other = O.loop_forward_act(W["h0"], W["e"], 5, W, cfg, w, -0.5, 0.99, follow_loops=never)
    early = int(np.count_nonzero(r.n_loops < 5))
    assert other.stats["halt_mismatch"] + other.stats["near_halts"] >= 1
    assert other.stats["halt_mismatch"] <= early
