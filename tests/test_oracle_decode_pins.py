"""Pins of the oracle's decode with a per-loop KV cache against the plain loop. Causality
makes position S of a full run over S + 1 positions depend on positions 0..S only, so a
prefill over S positions followed by one decode step must give the full run's h_T at S,
and the cache of loop t must hold the keys and values the full run computes in loop t.
A cache shared by all loops, a rotation at the wrong position, a latent cached before its
RMSNorm, or a LoRA adapter of the wrong loop each fail one of them."""
import numpy as np
import pytest

import oracle as O
from workloads import Workload, generate


def small_gqa(**kw) -> Workload:
    base = dict(name="pin-dec-gqa", dtype="f32", batch=2, seq=11, dim=32, attn="gqa", n_heads=4,
                n_kv_heads=2, head_dim=8, n_experts=4, top_k=2, expert_hidden=16,
                b_kind="diag", loops=(3,), seed=21)
    base.update(kw)
    return Workload(**base)


def small_mla(**kw) -> Workload:
    base = dict(name="pin-dec-mla", dtype="f32", batch=2, seq=9, dim=32, attn="mla", n_heads=4,
                q_lora_rank=24, kv_lora_rank=16, qk_nope_dim=8, qk_rope_dim=4, v_head_dim=8,
                n_experts=4, top_k=2, expert_hidden=16, b_kind="diag", loops=(3,), seed=22)
    base.update(kw)
    return Workload(**base)


CFGS = {
    "gqa": small_gqa(),
    "mla": small_mla(),
    "gqa-lora": small_gqa(lora_rank=4, n_lora=2, seed=23),
    "gqa-denseB-h0": small_gqa(b_kind="dense", seed=24),
}
T = 3


def _inputs(name):
    cfg = CFGS[name]
    W = generate(cfg, h0_independent=name.endswith("h0"))
    return cfg, W


def test_rope_at_equals_rope_on_slices():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 9, 3, 8))
    full = O.apply_rope(x, 1.0e4)
    for p0, p1 in ((0, 9), (4, 5), (3, 8), (8, 9)):
        got = O.apply_rope_at(x[:, p0:p1], np.arange(p0, p1), 1.0e4)
        np.testing.assert_allclose(got, full[:, p0:p1], rtol=0, atol=1e-14)


@pytest.mark.parametrize("name", list(CFGS))
def test_prefill_equals_loop_forward(name):
    cfg, W = _inputs(name)
    h, cache = O.loop_prefill(W["h0"], W["e"], T, W, cfg)
    assert cache.length == cfg.seq
    np.testing.assert_allclose(h, O.loop_forward(W["h0"], W["e"], T, W, cfg), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", list(CFGS))
def test_decode_step_equals_full_run_at_that_position(name):
    cfg, W = _inputs(name)
    S = cfg.seq - 1
    full = O.loop_forward(W["h0"], W["e"], T, W, cfg)
    _, cache = O.loop_prefill(W["h0"][:, :S], W["e"][:, :S], T, W, cfg)
    got = O.loop_decode(W["h0"][:, S:], W["e"][:, S:], T, W, cfg, cache)
    assert cache.length == S + 1
    np.testing.assert_allclose(got[:, 0], full[:, S], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["gqa", "mla"])
def test_successive_decode_steps(name):
    cfg, W = _inputs(name)
    S0 = cfg.seq - 3
    full = O.loop_forward(W["h0"], W["e"], T, W, cfg)
    _, cache = O.loop_prefill(W["h0"][:, :S0], W["e"][:, :S0], T, W, cfg)
    for s in range(S0, cfg.seq):
        got = O.loop_decode(W["h0"][:, s:s + 1], W["e"][:, s:s + 1], T, W, cfg, cache)
        np.testing.assert_allclose(got[:, 0], full[:, s], rtol=1e-12, atol=1e-12)


def test_cache_holds_each_loops_keys_and_values():
    cfg, W = _inputs("gqa-lora")
    tr = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], T, W, cfg, trace=tr)
    _, cache = O.loop_prefill(W["h0"], W["e"], T, W, cfg)
    for t in range(T):
        xn = O.rmsnorm(tr.h[t] + W["e"], W["norm1"], cfg.norm_eps)
        _, k, v = O.gqa_qkv(xn, W, cfg, t)
        np.testing.assert_allclose(cache.k[t], k, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(cache.v[t], v, rtol=1e-12, atol=1e-12)
    assert not np.allclose(cache.k[0], cache.k[1])          # every loop has keys of its own


def test_mla_cache_holds_the_latent():
    cfg, W = _inputs("mla")
    tr = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], T, W, cfg, trace=tr)
    _, cache = O.loop_prefill(W["h0"], W["e"], T, W, cfg)
    for t in range(T):
        assert cache.ckv[t].shape == (cfg.batch, cfg.seq, cfg.kv_lora_rank)
        assert cache.kr[t].shape == (cfg.batch, cfg.seq, cfg.qk_rope_dim)
        xn = O.rmsnorm(tr.h[t] + W["e"], W["norm1"], cfg.norm_eps)
        _, c_kv, k_rope = O.mla_latents(xn, W, cfg)
        np.testing.assert_allclose(cache.ckv[t], c_kv, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(cache.kr[t], k_rope[:, :, 0], rtol=1e-12, atol=1e-12)
