"""Decode with a per-loop KV cache (rdt_decode_prefill / rdt_decode_step) through the C ABI.

Against the fp64 oracle's cached decode (loop_prefill, then loop_decode one token at a
time): the prompt's h_T and every new token's h_T within the loop's bounds (max-abs 3e-2,
relative Frobenius 1e-2), for GQA, MLA (the latent cache) and depth-wise LoRA beyond its
adapters. Against the GPU's own plain loop over the longer sequence (causality: a new
token's result depends on the earlier positions only), and the step's CUDA-graph replay
against eager launches, bit for bit in deterministic mode. Invalid calls return errors.
"""
import numpy as np
import pytest

import oracle as O
from workloads import WORKLOADS, generate, round_bf16

from rdt_testlib import act, assert_close, errors, torch_mod

pytestmark = pytest.mark.gpu

C0, C1, C2, C3, C4 = WORKLOADS

CASES = {
    "gqa": (C1.replace(batch=2, seq=72), 3),
    "mla": (C2.replace(batch=2, seq=72), 3),
    "lora": (C4.replace(seq=64, n_lora=2), 3),       # loop 2 reuses adapter 1
}
STEPS = 3


def new_tokens(wl, steps, seed=99):
    """Inputs of the decoded tokens: e ~ N(0, 1) [steps, batch, dim], rounded like the prompt."""
    rng = np.random.default_rng(seed)
    e = rng.standard_normal((steps, wl.batch, wl.dim)).astype(np.float32)
    return round_bf16(e) if wl.dtype == "bf16" else e


def handle(wl, inputs, T, max_decode, deterministic=True):
    import recurrent_depth_transformer_b200 as R
    w = R.device_weights(inputs, wl.dtype == "bf16")
    return R.RDT(R.make_config(wl, max_loops=T, deterministic=deterministic, max_decode=max_decode), w)


def gpu_decode(wl, inputs, T, en, h=None, trace=False):
    """Prefill and decode steps; with trace, also the routing of every loop of the prefill
    ([T, N, k]) and of each step ([T, batch, k])."""
    torch = torch_mod()
    own = h is None
    if own:
        h = handle(wl, inputs, T, len(en))
    N, k = wl.batch * wl.seq, wl.top_k
    idx = torch.full((T, N, k), -1, dtype=torch.int32, device="cuda") if trace else None
    if trace:
        h.set_trace(idx, None, None)
    e = act(wl, inputs["e"])
    hp = h.decode_prefill(e, e, T).cpu().numpy()
    routes = [idx.cpu().numpy()] if trace else []
    outs = []
    for i in range(len(en)):
        x = act(wl, en[i])
        outs.append(h.decode_step(x, x, T).cpu().numpy())
        if trace:
            routes.append(idx.cpu().numpy()[:, :wl.batch].copy())
    torch.cuda.synchronize()
    if trace:
        h.set_trace(None, None, None)
    diag = h.diagnostics()
    if own:
        h.close()
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    return (hp, outs, routes) if trace else (hp, outs)


@pytest.mark.parametrize("name", list(CASES))
def test_decode_matches_oracle(name):
    wl, T = CASES[name]
    inputs = generate(wl)
    en = new_tokens(wl, STEPS)
    hp, outs, routes = gpu_decode(wl, inputs, T, en, trace=True)
    st = {}
    want_p, cache = O.loop_prefill(inputs["h0"], inputs["e"], T, inputs, wl,
                                   follow=[routes[0][t] for t in range(T)], stats=st)
    assert_close(hp, want_p, what=f"{name} prefill")
    for i in range(STEPS):
        x = en[i][:, None, :]
        want = O.loop_decode(x, x, T, inputs, wl, cache, follow=[routes[1 + i][t] for t in range(T)], stats=st)[:, 0]
        assert_close(outs[i], want, what=f"{name} decode step {i}")
    assert st["mismatch"] == 0, f"{st['mismatch']} routing differences outside near-ties"


def test_decode_equals_plain_loop_over_the_longer_sequence():
    """Positions S .. S + 2 decoded one at a time = the same positions of one plain loop over
    S + 3 positions (same kernels up to tile shapes and summation order)."""
    torch = torch_mod()
    wl, T = CASES["gqa"]
    inputs = generate(wl)
    en = new_tokens(wl, STEPS)
    hp, outs = gpu_decode(wl, inputs, T, en)
    long_wl = wl.replace(seq=wl.seq + STEPS)
    e_long = np.concatenate([inputs["e"], np.transpose(en, (1, 0, 2))], axis=1)
    lin = dict(inputs)
    lin["e"] = e_long
    lin["h0"] = e_long
    with handle(long_wl, lin, T, 0) as h:
        x = act(long_wl, e_long)
        full = h.loop_forward(x, x, T).cpu().numpy()
    torch.cuda.synchronize()
    assert errors(hp, full[:, :wl.seq])[0] < 1e-2
    for i in range(STEPS):
        assert errors(outs[i], full[:, wl.seq + i])[0] < 1e-2


def test_decode_graph_replay_equals_eager_bit_for_bit():
    """Steps after the first run from a captured CUDA graph (the position advances on the
    device); with per-kernel timing on, every step runs eagerly. Deterministic mode: equal."""
    wl, T = CASES["mla"]
    inputs = generate(wl)
    en = new_tokens(wl, 4)
    h = handle(wl, inputs, T, 4)
    hp_g, outs_g = gpu_decode(wl, inputs, T, en, h=h)
    h.profile(1)                                  # eager launches from here on
    hp_e, outs_e = gpu_decode(wl, inputs, T, en, h=h)
    h.close()
    np.testing.assert_array_equal(hp_g, hp_e)
    for a, b in zip(outs_g, outs_e):
        np.testing.assert_array_equal(a, b)


def test_decode_invalid_calls():
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    wl, T = CASES["gqa"]
    inputs = generate(wl)
    en = new_tokens(wl, 3)
    with handle(wl, inputs, T, 2) as h:
        x = act(wl, en[0])
        with pytest.raises(R.RdtError) as ex:
            h.decode_step(x, x, T)                    # no prefill yet
        assert ex.value.status == 1
        e = act(wl, inputs["e"])
        h.decode_prefill(e, e, T)
        with pytest.raises(R.RdtError) as ex:
            h.decode_step(x, x, T - 1)                # another number of loops
        assert ex.value.status == 1
        h.decode_step(x, x, T)
        h.decode_step(x, x, T)
        with pytest.raises(R.RdtError) as ex:
            h.decode_step(x, x, T)                    # the cache holds seq + 2 positions
        assert ex.value.status == 1
        torch.cuda.synchronize()
    with handle(wl, inputs, T, 0) as h:
        e = act(wl, inputs["e"])
        with pytest.raises(R.RdtError) as ex:
            h.decode_prefill(e, e, T)                 # no cache
        assert ex.value.status == 1
