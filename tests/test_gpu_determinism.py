"""Deterministic mode (rdt_config.deterministic = 1) and the bounded device waits.

Deterministic mode stores each expert row's weighted output in its own row and adds a
token's rows in a fixed order, with no K split reduced by atomics: three runs of
rdt_loop_forward (eager, graph capture, graph replay) must agree bit for bit, and still
match the fp64 oracle within the loop's bounds. The default mode reduces with fp32 atomics
and is only required to agree within rounding.

The bounded-wait probe waits on a barrier that nothing arrives on: the wait must give up
after its limit, the status must reach the host, and the context must stay usable.
"""
import time

import numpy as np
import pytest

from workloads import WORKLOADS, generate

from rdt_testlib import act, assert_close, oracle_follow, torch_mod

pytestmark = pytest.mark.gpu

C0, C1, C2, C3, C4 = WORKLOADS

CASES = {
    "tiny-f32": (C0, 3),                              # fp32 FMA router
    "gqa-s200": (C1.replace(batch=2, seq=200), 3),    # fused shared-memory router
    "mla-s136": (C2.replace(batch=2, seq=136), 2),
    "widemoe-s192": (C3.replace(batch=1, seq=192), 3),  # tensor-core router, shared expert
    "long-lora-s320": (C4.replace(seq=320), 3),       # tensor-core router, LoRA
}


def _runs(wl, inputs, T, deterministic, n=4, trace=False):
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    w = R.device_weights(inputs, wl.dtype == "bf16")
    outs = []
    idx = None
    with R.RDT(R.make_config(wl, max_loops=T, deterministic=deterministic), w) as h:
        if trace:
            idx = torch.full((T, wl.batch * wl.seq, wl.top_k), -1, dtype=torch.int32, device="cuda")
            h.set_trace(idx, None, None)
        e = act(wl, inputs["e"])
        out = torch.empty(e.shape, dtype=torch.float32, device="cuda")
        for _ in range(n):
            h.loop_forward(e, e, T, out=out)
            torch.cuda.synchronize()
            outs.append(out.cpu().numpy().copy())
        diag = h.diagnostics()
    assert diag["nonfinite"] == 0 and diag["timeout"] == 0
    return outs, (None if idx is None else idx.cpu().numpy())


@pytest.mark.parametrize("name", list(CASES))
def test_deterministic_mode_is_bit_identical_and_matches_oracle(name):
    wl, T = CASES[name]
    inputs = generate(wl)
    outs, _ = _runs(wl, inputs, T, True)                  # eager, capture, replay, replay
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])
    traced, idx = _runs(wl, inputs, T, True, n=1, trace=True)   # eager with the routing trace
    np.testing.assert_array_equal(traced[0], outs[0])
    want, mism, _, _ = oracle_follow(wl, inputs, T, idx)
    assert mism == 0
    assert_close(outs[0], want, what=f"{name} deterministic")


def test_deterministic_mode_equals_default_mode_within_rounding():
    """The two modes sum the same terms in different orders (and the default mode splits
    some K sums over CTAs): a last-bit difference can round a bf16 activation of the next
    loop the other way, so they agree within the loop's parity bounds, far inside them in
    the relative Frobenius norm."""
    wl, T = CASES["widemoe-s192"]
    inputs = generate(wl)
    det, _ = _runs(wl, inputs, T, True, n=1)
    dflt, _ = _runs(wl, inputs, T, False, n=1)
    assert_close(det[0], dflt[0], rel_fro=1e-3, what="deterministic vs default")


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    lib = R.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    for limit_ns in (1000, 1000000, 200000000):
        t0 = time.perf_counter()
        st = lib.rdt_wait_probe(limit_ns, stream)
        el = time.perf_counter() - t0
        assert st == 7, lib.rdt_last_error()              # RDT_ERR_DEVICE_TIMEOUT
        assert el < limit_ns * 1e-9 + 0.5, el             # it returned promptly after the limit
    assert lib.rdt_wait_probe(0, stream) == 1
    # the context still runs the block
    wl = C1.replace(batch=1, seq=128)
    inputs = generate(wl)
    outs, _ = _runs(wl, inputs, 2, True, n=1)
    assert np.isfinite(outs[0]).all()
