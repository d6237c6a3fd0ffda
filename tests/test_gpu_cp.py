"""Context parallelism (rdt_config.cp_size > 1) against the whole sequence on one handle.

Rank r of G holds positions [r S, (r + 1) S) of every sequence. Its QKV projection writes
its rotated keys and values into the gather buffers of ranks r .. G - 1 (its own included),
flag words in the ranks' memory order the push, the attention and the next loop's push.
Only one GPU is available here, so the ranks are separate handles on the same device and
stream, run one loop each in turn: rank 0's loop, rank 1's, ..., then the next loop. Every
flag a rank waits for has then been set by a kernel that already finished, so no kernel ever
waits for another that has not run. A loop is a call with T = 1, the state carried to the
next call in the element type; the reference chains its calls the same way.

In deterministic mode nothing in a row's arithmetic depends on how the sequence is split
(the projections, the attention over key blocks that start at position 0, the routing, the
expert rows, the fixed-order combine), so the ranks' outputs must equal the reference bit for
bit. The default mode (fp32 atomics) must agree within rounding.
"""
import numpy as np
import pytest

from workloads import WORKLOADS, generate

from rdt_testlib import act, assert_close, torch_mod

pytestmark = pytest.mark.gpu

C0, C1, C2, C3, C4 = WORKLOADS

CASES = {
    "gqa-g2": (C1, 2, 3),                                     # batch 4, 2 x 256 positions
    "gqa-g4": (C1, 4, 2),                                     # 4 x 128 positions
    "long-lora-g2": (C4.replace(seq=1024), 2, 2),             # 32/8 heads, LoRA, tensor-core router
    "widemoe-g4": (C3.replace(batch=1, seq=512), 4, 2),       # shared expert, 4 x 128 positions
}


def _reference(wl, inputs, T, det):
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    w = R.device_weights(inputs, True)
    with R.RDT(R.make_config(wl, max_loops=1, deterministic=det), w) as h:
        e = act(wl, inputs["e"])
        state = e.clone()
        out = torch.empty(e.shape, dtype=torch.float32, device="cuda")
        for _ in range(T):
            h.loop_forward(state, e, 1, out=out)
            state = out.to(torch.bfloat16)
        torch.cuda.synchronize()
        d = h.diagnostics()
        assert d["timeout"] == 0 and d["nonfinite"] == 0
        return out.cpu().numpy()


def _ranks(wl, inputs, T, G, det):
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    S = wl.seq // G
    local = wl.replace(seq=S)
    w = R.device_weights(inputs, True)
    hs = [R.RDT(R.make_config(local, max_loops=1, deterministic=det, cp_size=G, cp_rank=r), w) for r in range(G)]
    try:
        bufs = [h.cp_buffers() for h in hs]
        for h in hs:
            h.cp_connect([b[0] for b in bufs], [b[2] for b in bufs])
        e = act(wl, inputs["e"])
        es = [e[:, r * S:(r + 1) * S].contiguous() for r in range(G)]
        states = [x.clone() for x in es]
        outs = [torch.empty(x.shape, dtype=torch.float32, device="cuda") for x in es]
        for _ in range(T):
            for r in range(G):
                hs[r].loop_forward(states[r], es[r], 1, out=outs[r])
            states = [o.to(torch.bfloat16) for o in outs]
        torch.cuda.synchronize()
        for h in hs:
            d = h.diagnostics()
            assert d["timeout"] == 0 and d["nonfinite"] == 0
        return torch.cat(outs, dim=1).cpu().numpy()
    finally:
        for h in hs:
            h.close()


@pytest.mark.parametrize("name", list(CASES))
def test_context_parallel_ranks_equal_the_whole_sequence_bit_for_bit(name):
    wl, G, T = CASES[name]
    inputs = generate(wl)
    want = _reference(wl, inputs, T, True)
    got = _ranks(wl, inputs, T, G, True)
    assert got.shape == want.shape
    diff = np.abs(got - want)
    assert np.array_equal(got, want), (f"{int((diff > 0).sum())} of {diff.size} elements differ, "
                                       f"max {diff.max():.3e}")


@pytest.mark.parametrize("name", ["gqa-g2", "long-lora-g2"])
def test_context_parallel_default_mode_within_rounding(name):
    wl, G, T = CASES[name]
    inputs = generate(wl)
    want = _reference(wl, inputs, T, False)
    got = _ranks(wl, inputs, T, G, False)
    # the state is carried between calls in bf16: a rounding that falls the other way (the
    # atomics' order differs) moves an element by a bf16 ulp of its magnitude, 2^-8 of it,
    # and the next loop carries that on; 4 ulps of the largest element bound it
    assert_close(got, want, max_abs=2.0 ** -6 * float(np.abs(want).max()), rel_fro=1e-3,
                 what=f"{name} context-parallel vs whole sequence")


def test_context_parallel_needs_connect_and_rejects_single_block_and_bad_configs():
    torch = torch_mod()
    import recurrent_depth_transformer_b200 as R
    wl = C1.replace(batch=1, seq=256)
    inputs = generate(wl)
    w = R.device_weights(inputs, True)
    with R.RDT(R.make_config(wl.replace(seq=128), max_loops=2, cp_size=2, cp_rank=1), w) as h:
        e = act(wl, inputs["e"])[:, 128:].contiguous()
        out = torch.empty(e.shape, dtype=torch.float32, device="cuda")
        with pytest.raises(R.RdtError, match="INVALID_ARG"):
            h.loop_forward(e, e, 1, out=out)                     # not connected
        with pytest.raises(R.RdtError, match="UNSUPPORTED"):
            h.attn_forward(e, 0)                                  # single block: no peers' keys
        with pytest.raises(R.RdtError, match="INVALID_ARG"):
            h.cp_connect([0, 0], [0, 0])                          # rank 0's buffers missing
    with pytest.raises(R.RdtError, match="UNSUPPORTED"):
        R.RDT(R.make_config(wl.replace(seq=96), max_loops=1, cp_size=2, cp_rank=0), w)   # seq % 128
    with pytest.raises(R.RdtError, match="INVALID_ARG"):
        R.RDT(R.make_config(wl.replace(seq=128), max_loops=1, cp_size=2, cp_rank=2), w)  # rank >= size
