"""rdt_moe_route_noalloc: the MoE router for callers that cannot allocate device memory
(a framework's memory pool owns the device, allocation is forbidden after start-up, or the
host captures the work into its own CUDA graphs), so they cannot create a handle. It runs
the router kernel of rdt_moe_forward with its scratch in a static device array.

Checked through the C ABI against rdt_moe_forward's top-k outputs on two calls in a row
(the shared scratch keeps the previous call's contents; the counters must restart at 0),
and against the fp64 oracle's router on every kernel path the entry point can take: the
fused shared-memory router, the bf16 tensor-core router and the fp32 FMA router.
This file sorts last so that a stop-at-first-failure run has run every other test first.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from workloads import WORKLOADS, generate, round_bf16

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("wl", [WORKLOADS[1].replace(batch=1, seq=256),
                                WORKLOADS[3].replace(batch=1, seq=128),
                                WORKLOADS[0]])
def test_noalloc_router_matches_moe_forward_twice(wl):
    import torch
    import recurrent_depth_transformer_b200 as R
    from rdt_testlib import handle

    lib = R.load_library()
    inputs = generate(wl)
    N, k, E = wl.batch * wl.seq, wl.top_k, wl.n_experts
    bf = wl.dtype == "bf16"
    wr = torch.from_numpy(inputs["w_router"])
    wr = (wr.to(torch.bfloat16) if bf else wr).cuda()
    g2 = torch.from_numpy(inputs["norm2"]).cuda()
    bias = torch.from_numpy(np.linspace(-0.05, 0.05, E).astype(np.float32)).cuda()
    dt = 1 if bf else 0
    with handle(wl, {**inputs, "router_bias": bias.cpu().numpy()}) as h:
        for call, scale in enumerate((3.0, -1.7)):
            y = torch.from_numpy(inputs["e"].reshape(N, wl.dim) * scale).cuda()
            ref_i = torch.empty((N, k), dtype=torch.int32, device="cuda")
            ref_w = torch.empty((N, k), dtype=torch.float32, device="cuda")
            h.moe_forward(y, idx=ref_i, w=ref_w)
            got_i = torch.full((N, k), -1, dtype=torch.int32, device="cuda")
            got_w = torch.zeros((N, k), dtype=torch.float32, device="cuda")
            cnt = torch.full((E,), -1, dtype=torch.int32, device="cuda")
            st = lib.rdt_moe_route_noalloc(dt, _p(y), _p(g2), _p(wr), _p(bias), N, wl.dim, E, k,
                                           ctypes.c_float(wl.norm_eps), _p(got_i), _p(got_w), _p(cnt),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert st == 0, lib.rdt_last_error()
            torch.cuda.synchronize()
            np.testing.assert_array_equal(got_i.cpu().numpy(), ref_i.cpu().numpy(), err_msg=f"call {call}")
            np.testing.assert_allclose(got_w.cpu().numpy(), ref_w.cpu().numpy(), atol=1e-5, rtol=0)
            np.testing.assert_array_equal(cnt.cpu().numpy(),
                                          np.bincount(got_i.cpu().numpy().ravel(), minlength=E))


def test_noalloc_router_rejects_sizes_beyond_its_scratch():
    import torch
    import recurrent_depth_transformer_b200 as R
    lib = R.load_library()
    d, E = 2048, 64
    big = torch.empty(16, dtype=torch.float32, device="cuda")
    st = lib.rdt_moe_route_noalloc(1, _p(big), _p(big), _p(big), None, 4096, d, E, 8,
                                   ctypes.c_float(1e-6), _p(big), _p(big), None, None)
    assert st == 2 and b"scratch" in lib.rdt_last_error()


def _oracle_check(y, g2, wr, bias, k, eps, got_i, got_w, cnt):
    """Indices identical wherever the oracle's k-th/(k+1)-th score gap exceeds 1e-3, gate
    weights within 1e-4 there, counts = histogram of the indices."""
    yn = O.rmsnorm(y, g2, eps)
    r = O.router_topk(yn @ np.asarray(wr, np.float64).T, bias, k)
    clear = r.gap > O.NEAR_TIE
    assert clear.mean() > 0.9
    # the chosen set is unique outside near-ties; the order of two chosen experts with
    # (nearly) equal scores is not, so both sides are compared sorted by expert index
    go, ro = np.argsort(got_i, axis=1), np.argsort(r.idx, axis=1)
    np.testing.assert_array_equal(np.take_along_axis(got_i, go, 1)[clear], np.take_along_axis(r.idx, ro, 1)[clear])
    np.testing.assert_allclose(np.take_along_axis(got_w, go, 1)[clear], np.take_along_axis(r.w, ro, 1)[clear],
                               atol=1e-4, rtol=0)
    np.testing.assert_array_equal(cnt, np.bincount(got_i.ravel(), minlength=wr.shape[0]))


@pytest.mark.parametrize("dtype,ntok,dim,E,k", [
    ("bf16", 256, 1024, 16, 2),     # fused shared-memory router
    ("bf16", 192, 256, 128, 8),     # bf16 tensor-core router with its top-k epilogue
    ("f32", 160, 512, 64, 8),       # fp32 FMA router (weight above the shared-memory limit)
    ("bf16", 2048, 1024, 16, 2),    # the fused path at 2048 rows: no row scratch at all
])
def test_noalloc_router_matches_oracle_on_every_path(dtype, ntok, dim, E, k):
    import torch
    import recurrent_depth_transformer_b200 as R
    lib = R.load_library()
    rng = np.random.default_rng(ntok + dim + E)
    y = (rng.standard_normal((ntok, dim)) * 2.0).astype(np.float32)
    wr = (rng.standard_normal((E, dim)) * 0.02).astype(np.float32)
    if dtype == "bf16":
        wr = round_bf16(wr)
    g2 = (1.0 + 0.1 * rng.standard_normal(dim)).astype(np.float32)
    bias = np.linspace(-0.02, 0.02, E).astype(np.float32)
    wr_d = torch.from_numpy(wr)
    wr_d = (wr_d.to(torch.bfloat16) if dtype == "bf16" else wr_d).cuda()
    y_d, g2_d, b_d = (torch.from_numpy(a).cuda() for a in (y, g2, bias))
    for call in range(2):
        got_i = torch.full((ntok, k), -1, dtype=torch.int32, device="cuda")
        got_w = torch.zeros((ntok, k), dtype=torch.float32, device="cuda")
        cnt = torch.full((E,), -1, dtype=torch.int32, device="cuda")
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        st = lib.rdt_moe_route_noalloc(1 if dtype == "bf16" else 0, _p(y_d), _p(g2_d), _p(wr_d), _p(b_d),
                                       ntok, dim, E, k, ctypes.c_float(1e-6), _p(got_i), _p(got_w), _p(cnt),
                                       stream)
        assert st == 0, lib.rdt_last_error()
        assert lib.rdt_moe_route_noalloc_status(stream) == 0, lib.rdt_last_error()
        _oracle_check(y, g2, wr, bias, k, 1e-6, got_i.cpu().numpy(), got_w.cpu().numpy(), cnt.cpu().numpy())
