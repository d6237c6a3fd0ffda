"""rdt_moe_route_noalloc: the MoE router for callers that cannot allocate device memory
(a framework's memory pool owns the device, allocation is forbidden after start-up, or the
host captures the work into its own CUDA graphs), so they cannot create a handle. It runs
the router kernel of rdt_moe_forward with its scratch in a static device array.

Checked through the C ABI against rdt_moe_forward's top-k outputs on two calls in a row
(the shared scratch keeps the previous call's contents; the counters must restart at 0).
This file sorts last so that a stop-at-first-failure run has run every other test first.
"""
import ctypes

import numpy as np
import pytest

from workloads import WORKLOADS, generate

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
