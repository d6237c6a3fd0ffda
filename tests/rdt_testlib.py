"""Shared helpers of the GPU parity tests: create a handle from a seeded workload, run it,
read back the trace, and measure errors against the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle as O
from workloads import Workload, generate

MAX_ABS = 3.0e-2      # hidden-state bound after T loops (bf16 storage, fp32 accumulation)
REL_FRO = 1.0e-2


def torch_mod():
    import torch
    return torch


def handle(wl: Workload, inputs, max_loops: int = 16, gemm_tiles: int = 0, deterministic: bool = False):
    import recurrent_depth_transformer_b200 as R
    w = R.device_weights(inputs, wl.dtype == "bf16")
    return R.RDT(R.make_config(wl, max_loops=max_loops, gemm_tiles=gemm_tiles, deterministic=deterministic), w)


def act(wl: Workload, arr):
    """Upload an activation [B, S, d] in the workload's element type."""
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    if wl.dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def run_loop(wl: Workload, inputs, T: int, trace: bool = True, traj: bool = False, h=None,
             gemm_tiles: int = 0):
    """Run rdt_loop_forward; returns (h_T [B,S,d] fp32, idx [T,N,k], w [T,N,k], traj or None)."""
    torch = torch_mod()
    own = h is None
    if own:
        h = handle(wl, inputs, max_loops=max(T, 1), gemm_tiles=gemm_tiles)
    N = wl.batch * wl.seq
    idx = torch.full((max(T, 1), N, wl.top_k), -1, dtype=torch.int32, device="cuda") if trace else None
    wts = torch.zeros((max(T, 1), N, wl.top_k), dtype=torch.float32, device="cuda") if trace else None
    tr = torch.zeros((T + 1, N, wl.dim), dtype=torch.float32, device="cuda") if traj else None
    h.set_trace(idx, wts, tr)
    e = act(wl, inputs["e"])
    h0 = e if inputs["h0"] is inputs["e"] else act(wl, inputs["h0"])
    out = h.loop_forward(h0, e, T)
    torch.cuda.synchronize()
    diag = h.diagnostics()
    h.set_trace(None, None, None)
    res = (out.cpu().numpy(),
           None if idx is None else idx.cpu().numpy(),
           None if wts is None else wts.cpu().numpy(),
           None if tr is None else tr.cpu().numpy(),
           diag)
    if own:
        h.close()
    return res


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    d = got - want
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(want), 1e-300))


def assert_close(got, want, max_abs=MAX_ABS, rel_fro=REL_FRO, what=""):
    ma, rf = errors(got, want)
    assert ma <= max_abs and rf <= rel_fro, f"{what}: max|err| {ma:.3e} (<= {max_abs}), rel-Frobenius {rf:.3e} (<= {rel_fro})"
    return ma, rf


def oracle_follow(wl: Workload, inputs, T: int, gpu_idx):
    """Oracle run that adopts the GPU's routing on near-ties (gap <= 1e-3) only."""
    N = wl.batch * wl.seq
    follow = [gpu_idx[t].reshape(N, wl.top_k) for t in range(T)]
    tr = O.LoopTrace()
    h = O.loop_forward(inputs["h0"], inputs["e"], T, inputs, wl, follow=follow, trace=tr)
    mism = sum(s["mismatch"] for s in tr.stats)
    ties = sum(s["near_ties"] for s in tr.stats)
    return h, mism, ties, tr
