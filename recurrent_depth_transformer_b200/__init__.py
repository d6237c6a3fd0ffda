"""Python binding of librdt, the B200 (sm_100a) recurrent-depth block library.

Argument marshalling only: every step of the forward pass runs in the CUDA kernels of
``librdt.so`` behind the C ABI of ``include/rdt.h``. PyTorch provides device memory and
streams. There is no CPU path: without the built library (or a CUDA device) the calls
raise.

    from recurrent_depth_transformer_b200 import RDT
    m = RDT(config, weights)             # weights: dict name -> CUDA tensor
    out = m.loop_forward(h0, e, T)       # fp32 [batch, seq, dim] = h_T
    m.set_act(w_halt, b_halt, 0.99)      # ACT halting head: fp32 [dim] CUDA tensor
    out, n_loops = m.loop_forward_act(h0, e, T)   # weighted states, loops per position
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

__all__ = ["RDT", "RdtError", "library_path", "load_library", "make_config", "device_weights",
           "EXPORTED", "ipc_get_handle", "ipc_open_handle", "ipc_close_handle", "cp_connect_ranks"]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "librdt.so")

RDT_F32, RDT_BF16 = 0, 1
RDT_GQA, RDT_MLA = 0, 1
RDT_B_DIAG, RDT_B_DENSE = 0, 1

STATUS = {0: "RDT_OK", 1: "RDT_ERR_INVALID_ARG", 2: "RDT_ERR_UNSUPPORTED", 3: "RDT_ERR_MISALIGNED",
          4: "RDT_ERR_UNSTABLE_A", 5: "RDT_ERR_OOM", 6: "RDT_ERR_CUDA", 7: "RDT_ERR_DEVICE_TIMEOUT",
          8: "RDT_ERR_NONFINITE"}

EXPORTED = ("rdt_create", "rdt_attn_forward", "rdt_moe_forward", "rdt_loop_forward",
            "rdt_loop_forward_host", "rdt_set_trace", "rdt_get_diagnostics", "rdt_memory_bytes",
            "rdt_status_string", "rdt_last_error", "rdt_destroy", "rdt_matmul", "rdt_attention",
            "rdt_profile", "rdt_profile_read", "rdt_moe_route_noalloc", "rdt_moe_route_noalloc_status",
            "rdt_set_act", "rdt_loop_forward_act", "rdt_wait_probe", "rdt_decode_prefill",
            "rdt_decode_step", "rdt_cp_buffers", "rdt_cp_connect", "rdt_ipc_get_handle",
            "rdt_ipc_open_handle", "rdt_ipc_close_handle")


class RdtError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class RdtConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "dtype", "batch", "seq", "dim", "attn_type", "n_heads", "n_kv_heads", "head_dim",
        "q_lora_rank", "kv_lora_rank", "qk_nope_dim", "qk_rope_dim", "v_head_dim")] + [
        ("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float)] + [
        (n, ctypes.c_int32) for n in ("n_experts", "top_k", "n_shared", "expert_hidden",
                                      "lora_rank", "n_lora", "b_kind", "inject_e", "max_loops",
                                      "gemm_tiles", "deterministic", "max_decode", "da_heads",
                                      "da_kv_heads", "cp_size", "cp_rank")]


WEIGHT_FIELDS = ("A", "B", "norm1", "norm2", "wq", "wk", "wv", "wo", "w_dq", "q_norm", "w_uq",
                 "w_dkv", "kv_norm", "w_kr", "w_uk", "w_uv", "w_router", "router_bias", "w1",
                 "w3", "w2", "ws1", "ws3", "ws2", "lq_a", "lq_b", "lo_a", "lo_b", "norm_da", "wq_d",
                 "wk_d", "wv_d", "wo_d")
FP32_FIELDS = ("A", "B", "norm1", "norm2", "q_norm", "kv_norm", "router_bias", "norm_da")


class RdtWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class RdtKernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


class RdtDiag(ctypes.Structure):
    _fields_ = [("rho_A", ctypes.c_float), ("nonfinite", ctypes.c_int32), ("timeout", ctypes.c_int32),
                ("last_routed_rows", ctypes.c_int32), ("expert_counts", ctypes.c_int32 * 256)]


_LIB = None


def load_library() -> ctypes.CDLL:
    """Load the in-tree librdt.so (build it with ``python -m recurrent_depth_transformer_b200.build``)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(library_path):
        raise RuntimeError(f"{library_path} is missing: build it with "
                           "`python -m recurrent_depth_transformer_b200.build`")
    lib = ctypes.CDLL(library_path)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.rdt_create.argtypes = [ctypes.POINTER(RdtConfig), ctypes.POINTER(RdtWeights), vp,
                               ctypes.POINTER(vp)]
    lib.rdt_attn_forward.argtypes = [vp, vp, i32, vp, vp]
    lib.rdt_moe_forward.argtypes = [vp, vp, vp, vp, vp, vp]
    lib.rdt_loop_forward.argtypes = [vp, vp, vp, i32, vp, vp]
    lib.rdt_loop_forward_host.argtypes = [vp, vp, vp, i32, vp, vp]
    lib.rdt_set_trace.argtypes = [vp, vp, vp, vp]
    lib.rdt_set_act.argtypes = [vp, vp, ctypes.c_float, ctypes.c_float, vp]
    lib.rdt_loop_forward_act.argtypes = [vp, vp, vp, i32, vp, vp, vp]
    lib.rdt_get_diagnostics.argtypes = [vp, ctypes.POINTER(RdtDiag)]
    lib.rdt_memory_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t)]
    lib.rdt_status_string.argtypes = [i32]
    lib.rdt_status_string.restype = ctypes.c_char_p
    lib.rdt_last_error.argtypes = []
    lib.rdt_last_error.restype = ctypes.c_char_p
    lib.rdt_destroy.argtypes = [vp]
    lib.rdt_destroy.restype = None
    lib.rdt_matmul.argtypes = [i32, vp, vp, vp, i32, i32, i32, vp]
    lib.rdt_moe_route_noalloc.argtypes = [i32, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                          vp, vp, vp, vp]
    lib.rdt_moe_route_noalloc_status.argtypes = [vp]
    lib.rdt_wait_probe.argtypes = [ctypes.c_int64, vp]
    lib.rdt_decode_prefill.argtypes = [vp, vp, vp, i32, vp, vp]
    lib.rdt_decode_step.argtypes = [vp, vp, vp, i32, vp, vp]
    lib.rdt_profile.argtypes = [vp, i32]
    lib.rdt_profile_read.argtypes = [vp, ctypes.POINTER(RdtKernelStat), i32, ctypes.POINTER(i32),
                                     ctypes.POINTER(ctypes.c_int64)]
    lib.rdt_attention.argtypes = [i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                  ctypes.c_float, vp]
    sz = ctypes.POINTER(ctypes.c_size_t)
    lib.rdt_cp_buffers.argtypes = [vp, ctypes.POINTER(vp), sz, ctypes.POINTER(vp), sz]
    lib.rdt_cp_connect.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp)]
    lib.rdt_ipc_get_handle.argtypes = [vp, vp]
    lib.rdt_ipc_open_handle.argtypes = [vp, ctypes.POINTER(vp)]
    lib.rdt_ipc_close_handle.argtypes = [vp]
    for f in ("rdt_create", "rdt_attn_forward", "rdt_moe_forward", "rdt_loop_forward",
              "rdt_loop_forward_host", "rdt_set_trace", "rdt_get_diagnostics", "rdt_memory_bytes",
              "rdt_matmul", "rdt_attention", "rdt_profile", "rdt_profile_read", "rdt_moe_route_noalloc",
              "rdt_set_act", "rdt_loop_forward_act", "rdt_moe_route_noalloc_status", "rdt_wait_probe",
              "rdt_decode_prefill", "rdt_decode_step", "rdt_cp_buffers", "rdt_cp_connect",
              "rdt_ipc_get_handle", "rdt_ipc_open_handle", "rdt_ipc_close_handle"):
        getattr(lib, f).restype = i32
    _LIB = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        lib = load_library()
        raise RdtError(status, lib.rdt_last_error().decode(errors="replace"))


def make_config(wl, max_loops: int = 16, batch: Optional[int] = None, seq: Optional[int] = None,
                gemm_tiles: int = 0, deterministic: bool = False, max_decode: int = 0,
                cp_size: int = 0, cp_rank: int = 0) -> RdtConfig:
    """Fill the C config from any object with the block's hyper-parameters as attributes.
    With cp_size > 1, seq is this rank's share of each sequence."""
    c = RdtConfig()
    c.dtype = RDT_BF16 if wl.dtype == "bf16" else RDT_F32
    c.batch = wl.batch if batch is None else batch
    c.seq = wl.seq if seq is None else seq
    c.dim = wl.dim
    c.attn_type = RDT_GQA if wl.attn == "gqa" else RDT_MLA
    c.n_heads = wl.n_heads
    c.n_kv_heads = wl.n_kv_heads
    c.head_dim = wl.head_dim
    c.q_lora_rank = wl.q_lora_rank
    c.kv_lora_rank = wl.kv_lora_rank
    c.qk_nope_dim = wl.qk_nope_dim
    c.qk_rope_dim = wl.qk_rope_dim
    c.v_head_dim = wl.v_head_dim
    c.rope_base = wl.rope_base
    c.norm_eps = wl.norm_eps
    c.n_experts = wl.n_experts
    c.top_k = wl.top_k
    c.n_shared = wl.n_shared
    c.expert_hidden = wl.expert_hidden
    c.lora_rank = wl.lora_rank
    c.n_lora = wl.n_lora
    c.b_kind = RDT_B_DIAG if wl.b_kind == "diag" else RDT_B_DENSE
    c.inject_e = 1 if wl.inject_e else 0
    c.max_loops = max_loops
    c.gemm_tiles = gemm_tiles
    c.deterministic = 1 if deterministic else 0
    c.max_decode = max_decode
    c.da_heads = getattr(wl, "da_heads", 0)
    c.da_kv_heads = getattr(wl, "da_kv_heads", 0)
    c.cp_size = cp_size
    c.cp_rank = cp_rank
    return c


def ipc_get_handle(dev_ptr: int) -> bytes:
    """The 64-byte inter-process handle of a device allocation (rdt_ipc_get_handle)."""
    lib = load_library()
    buf = ctypes.create_string_buffer(64)
    _check(lib.rdt_ipc_get_handle(ctypes.c_void_p(dev_ptr), buf))
    return buf.raw


def ipc_open_handle(handle: bytes) -> int:
    """Map another process's allocation; returns its device address here."""
    lib = load_library()
    if len(handle) != 64:
        raise ValueError("an IPC handle has 64 bytes")
    ptr = ctypes.c_void_p()
    _check(lib.rdt_ipc_open_handle(ctypes.create_string_buffer(handle, 64), ctypes.byref(ptr)))
    return ptr.value


def ipc_close_handle(dev_ptr: int) -> None:
    _check(load_library().rdt_ipc_close_handle(ctypes.c_void_p(dev_ptr)))


def cp_connect_ranks(handle, rank: int, size: int, all_gather, get_handle=ipc_get_handle,
                     open_handle=ipc_open_handle):
    """Connect the context-parallel ranks of one sequence, one process per GPU.

    Every rank calls this collectively. all_gather(obj) returns the list of every rank's
    obj (torch.distributed.all_gather_object, for example). Each rank publishes the
    inter-process handles of its gather buffer and flag words, opens the other ranks',
    and passes the mapped addresses to rdt_cp_connect. Returns the opened addresses (close
    them with ipc_close_handle once the handle is destroyed)."""
    kv, kv_bytes, flags, flag_bytes = handle.cp_buffers()
    mine = (rank, get_handle(kv), get_handle(flags))
    every = all_gather(mine)
    if len(every) != size or sorted(r for r, _, _ in every) != list(range(size)):
        raise RuntimeError(f"context parallelism: expected ranks 0 .. {size - 1}, got "
                           f"{sorted(r for r, _, _ in every)}")
    peer_kv, peer_flags, opened = [0] * size, [0] * size, []
    for r, hkv, hfl in every:
        if r == rank:
            peer_kv[r], peer_flags[r] = kv, flags
            continue
        peer_kv[r] = open_handle(hkv)
        peer_flags[r] = open_handle(hfl)
        opened += [peer_kv[r], peer_flags[r]]
    handle.cp_connect(peer_kv, peer_flags)
    return opened


def device_weights(arrays: Dict[str, np.ndarray], bf16: bool, device="cuda"):
    """Upload host weight arrays (float32 holding element-type values) as CUDA tensors:
    fp32 for A, B, norm gains and the router bias; bf16 or fp32 for the matrices."""
    import torch
    out = {}
    for k in WEIGHT_FIELDS:
        if k not in arrays or arrays[k] is None:
            continue
        t = torch.from_numpy(np.ascontiguousarray(arrays[k], dtype=np.float32))
        if bf16 and k not in FP32_FIELDS:
            t = t.to(torch.bfloat16)
        out[k] = t.to(device)
    return out


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def matmul(A, B, C=None, stream=None):
    """C = A B^T (fp32) on the tensor-core GEMM; A [M, K], B [N, K] bf16 or fp32 CUDA tensors."""
    import torch
    lib = load_library()
    M, K = A.shape
    N = B.shape[0]
    C = torch.empty((M, N), dtype=torch.float32, device=A.device) if C is None else C
    dt = RDT_BF16 if A.dtype == torch.bfloat16 else RDT_F32
    _check(lib.rdt_matmul(dt, _ptr(A), _ptr(B), _ptr(C), M, N, K, _stream(stream)))
    return C


def attention(q, k, v, batch, seq, n_heads, n_kv_heads, dqk, dv, scale, o=None, stream=None):
    """Causal GQA attention on [batch*seq, heads*dim] CUDA tensors (see rdt_attention)."""
    import torch
    lib = load_library()
    o = torch.empty((batch * seq, n_heads * dv), dtype=q.dtype, device=q.device) if o is None else o
    dt = RDT_BF16 if q.dtype == torch.bfloat16 else RDT_F32
    _check(lib.rdt_attention(dt, _ptr(q), _ptr(k), _ptr(v), _ptr(o), batch, seq, n_heads, n_kv_heads,
                             dqk, dv, scale, _stream(stream)))
    return o


class RDT:
    """A created handle: weights copied into library memory, workspace for batch x seq tokens."""

    def __init__(self, config: RdtConfig, weights: Dict[str, "object"], stream=None):
        import torch
        self._lib = load_library()
        if not torch.cuda.is_available():
            raise RuntimeError("a CUDA device is required")
        self.cfg = config
        w = RdtWeights()
        for k in WEIGHT_FIELDS:
            setattr(w, k, _ptr(weights.get(k)))
        h = ctypes.c_void_p()
        _check(self._lib.rdt_create(ctypes.byref(config), ctypes.byref(w), _stream(stream), ctypes.byref(h)))
        self._h = h
        self.ntok = config.batch * config.seq
        self._trace = None

    # ---------------------------------------------------------------- calls
    def attn_forward(self, x, loop: int = 0, a_out=None, stream=None):
        import torch
        a_out = torch.empty_like(x, dtype=torch.float32) if a_out is None else a_out
        _check(self._lib.rdt_attn_forward(self._h, _ptr(x), loop, _ptr(a_out), _stream(stream)))
        return a_out

    def moe_forward(self, y, f_out=None, idx=None, w=None, stream=None):
        import torch
        f_out = torch.empty_like(y, dtype=torch.float32) if f_out is None else f_out
        _check(self._lib.rdt_moe_forward(self._h, _ptr(y), _ptr(f_out), _ptr(idx), _ptr(w), _stream(stream)))
        return f_out

    def loop_forward(self, h0, e, T: int, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty(e.shape, dtype=torch.float32, device=e.device)
        _check(self._lib.rdt_loop_forward(self._h, _ptr(h0), _ptr(e), T, _ptr(out), _stream(stream)))
        return out

    def decode_prefill(self, h0, e, T: int, out=None, stream=None):
        """The loop over the prompt [batch, seq, dim], filling every loop's KV cache."""
        import torch
        if out is None:
            out = torch.empty(e.shape, dtype=torch.float32, device=e.device)
        _check(self._lib.rdt_decode_prefill(self._h, _ptr(h0), _ptr(e), T, _ptr(out), _stream(stream)))
        return out

    def decode_step(self, h0, e, T: int, out=None, stream=None):
        """T loops for one new token per sequence (h0, e [batch, dim]); appends to the caches."""
        import torch
        if out is None:
            out = torch.empty(e.shape, dtype=torch.float32, device=e.device)
        _check(self._lib.rdt_decode_step(self._h, _ptr(h0), _ptr(e), T, _ptr(out), _stream(stream)))
        return out

    def set_act(self, w_halt, b_halt: float, threshold: float = 0.99, stream=None):
        """ACT halting head: w_halt a device fp32 [dim] tensor (copied)."""
        _check(self._lib.rdt_set_act(self._h, _ptr(w_halt), float(b_halt), float(threshold), _stream(stream)))

    def loop_forward_act(self, h0, e, T: int, out=None, n_loops=None, stream=None):
        """Looped block with ACT halting; returns (out fp32 [.., dim], n_loops int32 [..])."""
        import torch
        if out is None:
            out = torch.empty(e.shape, dtype=torch.float32, device=e.device)
        if n_loops is None:
            n_loops = torch.empty(e.shape[:-1], dtype=torch.int32, device=e.device)
        _check(self._lib.rdt_loop_forward_act(self._h, _ptr(h0), _ptr(e), T, _ptr(out), _ptr(n_loops),
                                              _stream(stream)))
        return out, n_loops

    def loop_forward_host(self, h0, e, T: int, out, stream=None):
        """Host (CPU, ideally pinned) tensors in, host fp32 tensor out; synchronous."""
        _check(self._lib.rdt_loop_forward_host(self._h, _ptr(h0), _ptr(e), T, _ptr(out), _stream(stream)))
        return out

    def set_trace(self, idx=None, w=None, h_traj=None):
        self._trace = (idx, w, h_traj)       # keep the buffers alive
        _check(self._lib.rdt_set_trace(self._h, _ptr(idx), _ptr(w), _ptr(h_traj)))

    def diagnostics(self) -> dict:
        d = RdtDiag()
        _check(self._lib.rdt_get_diagnostics(self._h, ctypes.byref(d)))
        E = self.cfg.n_experts + self.cfg.n_shared
        return {"rho_A": d.rho_A, "nonfinite": d.nonfinite, "timeout": d.timeout,
                "last_routed_rows": d.last_routed_rows, "expert_counts": list(d.expert_counts[:E])}

    def profile(self, mode=True):
        """Per-kernel event timing: True or 1 eager launches, 2 inside graph replay, 0 off."""
        _check(self._lib.rdt_profile(self._h, int(mode)))

    def profile_read(self):
        """(per-kernel {name: (launches, total_ms)}, kernels launched since create)."""
        arr = (RdtKernelStat * 64)()
        n = ctypes.c_int()
        tot = ctypes.c_int64()
        _check(self._lib.rdt_profile_read(self._h, arr, 64, ctypes.byref(n), ctypes.byref(tot)))
        return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n.value)}, tot.value

    def launch_count(self) -> int:
        tot = ctypes.c_int64()
        _check(self._lib.rdt_profile_read(self._h, None, 0, None, ctypes.byref(tot)))
        return tot.value

    def memory_bytes(self) -> int:
        n = ctypes.c_size_t()
        _check(self._lib.rdt_memory_bytes(self._h, ctypes.byref(n)))
        return n.value

    def cp_buffers(self):
        """(gather buffer address, its bytes, flag words address, their bytes) of this rank."""
        kv, fl = ctypes.c_void_p(), ctypes.c_void_p()
        kvb, flb = ctypes.c_size_t(), ctypes.c_size_t()
        _check(self._lib.rdt_cp_buffers(self._h, ctypes.byref(kv), ctypes.byref(kvb), ctypes.byref(fl),
                                        ctypes.byref(flb)))
        return kv.value, kvb.value, fl.value, flb.value

    def cp_connect(self, peer_kv, peer_flags):
        """Every rank's gather buffer and flag words as device addresses in this process."""
        n = len(peer_kv)
        kv = (ctypes.c_void_p * n)(*[ctypes.c_void_p(p) for p in peer_kv])
        fl = (ctypes.c_void_p * n)(*[ctypes.c_void_p(p) for p in peer_flags])
        _check(self._lib.rdt_cp_connect(self._h, kv, fl))

    def close(self):
        if getattr(self, "_h", None):
            self._lib.rdt_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()
