"""Seeded synthetic workloads for the recurrent-depth block.

This module holds shapes, sizes and random draws only: none of the block's
arithmetic. Both the CPU oracle and the CUDA path read their inputs from here,
so that the two see identical bytes.

Shapes follow the recurrent-block configurations that the OpenMythos pages
describe (getting-started page, "Passo 2" and "Passo 5": ``dim``, ``n_heads``,
``n_kv_heads``, ``kv_lora_rank``, ``q_lora_rank``, ``qk_rope_head_dim``,
``qk_nope_head_dim``, ``v_head_dim``, ``n_experts``, ``n_shared_experts``,
``n_experts_per_tok``, ``expert_dim``, ``lora_rank``), sized as the five
benchmark configurations (tiny fp32, GQA 1024, MLA 1024, wide MoE 2048,
long-context 2048 with depth-wise LoRA).

Recipe (fixed draw order, ``numpy.random.Generator(PCG64(seed))``):

1. ``e`` ~ N(0, 1), shape [batch, seq, dim]; ``h0`` is the same tensor as ``e``
   unless an independent ``h0`` is asked for (then drawn last).
2. ``u`` ~ U(u_low, 0), shape [dim]; ``A = exp(-exp(u))`` (diagonal, so
   rho(A) = max A < 1 by construction).
3. ``B``: diagonal N(b_mean, b_std) [dim], or dense N(0, 0.02) [dim, dim].
4. Projection, router, expert and LoRA matrices ~ N(0, weight_std), drawn in
   the order of :data:`WEIGHT_ORDER_GQA` / :data:`WEIGHT_ORDER_MLA`.
   Norm gains are 1 and the router bias is 0 (not drawn).

Draws are float32; for bf16 workloads every drawn tensor except ``A`` and
``B`` (which stay fp32, as the state arithmetic does) is rounded to the
nearest bf16 (ties to even) once, here.

The ACT halting head (:func:`act_head`) is drawn from a stream of its own, so
that adding it changes none of the draws above: ``w_halt`` ~ N(0, scale^2 / dim)
(fp32, a random direction of length about ``scale``), ``b_halt`` fixed, and the
threshold 0.99 of the getting-started page (troubleshooting item 4).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "by_name", "generate", "round_bf16", "bf16_bits",
    "WEIGHT_ORDER_GQA", "WEIGHT_ORDER_MLA", "weight_shapes", "act_head", "ACT_THRESHOLD",
    "DEPTH_WORKLOAD", "depth_weights",
]

# u range that makes A = exp(-exp(u)) <= 0.95 exactly at the upper end.
U_LOW_RHO_095 = math.log(-math.log(0.95))


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # "f32" or "bf16" (storage of e, h0 and weights)
    batch: int
    seq: int
    dim: int
    attn: str                  # "gqa" or "mla"
    n_heads: int
    n_experts: int
    top_k: int
    expert_hidden: int
    n_kv_heads: int = 0        # GQA
    head_dim: int = 0          # GQA
    q_lora_rank: int = 0       # MLA: compressed query width
    kv_lora_rank: int = 0      # MLA: latent KV width
    qk_nope_dim: int = 0       # MLA
    qk_rope_dim: int = 0       # MLA
    v_head_dim: int = 0        # MLA
    rope_base: float = 1.0e4
    norm_eps: float = 1.0e-6
    n_shared: int = 0
    lora_rank: int = 0
    n_lora: int = 0            # number of per-loop adapters (0: no LoRA)
    b_kind: str = "diag"       # "diag" or "dense"
    b_mean: float = 1.0
    b_std: float = 0.1
    u_low: float = -3.0
    loops: Tuple[int, ...] = (4,)
    seed: int = 0
    inject_e: bool = True
    weight_std: float = 0.02
    da_heads: int = 0          # depth attention: query heads (0: no depth attention)
    da_kv_heads: int = 0       # depth attention: KV heads (head width = head_dim)

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def q_width(self) -> int:
        """Width of the concatenated per-head attention output o."""
        if self.attn == "gqa":
            return self.n_heads * self.head_dim
        return self.n_heads * self.v_head_dim

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Tuple[Workload, ...] = (
    Workload(name="tiny-f32-b1s64-d128-gqa4x2-e4k2", dtype="f32", batch=1, seq=64, dim=128,
             attn="gqa", n_heads=4, n_kv_heads=2, head_dim=32,
             n_experts=4, top_k=2, expert_hidden=256,
             b_kind="dense", u_low=-3.0, loops=(4,), seed=0),
    Workload(name="gqa-bf16-b4s512-d1024-h16x4-e16k2", dtype="bf16", batch=4, seq=512, dim=1024,
             attn="gqa", n_heads=16, n_kv_heads=4, head_dim=64,
             n_experts=16, top_k=2, expert_hidden=1024,
             b_kind="diag", u_low=-3.0, loops=(8,), seed=1),
    Workload(name="mla-bf16-b4s512-d1024-h16-lat128-e16k2", dtype="bf16", batch=4, seq=512, dim=1024,
             attn="mla", n_heads=16, q_lora_rank=384, kv_lora_rank=128, qk_nope_dim=64,
             qk_rope_dim=32, v_head_dim=64,
             n_experts=16, top_k=2, expert_hidden=1024,
             b_kind="diag", u_low=-3.0, loops=(3, 8), seed=2),
    Workload(name="widemoe-bf16-b2s2048-d2048-h32x8-e64k8s1", dtype="bf16", batch=2, seq=2048, dim=2048,
             attn="gqa", n_heads=32, n_kv_heads=8, head_dim=64,
             n_experts=64, top_k=8, n_shared=1, expert_hidden=512,
             b_kind="diag", u_low=U_LOW_RHO_095, loops=(1, 4, 8, 16), seed=3),
    Workload(name="long-bf16-b1s8192-d2048-h32x8-e64k8-lora16", dtype="bf16", batch=1, seq=8192, dim=2048,
             attn="gqa", n_heads=32, n_kv_heads=8, head_dim=64,
             n_experts=64, top_k=8, expert_hidden=512, lora_rank=16, n_lora=16,
             b_kind="diag", u_low=U_LOW_RHO_095, loops=(16,), seed=4),
)

# The GQA configuration with a depth-attention sublayer (16 query / 4 KV heads of 64) before
# the sequence attention: the fifth item of the work list beyond the benchmark set.
DEPTH_WORKLOAD = Workload(name="gqa-da-bf16-b4s512-d1024-h16x4-e16k2-da16x4", dtype="bf16", batch=4, seq=512,
                          dim=1024, attn="gqa", n_heads=16, n_kv_heads=4, head_dim=64,
                          n_experts=16, top_k=2, expert_hidden=1024, b_kind="diag", u_low=-3.0,
                          loops=(8,), seed=5, da_heads=16, da_kv_heads=4)


def by_name(name: str) -> Workload:
    for w in WORKLOADS + (DEPTH_WORKLOAD,):
        if w.name == name:
            return w
    raise KeyError(name)


WEIGHT_ORDER_GQA = ("wq", "wk", "wv", "wo", "w_router", "w1", "w3", "w2",
                    "ws1", "ws3", "ws2", "lq_a", "lq_b", "lo_a", "lo_b")
WEIGHT_ORDER_MLA = ("w_dq", "w_uq", "w_dkv", "w_kr", "w_uk", "w_uv", "wo", "w_router",
                    "w1", "w3", "w2", "ws1", "ws3", "ws2", "lq_a", "lq_b", "lo_a", "lo_b")


def weight_shapes(wl: Workload) -> Dict[str, Tuple[int, ...]]:
    """Shapes of the drawn matrices, row-major [out, in] (per expert / per loop first)."""
    d, E, hid, S = wl.dim, wl.n_experts, wl.expert_hidden, wl.n_shared
    s: Dict[str, Tuple[int, ...]] = {}
    if wl.attn == "gqa":
        hq, hkv, dh = wl.n_heads, wl.n_kv_heads, wl.head_dim
        s["wq"] = (hq * dh, d)
        s["wk"] = (hkv * dh, d)
        s["wv"] = (hkv * dh, d)
        s["wo"] = (d, hq * dh)
        qout = hq * dh
    else:
        H = wl.n_heads
        s["w_dq"] = (wl.q_lora_rank, d)
        s["w_uq"] = (H * (wl.qk_nope_dim + wl.qk_rope_dim), wl.q_lora_rank)
        s["w_dkv"] = (wl.kv_lora_rank, d)
        s["w_kr"] = (wl.qk_rope_dim, d)
        s["w_uk"] = (H * wl.qk_nope_dim, wl.kv_lora_rank)
        s["w_uv"] = (H * wl.v_head_dim, wl.kv_lora_rank)
        s["wo"] = (d, H * wl.v_head_dim)
        qout = H * (wl.qk_nope_dim + wl.qk_rope_dim)
    s["w_router"] = (E, d)
    s["w1"] = (E, hid, d)
    s["w3"] = (E, hid, d)
    s["w2"] = (E, d, hid)
    if S:
        s["ws1"] = (S, hid, d)
        s["ws3"] = (S, hid, d)
        s["ws2"] = (S, d, hid)
    if wl.n_lora:
        if wl.attn != "gqa":
            raise ValueError("depth-wise LoRA is defined here for the GQA projections only")
        L, r = wl.n_lora, wl.lora_rank
        s["lq_a"] = (L, r, d)
        s["lq_b"] = (L, qout, r)
        s["lo_a"] = (L, r, wl.q_width)
        s["lo_b"] = (L, d, r)
    return s


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32).reshape(np.shape(x))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    if np.any(b & np.uint32(0xFFFF)):
        raise ValueError("values are not bf16-representable; call round_bf16 first")
    return (b >> np.uint32(16)).astype(np.uint16).reshape(np.shape(x))


def _normal(rng: np.random.Generator, shape, mean: float, std: float) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def generate(wl: Workload, *, seed: Optional[int] = None, h0_independent: bool = False,
             zero_block: bool = False, lora_b_zero: bool = False) -> Dict[str, np.ndarray]:
    """Draw every input of ``wl`` in the fixed order; return float32 arrays.

    Keys: ``e``, ``h0`` ([batch, seq, dim]), ``A`` [dim], ``B`` ([dim] or
    [dim, dim]), ``norm1``, ``norm2`` (and ``q_norm``, ``kv_norm`` for MLA),
    ``router_bias`` (zeros) and the matrices of :func:`weight_shapes`.
    ``zero_block`` zeroes every projection/expert matrix after drawing (the
    draws still happen, so other tensors are unchanged); ``lora_b_zero``
    zeroes the LoRA up-projections.
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    bf = wl.dtype == "bf16"
    out: Dict[str, np.ndarray] = {}
    e = _normal(rng, (wl.batch, wl.seq, wl.dim), 0.0, 1.0)
    out["e"] = round_bf16(e) if bf else e
    u = rng.uniform(wl.u_low, 0.0, size=wl.dim)
    out["A"] = np.exp(-np.exp(u)).astype(np.float32)
    if wl.b_kind == "diag":
        out["B"] = _normal(rng, (wl.dim,), wl.b_mean, wl.b_std)
    elif wl.b_kind == "dense":
        out["B"] = _normal(rng, (wl.dim, wl.dim), 0.0, 0.02)
    else:
        raise ValueError(wl.b_kind)
    shapes = weight_shapes(wl)
    order = WEIGHT_ORDER_GQA if wl.attn == "gqa" else WEIGHT_ORDER_MLA
    for k in order:
        if k not in shapes:
            continue
        w = _normal(rng, shapes[k], 0.0, wl.weight_std)
        if zero_block:
            w[...] = 0.0
        if lora_b_zero and k in ("lq_b", "lo_b"):
            w[...] = 0.0
        out[k] = round_bf16(w) if bf else w
    one = np.ones(wl.dim, dtype=np.float32)
    out["norm1"] = one.copy()
    out["norm2"] = one.copy()
    if wl.attn == "mla":
        out["q_norm"] = np.ones(wl.q_lora_rank, dtype=np.float32)
        out["kv_norm"] = np.ones(wl.kv_lora_rank, dtype=np.float32)
    out["router_bias"] = np.zeros(wl.n_experts, dtype=np.float32)
    if wl.da_heads:
        out.update(depth_weights(wl, seed=seed, zero=zero_block))
    if h0_independent:
        h0 = _normal(rng, (wl.batch, wl.seq, wl.dim), 0.0, 1.0)
        out["h0"] = round_bf16(h0) if bf else h0
    else:
        out["h0"] = out["e"]
    return out


def prefix(inputs: Dict[str, np.ndarray], n_tok: int) -> Dict[str, np.ndarray]:
    """Keep the first ``n_tok`` positions of every sequence (weights unchanged)."""
    d = dict(inputs)
    d["e"] = np.ascontiguousarray(inputs["e"][:, :n_tok])
    d["h0"] = np.ascontiguousarray(inputs["h0"][:, :n_tok])
    return d


def depth_weights(wl: Workload, *, seed: Optional[int] = None, zero: bool = False) -> Dict[str, np.ndarray]:
    """Depth-attention weights, from the PCG64 stream keyed by (seed, 2) so that the draws of
    :func:`generate` stay as they are: ``norm_da`` = 1, ``wq_d`` [da_heads * head_dim, dim],
    ``wk_d``, ``wv_d`` [da_kv_heads * head_dim, dim], ``wo_d`` [dim, da_heads * head_dim],
    each ~ N(0, weight_std), rounded like the other matrices."""
    rng = np.random.Generator(np.random.PCG64([wl.seed if seed is None else seed, 2]))
    bf = wl.dtype == "bf16"
    dh, d = wl.head_dim, wl.dim
    out = {"norm_da": np.ones(d, dtype=np.float32)}
    for k, shp in (("wq_d", (wl.da_heads * dh, d)), ("wk_d", (wl.da_kv_heads * dh, d)),
                   ("wv_d", (wl.da_kv_heads * dh, d)), ("wo_d", (d, wl.da_heads * dh))):
        w = _normal(rng, shp, 0.0, wl.weight_std)
        if zero:
            w[...] = 0.0
        out[k] = round_bf16(w) if bf else w
    return out


ACT_THRESHOLD = 0.99


def act_head(wl: Workload, *, scale: float = 0.5, bias: float = -1.0,
             seed: Optional[int] = None) -> Dict[str, object]:
    """Halting head of the ACT loop: ``w_halt`` [dim] fp32 ~ N(0, scale^2 / dim),
    ``b_halt`` = bias, ``threshold`` = 0.99. Drawn from the PCG64 stream keyed by
    (seed, 1), apart from :func:`generate`'s."""
    rng = np.random.Generator(np.random.PCG64([wl.seed if seed is None else seed, 1]))
    w = _normal(rng, (wl.dim,), 0.0, scale / math.sqrt(wl.dim))
    return {"w_halt": w, "b_halt": float(bias), "threshold": ACT_THRESHOLD}
