"""Plain fp64 CPU oracle of the recurrent-depth block's forward pass.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this module; only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg (and its ``--impl reference`` arm) may use it. It shares no
code with the CUDA path: both read their inputs from the ``workloads`` module
and nothing else.

Every function is written for a reader to check by eye: NumPy float64, no
blocking, fusion or reordering beyond the definition (attention over very long
sequences is evaluated one block of query rows at a time, which changes memory
use, not the arithmetic of any output).

Sources (pages about the OpenMythos recurrent-depth transformer):

* [TB]  techbriefly article "Projeto OpenMythos afirma que Claude Mythos e um
        transformador de profundidade recorrente": Prelude / Recurrent Block /
        Coda with up to 16 loops; the update equation
        h_{t+1} = A.h_t + B.e + Transformer(h_t, e); MoE per iteration; MLA;
        rho(A) < 1 (Parcae); depth-wise LoRA.
* [GS]  openclawapi getting-started page "Introducao ao OpenMythos": Passo 2
        (MythosConfig fields), Passo 3 (n_loops, depth extrapolation),
        Passo 5 (MLA vs GQA fields and the per-step K/V rebuild),
        Passo 6 (spectral radius of the diagonal A from get_A()), and the
        troubleshooting items on router_bias and on not clipping A.
* [RV]  bigsaas article "A Revolucao do Recurrent-Depth": MLA (latent KV,
        DeepSeek-V3) vs GQA (Llama 3) section; spectral-radius section.
* [CB]  hamidun article "OpenMythos: criando transformadores avancados com MLA
        e GQA no Colab": Sparse MoE section (router picks a few experts).
* [DR]  gist.science summary of "Dreamer" (depth-recurrent attention mixtures):
        depth attention, attention over a token's earlier depths with depth as the
        sequence and tokens as the batch, RoPE over depth with a reversed half, applied
        before sequence attention and the experts (DA -> SA -> EA).

Readings where the pages are silent (each is listed with its reason in the
design notes of the repository):

* the block input is x = h + e (``inject_e``), and Transformer(h, e) returns
  the residual increment a + f, so that the linear part of the update stays A;
* A and B are diagonal (B may be dense), rho(A) = max |A_i|;
* RMSNorm eps 1e-6, gains 1; RoPE rotates the pairs (i, i + r/2) by
  pos * base^(-2i/r); causal mask key <= query; GQA head h reads KV head
  floor(h * Hkv / Hq);
* router: top-k of (logits + bias), ties to the lower expert index, softmax of
  the selected logits (bias excluded); shared experts weight 1; dropless;
* depth-wise LoRA: W_t = W + B_t A_t on the Q and O projections, adapter
  min(t, L - 1) at loop t;
* MLA: latent RMSNorms on c_q and c_kv, decoupled RoPE key shared by all
  heads, score scale 1/sqrt(nope + rope);
* decode with a per-loop KV cache ([GS] Passo 4: the prompt is processed
  once, then one token per call; troubleshooting item 1: every loop keeps the
  KV state of all tokens): loop t of a new token attends over the keys and
  values that loop t produced for the earlier positions; GQA caches its
  rotated keys and values, MLA its normalised latent and rotated shared key,
  from which K/V are rebuilt at every step ([GS] Passo 5);
* ACT halting ([TB] names it; [GS] troubleshooting item 4 gives the 0.99
  threshold and that a position leaves once its accumulated halting probability
  reaches it): halting head p = sigmoid(w . h_{t+1} + b) on the new state;
  a position halts at the first loop where its running sum of p reaches the
  threshold (or at the last loop), taking the remainder 1 - (sum before) as
  that loop's weight; the output is the weighted sum of its states; a halted
  position keeps its state and still serves as a key, and is routed to no
  expert;
* depth attention (an optional sublayer, ``da_heads`` > 0): before the sequence
  attention, x' = x + DA(RMSNorm_da(x)), where a token's query at loop t attends over
  its own keys and values of loops 0 .. t (computed from its block inputs at those
  loops); RoPE over the loop index, the first half of the rotation pairs at t, the
  second half at T - 1 - t; the sequence attention then takes x', and the block's
  increment is d + a + f.

Parity status: every function below is pinned (closed forms, library special cases,
hand-computed fixtures, identities, brute force): the block and the loop by
``tests/test_oracle_pins.py``, ACT halting by ``tests/test_oracle_act_pins.py``, the
cached decode by ``tests/test_oracle_decode_pins.py``, depth attention by
``tests/test_oracle_depth_pins.py``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

F = np.float64
NEAR_TIE = 1.0e-3          # logit gap under which the oracle may follow the GPU's routing
NEAR_HALT = 2.0e-2         # |sum of p - threshold| under which it may follow the GPU's halting
ATTN_QBLOCK = 1024         # query rows per block when evaluating long sequences


def _f(x) -> np.ndarray:
    return np.asarray(x, dtype=F)


# --------------------------------------------------------------------------------------
# Elementary operations
# --------------------------------------------------------------------------------------

def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis (pre-norm of the block)."""
    x = _f(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * _f(gamma)


def rope_angles(n_pos: int, rot_dim: int, base: float) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin of pos * base^(-2i/rot_dim), shape [n_pos, rot_dim/2] ([GS] Passo 2: RoPE
    precomputed up to max_seq_len)."""
    i = np.arange(rot_dim // 2, dtype=F)
    inv_freq = np.power(F(base), -2.0 * i / rot_dim)
    ang = np.outer(np.arange(n_pos, dtype=F), inv_freq)
    return np.cos(ang), np.sin(ang)


def apply_rope(x, base: float) -> np.ndarray:
    """Rotate-half RoPE on the last axis of x [B, S, H, r]; position = index along S."""
    x = _f(x)
    r = x.shape[-1]
    cos, sin = rope_angles(x.shape[1], r, base)
    cos = cos[None, :, None, :]
    sin = sin[None, :, None, :]
    x1, x2 = x[..., : r // 2], x[..., r // 2:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def silu(x) -> np.ndarray:
    x = _f(x)
    return x / (1.0 + np.exp(-x))


def swiglu_ffn(z, w1, w3, w2) -> np.ndarray:
    """One SwiGLU expert: W2 (silu(W1 z) * (W3 z)); weights [hid, d], [hid, d], [d, hid]."""
    z = _f(z)
    u = silu(z @ _f(w1).T) * (z @ _f(w3).T)
    return u @ _f(w2).T


def causal_attention(q, k, v, scale: float, q_pos: Optional[np.ndarray] = None) -> np.ndarray:
    """softmax(q k^T * scale, keys after the query masked) v for one (sequence, head).

    q [Sq, dq] at positions ``q_pos`` (default 0..Sq-1), k [Sk, dq], v [Sk, dv].
    """
    q, k, v = _f(q), _f(k), _f(v)
    if q_pos is None:
        q_pos = np.arange(q.shape[0])
    out = np.empty((q.shape[0], v.shape[1]), dtype=F)
    kpos = np.arange(k.shape[0])
    for i0 in range(0, q.shape[0], ATTN_QBLOCK):
        qp = q_pos[i0:i0 + ATTN_QBLOCK]
        kmax = int(qp.max()) + 1
        s = (q[i0:i0 + ATTN_QBLOCK] @ k[:kmax].T) * scale
        s = np.where(kpos[None, :kmax] > qp[:, None], -np.inf, s)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[i0:i0 + ATTN_QBLOCK] = p @ v[:kmax]
    return out


def gqa_attention(q, k, v, scale: float, q_pos: Optional[np.ndarray] = None) -> np.ndarray:
    """Grouped-query causal attention ([RV] GQA section; [GS] Passo 5).

    q [B, Sq, Hq, dq]; k [B, Sk, Hkv, dq]; v [B, Sk, Hkv, dv]. Query head h reads
    KV head floor(h * Hkv / Hq). Returns [B, Sq, Hq, dv].
    """
    q, k, v = _f(q), _f(k), _f(v)
    Bn, Sq, Hq, _ = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv:
        raise ValueError("n_heads must be a multiple of n_kv_heads")
    o = np.empty((Bn, Sq, Hq, v.shape[3]), dtype=F)
    for b in range(Bn):
        for h in range(Hq):
            g = (h * Hkv) // Hq
            o[b, :, h] = causal_attention(q[b, :, h], k[b, :, g], v[b, :, g], scale, q_pos)
    return o


# --------------------------------------------------------------------------------------
# Router and mixture of experts
# --------------------------------------------------------------------------------------

@dataclass
class Routing:
    idx: np.ndarray       # [N, k] selected experts, by (score desc, index asc)
    w: np.ndarray         # [N, k] softmax over the selected logits
    gap: np.ndarray       # [N] k-th minus (k+1)-th selection score (inf when k == E)
    logits: np.ndarray    # [N, E]


def router_topk(logits, bias, k: int) -> Routing:
    """Top-k routing ([GS] Passo 2 n_experts_per_tok; troubleshooting item on router_bias).

    Selection ranks logits + bias; ties go to the lower expert index. Gate weights are
    the softmax of the selected logits alone (bias excluded), i.e. the full softmax
    renormalised over the k chosen experts.
    """
    logits = _f(logits)
    score = logits + (0.0 if bias is None else _f(bias))
    order = np.argsort(-score, axis=-1, kind="stable")
    idx = order[:, :k]
    srt = np.take_along_axis(score, order, axis=-1)
    gap = srt[:, k - 1] - srt[:, k] if k < score.shape[1] else np.full(score.shape[0], np.inf)
    sel = np.take_along_axis(logits, idx, axis=-1)
    ex = np.exp(sel - sel.max(axis=-1, keepdims=True))
    w = ex / ex.sum(axis=-1, keepdims=True)
    return Routing(idx=idx, w=w, gap=gap, logits=logits)


def moe_combine(yn, idx, w, w1, w3, w2, ws1=None, ws3=None, ws2=None) -> np.ndarray:
    """f[n] = sum_j w[n,j] * Expert_{idx[n,j]}(yn[n]) + sum_s Shared_s(yn[n]).

    Sparse MoE FFN ([TB] MoE per iteration; [GS] Passo 2 n_shared_experts always active;
    [CB] Sparse MoE section). Dropless: every (token, slot) is computed.
    """
    yn = _f(yn)
    idx = np.asarray(idx)
    f = np.zeros_like(yn)
    for e in range(w1.shape[0]):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        f[rows] += _f(w)[rows, slots][:, None] * swiglu_ffn(yn[rows], w1[e], w3[e], w2[e])
    if ws1 is not None:
        for s in range(ws1.shape[0]):
            f += swiglu_ffn(yn, ws1[s], ws3[s], ws2[s])
    return f


# --------------------------------------------------------------------------------------
# Attention sublayers
# --------------------------------------------------------------------------------------

def _lora_index(cfg, t: int) -> int:
    return min(t, cfg.n_lora - 1)


def gqa_qkv(xn, W, cfg, t: int):
    """Q, K, V projections with RoPE on Q and K, and the loop-t LoRA delta on Q."""
    Bn, S, _ = xn.shape
    hq, hkv, dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    q = xn @ _f(W["wq"]).T
    if cfg.n_lora:
        li = _lora_index(cfg, t)
        q = q + (xn @ _f(W["lq_a"][li]).T) @ _f(W["lq_b"][li]).T
    k = xn @ _f(W["wk"]).T
    v = xn @ _f(W["wv"]).T
    q = apply_rope(q.reshape(Bn, S, hq, dh), cfg.rope_base)
    k = apply_rope(k.reshape(Bn, S, hkv, dh), cfg.rope_base)
    return q, k, v.reshape(Bn, S, hkv, dh)


def out_proj(o, W, cfg, t: int) -> np.ndarray:
    """a = o Wo^T (+ the loop-t LoRA delta (o A'_t^T) B'_t^T)."""
    a = o @ _f(W["wo"]).T
    if cfg.n_lora:
        li = _lora_index(cfg, t)
        a = a + (o @ _f(W["lo_a"][li]).T) @ _f(W["lo_b"][li]).T
    return a


def mla_latents(xn, W, cfg):
    """c_q = RMSNorm(xn W_dq^T), c_kv = RMSNorm(xn W_dkv^T), k_rope = RoPE(xn W_kr^T).

    [GS] Passo 5 (q_lora_rank, kv_lora_rank, qk_rope_head_dim); [RV] MLA section
    (keys and values projected to a low-dimensional latent, as in DeepSeek-V3).
    """
    Bn, S, _ = xn.shape
    c_q = rmsnorm(xn @ _f(W["w_dq"]).T, W["q_norm"], cfg.norm_eps)
    c_kv = rmsnorm(xn @ _f(W["w_dkv"]).T, W["kv_norm"], cfg.norm_eps)
    k_rope = apply_rope((xn @ _f(W["w_kr"]).T).reshape(Bn, S, 1, cfg.qk_rope_dim), cfg.rope_base)
    return c_q, c_kv, k_rope


def mla_attention_explicit(xn, W, cfg) -> np.ndarray:
    """MLA with K and V rebuilt from the latent by their up-projections ([GS] Passo 5:
    K/V reconstructed by a linear projection at every step). Returns o [B, S, H*v]."""
    Bn, S, _ = xn.shape
    H, nope, rope, vd = cfg.n_heads, cfg.qk_nope_dim, cfg.qk_rope_dim, cfg.v_head_dim
    c_q, c_kv, k_rope = mla_latents(xn, W, cfg)
    qf = (c_q @ _f(W["w_uq"]).T).reshape(Bn, S, H, nope + rope)
    q = np.concatenate([qf[..., :nope], apply_rope(qf[..., nope:], cfg.rope_base)], axis=-1)
    k_nope = (c_kv @ _f(W["w_uk"]).T).reshape(Bn, S, H, nope)
    v = (c_kv @ _f(W["w_uv"]).T).reshape(Bn, S, H, vd)
    k = np.concatenate([k_nope, np.broadcast_to(k_rope, (Bn, S, H, rope))], axis=-1)
    o = gqa_attention(q, k, v, 1.0 / np.sqrt(nope + rope))
    return o.reshape(Bn, S, H * vd)


def mla_attention_absorbed(xn, W, cfg) -> np.ndarray:
    """The same MLA output with W_uk folded into the query and W_uv applied after the
    attention average: every head attends over the shared key [c_kv ; k_rope] and the
    shared value c_kv (one KV head). Algebraically equal to the explicit form."""
    Bn, S, _ = xn.shape
    H, nope, rope, vd = cfg.n_heads, cfg.qk_nope_dim, cfg.qk_rope_dim, cfg.v_head_dim
    L = cfg.kv_lora_rank
    c_q, c_kv, k_rope = mla_latents(xn, W, cfg)
    qf = (c_q @ _f(W["w_uq"]).T).reshape(Bn, S, H, nope + rope)
    w_uk = _f(W["w_uk"]).reshape(H, nope, L)
    w_uv = _f(W["w_uv"]).reshape(H, vd, L)
    q_lat = np.einsum("bshn,hnc->bshc", qf[..., :nope], w_uk)
    q_t = np.concatenate([q_lat, apply_rope(qf[..., nope:], cfg.rope_base)], axis=-1)
    key = np.concatenate([c_kv[:, :, None, :], k_rope], axis=-1)       # [B, S, 1, L + rope]
    o_lat = gqa_attention(q_t, key, c_kv[:, :, None, :], 1.0 / np.sqrt(nope + rope))
    o = np.einsum("bshc,hvc->bshv", o_lat, w_uv)
    return o.reshape(Bn, S, H * vd)


def attention_sublayer(x, W, cfg, t: int, mla_form: str = "explicit") -> np.ndarray:
    """a = Attn(RMSNorm1(x)) including the output projection (pre-norm block)."""
    x = _f(x)
    xn = rmsnorm(x, W["norm1"], cfg.norm_eps)
    Bn, S, _ = x.shape
    if cfg.attn == "gqa":
        q, k, v = gqa_qkv(xn, W, cfg, t)
        o = gqa_attention(q, k, v, 1.0 / np.sqrt(cfg.head_dim)).reshape(Bn, S, -1)
    elif mla_form == "explicit":
        o = mla_attention_explicit(xn, W, cfg)
    else:
        o = mla_attention_absorbed(xn, W, cfg)
    return out_proj(o, W, cfg, t)


def moe_sublayer(y, W, cfg, follow_idx=None, tie_band: float = NEAR_TIE) -> Tuple[np.ndarray, Routing, Dict[str, int]]:
    """f = MoE(RMSNorm2(y)). With ``follow_idx`` (another implementation's selection),
    tokens whose k-th/(k+1)-th score gap is at most ``tie_band`` (NEAR_TIE by default)
    adopt that selection; every other token keeps its own and is counted if the two sets
    differ. ``tie_band = inf`` adopts the other selection everywhere (gate weights still
    from this oracle's logits)."""
    y = _f(y)
    shp = y.shape
    yn = rmsnorm(y, W["norm2"], cfg.norm_eps).reshape(-1, shp[-1])
    r = router_topk(yn @ _f(W["w_router"]).T, W.get("router_bias"), cfg.top_k)
    stats = {"near_ties": 0, "mismatch": 0}
    idx = r.idx
    if follow_idx is not None:
        fi = np.asarray(follow_idx).reshape(idx.shape)
        near = r.gap <= tie_band
        same = np.all(np.sort(fi, axis=1) == np.sort(idx, axis=1), axis=1)
        stats["near_ties"] = int(np.count_nonzero(near & ~same))
        stats["mismatch"] = int(np.count_nonzero(~near & ~same))
        idx = np.where(near[:, None], fi, idx)
        sel = np.take_along_axis(r.logits, idx, axis=-1)
        ex = np.exp(sel - sel.max(axis=-1, keepdims=True))
        r = Routing(idx=idx, w=ex / ex.sum(axis=-1, keepdims=True), gap=r.gap, logits=r.logits)
    f = moe_combine(yn, r.idx, r.w, W["w1"], W["w3"], W["w2"],
                    W.get("ws1"), W.get("ws3"), W.get("ws2"))
    return f.reshape(shp), r, stats


# --------------------------------------------------------------------------------------
# Depth attention (attention over a token's earlier loop states)
# --------------------------------------------------------------------------------------

def depth_rope_angles(depth: int, n_depths: int, rot_dim: int, base: float) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin [rot/2] of the rotation at loop `depth` of `n_depths` ([DR] Dreamer summary,
    depth attention: RoPE over depth, with half of it reversed towards the last depth): pairs
    i < rot/4 turn by depth * theta_i, pairs i >= rot/4 by (n_depths - 1 - depth) * theta_i,
    theta_i = base^(-2i/rot)."""
    i = np.arange(rot_dim // 2, dtype=F)
    theta = np.power(F(base), -2.0 * i / rot_dim)
    pos = np.where(i < rot_dim // 4, F(depth), F(n_depths - 1 - depth))
    ang = pos * theta
    return np.cos(ang), np.sin(ang)


def apply_depth_rope(x, depth: int, n_depths: int, base: float) -> np.ndarray:
    """Rotate-half RoPE of x [..., r] at loop `depth` (see :func:`depth_rope_angles`)."""
    x = _f(x)
    r = x.shape[-1]
    cos, sin = depth_rope_angles(depth, n_depths, r, base)
    x1, x2 = x[..., : r // 2], x[..., r // 2:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


@dataclass
class DepthKV:
    """Keys and values of the depth attention at every loop so far, per token:
    ``k[s]``, ``v[s]`` [B, S, Hkv, dh] for loops s = 0 .. t."""
    k: List[np.ndarray] = field(default_factory=list)
    v: List[np.ndarray] = field(default_factory=list)


def depth_attention_sublayer(x, W, cfg, t: int, n_depths: int, kv: DepthKV) -> np.ndarray:
    """d = DA(RMSNorm_da(x)) at loop t ([DR] depth attention: the sequence dimension is the
    batch and the depth is the sequence): every token's query attends over its own keys of
    loops 0 .. t (causal over depth), heads grouped as in GQA, scale 1/sqrt(head_dim);
    appends loop t's keys and values to ``kv``. Returns d [B, S, dim]."""
    x = _f(x)
    Bn, S, _ = x.shape
    hq, hkv, dh = cfg.da_heads, cfg.da_kv_heads, cfg.head_dim
    xn = rmsnorm(x, W["norm_da"], cfg.norm_eps)
    q = apply_depth_rope((xn @ _f(W["wq_d"]).T).reshape(Bn, S, hq, dh), t, n_depths, cfg.rope_base)
    kv.k.append(apply_depth_rope((xn @ _f(W["wk_d"]).T).reshape(Bn, S, hkv, dh), t, n_depths, cfg.rope_base))
    kv.v.append((xn @ _f(W["wv_d"]).T).reshape(Bn, S, hkv, dh))
    K = np.stack(kv.k, axis=2)                      # [B, S, t + 1, hkv, dh]
    V = np.stack(kv.v, axis=2)
    o = np.empty((Bn, S, hq, dh), dtype=F)
    for h in range(hq):
        g = (h * hkv) // hq
        s = np.einsum("bnd,bnkd->bnk", q[:, :, h], K[:, :, :, g]) / np.sqrt(dh)   # keys: loops 0 .. t
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=-1, keepdims=True)
        o[:, :, h] = np.einsum("bnk,bnkd->bnd", p, V[:, :, :, g])
    return o.reshape(Bn, S, hq * dh) @ _f(W["wo_d"]).T


# --------------------------------------------------------------------------------------
# The loop
# --------------------------------------------------------------------------------------

def input_injection(e, B) -> np.ndarray:
    """B.e ([TB] update equation): elementwise for a diagonal B [d], e B^T for dense [d, d]."""
    e, B = _f(e), _f(B)
    return B * e if B.ndim == 1 else e @ B.T


def spectral_radius(A) -> float:
    """rho(A) for the diagonal A returned as a (dim,) vector ([GS] Passo 6): max |A_i|."""
    return float(np.max(np.abs(_f(A))))


@dataclass
class LoopTrace:
    h: List[np.ndarray] = field(default_factory=list)        # h_0 .. h_T
    delta: List[np.ndarray] = field(default_factory=list)    # Delta_0 .. Delta_{T-1}
    attn: List[np.ndarray] = field(default_factory=list)
    moe: List[np.ndarray] = field(default_factory=list)
    routing: List[Routing] = field(default_factory=list)
    stats: List[Dict[str, int]] = field(default_factory=list)


def loop_forward(h0, e, T: int, W, cfg, follow: Optional[Sequence[np.ndarray]] = None,
                 trace: Optional[LoopTrace] = None, mla_form: str = "explicit",
                 tie_band: float = NEAR_TIE) -> np.ndarray:
    """h_{t+1} = A.h_t + B.e + Transformer(h_t, e) for t = 0..T-1 ([TB] update equation;
    [GS] Passo 3: the same block repeated n_loops times).

    Transformer(h, e) = a + f with x = h + e (or x = h), a = Attn(RMSNorm1(x)),
    y = x + a, f = MoE(RMSNorm2(y)); with depth attention (``cfg.da_heads`` > 0) first
    d = DA(x) at loop t of T, x <- x + d, and Transformer(h, e) = d + a + f. ``follow[t]`` is an optional [N, k] selection to
    adopt on near-ties at loop t, those within ``tie_band`` (see :func:`moe_sublayer`).
    """
    A = _f(W["A"])
    e = _f(e)
    Be = input_injection(e, W["B"])
    h = _f(h0)
    depth = DepthKV() if getattr(cfg, "da_heads", 0) else None
    if trace is not None:
        trace.h.append(h.copy())
    for t in range(T):
        x = h + e if cfg.inject_e else h
        d = 0.0
        if depth is not None:
            d = depth_attention_sublayer(x, W, cfg, t, T, depth)
            x = x + d
        a = attention_sublayer(x, W, cfg, t, mla_form)
        y = x + a
        f, r, st = moe_sublayer(y, W, cfg, None if follow is None else follow[t], tie_band)
        delta = d + a + f
        h = A * h + Be + delta
        if trace is not None:
            trace.h.append(h.copy())
            trace.delta.append(delta)
            trace.attn.append(a)
            trace.moe.append(f)
            trace.routing.append(r)
            trace.stats.append(st)
    return h


# --------------------------------------------------------------------------------------
# One loop step evaluated at chosen positions only (for checks at full size)
# --------------------------------------------------------------------------------------

def loop_step_rows(h, e, W, cfg, t: int, rows: Sequence[Tuple[int, int]],
                   follow_idx: Optional[np.ndarray] = None):
    """h_{t+1} at the (batch, position) pairs ``rows``, given the full state h_t [B, S, d].

    Causality makes position s depend on positions 0..s of its own sequence only, so
    each output is evaluated from that prefix. Returns (h_next [R, d], routing, stats).
    ``follow_idx`` [R, k] is another implementation's selection at those rows.
    """
    A = _f(W["A"])
    h, e = _f(h), _f(e)
    rows = [(int(b), int(s)) for b, s in rows]
    a_rows = np.empty((len(rows), h.shape[2]), dtype=F)
    x_rows = np.empty_like(a_rows)
    for b in sorted({b for b, _ in rows}):
        sel = [i for i, (bb, _) in enumerate(rows) if bb == b]
        smax = max(rows[i][1] for i in sel) + 1
        x = (h[b:b + 1, :smax] + e[b:b + 1, :smax]) if cfg.inject_e else h[b:b + 1, :smax]
        xn = rmsnorm(x, W["norm1"], cfg.norm_eps)
        pos = np.array([rows[i][1] for i in sel])
        if cfg.attn == "gqa":
            q, k, v = gqa_qkv(xn, W, cfg, t)
            o = gqa_attention(q[:, pos], k, v, 1.0 / np.sqrt(cfg.head_dim), q_pos=pos)
            o = o.reshape(len(sel), -1)
        else:
            o = mla_attention_explicit(xn, W, cfg)[0, pos]
        a_rows[sel] = out_proj(o, W, cfg, t)
        x_rows[sel] = x[0, pos]
    y = x_rows + a_rows
    f, r, st = moe_sublayer(y, W, cfg, follow_idx)
    bidx = np.array([b for b, _ in rows])
    sidx = np.array([s for _, s in rows])
    Be = input_injection(e[bidx, sidx], W["B"])
    h_next = A * h[bidx, sidx] + Be + a_rows + f
    return h_next, r, st


# --------------------------------------------------------------------------------------
# ACT halting inside the loop
# --------------------------------------------------------------------------------------

def halting_probability(h, w_halt, b_halt) -> np.ndarray:
    """p = sigmoid(h . w_halt + b_halt) over the last axis: the halting head. [TB] names
    ACT halting and [GS] troubleshooting item 4 its threshold, but neither gives the head;
    this is the plainest one, a linear map of the state to one logit."""
    z = _f(h) @ _f(w_halt) + F(b_halt)
    return 1.0 / (1.0 + np.exp(-z))


@dataclass
class ActResult:
    out: np.ndarray          # [B, S, d]: sum over t of weights[t] * h_{t+1}
    n_loops: np.ndarray      # [B, S]: loops each position ran (its halting loop, 1-based)
    weights: np.ndarray      # [T, B, S]: weight of h_{t+1} in out (sums to 1 over t)
    stats: Dict[str, int]


def loop_forward_act(h0, e, T: int, W, cfg, w_halt, b_halt: float, threshold: float,
                     follow: Optional[Sequence[np.ndarray]] = None,
                     follow_loops: Optional[np.ndarray] = None,
                     trace: Optional[LoopTrace] = None, mla_form: str = "explicit") -> ActResult:
    """The loop of :func:`loop_forward` with ACT halting per position ([TB] "Dynamic
    Adaptive Computation Time"; [GS] troubleshooting item 4, act_threshold = 0.99).

    At loop t every position computes attention as usual (a halted position keeps its
    state, so its keys and values are those of its last state); positions still running
    are routed through the MoE and update h_{t+1} = A.h_t + B.e + a + f, halted ones keep
    h_{t+1} = h_t. Then each running position takes p_t = sigmoid(w . h_{t+1} + b); with
    c the sum of its earlier p, it halts at this loop if c + p_t >= threshold or t = T - 1,
    and h_{t+1} enters the output with weight 1 - c (the remainder); otherwise with weight
    p_t, and c grows by p_t.

    ``follow[t]`` ([N, k]) is another implementation's routing, adopted on near-ties as in
    :func:`moe_sublayer`; ``follow_loops`` ([B, S]) its halting loops, adopted where
    |c + p_t - threshold| <= NEAR_HALT; every other difference is counted in ``stats``.
    """
    A = _f(W["A"])
    e = _f(e)
    Be = input_injection(e, W["B"])
    h = _f(h0)
    bs = h.shape[:2]
    cum = np.zeros(bs, dtype=F)
    halted = np.zeros(bs, dtype=bool)
    n_loops = np.zeros(bs, dtype=np.int64)
    out = np.zeros_like(h)
    weights = np.zeros((T,) + bs, dtype=F)
    stats = {"near_ties": 0, "mismatch": 0, "near_halts": 0, "halt_mismatch": 0}
    theirs_loops = None if follow_loops is None else np.asarray(follow_loops).reshape(bs)
    if trace is not None:
        trace.h.append(h.copy())
    for t in range(T):
        x = h + e if cfg.inject_e else h
        a = attention_sublayer(x, W, cfg, t, mla_form)
        y = x + a
        run = ~halted
        f = np.zeros_like(y)
        if run.any():
            fi = None
            if follow is not None:
                fi = np.asarray(follow[t]).reshape(bs + (-1,))[run]
            f_run, r, st = moe_sublayer(y[run], W, cfg, fi)
            f[run] = f_run
            stats["near_ties"] += st["near_ties"]
            stats["mismatch"] += st["mismatch"]
        h_new = A * h + Be + a + f
        h_new[halted] = h[halted]                       # a halted position keeps its state
        p = halting_probability(h_new, w_halt, b_halt)
        reach = cum + p
        if t == T - 1:
            stop = run.copy()
        else:
            stop = run & (reach >= threshold)
            if theirs_loops is not None:
                theirs = run & (theirs_loops == t + 1)
                near = run & (np.abs(reach - threshold) <= NEAR_HALT)
                stats["near_halts"] += int(np.count_nonzero(near & (theirs != stop)))
                stats["halt_mismatch"] += int(np.count_nonzero(~near & (theirs != stop)))
                stop = np.where(near, theirs, stop)
        w = np.where(stop, 1.0 - cum, np.where(run, p, 0.0))
        out += w[..., None] * h_new
        weights[t] = w
        cum = np.where(run, reach, cum)
        n_loops[stop] = t + 1
        halted |= stop
        h = h_new
        if trace is not None:
            trace.h.append(h.copy())
            trace.attn.append(a)
            trace.moe.append(f)
    return ActResult(out=out, n_loops=n_loops, weights=weights, stats=stats)


# --------------------------------------------------------------------------------------
# Decode with a per-loop KV cache
# --------------------------------------------------------------------------------------

def apply_rope_at(x, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE of x [B, Sn, H, r] with row j of axis 1 at position pos[j]
    (:func:`apply_rope` is the case pos = 0..Sn-1)."""
    x = _f(x)
    r = x.shape[-1]
    pos = np.asarray(pos)
    cos, sin = rope_angles(int(pos.max()) + 1, r, base)
    cos = cos[pos][None, :, None, :]
    sin = sin[pos][None, :, None, :]
    x1, x2 = x[..., : r // 2], x[..., r // 2:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


@dataclass
class LoopKVCache:
    """What each loop keeps for the positions processed so far ([GS] Passo 4 and
    troubleshooting item 1). Per loop t: GQA ``k[t]`` (after RoPE) and ``v[t]``
    [B, length, Hkv, dh]; MLA ``ckv[t]`` [B, length, kv_lat] (after its RMSNorm) and
    ``kr[t]`` [B, length, rope] (after RoPE), from which K and V are rebuilt ([GS] Passo 5)."""
    length: int = 0
    k: Dict[int, np.ndarray] = field(default_factory=dict)
    v: Dict[int, np.ndarray] = field(default_factory=dict)
    ckv: Dict[int, np.ndarray] = field(default_factory=dict)
    kr: Dict[int, np.ndarray] = field(default_factory=dict)


def _append(store: Dict[int, np.ndarray], t: int, new: np.ndarray) -> np.ndarray:
    store[t] = new if t not in store else np.concatenate([store[t], new], axis=1)
    return store[t]


def attention_cached(x, W, cfg, t: int, cache: LoopKVCache) -> np.ndarray:
    """a = Attn(RMSNorm1(x)) for x [B, Sn, d] at positions cache.length .. + Sn - 1,
    attending over loop t's cached keys and values of the earlier positions and its own;
    appends this loop's new keys and values to the cache (the caller advances
    ``cache.length`` once every loop has run)."""
    x = _f(x)
    Bn, Sn, _ = x.shape
    pos = cache.length + np.arange(Sn)
    xn = rmsnorm(x, W["norm1"], cfg.norm_eps)
    if cfg.attn == "gqa":
        hq, hkv, dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
        q = xn @ _f(W["wq"]).T
        if cfg.n_lora:
            li = _lora_index(cfg, t)
            q = q + (xn @ _f(W["lq_a"][li]).T) @ _f(W["lq_b"][li]).T
        q = apply_rope_at(q.reshape(Bn, Sn, hq, dh), pos, cfg.rope_base)
        k = apply_rope_at((xn @ _f(W["wk"]).T).reshape(Bn, Sn, hkv, dh), pos, cfg.rope_base)
        v = (xn @ _f(W["wv"]).T).reshape(Bn, Sn, hkv, dh)
        k_all = _append(cache.k, t, k)
        v_all = _append(cache.v, t, v)
        o = gqa_attention(q, k_all, v_all, 1.0 / np.sqrt(dh), q_pos=pos).reshape(Bn, Sn, -1)
    else:
        H, nope, rope, vd = cfg.n_heads, cfg.qk_nope_dim, cfg.qk_rope_dim, cfg.v_head_dim
        c_q = rmsnorm(xn @ _f(W["w_dq"]).T, W["q_norm"], cfg.norm_eps)
        c_kv = rmsnorm(xn @ _f(W["w_dkv"]).T, W["kv_norm"], cfg.norm_eps)
        k_r = apply_rope_at((xn @ _f(W["w_kr"]).T).reshape(Bn, Sn, 1, rope), pos, cfg.rope_base)
        ckv_all = _append(cache.ckv, t, c_kv)
        kr_all = _append(cache.kr, t, k_r[:, :, 0])
        L = ckv_all.shape[1]
        qf = (c_q @ _f(W["w_uq"]).T).reshape(Bn, Sn, H, nope + rope)
        q = np.concatenate([qf[..., :nope], apply_rope_at(qf[..., nope:], pos, cfg.rope_base)], axis=-1)
        k_nope = (ckv_all @ _f(W["w_uk"]).T).reshape(Bn, L, H, nope)      # rebuilt from the latent
        v = (ckv_all @ _f(W["w_uv"]).T).reshape(Bn, L, H, vd)
        k = np.concatenate([k_nope, np.broadcast_to(kr_all[:, :, None, :], (Bn, L, H, rope))], axis=-1)
        o = gqa_attention(q, k, v, 1.0 / np.sqrt(nope + rope), q_pos=pos).reshape(Bn, Sn, -1)
    return out_proj(o, W, cfg, t)


def _loop_cached(h0, e, T: int, W, cfg, cache: LoopKVCache, follow=None, stats=None) -> np.ndarray:
    A = _f(W["A"])
    e = _f(e)
    Be = input_injection(e, W["B"])
    h = _f(h0)
    for t in range(T):
        x = h + e if cfg.inject_e else h
        a = attention_cached(x, W, cfg, t, cache)
        y = x + a
        f, _, st = moe_sublayer(y, W, cfg, None if follow is None else follow[t])
        if stats is not None:
            for k in st:
                stats[k] = stats.get(k, 0) + st[k]
        h = A * h + Be + a + f
    cache.length += h.shape[1]
    return h


def loop_prefill(h0, e, T: int, W, cfg, follow=None, stats=None) -> Tuple[np.ndarray, LoopKVCache]:
    """The loop over a whole prompt [B, S, d] ([GS] Passo 4, first call): h_T and the
    cache of every loop's keys and values for positions 0..S-1. ``follow[t]`` ([B*S, k])
    is another implementation's routing, adopted on near-ties as in :func:`moe_sublayer`;
    ``stats`` (a dict) collects the counts."""
    cache = LoopKVCache()
    h = _loop_cached(h0, e, T, W, cfg, cache, follow, stats)
    return h, cache


def loop_decode(h0, e, T: int, W, cfg, cache: LoopKVCache, follow=None, stats=None) -> np.ndarray:
    """T loops for new tokens h0, e [B, Sn, d] (Sn = 1 in a decode step) at positions
    cache.length .., each loop t attending over loop t's cache; extends the cache.
    ``follow`` and ``stats`` as in :func:`loop_prefill`."""
    return _loop_cached(h0, e, T, W, cfg, cache, follow, stats)
