"""Pins of the oracle's depth attention (attention over a token's earlier loop states) against
facts fixed outside it: the ordinary rotary embedding (itself pinned against a complex
rotation), PyTorch's scaled-dot-product attention with the depth as the sequence, the
closed form of the first loop (one key: the value itself), and the plain loop when the
sublayer's output projection is zero. A planted mistake in the reversed half or in the
residual wiring fails one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as tF

import oracle as O
from workloads import Workload, generate

TD = torch.float64


def _t(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64))


def small_da(**kw) -> Workload:
    base = dict(name="pin-da", dtype="f32", batch=2, seq=9, dim=32, attn="gqa", n_heads=4, n_kv_heads=2,
                head_dim=8, n_experts=4, top_k=2, expert_hidden=16, b_kind="diag", loops=(4,), seed=13,
                da_heads=4, da_kv_heads=2)
    base.update(kw)
    return Workload(**base)


def test_depth_rope_halves_are_ordinary_rope_at_forward_and_reversed_positions():
    rng = np.random.default_rng(0)
    r, n, base = 16, 7, 1e4
    x = rng.standard_normal((3, 2, r))
    for t in range(n):
        got = O.apply_depth_rope(x, t, n, base)
        seqx = np.repeat(x[None, None], n, axis=1).reshape(1, n, 6, r)    # [1, positions, 6, r]
        plain = O.apply_rope(seqx, base)[0]                                # position p in row p
        fwd = plain[t].reshape(3, 2, r)
        rev = plain[n - 1 - t].reshape(3, 2, r)
        q = r // 4                                                         # pairs (i, i + r/2), i < r/4
        for i in range(r // 2):
            src = fwd if i < q else rev
            np.testing.assert_allclose(got[..., i], src[..., i], atol=1e-13)
            np.testing.assert_allclose(got[..., i + r // 2], src[..., i + r // 2], atol=1e-13)


def test_first_loop_is_the_value_projection():
    """At loop 0 every token has one key (its own): softmax weight 1, d = v W_o^T."""
    cfg = small_da()
    W = generate(cfg)
    x = W["e"] * 1.4
    d = O.depth_attention_sublayer(x, W, cfg, 0, 4, O.DepthKV())
    xn = O.rmsnorm(x, W["norm_da"], cfg.norm_eps)
    v = (xn @ W["wv_d"].astype(np.float64).T).reshape(2, 9, 2, 8)
    o = np.repeat(v, 2, axis=2).reshape(2, 9, 32)                          # head h reads KV head h // 2
    np.testing.assert_allclose(d, o @ W["wo_d"].astype(np.float64).T, rtol=1e-12, atol=1e-13)


def _da_torch(xs, W, cfg, n):
    """Depth attention of loops 0 .. len(xs) - 1 with PyTorch: rms_norm, linear, the rotary
    halves as complex rotations, SDPA over the depth axis (tokens as the batch), causal."""
    hq, hkv, dh = cfg.da_heads, cfg.da_kv_heads, cfg.head_dim
    X = torch.stack([_t(x) for x in xs], dim=2)                             # [B, S, D, d]
    Bn, S, D, d = X.shape
    xn = tF.rms_norm(X, (d,), weight=_t(W["norm_da"]), eps=cfg.norm_eps)
    q = tF.linear(xn, _t(W["wq_d"])).view(Bn, S, D, hq, dh)
    k = tF.linear(xn, _t(W["wk_d"])).view(Bn, S, D, hkv, dh)
    v = tF.linear(xn, _t(W["wv_d"])).view(Bn, S, D, hkv, dh)
    i = torch.arange(dh // 2, dtype=TD)
    theta = cfg.rope_base ** (-2.0 * i / dh)
    depth = torch.arange(D, dtype=TD)[:, None]
    pos = torch.where(i[None, :] < dh // 4, depth, (n - 1) - depth)        # [D, dh/2]
    rot = torch.polar(torch.ones_like(pos), pos * theta)[None, None, :, None, :]

    def turn(u):
        z = torch.complex(u[..., : dh // 2], u[..., dh // 2:]) * rot
        return torch.cat([z.real, z.imag], dim=-1)

    q, k = turn(q), turn(k)
    # depth as the sequence, (batch, position) as the batch: [B*S, H, D, dh]
    q = q.reshape(Bn * S, D, hq, dh).transpose(1, 2)
    k = k.reshape(Bn * S, D, hkv, dh).transpose(1, 2)
    v = v.reshape(Bn * S, D, hkv, dh).transpose(1, 2)
    o = tF.scaled_dot_product_attention(q, k, v, is_causal=True, scale=1.0 / math.sqrt(dh), enable_gqa=True)
    o = o.transpose(1, 2).reshape(Bn, S, D, hq * dh)
    return tF.linear(o, _t(W["wo_d"])).numpy()                             # [B, S, D, d]


def test_depth_attention_matches_sdpa_over_depth():
    cfg = small_da()
    W = generate(cfg)
    rng = np.random.default_rng(3)
    n = 5
    xs = [W["e"] * (1.0 + 0.3 * t) + rng.standard_normal(W["e"].shape) * 0.5 for t in range(n)]
    want = _da_torch(xs, W, cfg, n)
    kv = O.DepthKV()
    for t in range(n):
        got = O.depth_attention_sublayer(xs[t], W, cfg, t, n, kv)
        np.testing.assert_allclose(got, want[:, :, t], rtol=1e-11, atol=1e-12)


def test_zero_output_projection_gives_the_plain_loop():
    cfg = small_da()
    W = generate(cfg)
    W["wo_d"] = np.zeros_like(W["wo_d"])
    with_da = O.loop_forward(W["h0"], W["e"], 4, W, cfg)
    plain = O.loop_forward(W["h0"], W["e"], 4, W, cfg.replace(da_heads=0, da_kv_heads=0))
    np.testing.assert_array_equal(with_da, plain)


def _gqa_sublayer_torch(x, W, cfg):
    from test_oracle_pins import _gqa_torch
    return _gqa_torch(x, W, cfg, 0)


def test_loop_composes_depth_then_sequence_attention_then_experts():
    """Three loops against a composition of independently pinned parts: depth attention by
    PyTorch over the block inputs so far, x' = x + d, the sequence-attention sublayer by
    PyTorch, the experts by the oracle's MoE (pinned on its own), the update equation."""
    cfg = small_da()
    W = generate(cfg)
    T = 3
    tr = O.LoopTrace()
    O.loop_forward(W["h0"], W["e"], T, W, cfg, trace=tr)
    A, Be = W["A"].astype(np.float64), W["B"].astype(np.float64) * W["e"]
    h = W["h0"].astype(np.float64)
    xs = []
    for t in range(T):
        x = h + W["e"]
        xs.append(x)
        d = _da_torch(xs, W, cfg, T)[:, :, t]
        x2 = x + d
        a = _gqa_sublayer_torch(x2, W, cfg)
        y = x2 + a
        f, _, _ = O.moe_sublayer(y, W, cfg)
        h = A * h + Be + d + a + f
        np.testing.assert_allclose(tr.h[t + 1], h, rtol=1e-10, atol=1e-10)


def test_pins_catch_planted_mistakes(monkeypatch):
    cfg = small_da()
    W = generate(cfg)
    n = 4
    rng = np.random.default_rng(5)
    xs = [W["e"] + rng.standard_normal(W["e"].shape) for _ in range(n)]
    want = _da_torch(xs, W, cfg, n)

    def run():
        kv = O.DepthKV()
        return [O.depth_attention_sublayer(xs[t], W, cfg, t, n, kv) for t in range(n)]

    # the reversed half turned forward
    def fwd_only(depth, n_depths, rot_dim, base):
        return O.rope_angles(depth + 1, rot_dim, base)[0][depth], O.rope_angles(depth + 1, rot_dim, base)[1][depth]

    monkeypatch.setattr(O.rdt_oracle, "depth_rope_angles", fwd_only)
    got = run()
    assert max(np.max(np.abs(g - want[:, :, t])) for t, g in enumerate(got)) > 1e-6
