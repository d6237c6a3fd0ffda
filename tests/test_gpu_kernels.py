"""The tensor-core GEMM and the attention kernel alone (rdt_matmul, rdt_attention) against
fp64 references on the same rounded inputs."""
import math

import numpy as np
import pytest

import oracle as O

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (300, 256, 1024), (2048, 1536, 1024),
                                   (77, 96, 128), (1, 32, 64), (4096, 2048, 2048)])
def test_matmul_bf16(M, N, K):
    torch = _torch()
    import recurrent_depth_transformer_b200 as R
    g = torch.Generator().manual_seed(M * 7 + N)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    C = R.matmul(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    ref = A.double() @ B.double().T
    err = (C.cpu().double() - ref).abs().max().item()
    assert err <= 2e-5 * K, err          # fp32 accumulation of exact bf16 products


@pytest.mark.parametrize("M,N,K", [(64, 128, 128), (200, 256, 512)])
def test_matmul_tf32(M, N, K):
    torch = _torch()
    import recurrent_depth_transformer_b200 as R
    g = torch.Generator().manual_seed(M + N)
    A = torch.randn(M, K, generator=g)
    B = torch.randn(N, K, generator=g)
    C = R.matmul(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    ref = A.double() @ B.double().T
    err = (C.cpu().double() - ref).abs().max().item()
    # tf32 keeps 10 mantissa bits: relative error 2^-11 per operand
    assert err <= 6 * 2.0 ** -11 * math.sqrt(K) * 4, err


@pytest.mark.parametrize("batch,seq,hq,hkv,dqk,dv", [(2, 200, 4, 2, 64, 64), (1, 64, 2, 2, 64, 64),
                                                     (1, 1, 2, 1, 64, 64), (2, 130, 4, 1, 160, 128),
                                                     (1, 513, 16, 4, 64, 64)])
def test_attention_bf16(batch, seq, hq, hkv, dqk, dv):
    torch = _torch()
    import recurrent_depth_transformer_b200 as R
    g = torch.Generator().manual_seed(seq * 3 + dqk)
    q = torch.randn(batch * seq, hq * dqk, generator=g).to(torch.bfloat16)
    k = torch.randn(batch * seq, hkv * dqk, generator=g).to(torch.bfloat16)
    v = torch.randn(batch * seq, hkv * dv, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(dqk)
    o = R.attention(q.cuda(), k.cuda(), v.cuda(), batch, seq, hq, hkv, dqk, dv, scale)
    torch.cuda.synchronize()
    ref = O.gqa_attention(q.float().numpy().reshape(batch, seq, hq, dqk),
                          k.float().numpy().reshape(batch, seq, hkv, dqk),
                          v.float().numpy().reshape(batch, seq, hkv, dv), scale)
    err = np.abs(o.cpu().float().numpy().reshape(ref.shape) - ref).max()
    assert err < 2e-2, err


def test_attention_f32():
    torch = _torch()
    import recurrent_depth_transformer_b200 as R
    batch, seq, hq, hkv, d = 1, 64, 4, 2, 32
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(batch * seq, h * d, generator=g) for h in (hq, hkv, hkv))
    o = R.attention(q.cuda(), k.cuda(), v.cuda(), batch, seq, hq, hkv, d, d, 0.2)
    torch.cuda.synchronize()
    ref = O.gqa_attention(q.numpy().reshape(1, seq, hq, d), k.numpy().reshape(1, seq, hkv, d),
                          v.numpy().reshape(1, seq, hkv, d), 0.2)
    assert np.abs(o.cpu().numpy().reshape(ref.shape) - ref).max() < 1e-4


@pytest.mark.parametrize("batch,seq,hq", [(2, 130, 4), (1, 300, 16)])
def test_attention_shared_latent_kv(batch, seq, hq):
    """Absorbed MLA: every head attends over the shared 160-wide key [c_kv ; k_rope] with the
    value c_kv = the key's first 128 columns (v passed as the key tensor itself)."""
    torch = _torch()
    import recurrent_depth_transformer_b200 as R
    g = torch.Generator().manual_seed(seq + hq)
    q = torch.randn(batch * seq, hq * 160, generator=g).to(torch.bfloat16)
    k = torch.randn(batch * seq, 160, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(96)
    kc = k.cuda()
    o = R.attention(q.cuda(), kc, kc, batch, seq, hq, 1, 160, 128, scale)
    torch.cuda.synchronize()
    kf = k.float().numpy().reshape(batch, seq, 1, 160)
    ref = O.gqa_attention(q.float().numpy().reshape(batch, seq, hq, 160), kf, kf[..., :128], scale)
    err = np.abs(o.cpu().float().numpy().reshape(ref.shape) - ref).max()
    assert err < 2e-2, err


@pytest.mark.parametrize("kind", ["gqa", "mla"])
def test_attention_long_sequence_rows_from_every_tile(kind):
    """Causal attention at the long configuration's length (8192 positions): about 256 query
    rows drawn from every 128-row query tile, for two heads, element by element against the
    oracle's attention at those positions (keys 0 .. position)."""
    torch = _torch()
    import recurrent_depth_transformer_b200 as R
    S = 8192
    if kind == "gqa":
        hq, hkv, dqk, dv = 32, 8, 64, 64
    else:
        hq, hkv, dqk, dv = 16, 1, 160, 128
    g = torch.Generator().manual_seed(S + dqk)
    q = torch.randn(S, hq * dqk, generator=g).to(torch.bfloat16)
    k = torch.randn(S, hkv * dqk, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(64 if kind == "gqa" else 96)
    kc = k.cuda()
    if kind == "gqa":
        v = torch.randn(S, hkv * dv, generator=g).to(torch.bfloat16)
        o = R.attention(q.cuda(), kc, v.cuda(), 1, S, hq, hkv, dqk, dv, scale)
    else:
        v = k[:, :dv]
        o = R.attention(q.cuda(), kc, kc, 1, S, hq, 1, dqk, dv, scale)
    torch.cuda.synchronize()
    got = o.cpu().float().numpy().reshape(S, hq, dv)
    rng = np.random.default_rng(11)
    pos = np.sort(np.concatenate([np.arange(0, S, 128) + rng.integers(0, 128, S // 128),
                                  rng.integers(0, S, 192), [0, 127, 128, S - 1]]))
    qf = q.float().numpy().reshape(S, hq, dqk)
    kf = k.float().numpy().reshape(S, hkv, dqk)
    vf = v.float().numpy().reshape(S, hkv, dv)
    for h in (0, hq - 1):
        kv = (h * hkv) // hq
        ref = O.causal_attention(qf[pos, h], kf[:, kv], vf[:, kv], scale, q_pos=pos)
        err = np.abs(got[pos, h] - ref).max()
        assert err < 2e-2, (h, err)
