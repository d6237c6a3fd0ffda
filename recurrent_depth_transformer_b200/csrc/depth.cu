// Depth attention: attention over a token's own earlier loop states (gist.science summary
// of "Dreamer", depth attention: the sequence dimension is treated as the batch and the
// depth as the sequence).
//
// At loop t every token has one query per depth head and the keys and values that the
// depth-attention projection produced from its block inputs at loops 0 .. t (kept in a
// per-token depth cache, loop t's row appended just before). The number of keys is at most
// the loop count, so the kernel is a short, memory-light reduction: one warp per
// (token, head), each lane holding two of the head's 64 columns; scores are warp sums,
// the softmax runs online over the depths in log2 units.
#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr int kDepthWarps = 8;

__global__ void __launch_bounds__(kDepthWarps * 32) depth_attn_kernel(const DepthAttnArgs a) {
    pdl_trigger();
    pdl_wait();
    const int w = blockIdx.x * kDepthWarps + (threadIdx.x >> 5);     // token * hq + head
    const int lane = threadIdx.x & 31;
    if (w >= a.ntok * a.hq) return;
    const int n = w / a.hq, h = w % a.hq;
    const int g = (h * a.hkv) / a.hq;
    const __nv_bfloat162 qb = *reinterpret_cast<const __nv_bfloat162*>(a.q + static_cast<size_t>(n) * a.q_ld +
                                                                       h * 64 + 2 * lane);
    const float2 q = __bfloat1622float2(qb);
    const bf16* rows = a.cache + static_cast<size_t>(n) * a.max_depth * a.cache_w;
    float m = -INFINITY, l = 0.0f, o0 = 0.0f, o1 = 0.0f;
#pragma unroll 1
    for (int s = 0; s <= a.t; ++s) {
        const bf16* row = rows + static_cast<size_t>(s) * a.cache_w;
        const float2 k = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + g * 64 + 2 * lane));
        const float2 v =
            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + a.v_col0 + g * 64 + 2 * lane));
        const float sc = warp_sum(fmaf(q.x, k.x, q.y * k.y)) * a.scale_log2;
        const float m_new = fmaxf(m, sc);
        const float corr = exp2f(m - m_new);
        const float p = exp2f(sc - m_new);
        l = l * corr + p;
        o0 = fmaf(o0, corr, p * v.x);
        o1 = fmaf(o1, corr, p * v.y);
        m = m_new;
    }
    const float inv = 1.0f / l;
    *reinterpret_cast<__nv_bfloat162*>(a.o + static_cast<size_t>(n) * a.o_ld + h * 64 + 2 * lane) =
        __floats2bfloat162_rn(o0 * inv, o1 * inv);
}

}  // namespace

rdt_status depth_attention(const DepthAttnArgs& a, cudaStream_t st) {
    const long warps = static_cast<long>(a.ntok) * a.hq;
    RDT_CUDA_TRY(launch_pdl(depth_attn_kernel, dim3(static_cast<unsigned>((warps + kDepthWarps - 1) / kDepthWarps)),
                            dim3(kDepthWarps * 32), 0, st, a));
    return RDT_OK;
}

}  // namespace rdt
