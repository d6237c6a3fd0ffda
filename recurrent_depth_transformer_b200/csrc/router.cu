// RMSNorm2 fused with the MoE router for routers whose weight fits in shared memory:
// each block stages W_r (n_experts x dim) once, then every warp takes one row: RMSNorm2 in
// fp32 (stored in the element type as the experts' input), the n_experts logits of the fp32
// normalised row, top-k of logits + bias with ties to the lower expert index, softmax over
// the k chosen logits, per-expert histogram.
#include <algorithm>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

// ----------------------------------------------------------------------------- norm2 + router (W_r in shared memory)

// For routers whose weight fits in shared memory: each block stages W_r once, then every
// warp takes rows in turn: RMSNorm2 (fp32, stored in the element type for the experts), the
// n_exp logits of the fp32 row against W_r, top-k of logits + bias (ties to the lower expert
// index), softmax over the k chosen logits, histogram.
constexpr int kRouterThreads = 512;   // 16 rows in flight per staged copy of W_r

template <typename T, int NV, int EMAX, int KMAX>
__global__ void __launch_bounds__(kRouterThreads) norm2_router_smem_kernel(const RouterArgs a) {
    extern __shared__ __align__(16) uint8_t smem_w[];
    T* Ws = reinterpret_cast<T*>(smem_w);
    pdl_trigger();
    pdl_wait();
    {
        const int nvec = a.n_exp * a.dim * static_cast<int>(sizeof(T)) / 16;
        const uint4* src = static_cast<const uint4*>(a.w_router);
        uint4* dst = reinterpret_cast<uint4*>(smem_w);
        for (int i = threadIdx.x; i < nvec; i += blockDim.x) dst[i] = src[i];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (kRouterThreads / 32);
#pragma unroll 1
    for (int row = blockIdx.x * (kRouterThreads / 32) + (threadIdx.x >> 5); row < a.ntok; row += warps_total) {
        const size_t base = static_cast<size_t>(row) * a.dim;
        float y[NV][4];
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            load4(a.y + base + i * 128 + lane * 4, y[i]);
#pragma unroll
            for (int j = 0; j < 4; ++j) ss = fmaf(y[i][j], y[i][j], ss);
        }
        ss = warp_sum(ss);
        const float inv = rsqrtf(ss / a.dim + a.eps);
        T* yn = static_cast<T*>(a.yn) + base;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int col = i * 128 + lane * 4;
            float g[4];
            load4(a.gamma + col, g);
#pragma unroll
            for (int j = 0; j < 4; ++j) y[i][j] *= inv * g[j];
            if (a.store_yn) store4(yn + col, y[i]);   // element-type copy; the router keeps fp32
        }
        float lg[EMAX];
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            float p = 0.0f;
            if (e < a.n_exp) {
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    float w[4];
                    load4(Ws + static_cast<size_t>(e) * a.dim + i * 128 + lane * 4, w);
#pragma unroll
                    for (int j = 0; j < 4; ++j) p = fmaf(y[i][j], w[j], p);
                }
            }
            lg[e] = p;
        }
#pragma unroll
        for (int e = 0; e < EMAX; ++e) lg[e] = warp_sum(lg[e]);   // every lane holds every logit
        // top-k by (score desc, index asc), kept sorted in registers (lane-redundant)
        float bs[KMAX], bl[KMAX];
        int bi[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            bs[j] = -INFINITY;
            bl[j] = 0.0f;
            bi[j] = -1;
        }
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            if (e >= a.n_exp) break;
            float cs = lg[e] + (a.bias ? a.bias[e] : 0.0f), cl = lg[e];
            int ci = e;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < a.top_k && cs > bs[j]) {
                    const float ts = bs[j], tl = bl[j];
                    const int ti = bi[j];
                    bs[j] = cs; bl[j] = cl; bi[j] = ci;
                    cs = ts; cl = tl; ci = ti;
                }
            }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < a.top_k && bi[j] >= 0) mx = fmaxf(mx, bl[j]);
        float den = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < a.top_k && bi[j] >= 0) den += expf(bl[j] - mx);
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= a.top_k) break;
            int rr = 0;
            if (lane == j) {
                const int e = bi[j] < 0 ? 0 : bi[j];
                const float wv = bi[j] < 0 ? 0.0f : expf(bl[j] - mx) / den;
                const size_t o = static_cast<size_t>(row) * a.top_k + j;
                a.idx[o] = e;
                a.w[o] = wv;
                if (a.trace_idx) a.trace_idx[o] = e;
                if (a.trace_w) a.trace_w[o] = wv;
                const int pos = atomicAdd(a.counts + e, 1);     // histogram and row claim
                rr = e * a.cap + pos;
                if (a.row_token) {
                    a.row_token[rr] = row;
                    a.row_w[rr] = wv;
                }
            }
            if (a.xperm) {                                       // the expert's copy of yn
                rr = __shfl_sync(0xffffffffu, rr, j);
                T* dst = static_cast<T*>(a.xperm) + static_cast<size_t>(a.a_routed_base + rr) * a.dim;
#pragma unroll
                for (int i = 0; i < NV; ++i) store4(dst + i * 128 + lane * 4, y[i]);
            }
        }
    }
}

}  // namespace

bool router_fits_smem(bool bf, int n_exp, int top_k, int dim) {
    const bool width_ok = dim == 128 || dim == 1024 || dim == 2048;
    return width_ok && n_exp <= 64 && top_k <= 8 && static_cast<long>(n_exp) * dim * (bf ? 2 : 4) <= 64 * 1024;
}

namespace {

template <typename T, int NV, int EMAX, int KMAX>
rdt_status launch_router_smem_k(const RouterArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(a.n_exp) * a.dim * sizeof(T);
    const int rows_per_block = kRouterThreads / 32;
    const int grid = (a.ntok + rows_per_block - 1) / rows_per_block;
    auto k = norm2_router_smem_kernel<T, NV, EMAX, KMAX>;
    RDT_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024));
    RDT_CUDA_TRY(launch_pdl(k, dim3(grid), dim3(kRouterThreads), smem, st, a));
    return RDT_OK;
}

template <typename T, int NV, int EMAX>
rdt_status launch_router_smem_e(const RouterArgs& a, cudaStream_t st) {
    if (a.top_k <= 2) return launch_router_smem_k<T, NV, EMAX, 2>(a, st);
    return launch_router_smem_k<T, NV, EMAX, 8>(a, st);
}

template <typename T, int NV>
rdt_status launch_router_smem(const RouterArgs& a, cudaStream_t st) {
    if (a.n_exp <= 16) return launch_router_smem_e<T, NV, 16>(a, st);
    return launch_router_smem_e<T, NV, 64>(a, st);
}

}  // namespace

rdt_status norm2_router_smem(bool bf, const RouterArgs& a, cudaStream_t st) {
    if (!router_fits_smem(bf, a.n_exp, a.top_k, a.dim)) {
        set_error("router weight does not fit in shared memory");
        return RDT_ERR_UNSUPPORTED;
    }
    switch (a.dim / 128) {
        case 1: return bf ? launch_router_smem<bf16, 1>(a, st) : launch_router_smem<float, 1>(a, st);
        case 8: return bf ? launch_router_smem<bf16, 8>(a, st) : launch_router_smem<float, 8>(a, st);
        case 16: return bf ? launch_router_smem<bf16, 16>(a, st) : launch_router_smem<float, 16>(a, st);
        default: set_error("router: unsupported width"); return RDT_ERR_UNSUPPORTED;
    }
}


}  // namespace rdt
