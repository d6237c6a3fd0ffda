// RMSNorm2 fused with the MoE router for routers whose weight fits in shared memory:
// each block stages W_r (n_experts x dim) once, then every warp takes rows in turn:
// RMSNorm2 in fp32 (stored in the element type as the experts' input), the n_experts logits
// of the fp32 normalised row, top-k of logits + bias with ties to the lower expert index,
// softmax over the k chosen logits, per-expert histogram.
#include <algorithm>
#include <type_traits>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

// ----------------------------------------------------------------------------- norm2 + router (W_r in shared memory)

// For routers whose weight fits in shared memory: each block stages W_r once, then every warp
// takes rows in turn: RMSNorm2 (fp32, stored in the element type for the experts),
// the n_exp logits of the fp32 row against W_r, top-k of logits + bias (ties to the lower
// expert index), softmax over the k chosen logits, histogram, and the row's copies for the
// chosen experts.
//
// The work per row is a few hundred instructions, so the kernel is bound by instruction
// issue and latency, not bytes: each lane owns 4 * NV columns of the row, forms its partial
// logits with packed fp32 FMAs from shared loads of 4 weights, and the warp reduces the EMAX
// partials with a transposing butterfly (EMAX - 1 + 1 shuffles instead of 5 per logit) that
// leaves lane l holding whole logits (expert l / 2 for 16 experts, experts 2l, 2l + 1 for 64).
// Top-k is then k warp-wide argmax rounds over (score desc, index asc).
constexpr int kRouterMaxThreads = 256;

// Butterfly transpose-reduce of v[0..E) over the warp. On return v[0 .. max(E/32, 1)) hold
// full sums; router_expert() gives their expert indices.
template <int E>
__device__ __forceinline__ void transpose_reduce(float (&v)[E], int lane) {
    int n = E;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (n > 1) {
            const int half = n / 2;
            const bool up = (lane & off) != 0;
#pragma unroll
            for (int j = 0; j < E / 2; ++j) {
                if (j < half) {
                    const float send = up ? v[j] : v[j + half];
                    const float keep = up ? v[j + half] : v[j];
                    v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            n = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
        }
    }
}
// Expert index of v[j] after transpose_reduce<E>.
template <int E>
__device__ __forceinline__ int router_expert(int lane, int j) {
    int e = j, n = E;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (n > 1) {
            n /= 2;
            if (lane & off) e += n;
        }
    }
    return e;
}

// (score, index) order: higher score first, then lower index; invalid entries last.
__device__ __forceinline__ bool router_better(float s, int e, float so, int eo) {
    return s > so || (s == so && e < eo);
}

template <typename T, int NV, int EMAX, int KMAX>
__global__ void __launch_bounds__(kRouterMaxThreads, 2) norm2_router_smem_kernel(const RouterArgs a) {
    extern __shared__ __align__(16) uint8_t ws_raw[];   // W_r [n_exp][dim] in the element type
    const T* Ws = reinterpret_cast<const T*>(ws_raw);
    constexpr int NL = EMAX >= 32 ? EMAX / 32 : 1;  // logits held per lane after the reduce
    const int lane = threadIdx.x & 31;
    const int nthreads = blockDim.x;
    // W_r is copied as is (16-byte chunks) and converted where it is read: the copy is half
    // the size of an fp32 one, small enough for a block to sit beside the projection GEMM's
    // CTAs and stage it while they run
    auto stage = [&]() {
        const int n16 = a.n_exp * a.dim * static_cast<int>(sizeof(T)) / 16;
        const uint4* src = static_cast<const uint4*>(a.w_router);
        uint4* dst = reinterpret_cast<uint4*>(ws_raw);
        for (int i = threadIdx.x; i < n16; i += nthreads) dst[i] = src[i];
    };
    pdl_trigger();
    if (a.weights_static) stage();      // overlaps the tail of the previous kernel
    pdl_wait();
    if (!a.weights_static) stage();
    __syncthreads();
    const int warps_total = gridDim.x * (nthreads / 32);
    float bias_l[NL];
    int ex_l[NL];
#pragma unroll
    for (int j = 0; j < NL; ++j) {
        ex_l[j] = router_expert<EMAX>(lane, j);
        bias_l[j] = (a.bias && ex_l[j] < a.n_exp) ? a.bias[ex_l[j]] : 0.0f;
    }
    // gamma stays in registers when they allow it (128 per thread: two 256-thread blocks per SM)
    constexpr bool kHoistGamma = NV * 4 + EMAX <= 64;
    float g[kHoistGamma ? NV : 1][4];
    if constexpr (kHoistGamma) {
#pragma unroll
        for (int i = 0; i < NV; ++i) load4(a.gamma + i * 128 + lane * 4, g[i]);
    }
#pragma unroll 1
    for (int row = blockIdx.x * (nthreads / 32) + (threadIdx.x >> 5); row < a.ntok; row += warps_total) {
        const size_t base = static_cast<size_t>(row) * a.dim;
        float y[NV][4];
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < NV; ++i) load4(a.y + base + i * 128 + lane * 4, y[i]);
#pragma unroll
        for (int i = 0; i < NV; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) ss = fmaf(y[i][j], y[i][j], ss);
        ss = warp_sum(ss);
        const float inv = rsqrtf(ss / a.dim + a.eps);
        T* yn = static_cast<T*>(a.yn) + base;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            float gi[4];
            if constexpr (kHoistGamma) {
                gi[0] = g[i][0]; gi[1] = g[i][1]; gi[2] = g[i][2]; gi[3] = g[i][3];
            } else {
                load4(a.gamma + i * 128 + lane * 4, gi);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) y[i][j] *= inv * gi[j];
            if (a.store_yn) store4(yn + i * 128 + lane * 4, y[i]);   // element-type copy; logits use fp32
        }
        if (a.halted && a.halted[row]) {          // ACT: a halted token is routed nowhere
            if (lane < a.top_k) {
                const size_t o = static_cast<size_t>(row) * a.top_k + lane;
                a.idx[o] = -1;
                a.w[o] = 0.0f;
                if (a.trace_idx) a.trace_idx[o] = -1;
                if (a.trace_w) a.trace_w[o] = 0.0f;
                if (a.slot_row) a.slot_row[o] = -1;
            }
            continue;
        }
        float lg[EMAX];
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            float2 acc = make_float2(0.0f, 0.0f);
            if (e < a.n_exp) {
                const T* wrow = Ws + static_cast<size_t>(e) * a.dim + lane * 4;
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    float4 w;
                    if constexpr (std::is_same<T, bf16>::value) {
                        const uint2 u = *reinterpret_cast<const uint2*>(wrow + i * 128);
                        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
                        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
                        w = make_float4(lo.x, lo.y, hi.x, hi.y);
                    } else {
                        w = *reinterpret_cast<const float4*>(wrow + i * 128);
                    }
                    acc = __ffma2_rn(make_float2(y[i][0], y[i][1]), make_float2(w.x, w.y), acc);
                    acc = __ffma2_rn(make_float2(y[i][2], y[i][3]), make_float2(w.z, w.w), acc);
                }
            }
            lg[e] = acc.x + acc.y;
        }
        transpose_reduce<EMAX>(lg, lane);
        // this lane's candidates: score = logit + bias, NaN scores rank below every number
        float sc[NL];
        bool taken[NL];
#pragma unroll
        for (int j = 0; j < NL; ++j) {
            const float s = lg[j] + bias_l[j];
            sc[j] = (ex_l[j] < a.n_exp && !isnan(s)) ? s : -INFINITY;
            taken[j] = ex_l[j] >= a.n_exp;
        }
        int ci[KMAX];
        float cl[KMAX];
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
            if (r >= a.top_k) break;
            // lane-local best untaken candidate, then the warp's best
            float bs = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < NL; ++j)
                if (!taken[j] && router_better(sc[j], ex_l[j], bs, be)) {
                    bs = sc[j];
                    be = ex_l[j];
                }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const float os = __shfl_xor_sync(0xffffffffu, bs, off);
                const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                if (router_better(os, oe, bs, be)) {
                    bs = os;
                    be = oe;
                }
            }
            if (be >= a.n_exp) be = 0;                 // only if every expert was taken (k > E)
            float l = 0.0f;
#pragma unroll
            for (int j = 0; j < NL; ++j)
                if (ex_l[j] == be) {
                    taken[j] = true;
                    l = lg[j];
                }
            // the logit of the winner from a lane that holds it
            const int owner = EMAX >= 32 ? be / NL : 2 * be;
            ci[r] = be;
            cl[r] = __shfl_sync(0xffffffffu, l, owner & 31);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int r = 0; r < KMAX; ++r)
            if (r < a.top_k) mx = fmaxf(mx, cl[r]);
        float den = 0.0f;
#pragma unroll
        for (int r = 0; r < KMAX; ++r)
            if (r < a.top_k) den += expf(cl[r] - mx);
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
            if (r >= a.top_k) break;
            int rr = 0;
            if (lane == r) {
                const int e = ci[r];
                const float wv = expf(cl[r] - mx) / den;
                const size_t o = static_cast<size_t>(row) * a.top_k + r;
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
                if (a.slot_row) a.slot_row[o] = rr;
            }
            if (a.xperm) {                                       // the expert's copy of yn
                rr = __shfl_sync(0xffffffffu, rr, r);
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

// Blocks of 8 warps, one row per warp: small enough (W_r copy <= 64 KB, 256 threads of at most
// 128 registers) to run beside a GEMM CTA, so that blocks stage W_r while the previous kernel
// runs (programmatic dependent launch) and the next kernel's prologue can start beside them.
template <typename T, int NV, int EMAX, int KMAX>
rdt_status launch_router_smem_k(const RouterArgs& a, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(a.n_exp) * a.dim * sizeof(T);
    const int warps = kRouterMaxThreads / 32;
    const int grid = (a.ntok + warps - 1) / warps;
    auto k = norm2_router_smem_kernel<T, NV, EMAX, KMAX>;
    RDT_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024));
    RDT_CUDA_TRY(launch_pdl(k, dim3(grid), dim3(warps * 32), smem, st, a));
    return RDT_OK;
}

template <typename T, int NV, int EMAX>
rdt_status launch_router_smem_e(const RouterArgs& a, cudaStream_t st) {
    if (a.top_k <= 2) return launch_router_smem_k<T, NV, EMAX, 2>(a, st);
    return launch_router_smem_k<T, NV, EMAX, 8>(a, st);
}

// Only the expert-count classes that router_fits_smem admits at this width are built.
template <typename T, int NV>
rdt_status launch_router_smem(const RouterArgs& a, cudaStream_t st) {
    constexpr long kRow = 128L * NV * static_cast<long>(sizeof(T));   // bytes of one W_r row
    if (a.n_exp <= 16) return launch_router_smem_e<T, NV, 16>(a, st);
    if constexpr (17 * kRow <= 64 * 1024) {
        if (a.n_exp <= 32) return launch_router_smem_e<T, NV, 32>(a, st);
    }
    if constexpr (33 * kRow <= 64 * 1024) {
        if (a.n_exp <= 64) return launch_router_smem_e<T, NV, 64>(a, st);
    }
    set_error("router: expert count does not fit the shared-memory router");
    return RDT_ERR_UNSUPPORTED;
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
