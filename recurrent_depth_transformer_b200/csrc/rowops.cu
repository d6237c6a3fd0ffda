// Memory-bound row kernels of the recurrent block (one warp per token row, 16-byte
// vectorised, coalesced across the warp):
//   hoist          h <- h0 (fp32 state), Be <- B (.) e      (once per call)
//   norm1          x = h + e, xn = RMSNorm1(x)
//   norm2_router   yn = RMSNorm2(y) (fp32 in registers, stored in the element type for the
//                  experts), router logits yn W_r^T in fp32, top-k of logits + bias with
//                  ties to the lower expert index, softmax over the k chosen logits,
//                  per-expert histogram
//   moe_copy       the copy of each token's normalised row into the expert rows its
//                  router claimed (capacity layout), for routers that do not write them
//   moe_combine    deterministic mode: a token's expert-row outputs added in a fixed order
//   mla_latent_norm  RMSNorm of c_q and c_kv, RoPE of the decoupled key
//   act_step       ACT halting after a loop: halting probability of the new state,
//                  the halting decision, the weighted output sum, frozen halted states
// plus the weight-preparation matmul and a finite-value check.
#include <algorithm>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr int kRowThreads = 256;   // 8 rows (warps) per block

template <typename T>
__device__ __forceinline__ void store_t(T* p, float v) { *p = from_f<T>(v); }

// ----------------------------------------------------------------------------- hoist

template <typename T>
__global__ void hoist_kernel(const T* __restrict__ h0, const T* __restrict__ e, const float* __restrict__ Bd,
                             float* __restrict__ h, float* __restrict__ Be, size_t n4, int dim) {
    pdl_trigger();
    pdl_wait();
    // (restrict: the unrolled iterations' loads may be issued before the earlier stores)
#pragma unroll 4
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t off = i * 4;
        float a[4], b[4];
        load4(h0 + off, a);
        store4(h + off, a);
        if (Bd) {
            float bd[4];
            load4(e + off, b);
            load4(Bd + off % dim, bd);
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] *= bd[j];
            store4(Be + off, b);
        }
    }
}

// C[M,N] = A[M,K] B[N,K]^T, fp32 sums, 16x16 tiles (once-per-call dense B.e only).
template <typename T>
__global__ void matmul_nt_kernel(const T* A, const float* B, float* C, int M, int N, int K) {
    __shared__ float sa[16][17], sb[16][17];
    pdl_trigger();
    pdl_wait();
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int row = blockIdx.y * 16 + ty, col = blockIdx.x * 16 + tx;
    float acc = 0.0f;
    for (int k0 = 0; k0 < K; k0 += 16) {
        sa[ty][tx] = (row < M && k0 + tx < K) ? to_f(A[static_cast<size_t>(row) * K + k0 + tx]) : 0.0f;
        const int bn = blockIdx.x * 16 + ty;
        sb[ty][tx] = (bn < N && k0 + tx < K) ? B[static_cast<size_t>(bn) * K + k0 + tx] : 0.0f;
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(sa[ty][k], sb[tx][k], acc);
        __syncthreads();
    }
    if (row < M && col < N) C[static_cast<size_t>(row) * N + col] = acc;
}

// ----------------------------------------------------------------------------- norm1

// Wide rows are split over WR warps (each lane then holds PV = NV / WR vectors of 4): a row
// of 2048 elements held by one warp took 138 registers a thread, one block per SM, and the
// norms ran at a quarter of the HBM bandwidth. Warp w of a row takes the vectors
// (i WR + w) 128 + 4 lane, so each warp-wide access still covers one contiguous segment; the
// row's sum of squares is the WR warps' partial sums added in warp order.
template <int NV>
struct RowSplit {
    static constexpr int WR = NV >= 8 ? NV / 4 : 1;        // warps per row
    static constexpr int PV = NV / WR;                      // vectors of 4 per lane
    static constexpr int ROWS = (kRowThreads / 32) / WR;    // rows per block
    static_assert(WR * PV == NV && ROWS >= 1, "row split");
};

// Sum over the WR warps of a row (every thread of the block must call it: it synchronises
// the block when WR > 1).
template <int WR>
__device__ __forceinline__ float row_sum(float v, float* part) {
    v = warp_sum(v);
    if constexpr (WR > 1) {
        const int warp = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) part[warp] = v;
        __syncthreads();
        const int w0 = warp / WR * WR;
        v = 0.0f;
#pragma unroll
        for (int w = 0; w < WR; ++w) v += part[w0 + w];
    }
    return v;
}

template <typename T, int NV>
__global__ void __launch_bounds__(kRowThreads) norm1_kernel(const Norm1Args a) {
    using RS = RowSplit<NV>;
    constexpr int PV = RS::PV;
    __shared__ float part[kRowThreads / 32];
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x == 0 && a.zero_counts)
        for (int i = threadIdx.x; i < a.n_zero; i += blockDim.x) a.zero_counts[i] = 0;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * RS::ROWS + warp / RS::WR;
    const int wr = warp % RS::WR;
    const bool live = row < a.ntok;
    const size_t base = static_cast<size_t>(live ? row : 0) * a.dim;
    const T* e = static_cast<const T*>(a.e);
    float x[PV][4];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        const int col = (i * RS::WR + wr) * 128 + lane * 4;
        if (a.h && live) {
            load4(a.h + base + col, x[i]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) x[i][j] = 0.0f;
        }
    }
    if (e && live) {
#pragma unroll
        for (int i = 0; i < PV; ++i) {
            float ev[4];
            load4(e + base + (i * RS::WR + wr) * 128 + lane * 4, ev);
#pragma unroll
            for (int j = 0; j < 4; ++j) x[i][j] += ev[j];
        }
    }
#pragma unroll
    for (int i = 0; i < PV; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) ss = fmaf(x[i][j], x[i][j], ss);
    ss = row_sum<RS::WR>(ss, part);
    if (!live) return;
    const float inv = rsqrtf(ss / a.dim + a.eps);
    T* xn = static_cast<T*>(a.xn) + base;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        const int col = (i * RS::WR + wr) * 128 + lane * 4;
        float gi[4];
        load4(a.gamma + col, gi);
#pragma unroll
        for (int j = 0; j < 4; ++j) x[i][j] = to_f(from_f<T>(x[i][j] * inv * gi[j]));
        store4(xn + col, x[i]);
    }
}

// ----------------------------------------------------------------------------- norm2 + router

template <typename T, int NV, int ESLOT>
__global__ void __launch_bounds__(kRowThreads) norm2_router_kernel(const RouterArgs a) {
    const int row = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.ntok) return;
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
        store4(yn + col, y[i]);   // rounded copy for the experts; the router keeps fp32
    }
    if (a.halted && a.halted[row]) {              // ACT: a halted token is routed nowhere
        if (lane < a.top_k) {
            const size_t o = static_cast<size_t>(row) * a.top_k + lane;
            a.idx[o] = -1;
            a.w[o] = 0.0f;
            if (a.trace_idx) a.trace_idx[o] = -1;
            if (a.trace_w) a.trace_w[o] = 0.0f;
            if (a.row_token) a.slot_row[o] = -1;
        }
        return;
    }

    // logits: lane (e % 32) keeps expert e in slot e / 32
    const T* W = static_cast<const T*>(a.w_router);
    float lg[ESLOT];
#pragma unroll
    for (int s = 0; s < ESLOT; ++s) lg[s] = -INFINITY;
#pragma unroll 1
    for (int ex = 0; ex < a.n_exp; ++ex) {
        float p = 0.0f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            float w[4];
            load4(W + static_cast<size_t>(ex) * a.dim + i * 128 + lane * 4, w);
#pragma unroll
            for (int j = 0; j < 4; ++j) p = fmaf(y[i][j], w[j], p);
        }
        p = warp_sum(p);
#pragma unroll
        for (int s = 0; s < ESLOT; ++s)
            if (lane == (ex & 31) && s == (ex >> 5)) lg[s] = p;
    }
    float score[ESLOT];
    bool taken[ESLOT];
#pragma unroll
    for (int s = 0; s < ESLOT; ++s) {
        const int ex = s * 32 + lane;
        const float sc = ex < a.n_exp ? lg[s] + (a.bias ? a.bias[ex] : 0.0f) : -INFINITY;
        score[s] = isnan(sc) ? -INFINITY : sc;   // a NaN never wins; indices stay in range
        taken[s] = ex >= a.n_exp;
    }
    // top-k by (score desc, index asc)
    int sel_idx = -1;
    float sel_logit = 0.0f;
#pragma unroll 1
    for (int k = 0; k < a.top_k; ++k) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        float bl = 0.0f;
#pragma unroll
        for (int s = 0; s < ESLOT; ++s) {
            const int ex = s * 32 + lane;
            if (!taken[s] && (score[s] > bv || (score[s] == bv && ex < bi))) {
                bv = score[s];
                bi = ex;
                bl = lg[s];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
                bl = ol;
            }
        }
#pragma unroll
        for (int s = 0; s < ESLOT; ++s)
            if (s * 32 + lane == bi) taken[s] = true;
        if (lane == k) {
            sel_idx = min(max(bi, 0), a.n_exp - 1);
            sel_logit = bl;
        }
    }
    // softmax over the k selected logits (lanes 0..k-1 hold one each)
    const bool mine = lane < a.top_k;
    float mx = mine ? sel_logit : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float ex = mine ? expf(sel_logit - mx) : 0.0f;
    const float den = warp_sum(ex);
    if (mine) {
        const float wv = ex / den;
        const size_t o = static_cast<size_t>(row) * a.top_k + lane;
        a.idx[o] = sel_idx;
        a.w[o] = wv;
        if (a.trace_idx) a.trace_idx[o] = sel_idx;
        if (a.trace_w) a.trace_w[o] = wv;
        const int pos = atomicAdd(a.counts + sel_idx, 1);     // histogram and row claim
        if (a.row_token) {
            const int rr = sel_idx * a.cap + pos;
            a.row_token[rr] = row;
            a.row_w[rr] = wv;
            a.slot_row[o] = rr;
        }
    }
}

// ----------------------------------------------------------------------------- norm2 (hi/lo)

// hi = yn rounded to the element type (bf16; for fp32 the tf32 precision the tensor cores
// read), lo = the element-type value of yn - hi.
__device__ __forceinline__ void split_hi_lo(float v, bf16& hi, bf16& lo) {
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}
__device__ __forceinline__ void split_hi_lo(float v, float& hi, float& lo) {
    hi = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    lo = v - hi;
}

template <typename T, int NV>
__global__ void __launch_bounds__(kRowThreads) norm2_split_kernel(const Norm2Args a) {
    using RS = RowSplit<NV>;
    constexpr int PV = RS::PV;
    __shared__ float part[kRowThreads / 32];
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * RS::ROWS + warp / RS::WR;
    const int wr = warp % RS::WR;
    const bool live = row < a.ntok;
    const size_t base = static_cast<size_t>(live ? row : 0) * a.dim;
    float y[PV][4];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        if (live) {
            load4(a.y + base + (i * RS::WR + wr) * 128 + lane * 4, y[i]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) y[i][j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) ss = fmaf(y[i][j], y[i][j], ss);
    }
    ss = row_sum<RS::WR>(ss, part);
    if (!live) return;
    const float inv = rsqrtf(ss / a.dim + a.eps);
    if (a.zero_rows)
        for (int i = wr * 32 + lane; i < a.zero_width; i += RS::WR * 32)
            a.zero_rows[static_cast<size_t>(row) * a.zero_width + i] = 0.0f;
    T* yn = static_cast<T*>(a.yn) + base;
    T* lo = static_cast<T*>(a.yn_lo) + base;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        const int col = (i * RS::WR + wr) * 128 + lane * 4;
        float g[4], hv[4], lv[4];
        load4(a.gamma + col, g);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            T h, l;
            split_hi_lo(y[i][j] * inv * g[j], h, l);
            hv[j] = to_f(h);
            lv[j] = to_f(l);
        }
        store4(yn + col, hv);
        store4(lo + col, lv);
    }
}

// ----------------------------------------------------------------------------- MoE dispatch copy

// One warp per token: the normalised row yn[token] is read once (eight 16-byte vectors of the
// lane in flight) and stored into each row the router claimed for it (capacity layout). A
// warp per (token, slot) re-read the row k times from L2 and ran at ~4.6 TB/s of stores.
template <typename T>
__global__ void __launch_bounds__(kRowThreads) moe_copy_kernel(T* xperm, const int* slot_row, int ntok,
                                                               int top_k, int dim, int a_routed_base) {
    pdl_trigger();
    pdl_wait();
    const int n = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (n >= ntok) return;
    const uint4* src = reinterpret_cast<const uint4*>(xperm + static_cast<size_t>(n) * dim);
    const int nvec = dim * static_cast<int>(sizeof(T)) / 16;
    for (int i0 = lane; i0 < nvec; i0 += 8 * 32) {
        uint4 t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (i0 + 32 * u < nvec) t[u] = src[i0 + 32 * u];
#pragma unroll 1
        for (int s = 0; s < top_k; ++s) {
            const int sr = slot_row[static_cast<size_t>(n) * top_k + s];
            if (sr < 0) continue;                 // halted token: no row claimed
            uint4* dst = reinterpret_cast<uint4*>(xperm + static_cast<size_t>(a_routed_base + sr) * dim);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + 32 * u < nvec) dst[i0 + 32 * u] = t[u];
        }
    }
}

// ----------------------------------------------------------------------------- deterministic combine

// One warp per token: the token's expert outputs (each stored in its own row by the
// down-projection) are added into dst in a fixed order - shared experts first, then the
// routed slots 0 .. top_k - 1 - so that the fp32 sums do not depend on scheduling.
template <int NV>
__global__ void __launch_bounds__(kRowThreads) moe_combine_kernel(const float* rows, const int* slot_row,
                                                                  int ntok, int top_k, int n_shared, int cap,
                                                                  float* dst) {
    pdl_trigger();
    pdl_wait();
    const int n = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (n >= ntok) return;
    constexpr int dim = NV * 128;
    float acc[NV][4];
    float* d = dst + static_cast<size_t>(n) * dim;
#pragma unroll
    for (int i = 0; i < NV; ++i) load4(d + i * 128 + lane * 4, acc[i]);
    auto add_row = [&](size_t r) {
        const float* src = rows + r * dim;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            float v[4];
            load4(src + i * 128 + lane * 4, v);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] += v[j];
        }
    };
    for (int s = 0; s < n_shared; ++s) add_row(static_cast<size_t>(s) * cap + n);
    for (int j = 0; j < top_k; ++j) {
        const int r = slot_row[static_cast<size_t>(n) * top_k + j];
        if (r >= 0) add_row(static_cast<size_t>(n_shared) * cap + r);
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) store4(d + i * 128 + lane * 4, acc[i]);
}

// ----------------------------------------------------------------------------- MLA latents

template <typename T>
__global__ void __launch_bounds__(kRowThreads) mla_latent_norm_kernel(const MlaNormArgs a) {
    pdl_trigger();
    pdl_wait();
    const int row = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.ntok) return;
    const float* L = a.lat + static_cast<size_t>(row) * a.ld_lat;
    // c_q
    float ss = 0.0f;
    for (int i = lane; i < a.q_lat; i += 32) ss = fmaf(L[i], L[i], ss);
    ss = warp_sum(ss);
    float inv = rsqrtf(ss / a.q_lat + a.eps);
    T* cq = static_cast<T*>(a.cq) + static_cast<size_t>(row) * a.q_lat;
    for (int i = lane; i < a.q_lat; i += 32) store_t(cq + i, L[i] * inv * a.q_norm[i]);
    // c_kv
    const float* C = L + a.q_lat;
    ss = 0.0f;
    for (int i = lane; i < a.kv_lat; i += 32) ss = fmaf(C[i], C[i], ss);
    ss = warp_sum(ss);
    inv = rsqrtf(ss / a.kv_lat + a.eps);
    T* kv = static_cast<T*>(a.kv) + static_cast<size_t>(row) * (a.kv_lat + a.rope);
    for (int i = lane; i < a.kv_lat; i += 32) store_t(kv + i, C[i] * inv * a.kv_norm[i]);
    // decoupled RoPE key
    const float* R = C + a.kv_lat;
    const int half = a.rope / 2;
    const int pos = row % a.seq + (a.pos_dev ? *a.pos_dev : 0);
    for (int i = lane; i < half; i += 32) {
        const float c = a.rope_cos[i * a.rope_ld + pos], s = a.rope_sin[i * a.rope_ld + pos];
        const float x1 = R[i], x2 = R[i + half];
        store_t(kv + a.kv_lat + i, x1 * c - x2 * s);
        store_t(kv + a.kv_lat + half + i, x2 * c + x1 * s);
    }
}

// ----------------------------------------------------------------------------- weight prep / checks

template <typename T>
__global__ void prep_matmul_kernel(const T* A, long sam, long sak, const T* B, long sbk, long sbn,
                                   T* C, int ldc, int M, int N, int K, const T* add, int ld_add) {
    const int m = blockIdx.y * blockDim.y + threadIdx.y;
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M || n >= N) return;
    float acc = add ? to_f(add[static_cast<size_t>(m) * ld_add + n]) : 0.0f;
    for (int k = 0; k < K; ++k) acc = fmaf(to_f(A[m * sam + k * sak]), to_f(B[k * sbk + n * sbn]), acc);
    C[static_cast<size_t>(m) * ldc + n] = from_f<T>(acc);
}

// ----------------------------------------------------------------------------- ACT halting

// ACT (Dynamic Adaptive Computation Time) after loop t, one warp per token: a token halted
// before this loop copies its state forward; a running one takes its halting probability
// p = sigmoid(w . h_next + b) from the new state, halts once its summed p reaches the
// threshold (or at the last loop) with the remainder as weight, and adds its weighted state
// to the output. Reads and writes 2-3 fp32 rows per token: bound by HBM bandwidth.
template <int NV>
__global__ void __launch_bounds__(kRowThreads) act_step_kernel(const ActArgs a) {
    pdl_trigger();
    pdl_wait();
    const int row = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.ntok) return;
    const size_t base = static_cast<size_t>(row) * a.dim;
    if (a.t > 0 && a.loops[row] > 0) {            // halted earlier: the state stays put
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            float v[4];
            load4(a.h_cur + base + i * 128 + lane * 4, v);
            store4(a.h_next + base + i * 128 + lane * 4, v);
        }
        return;
    }
    float v[NV][4];
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        float w[4];
        load4(a.h_next + base + i * 128 + lane * 4, v[i]);
        load4(a.w_halt + i * 128 + lane * 4, w);
#pragma unroll
        for (int j = 0; j < 4; ++j) z = fmaf(v[i][j], w[j], z);
    }
    z = warp_sum(z) + a.b_halt;
    const float p = 1.0f / (1.0f + expf(-z));
    const float c = a.t > 0 ? a.cum[row] : 0.0f;
    const bool halt = a.last || c + p >= a.threshold;
    const float wgt = halt ? 1.0f - c : p;
    if (lane == 0) {
        a.cum[row] = c + p;
        a.loops[row] = halt ? a.t + 1 : 0;
    }
    float* out = a.out + base;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (a.t > 0) load4(out + i * 128 + lane * 4, o);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = fmaf(wgt, v[i][j], o[j]);
        store4(out + i * 128 + lane * 4, o);
    }
}

// 16-byte loads, four of a thread in flight (one 4-byte load at a time left it at a third of
// the HBM bandwidth); scalar loads for a misaligned start and the tail.
__global__ void check_finite_kernel(const float* __restrict__ x, size_t n, int* flags) {
    pdl_trigger();
    pdl_wait();
    bool bad = false;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t tid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    size_t tail = 0;
    if ((reinterpret_cast<uintptr_t>(x) & 15) == 0) {
        const float4* x4 = reinterpret_cast<const float4*>(x);
        const size_t n4 = n / 4;
#pragma unroll 4
        for (size_t i = tid; i < n4; i += stride) {
            const float4 v = x4[i];
            bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
        }
        tail = n4 * 4;
    }
    for (size_t i = tail + tid; i < n; i += stride) bad |= !isfinite(x[i]);
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicExch(flags + FLAG_NONFINITE, 1);
}

template <typename T, template <typename, int> class K, typename... Args>
rdt_status launch_rows(int nv, int rows, cudaStream_t st, Args... args) {
    const dim3 grid((rows + kRowThreads / 32 - 1) / (kRowThreads / 32));
    switch (nv) {
        case 1: K<T, 1>::run(grid, st, args...); break;
        case 2: K<T, 2>::run(grid, st, args...); break;
        case 4: K<T, 4>::run(grid, st, args...); break;
        case 8: K<T, 8>::run(grid, st, args...); break;
        case 16: K<T, 16>::run(grid, st, args...); break;
        case 32: K<T, 32>::run(grid, st, args...); break;
        default: set_error("row kernel: unsupported width"); return RDT_ERR_UNSUPPORTED;
    }
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

template <typename T, int NV>
struct Norm1L {
    static void run(dim3, cudaStream_t st, Norm1Args a) {
        const dim3 g((a.ntok + RowSplit<NV>::ROWS - 1) / RowSplit<NV>::ROWS);
        launch_pdl(norm1_kernel<T, NV>, g, dim3(kRowThreads), 0, st, a);
    }
};
template <typename T, int NV>
struct ActL {
    static void run(dim3 g, cudaStream_t st, ActArgs a) {
        launch_pdl(act_step_kernel<NV>, g, dim3(kRowThreads), 0, st, a);
    }
};
template <typename T, int NV>
struct CombineL {
    static void run(dim3 g, cudaStream_t st, const float* rows, const int* slot_row, int ntok, int top_k,
                    int n_shared, int cap, float* dst) {
        launch_pdl(moe_combine_kernel<NV>, g, dim3(kRowThreads), 0, st, rows, slot_row, ntok, top_k, n_shared,
                   cap, dst);
    }
};
template <typename T, int NV>
struct Norm2L {
    static void run(dim3, cudaStream_t st, Norm2Args a) {
        const dim3 g((a.ntok + RowSplit<NV>::ROWS - 1) / RowSplit<NV>::ROWS);
        launch_pdl(norm2_split_kernel<T, NV>, g, dim3(kRowThreads), 0, st, a);
    }
};
template <typename T, int NV>
struct RouterL {
    static void run(dim3 g, cudaStream_t st, RouterArgs a) {
        if (a.n_exp <= 32)
            norm2_router_kernel<T, NV, 1><<<g, kRowThreads, 0, st>>>(a);
        else if (a.n_exp <= 64)
            norm2_router_kernel<T, NV, 2><<<g, kRowThreads, 0, st>>>(a);
        else
            norm2_router_kernel<T, NV, 8><<<g, kRowThreads, 0, st>>>(a);
    }
};

}  // namespace

rdt_status hoist(bool bf, const void* h0, const void* e, const float* Bdiag, float* h, float* Be,
                 size_t n, int dim, cudaStream_t st) {
    const size_t n4 = n / 4;
    const int grid = static_cast<int>(std::min<size_t>((n4 + 255) / 256, 148 * 16));
    if (bf)
        RDT_CUDA_TRY(launch_pdl(hoist_kernel<bf16>, dim3(grid), dim3(256), 0, st, static_cast<const bf16*>(h0),
                                static_cast<const bf16*>(e), Bdiag, h, Be, n4, dim));
    else
        RDT_CUDA_TRY(launch_pdl(hoist_kernel<float>, dim3(grid), dim3(256), 0, st, static_cast<const float*>(h0),
                                static_cast<const float*>(e), Bdiag, h, Be, n4, dim));
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

rdt_status matmul_nt_simt(bool a_bf16, const void* A, const float* B, float* C, int M, int N,
                          int K, cudaStream_t st) {
    const dim3 blk(16, 16), grid((N + 15) / 16, (M + 15) / 16);
    if (a_bf16)
        RDT_CUDA_TRY(launch_pdl(matmul_nt_kernel<bf16>, grid, blk, 0, st, static_cast<const bf16*>(A), B, C, M, N, K));
    else
        RDT_CUDA_TRY(launch_pdl(matmul_nt_kernel<float>, grid, blk, 0, st, static_cast<const float*>(A), B, C, M, N, K));
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

rdt_status norm1(bool bf, const Norm1Args& a, cudaStream_t st) {
    const int nv = a.dim / 128;
    return bf ? launch_rows<bf16, Norm1L>(nv, a.ntok, st, a)
              : launch_rows<float, Norm1L>(nv, a.ntok, st, a);
}

rdt_status norm2_split(bool bf, const Norm2Args& a, cudaStream_t st) {
    const int nv = a.dim / 128;
    return bf ? launch_rows<bf16, Norm2L>(nv, a.ntok, st, a)
              : launch_rows<float, Norm2L>(nv, a.ntok, st, a);
}

rdt_status norm2_router(bool bf, const RouterArgs& a, cudaStream_t st) {
    const int nv = a.dim / 128;
    return bf ? launch_rows<bf16, RouterL>(nv, a.ntok, st, a)
              : launch_rows<float, RouterL>(nv, a.ntok, st, a);
}

rdt_status moe_copy(bool bf, void* xperm, const int* slot_row, int ntok, int top_k, int dim,
                    int a_routed_base, cudaStream_t st) {
    const dim3 grid((ntok + kRowThreads / 32 - 1) / (kRowThreads / 32));
    if (bf)
        RDT_CUDA_TRY(launch_pdl(moe_copy_kernel<bf16>, grid, dim3(kRowThreads), 0, st, static_cast<bf16*>(xperm),
                                slot_row, ntok, top_k, dim, a_routed_base));
    else
        RDT_CUDA_TRY(launch_pdl(moe_copy_kernel<float>, grid, dim3(kRowThreads), 0, st, static_cast<float*>(xperm),
                                slot_row, ntok, top_k, dim, a_routed_base));
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

rdt_status mla_latent_norm(bool bf, const MlaNormArgs& a, cudaStream_t st) {
    const dim3 grid((a.ntok + kRowThreads / 32 - 1) / (kRowThreads / 32));
    if (bf)
        RDT_CUDA_TRY(launch_pdl(mla_latent_norm_kernel<bf16>, grid, dim3(kRowThreads), 0, st, a));
    else
        RDT_CUDA_TRY(launch_pdl(mla_latent_norm_kernel<float>, grid, dim3(kRowThreads), 0, st, a));
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

rdt_status moe_combine(const float* rows, const int* slot_row, int ntok, int top_k, int n_shared, int cap,
                       float* dst, int dim, cudaStream_t st) {
    return launch_rows<float, CombineL>(dim / 128, ntok, st, rows, slot_row, ntok, top_k, n_shared, cap, dst);
}

rdt_status prep_matmul(bool bf, const void* A, long sam, long sak, const void* B, long sbk,
                       long sbn, void* C, int ldc, int M, int N, int K, cudaStream_t st, const void* add,
                       int ld_add) {
    const dim3 blk(32, 8), grid((N + 31) / 32, (M + 7) / 8);
    if (bf)
        prep_matmul_kernel<bf16><<<grid, blk, 0, st>>>(static_cast<const bf16*>(A), sam, sak,
                                                       static_cast<const bf16*>(B), sbk, sbn,
                                                       static_cast<bf16*>(C), ldc, M, N, K,
                                                       static_cast<const bf16*>(add), ld_add);
    else
        prep_matmul_kernel<float><<<grid, blk, 0, st>>>(static_cast<const float*>(A), sam, sak,
                                                        static_cast<const float*>(B), sbk, sbn,
                                                        static_cast<float*>(C), ldc, M, N, K,
                                                        static_cast<const float*>(add), ld_add);
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

rdt_status act_step(const ActArgs& a, cudaStream_t st) {
    if (a.dim % 128 != 0) {
        set_error("ACT step: dim must be a multiple of 128");
        return RDT_ERR_UNSUPPORTED;
    }
    return launch_rows<float, ActL>(a.dim / 128, a.ntok, st, a);
}

rdt_status check_finite(const float* x, size_t n, int* flags, cudaStream_t st) {
    const int grid = static_cast<int>(std::min<size_t>((n + 255) / 256, 148 * 8));
    RDT_CUDA_TRY(launch_pdl(check_finite_kernel, dim3(grid), dim3(256), 0, st, x, n, flags));
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

}  // namespace rdt
