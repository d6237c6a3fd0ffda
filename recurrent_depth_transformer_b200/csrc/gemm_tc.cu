// Dense and grouped GEMM on the sm_100a 5th-generation tensor cores, C = A * B^T.
//
// One CTA computes one 128 x BN output tile:
//   warp 0      one thread issues TMA loads of 128-byte-wide K slices of A and B into a
//               ring of shared-memory stages (128-byte swizzle, K-major);
//   warp 1      allocates the TMEM accumulator; one thread issues tcgen05.mma (M = 128,
//               N = BN, K = 16 bf16 / 8 tf32 per instruction) and frees each stage with
//               tcgen05.commit when its MMAs have read it;
//   warps 2-5   the epilogue: each warp reads its 32-lane quadrant of TMEM (one output row
//               per thread) and applies one of the fused epilogues below.
//
// The fused epilogues are where the block's element-wise work lives:
//   EPI_ROPE        Q/K/V projection + rotary embedding on the rotated heads;
//   EPI_OPROJ_LOOP  output projection fused with the residual (y = x + a) and the
//                   recurrent update h_next = A (.) h + B.e + a (the MoE adds f later);
//   EPI_SWIGLU      expert up-projection (gate and up rows interleaved per tile) -> silu(g)*u;
//   EPI_SCATTER     expert down-projection, gate weight, and reduction into h_next
//                   (h_{t+1} = A h + B e + a + sum_j w_j E_j(yn)).
// Grouped mode decodes its tiles from the per-expert row counters on the device (capacity
// layout: expert e's rows start at e * tokens), so the counts never travel to the host.
#include <algorithm>
#include <type_traits>

#include "rdt_internal.cuh"

namespace rdt {

namespace {

constexpr int BM = 128;
constexpr int kThreads = 192;

template <int BN>
struct TcCfg {
    static constexpr int STAGES = (BN <= 64) ? 8 : (BN <= 128) ? 6 : 4;
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // two accumulators of BN fp32 columns, rounded up to a power of two
    static constexpr int TMEM_COLS = 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
    // [stages][barriers][group tables]: all dynamic, so that the kernel (with the 1 KB the
    // driver reserves per CTA) stays within the 196 KB shared-memory carveout and keeps
    // 60 KB of L1 for the epilogue's loads
    static constexpr int BAR_BYTES = 192;
    static constexpr int GROUP_BYTES = 2064;
    static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + GROUP_BYTES;
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte alignment of stages");
};

__device__ __forceinline__ void ld_chunk(uint32_t taddr, int c, float (&v)[32]) {
    uint32_t r[32];
    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <typename OutT>
__device__ __forceinline__ void store_row32(OutT* p, const float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float t[4] = {v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]};
        store4(p + 4 * j, t);
    }
}

// ----------------------------------------------------------------------------- epilogues

// Router top-k: keep the KMAX best (score = logit + bias) in registers, visiting experts in
// ascending index so that strict comparisons leave ties to the lower index; gate weights
// are the softmax of the chosen logits.
template <int KMAX>
struct TopK {
    float bs[KMAX], bl[KMAX];
    int bi[KMAX];
    __device__ __forceinline__ TopK() {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            bs[j] = -INFINITY;
            bl[j] = 0.0f;
            bi[j] = -1;
        }
    }
    __device__ __forceinline__ void insert(float logit, float bias, int ex, int k) {
        float cs = logit + bias, cl = logit;
        int ci = ex;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < k && cs > bs[j]) {
                const float ts = bs[j], tl = bl[j];
                const int ti = bi[j];
                bs[j] = cs; bl[j] = cl; bi[j] = ci;
                cs = ts; cl = tl; ci = ti;
            }
        }
    }
    __device__ __forceinline__ void write(const EpiParams& p, int row) const {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < p.top_k && bi[j] >= 0) mx = fmaxf(mx, bl[j]);
        float ex[KMAX], den = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            ex[j] = (j < p.top_k && bi[j] >= 0) ? expf(bl[j] - mx) : 0.0f;
            den += ex[j];
        }
        const size_t o = static_cast<size_t>(row) * p.top_k;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= p.top_k) break;
            const int e = bi[j] < 0 ? 0 : bi[j];      // only when every score was NaN
            const float w = den > 0.0f ? ex[j] / den : 0.0f;
            p.idx_out[o + j] = e;
            p.w_out[o + j] = w;
            if (p.trace_idx) p.trace_idx[o + j] = e;
            if (p.trace_w) p.trace_w[o + j] = w;
            const int pos = atomicAdd(p.counts + e, 1);          // histogram and row claim
            if (p.route_token) {
                const int rr = e * p.cap + pos;
                p.route_token[rr] = row;
                p.route_w[rr] = w;
                p.slot_row[o + j] = rr;
            }
        }
    }
};

// Router epilogue. Unsplit: the thread's row holds all logits (BN >= n_exp) in TMEM.
// Split over K: every CTA adds its partial logits into p.logits; the CTA that arrives last
// on the row tile's counter (threadfence-reduction order: adds, fence, count) reads the
// complete rows back and selects.
template <int BN, int KMAX>
__device__ __forceinline__ void epilogue_topk(const EpiParams& p, uint32_t taddr, bool valid, int crow,
                                              int split, int mtile) {
    if (split <= 1) {
        TopK<KMAX> tk;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            ld_chunk(taddr, c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int ex = c * 32 + i;
                if (ex < p.n_exp) tk.insert(v[i], p.bias ? p.bias[ex] : 0.0f, ex, p.top_k);
            }
        }
        if (valid) tk.write(p, crow);
        return;
    }
    __shared__ int s_last;
    float* lrow = p.logits + static_cast<size_t>(crow) * p.n_exp;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        ld_chunk(taddr, c, v);
        if (!valid) continue;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int ex = c * 32 + i;
            if (ex < p.n_exp) atomicAdd(lrow + ex, v[i]);
        }
    }
    __threadfence();
    asm volatile("bar.sync 1, 128;" ::: "memory");     // the four epilogue warps
    if (threadIdx.x == 64) {
        const int old = atomicAdd(p.tile_count + mtile, 1);
        s_last = old == split - 1;
        if (s_last) p.tile_count[mtile] = 0;             // ready for the next launch
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!s_last) return;
    __threadfence();
    if (!valid) return;
    TopK<KMAX> tk;
#pragma unroll 1
    for (int ex = 0; ex < p.n_exp; ++ex)
        tk.insert(__ldcg(lrow + ex), p.bias ? p.bias[ex] : 0.0f, ex, p.top_k);
    tk.write(p, crow);
}

template <typename T, int BN, int KIND>
__device__ __forceinline__ void epilogue(const EpiParams& p, uint32_t taddr, bool valid, int crow,
                                         int n0, int split = 1, int mtile = 0) {
    if constexpr (KIND == EPI_STORE || KIND == EPI_STORE_F32 || KIND == EPI_OPROJ_PLAIN) {
        using OutT = std::conditional_t<KIND == EPI_STORE, T, float>;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            ld_chunk(taddr, c, v);
            const int col = n0 + c * 32;
            if (valid && col < p.ncols_valid)
                store_row32(static_cast<OutT*>(p.out) + static_cast<size_t>(crow) * p.ldo + col, v);
        }
    } else if constexpr (KIND == EPI_ROPE) {
        // Heads of width head_w tile the BN columns exactly (host checks BN % head_w == 0).
        // The angle tables are [rot/2][seq]: for a fixed frequency the lanes (consecutive
        // positions) read consecutive floats. One position per row: load its angles once.
        const int pos = crow % p.seq;
        const int hw_chunks = p.head_w / 32;
        const int rc0 = p.rot_off / 32;
        const int rch = p.rot_dim / 32;
        const int half = p.rot_dim / 2;
        float cs[32], sn[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            cs[i] = i < half ? p.rope_cos[static_cast<size_t>(i) * p.seq + pos] : 0.0f;
            sn[i] = i < half ? p.rope_sin[static_cast<size_t>(i) * p.seq + pos] : 0.0f;
        }
        T* out = static_cast<T*>(p.out) + static_cast<size_t>(crow) * p.ldo;
#pragma unroll 1
        for (int hc = 0; hc < BN / 32; hc += hw_chunks) {
            const int head_col0 = n0 + hc * 32;
            const bool rotate = head_col0 < p.rope_limit;
#pragma unroll 1
            for (int c = 0; c < hw_chunks; ++c) {
                const int col = head_col0 + c * 32;
                if (rotate && c == rc0) {
                    if (rch == 2) {
                        float v0[32], v1[32];
                        ld_chunk(taddr, hc + c, v0);
                        ld_chunk(taddr, hc + c + 1, v1);
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float x1 = v0[i], x2 = v1[i];
                            v0[i] = x1 * cs[i] - x2 * sn[i];
                            v1[i] = x2 * cs[i] + x1 * sn[i];
                        }
                        if (valid && col < p.ncols_valid) {
                            store_row32(out + col, v0);
                            store_row32(out + col + 32, v1);
                        }
                        c += 1;
                    } else {
                        float v[32];
                        ld_chunk(taddr, hc + c, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float x1 = v[i], x2 = v[i + 16];
                            v[i] = x1 * cs[i] - x2 * sn[i];
                            v[i + 16] = x2 * cs[i] + x1 * sn[i];
                        }
                        if (valid && col < p.ncols_valid) store_row32(out + col, v);
                    }
                } else {
                    float v[32];
                    ld_chunk(taddr, hc + c, v);
                    if (valid && col < p.ncols_valid) store_row32(out + col, v);
                }
            }
        }
    } else if constexpr (KIND == EPI_OPROJ_LOOP) {
        // All loads of a 32-column chunk are issued before any store (the stores could alias
        // them as far as the compiler knows, which would serialise every load behind them).
        const size_t rbase = static_cast<size_t>(crow) * p.ld;
        const T* e = static_cast<const T*>(p.e);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            ld_chunk(taddr, c, v);
            const int col = n0 + c * 32;
            if (!valid || col >= p.ncols_valid) continue;
            float hh[32], be[32], aa[32], ee[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const size_t off = rbase + col + 4 * j;
                float t[4];
                load4(p.h + off, t);
                hh[4 * j] = t[0]; hh[4 * j + 1] = t[1]; hh[4 * j + 2] = t[2]; hh[4 * j + 3] = t[3];
                load4(p.Be + off, t);
                be[4 * j] = t[0]; be[4 * j + 1] = t[1]; be[4 * j + 2] = t[2]; be[4 * j + 3] = t[3];
                load4(p.Adiag + col + 4 * j, t);
                aa[4 * j] = t[0]; aa[4 * j + 1] = t[1]; aa[4 * j + 2] = t[2]; aa[4 * j + 3] = t[3];
                if (e) {
                    load4(e + off, t);
                } else {
                    t[0] = t[1] = t[2] = t[3] = 0.0f;
                }
                ee[4 * j] = t[0]; ee[4 * j + 1] = t[1]; ee[4 * j + 2] = t[2]; ee[4 * j + 3] = t[3];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const size_t off = rbase + col + 4 * j;
                float yv[4], hn[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int q = 4 * j + i;
                    const float a = v[q];
                    yv[i] = hh[q] + ee[q] + a;
                    hn[i] = aa[q] * hh[q] + be[q] + a;
                }
                store4(p.y + off, yv);
                store4(p.h_next + off, hn);
            }
        }
    } else if constexpr (KIND == EPI_SWIGLU) {
        // Tile columns [0, BN/2) are gate rows (W1), [BN/2, BN) the matching up rows (W3).
        T* out = static_cast<T*>(p.out) + static_cast<size_t>(crow) * p.ldo + n0 / 2;
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
            float g[32], u[32];
            ld_chunk(taddr, c, g);
            ld_chunk(taddr, c + BN / 64, u);
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = g[i] / (1.0f + expf(-g[i])) * u[i];
            if (valid) store_row32(out + c * 32, g);
        }
    } else if constexpr (KIND == EPI_SCATTER) {
        int token = -1;
        float w = 0.0f;
        if (valid) {
            if (crow < p.shared_rows) {
                token = crow % p.ntok;
                w = 1.0f;
            } else {
                token = p.row_token[crow - p.shared_rows];
                w = p.row_w[crow - p.shared_rows];
            }
        }
        float* dst = p.dst + static_cast<size_t>(token < 0 ? 0 : token) * p.ld;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            ld_chunk(taddr, c, v);
            const int col = n0 + c * 32;
            if (token < 0 || col >= p.ncols_valid) continue;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float4 add = make_float4(w * v[4 * j], w * v[4 * j + 1], w * v[4 * j + 2],
                                         w * v[4 * j + 3]);
                atomicAdd(reinterpret_cast<float4*>(dst + col + 4 * j), add);
            }
        }
    } else if constexpr (KIND == EPI_TOPK) {
        if (p.top_k <= 2)
            epilogue_topk<BN, 2>(p, taddr, valid, crow, split, mtile);
        else if (p.top_k <= 4)
            epilogue_topk<BN, 4>(p, taddr, valid, crow, split, mtile);
        else if (p.top_k <= 8)
            epilogue_topk<BN, 8>(p, taddr, valid, crow, split, mtile);
        else
            epilogue_topk<BN, 16>(p, taddr, valid, crow, split, mtile);
    }
}

// ----------------------------------------------------------------------------- the kernel

struct TileCoord {
    int a_row0, c_row0, nrows, group, n0, mt, kb0, kb1;
};

// Grouped mode: s_pref[g] = first 128-row tile of group g (routed groups, then shared ones),
// s_pref[256] = tile count; s_cnt[g] = rows of group g.
struct GroupTables {
    int pref[257];
    int cnt[256];
};

__device__ __forceinline__ void build_group_tables(const GemmArgs& args, GroupTables& t, int lane) {
    const int G = args.n_routed + args.n_shared;
    int tiles[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int g = lane * 8 + i;
        const int c = g < args.n_routed ? args.counts[g] : (g < G ? args.M : 0);   // shared: all tokens
        t.cnt[g] = c;
        tiles[i] = (c + BM - 1) / BM;
        sum += tiles[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        t.pref[lane * 8 + i] = run;
        run += tiles[i];
    }
    if (lane == 31) t.pref[256] = incl;
}

// tile = (mt * n_ntiles + nt) * split + ks; split > 1 divides the K blocks evenly
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& args, const GroupTables* gt, int tile,
                                                int n_ntiles, int bn, int split, int num_kb) {
    TileCoord t;
    const int ks = tile % split;
    tile /= split;
    const int mt = tile / n_ntiles;
    t.mt = mt;
    t.n0 = (tile - mt * n_ntiles) * bn;
    const int per = (num_kb + split - 1) / split;
    t.kb0 = ks * per;
    t.kb1 = min(num_kb, t.kb0 + per);
    if (gt != nullptr) {
        const int G = args.n_routed + args.n_shared;
        int lo = 0, hi = G - 1;                      // last group whose first tile <= mt
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (gt->pref[mid] <= mt) lo = mid; else hi = mid - 1;
        }
        const int local = (mt - gt->pref[lo]) * BM;
        t.group = lo;
        t.nrows = min(BM, gt->cnt[lo] - local);
        if (lo < args.n_routed) {
            t.a_row0 = args.a_routed_base + lo * args.cap + local;
            t.c_row0 = (args.n_shared + lo) * args.cap + local;
        } else {
            t.a_row0 = local;
            t.c_row0 = (lo - args.n_routed) * args.cap + local;
        }
        if (args.a_from_c) t.a_row0 = t.c_row0;
    } else {
        t.group = 0;
        t.a_row0 = mt * BM;
        t.c_row0 = t.a_row0;
        t.nrows = min(BM, args.M - t.a_row0);
    }
    return t;
}

// Persistent: each CTA walks tiles blockIdx.x, blockIdx.x + gridDim.x, ... The TMA warp
// and the MMA warp run ahead through a ring of shared-memory stages; the accumulator is
// double-buffered in TMEM so the epilogue of one tile overlaps the MMAs of the next.
template <typename T, int BN, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                   const __grid_constant__ CUtensorMap tA2, const __grid_constant__ CUtensorMap tB2,
                   const GemmArgs args, const EpiParams epi) {
    using C = TcCfg<BN>;
    constexpr bool kBf16 = std::is_same<T, bf16>::value;
    constexpr int kElemsPerRow = 128 / static_cast<int>(sizeof(T));   // K elements per stage

    // The dynamic shared memory of a CTA without static shared memory starts 1024-aligned,
    // as the 128-byte swizzle atoms need; checked below rather than padded for.
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;      // accumulator b ready for the epilogue
    uint64_t* tempty = tfull + 2;             // accumulator b drained by the epilogue
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    GroupTables& s_groups = *reinterpret_cast<GroupTables*>(smem + C::STAGES * C::STAGE_BYTES + C::BAR_BYTES);
    static_assert(2 * C::STAGES * 8 + 4 * 8 + 4 <= C::BAR_BYTES, "barrier area");
    static_assert(sizeof(GroupTables) <= C::GROUP_BYTES, "group tables");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (smem_u32(smem) & 1023) {              // uniform per CTA: misaligned base, do nothing
        if (threadIdx.x == 0 && epi.flags) atomicExch(epi.flags + FLAG_TIMEOUT, 1);
        return;
    }

    if (threadIdx.x == 0) {
#pragma unroll 1
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);         // one arrival per epilogue warp
        }
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tA);
        tma_prefetch_desc(&tB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();
    pdl_wait();

    const GroupTables* gt = nullptr;
    if (args.counts != nullptr) {          // grouped: per-group tile offsets from the counters
        if (warp == 0) build_group_tables(args, s_groups, lane);
        __syncthreads();
        gt = &s_groups;
    }
    const int n_ntiles = (args.N + BN - 1) / BN;
    const int n_mtiles = gt != nullptr ? gt->pref[256] : (args.M + BM - 1) / BM;
    const int split = args.split_k > 1 ? args.split_k : 1;
    const int total = n_mtiles * n_ntiles * split;
    const int num_kb = args.kb_main + args.kb_ext;

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
#pragma unroll 1
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileCoord tc = tile_coord(args, gt, tile, n_ntiles, BN, split, num_kb);
                const int b_row0 = tc.group * args.N + tc.n0;
#pragma unroll 1
                for (int kb = tc.kb0; kb < tc.kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, epi.flags)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                    if (kb < args.kb_main) {
                        tma_load_2d(sa, &tA, &full[s], kb * kElemsPerRow, tc.a_row0);
                        tma_load_2d(sb, &tB, &full[s], kb * kElemsPerRow, b_row0);
                    } else {
                        const int kx = (kb - args.kb_main) * kElemsPerRow;
                        tma_load_2d(sa, &tA2, &full[s], kx, tc.a_row0);
                        tma_load_2d(sb, &tB2, &full[s], kx, args.b2_row0 + b_row0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(kBf16 ? 1 : 2, BM, BN);
            int it = 0, local = 0;
            bool ok = true;
#pragma unroll 1
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++local) {
                const int b = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1);
                if (!mbar_wait(&tempty[b], (use & 1) ^ 1, epi.flags)) break;
                tc_fence_after();
                const uint32_t dt = tmem + static_cast<uint32_t>(b * BN);
                const TileCoord tc = tile_coord(args, gt, tile, n_ntiles, BN, split, num_kb);
#pragma unroll 1
                for (int kb = tc.kb0; kb < tc.kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1;
                    if (!mbar_wait(&full[s], ph, epi.flags)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint64_t da = sw128_kmajor_desc(sa);
                    const uint64_t db = sw128_kmajor_desc(sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // each MMA consumes 32 bytes of K: advance the start address by 32 B (>> 4 = 2)
                        if constexpr (kBf16)
                            tc_mma_bf16(dt, da + 2 * k, db + 2 * k, idesc, (kb > tc.kb0) || k);
                        else
                            tc_mma_tf32(dt, da + 2 * k, db + 2 * k, idesc, (kb > tc.kb0) || k);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(&tfull[b]);
            }
        }
    } else {
        const int q = warp & 3;            // TMEM lane quadrant accessible to this warp
        const int r = q * 32 + lane;       // row inside the tile
        int local = 0;
#pragma unroll 1
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
            const int b = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1);
            if (!mbar_wait(&tfull[b], use & 1, epi.flags)) break;
            tc_fence_after();
            const TileCoord tc = tile_coord(args, gt, tile, n_ntiles, BN, split, num_kb);
            epilogue<T, BN, KIND>(epi, tmem + (static_cast<uint32_t>(q * 32) << 16) + b * BN,
                                  r < tc.nrows, tc.c_row0 + r, tc.n0, split, tc.mt);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <typename T, int BN, int KIND>
rdt_status launch(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                  const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                  cudaStream_t st) {
    using C = TcCfg<BN>;
    auto kern = gemm_tc_kernel<T, BN, KIND>;
    static bool configured = false;
    if (!configured) {
        RDT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          C::SMEM));
        configured = true;
    }
    const int n_ntiles = (args.N + BN - 1) / BN;
    const long mt = args.counts ? args.max_tiles : (args.M + BM - 1) / BM;
    const long total = mt * n_ntiles * (args.split_k > 1 ? args.split_k : 1);
    if (total <= 0) return RDT_OK;
    const int grid = static_cast<int>(std::min<long>(total, num_sms()));
    RDT_CUDA_TRY(launch_pdl(kern, dim3(grid), dim3(kThreads), C::SMEM, st, tA, tB, tA2 ? *tA2 : tA,
                            tB2 ? *tB2 : tB, args, epi));
    return RDT_OK;
}

template <typename T, int BN>
rdt_status dispatch_kind(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                         const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                         cudaStream_t st) {
    switch (epi.kind) {
        case EPI_STORE: return launch<T, BN, EPI_STORE>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_STORE_F32: return launch<T, BN, EPI_STORE_F32>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_ROPE: return launch<T, BN, EPI_ROPE>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_OPROJ_LOOP: return launch<T, BN, EPI_OPROJ_LOOP>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_OPROJ_PLAIN: return launch<T, BN, EPI_OPROJ_PLAIN>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_SWIGLU: return launch<T, BN, EPI_SWIGLU>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_SCATTER: return launch<T, BN, EPI_SCATTER>(tA, tB, tA2, tB2, args, epi, st);
        default: set_error("gemm_tc: unknown epilogue"); return RDT_ERR_INVALID_ARG;
    }
}

template <typename T, int BN>
rdt_status dispatch_router(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                           const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                           cudaStream_t st) {
    return launch<T, BN, EPI_TOPK>(tA, tB, tA2, tB2, args, epi, st);
}

}  // namespace

rdt_status gemm_tc(bool bf16_elems, int bn, const CUtensorMap& tA, const CUtensorMap& tB,
                   const CUtensorMap* tA2, const CUtensorMap* tB2, const GemmArgs& args,
                   const EpiParams& epi, cudaStream_t st) {
    if (epi.kind == EPI_TOPK) {
        if (bf16_elems) {
            if (bn == 64) return dispatch_router<bf16, 64>(tA, tB, tA2, tB2, args, epi, st);
            if (bn == 128) return dispatch_router<bf16, 128>(tA, tB, tA2, tB2, args, epi, st);
            if (bn == 256) return dispatch_router<bf16, 256>(tA, tB, tA2, tB2, args, epi, st);
        } else {
            if (bn == 64) return dispatch_router<float, 64>(tA, tB, tA2, tB2, args, epi, st);
        }
        set_error("router: unsupported expert count");
        return RDT_ERR_UNSUPPORTED;
    }
    if (bf16_elems) {
        if (bn == 128) return dispatch_kind<bf16, 128>(tA, tB, tA2, tB2, args, epi, st);
        if (bn == 160) return dispatch_kind<bf16, 160>(tA, tB, tA2, tB2, args, epi, st);
        if (bn == 256) return dispatch_kind<bf16, 256>(tA, tB, tA2, tB2, args, epi, st);
    } else {
        if (bn == 128) return dispatch_kind<float, 128>(tA, tB, tA2, tB2, args, epi, st);
    }
    set_error("gemm_tc: unsupported tile width");
    return RDT_ERR_UNSUPPORTED;
}

int num_sms() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

// ----------------------------------------------------------------------------- tensor maps

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}
}  // namespace

rdt_status make_tmap_2d(CUtensorMap* map, const void* base, bool bf16_elems, uint64_t inner,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                        uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        set_error("cuTensorMapEncodeTiled entry point unavailable");
        return RDT_ERR_CUDA;
    }
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_stride_bytes & 15)) {
        set_error("tensor map: base or row stride not 16-byte aligned");
        return RDT_ERR_MISALIGNED;
    }
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, bf16_elems ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed with code " + std::to_string(static_cast<int>(r)));
        return RDT_ERR_CUDA;
    }
    return RDT_OK;
}

}  // namespace rdt
