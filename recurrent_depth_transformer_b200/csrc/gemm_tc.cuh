// Dense and grouped GEMM on the sm_100a 5th-generation tensor cores, C = A * B^T.
//
// Kernel template shared by the single-CTA and the CTA-pair instantiations. A single CTA
// computes 128 x BN output tiles; a CTA pair (cluster of two, cta_group::2) computes
// 256 x BN tiles, each CTA loading its 128 rows of A and half of the tile's B rows, the even
// CTA issuing the M = 256 MMAs that read both halves, each CTA holding its 128 accumulator
// rows in its own TMEM. The pair loads half as many bytes per multiply-add as one CTA,
// which is what bounds these GEMMs (per-SM ingest from L2), not the tensor pipe.
//
// Roles inside a CTA:
//   warp 0      one thread issues TMA loads of 128-byte-wide K slices of A and B into a
//               ring of shared-memory stages (128-byte swizzle, K-major);
//   warp 1      allocates the TMEM accumulator; one thread issues tcgen05.mma (M = 128,
//               N = BN, K = 16 bf16 / 8 tf32 per instruction) and frees each stage with
//               tcgen05.commit when its MMAs have read it;
//   warps 2-9   the epilogue (warps 2-5 for the router's top-k): each warp reads its 32-lane
//               quadrant of TMEM (one output row per thread, 32 columns at a time; two warps
//               per quadrant take alternate column chunks), transposes the 32 x 32 chunk
//               through a private shared-memory buffer so that each global access of the warp
//               covers four whole row segments, and applies one of the fused epilogues below.
//
// The fused epilogues are where the block's element-wise work lives:
//   EPI_ROPE        Q/K/V projection + rotary embedding on the rotated heads;
//   EPI_OPROJ_LOOP  output projection forming the residual y = x + a and the recurrent
//                   update h_next = A (.) h + B.e + a from h and e (after depth attention:
//                   adding a into the y and h_next its O projection formed; the MoE adds f
//                   later);
//   EPI_SWIGLU      expert up-projection (gate and up rows interleaved per tile) -> silu(g)*u;
//   EPI_SCATTER     expert down-projection, gate weight, and reduction into h_next
//                   (h_{t+1} = A h + B e + a + sum_j w_j E_j(yn));
//   EPI_TOPK        router logits -> top-k, gate weights and the claim of each chosen
//                   expert's row (K split over CTAs: partial logits reduced, the last
//                   arrival picks); tokens halted by ACT are routed nowhere;
//   EPI_STORE, EPI_STORE_F32, EPI_OPROJ_PLAIN  plain stores (element type, fp32).
// Grouped mode decodes its tiles from the per-expert row counters on the device (capacity
// layout: group g's rows start at g * cap), so the counts never travel to the host.
#pragma once
#include <algorithm>
#include <type_traits>

#include "rdt_internal.cuh"

namespace rdt {

namespace {

constexpr int BM = 128;

// Epilogue warps per TMEM lane quadrant: two for the epilogues that work chunk by chunk
// (each warp takes every other 32-column chunk of the tile, so that one warp's TMEM loads,
// transposes and stores or reductions overlap the other's; four made the expert
// down-projection slower), one for the router's top-k (a warp needs its rows' whole logits).
template <int KIND>
__host__ __device__ constexpr int epi_split() { return KIND == EPI_TOPK ? 1 : 2; }
// warp 0: TMA, warp 1: MMA, then 4 x epi_split epilogue warps
template <int KIND>
__host__ __device__ constexpr int gemm_threads() { return 64 + 128 * epi_split<KIND>(); }

template <int BN, int CG, int ES>
struct TcCfg {
    static constexpr int B_ROWS = BN / CG;               // B rows this CTA loads per stage
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = B_ROWS * 128;
    static constexpr int BAR_BYTES = 192;
    static constexpr int GROUP_BYTES = 2064;
    static constexpr int STG_BYTES = 4 * ES * 32 * 32 * 4;   // one 32 x 32 fp32 chunk per epilogue warp
    // As many stages as keep the block (plus the 1 KB reserved per CTA) within the 196 KB
    // shared-memory carveout, at most 8: beyond it the driver takes the 228 KB carveout and
    // L1 shrinks from 60 to 28 KB, which measurably slows the epilogues' global traffic.
    static constexpr int STAGES_FIT = (195 * 1024 - BAR_BYTES - GROUP_BYTES - STG_BYTES) / (A_BYTES + B_BYTES);
    static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // two accumulators of BN fp32 columns, rounded up to a power of two
    static constexpr int TMEM_COLS = 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
    // [stages][barriers][group tables][epilogue staging], all dynamic (no static shared
    // memory, so that the dynamic block starts 1024-byte aligned)
    static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + GROUP_BYTES + STG_BYTES;
    static_assert((BAR_BYTES + GROUP_BYTES) % 16 == 0, "staging buffers must be 16-byte aligned");
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte alignment of stages");
    static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair");
    static_assert(STAGES >= 3, "too few pipeline stages");
};

__device__ __forceinline__ void ld_chunk(uint32_t taddr, int c, float (&v)[32]) {
    uint32_t r[32];
    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Transpose of one warp's 32 x 32 fp32 chunk through its private staging buffer. Before:
// lane l holds row l (as TMEM hands it out). After: pass it = 0..7 gives lane l row
// 4 * it + l / 8, columns 4 * (l % 8) .. + 3, so a warp-wide 16-byte access covers four
// contiguous row segments rather than 32 rows. The 16-byte slots of a row are XOR-swizzled
// by the row index: eight lanes of a quarter-warp always hit eight different bank groups,
// in both directions.
__device__ __forceinline__ void stage_put(float* stg, int lane, const float (&v)[32]) {
    __syncwarp();                                   // the previous chunk has been read
#pragma unroll
    for (int k = 0; k < 8; ++k)
        *reinterpret_cast<float4*>(stg + lane * 32 + ((k ^ (lane & 7)) << 2)) =
            make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    __syncwarp();
}

__device__ __forceinline__ void stage_get(const float* stg, int lane, int it, float (&o)[4]) {
    const int row = it * 4 + (lane >> 3);
    const float4 x = *reinterpret_cast<const float4*>(stg + row * 32 + (((lane & 7) ^ (row & 7)) << 2));
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
}

// Store a 32-column chunk of the warp's 32 rows (row-per-lane in v) to base[r * ld + c],
// r < nvalid.
template <typename OutT>
__device__ __forceinline__ void store_chunk(float* stg, int lane, const float (&v)[32], OutT* base,
                                            size_t ld, int nvalid) {
    stage_put(stg, lane, v);
    const int cc = (lane & 7) * 4;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int rr = it * 4 + (lane >> 3);
        float o[4];
        stage_get(stg, lane, it, o);
        if (rr < nvalid) store4(base + rr * ld + cc, o);
    }
}

// store_chunk for the QKV projection: the chunk goes to base as above and, when it holds key
// or value columns (col >= cp_col0) and context parallelism is on, also to every rank's
// gather buffer (this rank's and, over peer memory, its peers'), rows renumbered to the
// sequence positions of this rank: local row r -> (r / seq) * cp_seq_tot + cp_row_off +
// r % seq. One transpose serves all destinations.
template <typename OutT>
__device__ __forceinline__ void store_chunk_cp(const EpiParams& p, float* stg, int lane, const float (&v)[32],
                                               OutT* base, int nvalid, int row0, int col) {
    stage_put(stg, lane, v);
    const int cc = (lane & 7) * 4;
    const bool push = p.cp_n > 0 && col >= p.cp_col0;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int rr = it * 4 + (lane >> 3);
        float o[4];
        stage_get(stg, lane, it, o);
        if (rr >= nvalid) continue;
        store4(base + static_cast<size_t>(rr) * p.ldo + cc, o);
        if (push) {
            const int r = row0 + rr;
            const size_t grow = static_cast<size_t>(r / p.seq) * p.cp_seq_tot + p.cp_row_off + r % p.seq;
            const size_t off = grow * p.cp_w + (col - p.cp_col0) + cc;
#pragma unroll 1
            for (int q = 0; q < p.cp_n; ++q) store4(static_cast<OutT*>(p.cp_dst[q]) + off, o);
        }
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
    // Branch-free: the list stays sorted by score (entries past top_k are the runners-up).
    // The candidate goes to the first slot whose score it beats (strictly: of equal scores
    // the earlier expert stays ahead) and the slots after it shift down by one. Every slot's
    // new entry follows from the old list and the comparisons alone, so the slots update in
    // parallel rather than as a chain through the list.
    __device__ __forceinline__ void insert(float logit, float bias, int ex) {
        const float cs = logit + bias;
        bool c[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) c[j] = cs > bs[j];
#pragma unroll
        for (int j = KMAX - 1; j > 0; --j) {         // downwards: slot j - 1 is still the old one
            bs[j] = c[j] ? (c[j - 1] ? bs[j - 1] : cs) : bs[j];
            bl[j] = c[j] ? (c[j - 1] ? bl[j - 1] : logit) : bl[j];
            bi[j] = c[j] ? (c[j - 1] ? bi[j - 1] : ex) : bi[j];
        }
        bs[0] = c[0] ? cs : bs[0];
        bl[0] = c[0] ? logit : bl[0];
        bi[0] = c[0] ? ex : bi[0];
    }
    // four consecutive experts ex0 .. ex0 + 3, those from n on left out
    __device__ __forceinline__ void insert4(const float (&x)[4], const float* bias, int ex0, int n) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool in = ex0 + u < n;
            insert(in ? x[u] : -INFINITY, in && bias ? __ldg(bias + ex0 + u) : 0.0f, ex0 + u);
        }
    }
    // Warp-collective (every lane calls it; `valid`: the lane's row is a real one). The
    // rows claimed in each expert's capacity block are counted per warp in shared memory
    // first (sc: 2 n_exp ints of the warp's own staging buffer) and then taken from the
    // global counter with one atomic per expert the warp chose: a token's top-k claims,
    // one atomic each on n_exp counters that share two cache lines, serialised at the L2
    // and cost more than the router GEMM itself.
    __device__ __forceinline__ void write(const EpiParams& p, int row, bool valid, int lane, int* sc) const {
        const size_t o = static_cast<size_t>(row) * p.top_k;
        const bool halted = valid && p.halted && p.halted[row];
        const bool route = valid && !halted;
        if (halted) {                                // ACT: a halted token is routed nowhere
            for (int j = 0; j < p.top_k; ++j) {
                p.idx_out[o + j] = -1;
                p.w_out[o + j] = 0.0f;
                if (p.trace_idx) p.trace_idx[o + j] = -1;
                if (p.trace_w) p.trace_w[o + j] = 0.0f;
                if (p.route_token) p.slot_row[o + j] = -1;
            }
        }
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
        int* cnt = sc;
        int* base = sc + p.n_exp;
        for (int x = lane; x < p.n_exp; x += 32) cnt[x] = 0;
        __syncwarp();
        int pos[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            pos[j] = 0;
            if (j < p.top_k && route) pos[j] = atomicAdd(cnt + (bi[j] < 0 ? 0 : bi[j]), 1);
        }
        __syncwarp();
        for (int x = lane; x < p.n_exp; x += 32) {
            const int c = cnt[x];
            base[x] = c ? atomicAdd(p.counts + x, c) : 0;   // histogram and the warp's rows
        }
        __syncwarp();
        if (route) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j >= p.top_k) break;
                const int e = bi[j] < 0 ? 0 : bi[j];      // only when every score was NaN
                const float w = den > 0.0f ? ex[j] / den : 0.0f;
                p.idx_out[o + j] = e;
                p.w_out[o + j] = w;
                if (p.trace_idx) p.trace_idx[o + j] = e;
                if (p.trace_w) p.trace_w[o + j] = w;
                if (p.route_token) {
                    const int rr = e * p.cap + base[e] + pos[j];
                    p.route_token[rr] = row;
                    p.route_w[rr] = w;
                    p.slot_row[o + j] = rr;
                }
            }
        }
        __syncwarp();                                // the staging buffer is free again
    }
};

// Router epilogue. Unsplit: the thread's row holds all logits (BN >= n_exp) in TMEM.
// Split over K: every CTA adds its partial logits into p.logits; for each 32 rows, the warp
// that arrives last on their counter (threadfence-reduction order: adds, fence, count) reads
// the complete rows back and selects.
template <int BN, int KMAX>
__device__ __forceinline__ void epilogue_topk(const EpiParams& p, uint32_t taddr, float* stg, bool valid,
                                              int crow, int split, int mtile) {
    const int lane = threadIdx.x & 31;
    int* sc = reinterpret_cast<int*>(stg);
    // The selection runs as a short rolled loop (four logits per step): fully unrolled over
    // the experts it was tens of kilobytes of straight-line code that one warp per SM
    // sub-partition streamed through the instruction cache, ~60K cycles at 64 experts.
    const float* bias = p.bias;
    if (split <= 1) {
        TopK<KMAX> tk;
        uint32_t r[4];
#pragma unroll 1
        for (int ex = 0; ex < p.n_exp; ex += 4) {
            tmem_ld4(taddr + static_cast<uint32_t>(ex), r);
            tmem_wait_ld();
            const float x[4] = {__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]),
                                __uint_as_float(r[3])};
            tk.insert4(x, bias, ex, p.n_exp);
        }
        tk.write(p, crow, valid, lane, sc);
        return;
    }
    float* lrow = p.logits + static_cast<size_t>(crow) * p.n_exp;
    // the partial logits, transposed through the warp's staging buffer so that each vector
    // reduction of the warp covers four whole 128-byte row pieces (scalar atomics, one row
    // per lane, cost ~30 us at 8192 rows and delayed every later L2 access of the router)
    {
        const int crow0 = crow - lane;              // the warp's first row
        const int nrow = __reduce_add_sync(0xffffffffu, valid ? 1 : 0);
        const int cc = (lane & 7) * 4;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            ld_chunk(taddr, c, v);
            if (c * 32 >= p.n_exp) continue;
            stage_put(stg, lane, v);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int rr = it * 4 + (lane >> 3);
                float o[4];
                stage_get(stg, lane, it, o);
                if (rr >= nrow || c * 32 + cc >= p.n_exp) continue;
                atomicAdd(reinterpret_cast<float4*>(p.logits + static_cast<size_t>(crow0 + rr) * p.n_exp + c * 32 + cc),
                          make_float4(o[0], o[1], o[2], o[3]));
            }
        }
        __syncwarp();                               // the staging buffer is free again
    }
    // Each warp elects alone, on the counter of its 32 rows (no barrier between warps, so a
    // warp that left on a timeout cannot stall the others): adds, fence, count.
    __threadfence();
    __syncwarp();
    const int quad = (threadIdx.x >> 5) & 3;
    int last = 0;
    if (lane == 0) {
        int* cnt = p.tile_count + mtile * 4 + quad;
        last = atomicAdd(cnt, 1) == split - 1;
        if (last) *cnt = 0;                              // ready for the next launch
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    __threadfence();
    // the complete row from L2, four logits per step, the next two loads in flight
    // (n_exp is a multiple of 4: 16-byte pieces; a loop over eight loads at a time, unrolled,
    // measured slower: its code no longer stays in the instruction cache)
    TopK<KMAX> tk;
    if (valid) {
        const float4* row4 = reinterpret_cast<const float4*>(lrow);
        const int n4 = p.n_exp / 4;
        float4 a0 = __ldcg(row4);
        float4 a1 = n4 > 1 ? __ldcg(row4 + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int q = 0; q < n4; ++q) {
            const float x[4] = {a0.x, a0.y, a0.z, a0.w};
            a0 = a1;
            if (q + 2 < n4) a1 = __ldcg(row4 + q + 2);
            tk.insert4(x, bias, 4 * q, p.n_exp);
        }
    }
    tk.write(p, crow, valid, lane, sc);
}

// Operands of an epilogue that do not depend on the accumulator: loaded before the epilogue
// warps wait for it (they are idle during the tile's MMAs), so that their memory round trip
// is not added to the tile's exposed tail.
struct EpiPre {
    float cs[32], sn[32];   // RoPE: cos / sin of the row's position, one per rotary pair
    int token;              // scatter: the row's token (-1: padding row) and gate weight
    float w;
};

template <int KIND>
__device__ __forceinline__ void epilogue_pre(const EpiParams& p, int lane, int nvalid, int row0, EpiPre& pre) {
    if constexpr (KIND == EPI_ROPE) {
        // The angle tables are [rot/2][seq]: for a fixed frequency the lanes (consecutive
        // positions) read consecutive floats.
        const int pos = (row0 + lane) % p.seq + p.pos_off + (p.pos_dev ? *p.pos_dev : 0);
        const int half = p.rot_dim / 2;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            pre.cs[i] = i < half ? p.rope_cos[static_cast<size_t>(i) * p.rope_ld + pos] : 0.0f;
            pre.sn[i] = i < half ? p.rope_sin[static_cast<size_t>(i) * p.rope_ld + pos] : 0.0f;
        }
    } else if constexpr (KIND == EPI_SCATTER) {
        // Row r of the tile is expert output for token row_token[r] with gate weight row_w[r]
        // (shared experts: every token, weight 1)
        pre.token = -1;
        pre.w = 0.0f;
        if (lane < nvalid) {
            const int crow = row0 + lane;
            if (crow < p.shared_rows) {
                pre.token = crow % p.ntok;
                pre.w = 1.0f;
            } else {
                pre.token = p.row_token[crow - p.shared_rows];
                pre.w = p.row_w[crow - p.shared_rows];
            }
        }
    }
}

// One epilogue warp's share of a tile: rows row0 .. row0 + 31 of C (lane l owns row
// row0 + l in TMEM, the first nvalid of them are real), columns n0 .. n0 + BN - 1, the
// 32-column chunks ch0, ch0 + chs, ... of them (RoPE: of its heads).
template <typename T, int BN, int KIND>
__device__ __forceinline__ void epilogue(const EpiParams& p, const EpiPre& pre, uint32_t taddr, float* stg,
                                         int lane, int nvalid, int row0, int n0, int ch0, int chs, int split = 1,
                                         int mtile = 0) {
    const int cc = (lane & 7) * 4;                 // this lane's columns after the transpose
    if constexpr (KIND == EPI_STORE || KIND == EPI_STORE_F32 || KIND == EPI_OPROJ_PLAIN) {
        using OutT = std::conditional_t<KIND == EPI_STORE, T, float>;
        OutT* out = static_cast<OutT*>(p.out) + static_cast<size_t>(row0) * p.ldo;
#pragma unroll 1
        for (int c = ch0; c < BN / 32; c += chs) {
            float v[32];
            ld_chunk(taddr, c, v);
            const int col = n0 + c * 32;
            if (col < p.ncols_valid) store_chunk(stg, lane, v, out + col, p.ldo, nvalid);
        }
    } else if constexpr (KIND == EPI_ROPE) {
        // Heads of width head_w tile the BN columns exactly (host checks BN % head_w == 0).
        // The rotation pairs columns i and i + rot/2 of a head, so it runs row-per-lane
        // (before the transpose), with the row's angles loaded before the accumulator wait.
        const int hw_chunks = p.head_w / 32;
        const int rc0 = p.rot_off / 32;
        const int rch = p.rot_dim / 32;
        const float* cs = pre.cs;
        const float* sn = pre.sn;
        T* out = static_cast<T*>(p.out) + static_cast<size_t>(row0) * p.ldo;
#pragma unroll 1
        for (int hc = ch0 * hw_chunks; hc < BN / 32; hc += chs * hw_chunks) {
            const int head_col0 = n0 + hc * 32;
            const bool rotate = head_col0 < p.rope_limit;
#pragma unroll 1
            for (int c = 0; c < hw_chunks; ++c) {
                const int col = head_col0 + c * 32;
                const bool keep = col < p.ncols_valid;
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
                        if (keep) {
                            store_chunk_cp(p, stg, lane, v0, out + col, nvalid, row0, col);
                            store_chunk_cp(p, stg, lane, v1, out + col + 32, nvalid, row0, col + 32);
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
                        if (keep) store_chunk_cp(p, stg, lane, v, out + col, nvalid, row0, col);
                    }
                } else {
                    float v[32];
                    ld_chunk(taddr, hc + c, v);
                    if (keep) store_chunk_cp(p, stg, lane, v, out + col, nvalid, row0, col);
                }
            }
        }
    } else if constexpr (KIND == EPI_OPROJ_LOOP) {
        if (p.h_in) {
            // y = x + a and h_next = A (.) h + B.e + a, x = h (+ e), from h and e read here
            // (issued before the chunk's accumulator load); every output is stored once
            const T* e = static_cast<const T*>(p.e_in);
            const bool fuse_b = p.b_diag && e;
#pragma unroll 1
            for (int c = ch0; c < BN / 32; c += chs) {
                const int col = n0 + c * 32;
                if (col >= p.ncols_valid) continue;
                float hv[8][4], ev[8][4];
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int rr = it * 4 + (lane >> 3);
                    if (rr >= nvalid) continue;
                    const size_t off = static_cast<size_t>(row0 + rr) * p.ld + col + cc;
                    load4(p.h_in + off, hv[it]);
                    if (e) load4(e + off, ev[it]);
                    if (!fuse_b) {   // ev holds B.e itself; x = h + e then needs e as well
                        if (e) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) hv[it][j] += ev[it][j];   // x
                        }
                        load4(p.be + off, ev[it]);
                    }
                }
                float v[32], ad[4], bd[4];
                ld_chunk(taddr, c, v);
                stage_put(stg, lane, v);
                load4(p.a_diag + col + cc, ad);
                if (fuse_b) load4(p.b_diag + col + cc, bd);
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int rr = it * 4 + (lane >> 3);
                    float o[4];
                    stage_get(stg, lane, it, o);
                    if (rr >= nvalid) continue;
                    const size_t off = static_cast<size_t>(row0 + rr) * p.ld + col + cc;
                    float y[4], hn[4];
                    if (fuse_b) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float h = hv[it][j];
                            hn[j] = fmaf(ad[j], h, ev[it][j] * bd[j]) + o[j];
                            y[j] = (h + ev[it][j]) + o[j];
                        }
                    } else {
                        // hv holds x; A (.) h takes h, read again (the line is in L1)
                        float h[4];
                        load4(p.h_in + off, h);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            hn[j] = fmaf(ad[j], h[j], ev[it][j]) + o[j];
                            y[j] = hv[it][j] + o[j];
                        }
                    }
                    store4(p.y + off, y);
                    store4(p.h_next + off, hn);
                }
            }
            return;
        }
        // y and h_next were formed by an earlier O projection (depth attention's: x + d and
        // A (.) h + B.e + d); a is added into both. Vector atomics need no reads here, so the
        // epilogue never waits on memory.
#pragma unroll 1
        for (int c = ch0; c < BN / 32; c += chs) {
            float v[32];
            ld_chunk(taddr, c, v);
            const int col = n0 + c * 32;
            if (col >= p.ncols_valid) continue;
            stage_put(stg, lane, v);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int rr = it * 4 + (lane >> 3);
                float o[4];
                stage_get(stg, lane, it, o);
                if (rr >= nvalid) continue;
                const size_t off = static_cast<size_t>(row0 + rr) * p.ld + col + cc;
                const float4 add = make_float4(o[0], o[1], o[2], o[3]);
                atomicAdd(reinterpret_cast<float4*>(p.y + off), add);
                atomicAdd(reinterpret_cast<float4*>(p.h_next + off), add);
            }
        }
    } else if constexpr (KIND == EPI_SWIGLU) {
        // Tile columns [0, BN/2) are gate rows (W1), [BN/2, BN) the matching up rows (W3).
        T* out = static_cast<T*>(p.out) + static_cast<size_t>(row0) * p.ldo + n0 / 2;
#pragma unroll 1
        for (int c = ch0; c < BN / 64; c += chs) {
            float g[32], u[32];
            ld_chunk(taddr, c, g);
            ld_chunk(taddr, c + BN / 64, u);
            // silu(g) * u with the fast exponential and division intrinsics: the result is
            // stored in bf16, whose rounding (2^-8 relative) dwarfs their few-ulp fp32 error;
            // IEEE expf and division made this epilogue longer than a tile's MMAs on pairs
            // (for g -> -inf: exp -> inf, 1 / inf = 0, silu -> 0 as it should)
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = g[i] * __fdividef(1.0f, 1.0f + __expf(-g[i])) * u[i];
            store_chunk(stg, lane, g, out + c * 32, p.ldo, nvalid);
        }
    } else if constexpr (KIND == EPI_SCATTER) {
        // Row r of the tile (token and gate weight loaded before the accumulator wait) is added
        // into h_next with vector atomics.
        const int token = pre.token;
        const float w = pre.w;
        int tok[8];
        float wt[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            tok[it] = __shfl_sync(0xffffffffu, token, it * 4 + (lane >> 3));
            wt[it] = __shfl_sync(0xffffffffu, w, it * 4 + (lane >> 3));
        }
#pragma unroll 1
        for (int c = ch0; c < BN / 32; c += chs) {
            float v[32];
            ld_chunk(taddr, c, v);
            const int col = n0 + c * 32;
            if (col >= p.ncols_valid) continue;
            stage_put(stg, lane, v);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                float o[4];
                stage_get(stg, lane, it, o);
                if (tok[it] < 0) continue;
                const float4 add = make_float4(wt[it] * o[0], wt[it] * o[1], wt[it] * o[2], wt[it] * o[3]);
                if (p.rows_out) {          // deterministic mode: the row's own slot, combined later
                    const size_t r = static_cast<size_t>(row0 + it * 4 + (lane >> 3));
                    *reinterpret_cast<float4*>(p.rows_out + r * p.ld + col + cc) = add;
                } else {
                    atomicAdd(reinterpret_cast<float4*>(p.dst + static_cast<size_t>(tok[it]) * p.ld + col + cc), add);
                }
            }
        }
    } else if constexpr (KIND == EPI_TOPK) {
        const bool valid = lane < nvalid;
        const int crow = row0 + lane;
        if (p.top_k <= 2)
            epilogue_topk<BN, 2>(p, taddr, stg, valid, crow, split, mtile);
        else if (p.top_k <= 4)
            epilogue_topk<BN, 4>(p, taddr, stg, valid, crow, split, mtile);
        else if (p.top_k <= 8)
            epilogue_topk<BN, 8>(p, taddr, stg, valid, crow, split, mtile);
        else
            epilogue_topk<BN, 16>(p, taddr, stg, valid, crow, split, mtile);
    }
}

// ----------------------------------------------------------------------------- the kernel

struct TileCoord {
    int a_row0, c_row0, nrows, group, n0, mt, kb0, kb1;
};

// Grouped mode: pref[g] = first row tile of group g (routed groups, then shared ones),
// pref[256] = tile count; cnt[g] = rows of group g.
struct GroupTables {
    int pref[257];
    int cnt[256];
};

__device__ __forceinline__ void build_group_tables(const GemmArgs& args, GroupTables& t, int lane,
                                                   int tile_rows) {
    const int G = args.n_routed + args.n_shared;
    int tiles[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int g = lane * 8 + i;
        const int c = g < args.n_routed ? args.counts[g] : (g < G ? args.M : 0);   // shared: all tokens
        t.cnt[g] = c;
        tiles[i] = (c + tile_rows - 1) / tile_rows;
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

// tile = (mt * n_ntiles + nt) * split + ks; split > 1 divides the K blocks evenly.
// Rows are those of the whole (pair) tile: tile_rows = 128 or 256.
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& args, const GroupTables* gt, int tile,
                                                int n_ntiles, int bn, int split, int num_kb,
                                                int tile_rows) {
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
        const int local = (mt - gt->pref[lo]) * tile_rows;
        t.group = lo;
        t.nrows = min(tile_rows, gt->cnt[lo] - local);
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
        t.a_row0 = mt * tile_rows;
        t.c_row0 = t.a_row0;
        t.nrows = min(tile_rows, args.M - t.a_row0);
    }
    return t;
}

// Persistent: each CTA (pair) walks tiles cid, cid + n_clusters, ... The TMA warp and the
// MMA warp run ahead through a ring of shared-memory stages; the accumulator is
// double-buffered in TMEM so the epilogue of one tile overlaps the MMAs of the next.
//
// Pair protocol (CG = 2; "leader" = the even CTA):
//   full[s]   leader only: one arrival, the leader producer's expect_tx for the bytes of
//             both CTAs; both CTAs' TMA loads complete on it (the peer's bytes may land
//             before that arrival: the phase cannot complete while it is pending).
//   empty[s]  each CTA: the leader's commit arrives on both CTAs' barriers when the MMAs
//             that read stage s (in both CTAs) are done.
//   tfull[b]  each CTA: the leader's commit arrives on both when accumulator b is complete.
//   tempty[b] leader only: one arrival per epilogue warp of both CTAs.
// Every wait is bounded; on a timeout the roles stop and the kernel still passes its
// closing barriers.
template <typename T, int BN, int KIND, int CG>
__global__ void __launch_bounds__(gemm_threads<KIND>(), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                   const __grid_constant__ CUtensorMap tA2, const __grid_constant__ CUtensorMap tB2,
                   const GemmArgs args, const EpiParams epi) {
    constexpr int ES = epi_split<KIND>();
    using C = TcCfg<BN, CG, ES>;
    constexpr bool kBf16 = std::is_same<T, bf16>::value;
    constexpr int kElemsPerRow = 128 / static_cast<int>(sizeof(T));   // K elements per stage
    constexpr int kTileRows = BM * CG;
    static_assert(CG == 1 || kBf16, "pair tiles are bf16 only");

    // The dynamic shared memory of a CTA without static shared memory starts 1024-aligned,
    // as the 128-byte swizzle atoms need; checked below rather than padded for (the result
    // is the same in both CTAs of a pair).
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
    // A misaligned base (never expected) skips every tile but still passes the barriers
    // below, so that a CTA pair cannot be left waiting on one of its CTAs.
    const bool misaligned = (smem_u32(smem) & 1023) != 0;
    if (misaligned && threadIdx.x == 0 && epi.flags) atomicExch(epi.flags + FLAG_TIMEOUT, 1);
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0;
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
#pragma unroll 1
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4 * ES * CG);   // one arrival per epilogue warp of the pair
        }
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tA);
        tma_prefetch_desc(&tB);
    }
    if (warp == 1) {
        if constexpr (CG == 2) {
            tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (CG == 2) cluster_sync();    // the peer's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();
    pdl_wait();

    const GroupTables* gt = nullptr;
    if (args.counts != nullptr && !misaligned) {   // grouped: per-group tile offsets from the counters
        if (warp == 0) build_group_tables(args, s_groups, lane, kTileRows);
        __syncthreads();
        gt = &s_groups;
    }
    const int n_ntiles = (args.N + BN - 1) / BN;
    const int n_mtiles = gt != nullptr ? gt->pref[256]
                       : args.counts != nullptr ? 0 : (args.M + kTileRows - 1) / kTileRows;
    const int split = args.split_k > 1 ? args.split_k : 1;
    const int total = misaligned ? 0 : n_mtiles * n_ntiles * split;
    const int num_kb = args.kb_main + args.kb_ext;
    const int cid = static_cast<int>(blockIdx.x) / CG;
    const int ncl = static_cast<int>(gridDim.x) / CG;

    if (warp == 0) {
        if (lane == 0) {
            // the leader's full barriers, by cluster address (own address when CG == 1)
            const uint32_t full0 = CG == 2 ? mapa_shared(smem_u32(full), 0) : smem_u32(full);
            int it = 0;
            bool ok = true;
#pragma unroll 1
            for (int tile = cid; tile < total && ok; tile += ncl) {
                const TileCoord tc = tile_coord(args, gt, tile, n_ntiles, BN, split, num_kb, kTileRows);
                const int a_row = tc.a_row0 + static_cast<int>(rank) * BM;
                const int b_row = tc.group * args.N + tc.n0 + static_cast<int>(rank) * C::B_ROWS;
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
                    const bool ext = kb >= args.kb_main;
                    const CUtensorMap* ma = ext ? &tA2 : &tA;
                    const CUtensorMap* mb = ext ? &tB2 : &tB;
                    const int kx = (ext ? kb - args.kb_main : kb) * kElemsPerRow;
                    const int brow = ext ? args.b2_row0 + b_row : b_row;
                    if constexpr (CG == 2) {
                        const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8;
                        if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
                        tma_load_2d_pair(sa, ma, fb, kx, a_row);
                        tma_load_2d_pair(sb, mb, fb, kx, brow);
                    } else {
                        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                        tma_load_2d(sa, ma, &full[s], kx, a_row);
                        tma_load_2d(sb, mb, &full[s], kx, brow);
                    }
                }
            }
            // Tail: wait until the MMAs have released every stage this CTA filled, so that no
            // commit to this CTA's barriers, and no MMA read of its stages, is still in flight
            // when it leaves.
            // (fill i of stage i % STAGES is released by phase i / STAGES of its barrier).
#pragma unroll 1
            for (int i = it > C::STAGES ? it - C::STAGES : 0; ok && i < it; ++i)
                if (!mbar_wait(&empty[i % C::STAGES], (i / C::STAGES) & 1, epi.flags)) ok = false;
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = make_idesc(kBf16 ? 1 : 2, kTileRows, BN);
            int it = 0, local = 0;
            bool ok = true;
#pragma unroll 1
            for (int tile = cid; tile < total && ok; tile += ncl, ++local) {
                const int b = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1);
                if (!mbar_wait(&tempty[b], (use & 1) ^ 1, epi.flags)) break;
                tc_fence_after();
                const uint32_t dt = tmem + static_cast<uint32_t>(b * BN);
                const TileCoord tc = tile_coord(args, gt, tile, n_ntiles, BN, split, num_kb, kTileRows);
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
                        const uint32_t acc = (kb > tc.kb0) || k;
                        if constexpr (CG == 2)
                            tc_mma_bf16_pair(dt, da + 2 * k, db + 2 * k, idesc, acc);
                        else if constexpr (kBf16)
                            tc_mma_bf16(dt, da + 2 * k, db + 2 * k, idesc, acc);
                        else
                            tc_mma_tf32(dt, da + 2 * k, db + 2 * k, idesc, acc);
                    }
                    if constexpr (CG == 2) tc_commit_pair(&empty[s], 0x3);
                    else tc_commit(&empty[s]);
                }
                if (!ok) break;
                if constexpr (CG == 2) tc_commit_pair(&tfull[b], 0x3);
                else tc_commit(&tfull[b]);
            }
        }
    } else {
        const int q = warp & 3;            // TMEM lane quadrant accessible to this warp
        float* stg = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES + C::BAR_BYTES +
                                              C::GROUP_BYTES) + (warp - 2) * 32 * 32;
        const uint32_t tempty0 = CG == 2 ? mapa_shared(smem_u32(tempty), 0) : smem_u32(tempty);
        const int row_off = static_cast<int>(rank) * BM + q * 32;   // first row of this warp in the tile
        int local = 0;
#pragma unroll 1
        for (int tile = cid; tile < total; tile += ncl, ++local) {
            const int b = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1);
            const TileCoord tc = tile_coord(args, gt, tile, n_ntiles, BN, split, num_kb, kTileRows);
            const int nvalid = min(32, max(0, tc.nrows - row_off));
            EpiPre pre;
            epilogue_pre<KIND>(epi, lane, nvalid, tc.c_row0 + row_off, pre);
            if (!mbar_wait(&tfull[b], use & 1, epi.flags)) break;
            tc_fence_after();
            epilogue<T, BN, KIND>(epi, pre, tmem + (static_cast<uint32_t>(q * 32) << 16) + b * BN, stg, lane,
                                  nvalid, tc.c_row0 + row_off, tc.n0, (warp - 2) >> 2, ES, split, tc.mt);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 2) mbar_arrive_cluster(tempty0 + static_cast<uint32_t>(b) * 8);
                else mbar_arrive(&tempty[b]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (CG == 2) cluster_sync();    // neither CTA leaves while the other may touch it
    if (warp == 1) {
        tc_fence_after();
        if constexpr (CG == 2) tmem_dealloc_pair(tmem, C::TMEM_COLS);
        else tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <typename T, int BN, int KIND, int CG>
rdt_status launch(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                  const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                  cudaStream_t st) {
    using C = TcCfg<BN, CG, epi_split<KIND>()>;
    auto kern = gemm_tc_kernel<T, BN, KIND, CG>;
    constexpr int kTileRows = BM * CG;
    static int dev_ready[64] = {};         // per device: attributes set, co-resident clusters
    static int max_clusters[64] = {};
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) {
        set_error("gemm_tc: device index out of range");
        return RDT_ERR_UNSUPPORTED;
    }
    if (!dev_ready[dev]) {
        RDT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
        int mc = num_sms() / CG;
        if (CG > 1) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * mc);
            cfg.blockDim = dim3(gemm_threads<KIND>());
            cfg.dynamicSmemBytes = C::SMEM;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = CG;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            RDT_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
            if (n < 1) {
                set_error("gemm_tc: a CTA pair with this shared memory cannot be resident");
                return RDT_ERR_UNSUPPORTED;
            }
            mc = std::min(mc, n);
        }
        max_clusters[dev] = mc;
        dev_ready[dev] = 1;
    }
    const int n_ntiles = (args.N + BN - 1) / BN;
    const long mt = args.counts ? args.max_tiles : (args.M + kTileRows - 1) / kTileRows;
    const long total = mt * n_ntiles * (args.split_k > 1 ? args.split_k : 1);
    if (total <= 0) return RDT_OK;
    const int clusters = static_cast<int>(std::min<long>(total, max_clusters[dev]));
    RDT_CUDA_TRY(launch_pdl_cluster(kern, dim3(clusters * CG), dim3(gemm_threads<KIND>()), C::SMEM, st, CG, tA, tB,
                                    tA2 ? *tA2 : tA, tB2 ? *tB2 : tB, args, epi));
    return RDT_OK;
}

template <typename T, int BN, int CG>
rdt_status dispatch_kind(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                         const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                         cudaStream_t st) {
    switch (epi.kind) {
        case EPI_STORE: return launch<T, BN, EPI_STORE, CG>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_STORE_F32: return launch<T, BN, EPI_STORE_F32, CG>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_ROPE: return launch<T, BN, EPI_ROPE, CG>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_OPROJ_LOOP: return launch<T, BN, EPI_OPROJ_LOOP, CG>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_OPROJ_PLAIN: return launch<T, BN, EPI_OPROJ_PLAIN, CG>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_SWIGLU: return launch<T, BN, EPI_SWIGLU, CG>(tA, tB, tA2, tB2, args, epi, st);
        case EPI_SCATTER: return launch<T, BN, EPI_SCATTER, CG>(tA, tB, tA2, tB2, args, epi, st);
        default: set_error("gemm_tc: unknown epilogue"); return RDT_ERR_INVALID_ARG;
    }
}

}  // namespace
}  // namespace rdt
