// Causal attention forward on the sm_100a tensor cores (tcgen05), one CTA per
// (128 queries, query head, sequence), two CTAs per SM:
//
//   o = softmax(q k^T * scale, key > query masked) v
//
// For each block j of 128 keys:  S_j = Q K_j^T  (tcgen05.mma, M = 128 queries, N = 128 keys,
// fp32 in TMEM)  ->  eight softmax warps, two per 32 query rows (one per half of the key
// block), one query row per thread: row maximum (the two halves exchange theirs), then
// P_j = 2^(S_j * scale * log2 e - m_ref) in bf16, written to shared memory in the
// 128-byte-swizzled K-major layout, and the row sum l  ->  O += P_j V_j  (tcgen05.mma into a
// TMEM accumulator, N = dv; V read as an MN-major operand straight from its [key][dv] layout).
// m_ref is raised only when a row maximum exceeds it by more than 2^8; O (in TMEM) and l are
// then rescaled once. The division by l happens when o is written.
//
// Grouped-query heads read KV head floor(h * Hkv / Hq) ("Introducao ao OpenMythos" Passo 5).
// Absorbed MLA attends over the shared latent key [c_kv ; k_rope] (160 wide) with the value
// c_kv = the key's first 128 columns, so its V operand is the K tile itself.
//
// Roles: warp 0 issues TMA loads (Q once; K one stage and V two, or two stages of the shared
// latent key for MLA); warp 1 owns TMEM
// and issues the MMAs (S_{j+1} before P_j V_j); warps 2-9 do the softmax (two warps per 32
// query rows, one per half of the key block) and write o.
// Every wait is bounded.
#include <algorithm>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr int kBQ = 128;     // queries per CTA
constexpr int kBK = 128;     // keys per block
constexpr int kAtom = 16384; // one 128-row x 128-byte swizzled region

// 2^x by the hardware approximation (ex2.approx, flush-to-zero): the probabilities are
// rounded to bf16 for the P.V product, and P below 2^-126 contributes nothing there.
__device__ __forceinline__ float exp2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// K-major (a_major = b_major = 0) or K-major A with MN-major B (b_major = 1).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// MN-major operand with the 128-byte swizzle: 8 K-rows of 128 bytes per atom (stride byte
// offset 1024), consecutive 64-element MN atoms `lbo` bytes apart.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr, uint32_t lbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

template <int DQK, int DV, bool SHARE_KV>
struct AttnCfg {
    static constexpr int QA = (DQK + 63) / 64;     // 64-wide atoms of the query/key width
    static constexpr int VA = DV / 64;             // 64-wide atoms of the value width
    static constexpr int Q_BYTES = QA * kAtom;
    static constexpr int K_BYTES = QA * kAtom;     // one stage of K (128 keys)
    // Separate V: one K stage (K_{j+1} loads once S_j has read K_j, during softmax j) and two
    // V stages (V_{j+1} loads while P_j V_j runs). Shared latent V (= K): two K stages.
    static constexpr int KSTAGES = SHARE_KV ? 2 : 1;
    static constexpr int VSTAGES = SHARE_KV ? 0 : 2;
    static constexpr int V_BYTES = SHARE_KV ? 0 : VA * kAtom;
    static constexpr int P_BYTES = 2 * kAtom;      // 128 x 128 bf16 probabilities
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KSTAGES * K_BYTES;
    static constexpr int OFF_P = OFF_V + VSTAGES * V_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;
    static constexpr int OFF_X = OFF_BAR + 256;    // softmax exchange: row maxima [2][2][128], sums [2][128]
    static constexpr int SMEM = OFF_X + 3 * 2 * 128 * 4 + 1024;
    static constexpr int S_COL = 0;                 // S: columns [0, 128)
    static constexpr int O_COL = 128;               // O: columns [128, 128 + DV)
    static constexpr int TMEM_COLS = 128 + DV <= 256 ? 256 : 512;
};

struct AttnTcArgs {
    int seq, hq, hkv, q_hstride, k_hstride, v_hstride, ldo, dv_out;
    int nqb, batch, sms;   // query blocks per sequence; sequences; SMs (first-round CTA slots)
    float scale_log2;
    void* o;
    int* flags;
};

// O is accumulated in TMEM by the P.V MMAs. P_j is taken relative to a reference maximum
// m_ref that is raised only when a row's maximum exceeds it by more than 8 (in log2 units),
// so P <= 2^8; then O and l are rescaled once by 2^(m_ref_old - m_ref_new).
constexpr float kRescaleThreshold = 8.0f;

constexpr int kAttnThreads = 320;   // TMA warp, MMA warp, 8 softmax warps

template <int DQK, int DV, bool SHARE_KV>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnTcArgs a) {
    using C = AttnCfg<DQK, DV, SHARE_KV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q = bars + 0;
    uint64_t* kfull = bars + 1;    // [2]
    uint64_t* kempty = bars + 3;   // [2]
    auto vfull2 = [bars](int st) { return bars + (st ? 20 : 5); };    // per V stage
    auto vempty2 = [bars](int st) { return bars + (st ? 21 : 6); };
    uint64_t* sfull = bars + 7;    // S_j in TMEM
    uint64_t* sfree = bars + 8;    // S_j read by the softmax warps
    uint64_t* pfull = bars + 9;    // P_j in shared memory (and O rescaled if needed)
    uint64_t* ofull = bars + 10;   // P_j . V_j accumulated (P buffer and V stage free)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
    uint64_t* xchg = bars + 12;    // [4] per lane quadrant: both column halves posted their row maxima
    uint64_t* lfin = bars + 16;    // [4] per lane quadrant: both halves posted their row sums

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Work items ranked by cost, heaviest (last query block: most keys) first. CTAs start in
    // launch order, one per SM and then a second one per SM; when the grid needs more than
    // one CTA per SM but fits two, the CTA in position S + i takes the lightest item left,
    // so that an SM pairs a long query block with a short one instead of two long ones.
    const int W = a.nqb * a.hq * a.batch;
    const int L = blockIdx.x;
    const int rank = (W > a.sms && W <= 2 * a.sms && L >= a.sms) ? W - 1 - (L - a.sms) : L;
    const int per_qb = a.hq * a.batch;
    const int qb = a.nqb - 1 - rank / per_qb;
    const int h = (rank % per_qb) % a.hq;
    const int b = (rank % per_qb) / a.hq;
    const int g = (h * a.hkv) / a.hq;
    const int q0 = qb * kBQ;
    const int row0 = b * a.seq;                        // first token row of this sequence
    const int n_kb = min(qb + 1, (a.seq + kBK - 1) / kBK);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(vfull2(i), 1);
            mbar_init(vempty2(i), 1);
        }
        mbar_init(sfull, 1);
        mbar_init(sfree, 8);
        mbar_init(pfull, 8);
        mbar_init(ofull, 1);
        for (int q = 0; q < 4; ++q) {
            mbar_init(&xchg[q], 2);
            mbar_init(&lfin[q], 2);
        }
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        if (!SHARE_KV) tma_prefetch_desc(&tv);
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

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
            for (int t = 0; t < C::QA; ++t)
                tma_load_2d(smem + C::OFF_Q + t * kAtom, &tq, bar_q, h * a.q_hstride + 64 * t, row0 + q0);
            // K block j goes to stage j % KSTAGES (use j / KSTAGES of it), V block j to stage j & 1
            auto load_k = [&](int j) -> bool {
                const int s = j % C::KSTAGES;
                if (!mbar_wait(&kempty[s], ((j / C::KSTAGES) & 1) ^ 1, a.flags)) return false;
                mbar_arrive_expect_tx(&kfull[s], C::K_BYTES);
                for (int t = 0; t < C::QA; ++t)
                    tma_load_2d(smem + C::OFF_K + s * C::K_BYTES + t * kAtom, &tk, &kfull[s],
                                g * a.k_hstride + 64 * t, row0 + j * kBK);
                return true;
            };
            auto load_v = [&](int j) -> bool {
                const int s = j & 1;
                if (!mbar_wait(vempty2(s), ((j >> 1) & 1) ^ 1, a.flags)) return false;
                mbar_arrive_expect_tx(vfull2(s), C::V_BYTES);
                for (int t = 0; t < C::VA; ++t)
                    tma_load_2d(smem + C::OFF_V + s * C::V_BYTES + t * kAtom, &tv, vfull2(s),
                                g * a.v_hstride + 64 * t, row0 + j * kBK);
                return true;
            };
            bool ok = load_k(0);
#pragma unroll 1
            for (int j = 0; j < n_kb && ok; ++j) {
                // V_j first (its stage frees when P_{j-2} V_{j-2} is done, well before S_j),
                // then K_{j+1} (its stage frees when S_j has read K_j)
                if (!SHARE_KV) ok = load_v(j);
                if (ok && j + 1 < n_kb) ok = load_k(j + 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(kBQ, kBK, 0);
            constexpr uint32_t id_o = idesc_bf16(kBQ, DV, 1);
            const uint32_t sq = smem_u32(smem + C::OFF_Q);
            const uint32_t sp = smem_u32(smem + C::OFF_P);
            bool ok = mbar_wait(bar_q, 0, a.flags);
            auto issue_s = [&](int j) -> bool {
                const int s = j % C::KSTAGES;
                if (!mbar_wait(&kfull[s], (j / C::KSTAGES) & 1, a.flags)) return false;
                if (!mbar_wait(sfree, (j & 1) ^ 1, a.flags)) return false;
                tc_fence_after();
                const uint32_t sk = smem_u32(smem + C::OFF_K + s * C::K_BYTES);
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    tc_mma_bf16(tmem + C::S_COL, sw128_kmajor_desc(sq + off), sw128_kmajor_desc(sk + off),
                                id_s, kk > 0);
                }
                tc_commit(sfull);
                if (!SHARE_KV) tc_commit(&kempty[s]);     // K stage consumed
                return true;
            };
            auto issue_o = [&](int j) -> bool {
                const int s = SHARE_KV ? j % C::KSTAGES : j & 1;
                if (!mbar_wait(pfull, j & 1, a.flags)) return false;
                if (!SHARE_KV && !mbar_wait(vfull2(s), (j >> 1) & 1, a.flags)) return false;
                tc_fence_after();
                const uint32_t sv = SHARE_KV ? smem_u32(smem + C::OFF_K + s * C::K_BYTES)
                                             : smem_u32(smem + C::OFF_V + s * C::V_BYTES);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint32_t offp = (kk >> 2) * kAtom + (kk & 3) * 32;
                    tc_mma_bf16(tmem + C::O_COL, sw128_kmajor_desc(sp + offp),
                                sw128_mnmajor_desc(sv + kk * 16 * 128, kAtom), id_o, (j > 0) || kk);
                }
                tc_commit(ofull);
                if (SHARE_KV)
                    tc_commit(&kempty[s]);
                else
                    tc_commit(vempty2(s));
                return true;
            };
            if (ok) ok = issue_s(0);
#pragma unroll 1
            for (int j = 1; j < n_kb && ok; ++j) {
                ok = issue_s(j);
                if (ok) ok = issue_o(j - 1);
            }
            if (ok) issue_o(n_kb - 1);
        }
    } else {
        // Softmax warps 2..9: warp w covers TMEM lane quadrant w & 3 (32 query rows, a thread
        // per row) and column half (w - 2) / 4 of each key block and of O. The two halves of a
        // row exchange their block maxima (and, at the end, their sums) through shared memory,
        // paired by a per-quadrant mbarrier with bounded waits; both then take the same
        // rescaling decisions, and each rescales and finally writes its own half of O.
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        const int qpos = q0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const float sl = a.scale_log2;
        float m_ref = -INFINITY, l = 0.0f;
        uint8_t* arow = smem + C::OFF_P + half * kAtom + r * 128;    // this half's P atom
        float* mxx = reinterpret_cast<float*>(smem + C::OFF_X);      // [2 parity][2 half][128]
        float* lxx = mxx + 2 * 2 * 128;                              // [2 half][128]
        constexpr int HC = kBK / 64;                                 // 32-column chunks per half
        constexpr int OC = DV / 64;                                  // 32-column O chunks per half
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < n_kb && ok; ++j) {
            if (!mbar_wait(sfull, j & 1, a.flags)) { ok = false; break; }
            tc_fence_after();
            const int key0 = j * kBK;
            const bool need_mask = (j == qb) || (key0 + kBK > a.seq);
            const int kmax = need_mask ? min(qpos, a.seq - 1) - key0 : kBK - 1;  // last allowed key
            // pass 1: maximum of this half of the row (scaled to log2 units), then of the row
            float mx = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < HC; ++c) {
                const int col0 = half * 64 + c * 32;
                uint32_t v[32];
                tmem_ld32(lane_base + C::S_COL + col0, v);
                tmem_wait_ld();
                if (!need_mask) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(v[i]));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (col0 + i <= kmax) mx = fmaxf(mx, __uint_as_float(v[i]));
                }
            }
            mx *= sl;
            float* slot = mxx + (j & 1) * 256;
            slot[half * 128 + r] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xchg[quad]);
            if (!mbar_wait(&xchg[quad], j & 1, a.flags)) { ok = false; break; }
            mx = fmaxf(mx, slot[(half ^ 1) * 128 + r]);
            // O (accumulated by P_{j-1} V_{j-1}) is stable once that MMA has completed
            if (j > 0 && !mbar_wait(ofull, (j - 1) & 1, a.flags)) { ok = false; break; }
            tc_fence_after();
            if (mx > m_ref + kRescaleThreshold) {
                const float corr = exp2_ftz(m_ref - mx);
                if (j > 0) {
#pragma unroll
                    for (int c = 0; c < OC; ++c) {
                        const uint32_t ocol = C::O_COL + half * (DV / 2) + c * 32;
                        uint32_t v[32];
                        tmem_ld32(lane_base + ocol, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * corr);
                        tmem_st32(lane_base + ocol, v);
                    }
                    tmem_wait_st();
                }
                l *= corr;
                m_ref = mx;
            }
            // pass 2: P = 2^(S*sl - m_ref) in bf16 into this half's atom of the swizzled P buffer
            float rs = 0.0f;
#pragma unroll 1
            for (int c = 0; c < HC; ++c) {
                const int col0 = half * 64 + c * 32;
                uint32_t v[32];
                tmem_ld32(lane_base + C::S_COL + col0, v);
                tmem_wait_ld();
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float p0 = exp2_ftz(__uint_as_float(v[2 * i]) * sl - m_ref);
                    float p1 = exp2_ftz(__uint_as_float(v[2 * i + 1]) * sl - m_ref);
                    if (need_mask) {
                        if (col0 + 2 * i > kmax) p0 = 0.0f;
                        if (col0 + 2 * i + 1 > kmax) p1 = 0.0f;
                    }
                    rs += p0 + p1;
                    __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                    packed[i] = *reinterpret_cast<uint32_t*>(&pb);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int phys = (c * 4 + q) ^ (r & 7);
                    *reinterpret_cast<uint4*>(arow + phys * 16) =
                        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                }
            }
            l += rs;
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(sfree);
                mbar_arrive(pfull);
            }
        }
        if (ok) ok = mbar_wait(ofull, (n_kb - 1) & 1, a.flags);
        tc_fence_after();
        // the row sum is the two halves' partial sums
        lxx[half * 128 + r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&lfin[quad]);
        if (ok) ok = mbar_wait(&lfin[quad], 0, a.flags);
        const float inv = ok ? 1.0f / (l + lxx[(half ^ 1) * 128 + r]) : 0.0f;
        bf16* out = static_cast<bf16*>(a.o) + static_cast<size_t>(row0 + qpos) * a.ldo + h * a.dv_out +
                    half * (DV / 2);
#pragma unroll 1
        for (int c = 0; c < OC; ++c) {
            uint32_t v[32];
            tmem_ld32(lane_base + C::O_COL + half * (DV / 2) + c * 32, v);
            tmem_wait_ld();
            if (!ok || qpos >= a.seq) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * u]) * inv,
                                                              __uint_as_float(v[8 * q + 2 * u + 1]) * inv);
                    w[u] = *reinterpret_cast<uint32_t*>(&pb);
                }
                *reinterpret_cast<uint4*>(out + c * 32 + 8 * q) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int DQK, int DV, bool SHARE_KV>
rdt_status launch_tc(const AttnArgs& a, cudaStream_t st) {
    using C = AttnCfg<DQK, DV, SHARE_KV>;
    auto kern = attn_tc_kernel<DQK, DV, SHARE_KV>;
    static int configured[64] = {};        // per device: function attributes are set per device
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        RDT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
        RDT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    const long rows = static_cast<long>(a.batch) * a.seq;
    CUtensorMap tq, tk, tv;
    RDT_TRY(make_tmap_2d(&tq, a.q, true, a.ldq, rows, static_cast<uint64_t>(a.ldq) * 2, 64, 128));
    RDT_TRY(make_tmap_2d(&tk, a.k, true, a.ldk, rows, static_cast<uint64_t>(a.ldk) * 2, 64, 128));
    if (!SHARE_KV)
        RDT_TRY(make_tmap_2d(&tv, a.v, true, a.ldv, rows, static_cast<uint64_t>(a.ldv) * 2, 64, 128));
    else
        tv = tk;
    AttnTcArgs ta{};
    ta.seq = a.seq;
    ta.hq = a.hq;
    ta.hkv = a.hkv;
    ta.q_hstride = a.q_hstride;
    ta.k_hstride = a.k_hstride;
    ta.v_hstride = a.v_hstride;
    ta.ldo = a.ldo;
    ta.dv_out = a.dv;
    ta.scale_log2 = a.scale * 1.4426950408889634f;
    ta.o = a.o;
    ta.flags = a.flags;
    ta.nqb = (a.seq + kBQ - 1) / kBQ;
    ta.batch = a.batch;
    ta.sms = num_sms();
    const dim3 grid(static_cast<unsigned>(ta.nqb) * a.hq * a.batch);
    RDT_CUDA_TRY(launch_pdl(kern, grid, dim3(kAttnThreads), C::SMEM, st, tq, tk, tv, ta));
    return RDT_OK;
}

}  // namespace

rdt_status attention_tc(const AttnArgs& a, cudaStream_t st) {
    if (a.dqk == 64 && a.dv == 64) return launch_tc<64, 64, false>(a, st);
    if (a.dqk == 160 && a.dv == 128 && a.v == a.k) return launch_tc<160, 128, true>(a, st);
    set_error("tensor-core attention: unsupported head dimensions");
    return RDT_ERR_UNSUPPORTED;
}

}  // namespace rdt
