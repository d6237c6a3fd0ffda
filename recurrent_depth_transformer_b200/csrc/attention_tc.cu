// Causal attention forward on the sm_100a tensor cores (tcgen05):
//
//   o = softmax(q k^T * scale, key > query masked) v
//
// Two kernels. Per query tile t (128 consecutive query rows of one head) and key block j:
//
//   S_t(j) = Q_t K_j^T            tcgen05.mma, M = 128 queries, N = the block's keys, fp32
//                                 in TMEM
//   P_t(j) = 2^(S * scale * log2 e - m_ref)   one thread per query row (a warpgroup per
//            tile), written back into TMEM over S_t(j) as bf16 pairs
//   O_t   += P_t(j) V_j           tcgen05.mma with A = P read from TMEM, B = V from shared
//                                 memory (MN-major), fp32 accumulator in TMEM
//
// O_t is rescaled only when a row maximum grows by more than 2^8 over the reference m_ref
// (so P <= 2^8); the division by the row sum l happens when o is written.
//
// attn96_kernel (head width 64, the GQA shapes): blocks of 96 keys, two score buffers per
// tile so that S_t(j + 1) is computed while the softmax works on S_t(j), one MMA-issuing
// thread per tile, two softmax warps per query row (48 keys of every block each; they agree
// on the row maximum through shared memory), part of the exponentials on the FMA pipe.
//
// attn_tc_kernel (the 160-wide absorbed MLA keys, values of 128): blocks of 128 keys, one
// score buffer per tile, one MMA thread. Absorbed MLA attends over the shared latent key
// [c_kv ; k_rope] (160 wide) with the value c_kv = the key's first 128 columns, so its V
// operand is the K tile itself.
//
// Grouped-query heads read KV head floor(h * Hkv / Hq) ("Introducao ao OpenMythos" Passo 5).
//
// Roles: warpgroup 0 is control: warp 0 issues TMA loads (Q once; K and V in rings of
// stages), warp 1 owns TMEM and issues MMAs, the other warps only take part in set-up (in
// attn96_kernel warp 2 issues the second tile's MMAs). Warpgroups 1 .. QT are the softmax
// warpgroups (warpgroup 1 + t: tile t, one query row per thread, its scores held in
// registers) and write o. Registers are moved from the control warpgroup to the softmax
// warpgroups with setmaxnreg (the split adds up to the block's launch allocation). Every
// wait is bounded.
#include <algorithm>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr int kBQ = 128;     // queries per tile
constexpr int kBK = 128;     // keys per block
constexpr int kAtom = 16384; // one 128-row x 128-byte swizzled region

// 2^x by the hardware approximation (ex2.approx, flush-to-zero): the probabilities are
// rounded to bf16 for the P.V product, and P below 2^-126 contributes nothing there.
__device__ __forceinline__ float exp2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// max(a, b, c) in one instruction (three-input max of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x on the FMA pipe, for two values at once (x <= 8, as the probabilities here are).
// Cody-Waite range reduction: x = j + f with j = round(x), found by adding 1.5 * 2^23 (the
// sum's low mantissa bits then hold j) and f = x - j in [-0.5, 0.5]; 2^f by a cubic fitted
// for this kernel (least maximum relative error on [-0.5, 0.5]: 7.5e-5, far below the bf16
// rounding of P); j is added to the exponent field. x is clamped at -126 first, so a masked
// score (-inf) gives 2^-126 instead of 0: nothing, next to the row's largest term 1.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    const float2 xc = make_float2(fmaxf(x.x, -126.0f), fmaxf(x.y, -126.0f));
    const float2 t = __fadd2_rn(xc, make_float2(12582912.0f, 12582912.0f));
    const float2 j = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = __fadd2_rn(xc, make_float2(-j.x, -j.y));
    float2 q = __ffma2_rn(f, make_float2(0.05517132f, 0.05517132f), make_float2(0.24261054f, 0.24261054f));
    q = __ffma2_rn(q, f, make_float2(0.69326099f, 0.69326099f));
    q = __ffma2_rn(q, f, make_float2(0.99992811f, 0.99992811f));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
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

// D[tmem] (+)= A[tmem] * B[smem]: A (M x K, bf16 pairs per 32-bit TMEM cell, lower K in the
// low half) read from TMEM, B from a shared-memory descriptor; kind::f16, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

template <int DQK, int DV, bool SHARE_KV, int QT>
struct AttnCfg {
    static constexpr int QA = (DQK + 63) / 64;     // 64-wide atoms of the query/key width
    static constexpr int VA = DV / 64;             // 64-wide atoms of the value width
    static constexpr int Q_BYTES = QA * kAtom;     // one query tile
    static constexpr int K_BYTES = QA * kAtom;     // one stage of K (128 keys)
    static constexpr int KSTAGES = (QT == 2 && !SHARE_KV) ? 3 : 2;
    static constexpr int VSTAGES = SHARE_KV ? 0 : KSTAGES;
    static constexpr int V_BYTES = SHARE_KV ? 0 : VA * kAtom;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QT * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KSTAGES * K_BYTES;
    static constexpr int OFF_BAR = OFF_V + VSTAGES * V_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;   // + alignment slack
    // TMEM: score buffer t at columns [128 t, 128 t + 128) (P over the first 64 of its
    // score), then O_t for every tile
    static constexpr int NSBUF = QT;
    static constexpr int S_COL = 0;
    static constexpr int O_COL = 128 * NSBUF;
    static constexpr int COLS_USED = 128 * NSBUF + QT * DV;
    static constexpr int TMEM_COLS = COLS_USED <= 256 ? 256 : 512;
    static constexpr int THREADS = 128 + 128 * QT;
    static constexpr int BLOCKS_PER_SM = QT == 1 ? 2 : 1;
    // registers per thread at launch (65536 per SM over the resident threads, in units of 8)
    static constexpr int REGS_LAUNCH = (65536 / (THREADS * BLOCKS_PER_SM)) / 8 * 8;
    static constexpr int REGS_CONTROL = QT == 1 ? 40 : 64;
    // the softmax warpgroups take what the control warpgroup gives up
    static constexpr int REGS_SOFTMAX = ((REGS_LAUNCH * THREADS - 128 * REGS_CONTROL) / (128 * QT)) / 8 * 8;
    static_assert(128 * REGS_CONTROL + 128 * QT * REGS_SOFTMAX <= REGS_LAUNCH * THREADS, "register split");
    static_assert(REGS_SOFTMAX <= 256, "setmaxnreg limit");
    static_assert(COLS_USED <= 512, "TMEM budget");
    static_assert(NSBUF >= QT, "one score buffer per tile at least");
    static_assert(SMEM <= 227 * 1024, "shared-memory budget");
};

struct AttnTcArgs {
    int seq, hq, hkv, q_hstride, k_hstride, v_hstride, ldo, dv_out;
    int q_off, kv_seq;   // queries at positions q_off + 0 .. seq - 1 of kv_seq keys (attn96 only)
    int nqb, npairs, batch, sms;   // query blocks and CTA work items (of QT blocks) per sequence
    float scale_log2;
    void* o;
    int* flags;
};

// O rows are rescaled only when the running maximum exceeds the reference by more than this
// (log2 units), so P <= 2^8 and the bf16 probabilities keep their relative precision.
constexpr float kRescaleThreshold = 8.0f;

template <int DQK, int DV, bool SHARE_KV, int QT>
__global__ void __launch_bounds__(AttnCfg<DQK, DV, SHARE_KV, QT>::THREADS,
                                  AttnCfg<DQK, DV, SHARE_KV, QT>::BLOCKS_PER_SM)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnTcArgs a) {
    using C = AttnCfg<DQK, DV, SHARE_KV, QT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q = bars + 0;
    uint64_t* kfull = bars + 1;    // [3] per K stage
    uint64_t* kempty = bars + 4;   // [3]
    uint64_t* vfull = bars + 7;    // [3] per V stage
    uint64_t* vempty = bars + 10;  // [3]
    uint64_t* sfull = bars + 13;   // [QT] S_t(j) in TMEM
    uint64_t* pfull = bars + 15;   // [QT] P_t(j) in TMEM (and O_t rescaled if needed)
    uint64_t* oready = bars + 17;  // [QT] PV_t(j) complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
    constexpr int KS = C::KSTAGES;
    constexpr int VS = C::VSTAGES > 0 ? C::VSTAGES : 1;   // V stages (unused when V is the shared latent K)

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Work items ranked by cost, heaviest (last query blocks: most keys) first. With one
    // tile per CTA and two CTAs per SM, when the grid needs more than one CTA per SM but fits
    // two, the CTA in position S + i takes the lightest item left, so that an SM pairs a long
    // query block with a short one.
    const int W = a.npairs * a.hq * a.batch;
    const int L = blockIdx.x;
    const int rank = (QT == 1 && W > a.sms && W <= 2 * a.sms && L >= a.sms) ? W - 1 - (L - a.sms) : L;
    const int per_p = a.hq * a.batch;
    const int pr = a.npairs - 1 - rank / per_p;
    const int h = (rank % per_p) % a.hq;
    const int b = (rank % per_p) / a.hq;
    const int g = (h * a.hkv) / a.hq;
    const int row0 = b * a.seq;                          // first token row of this sequence
    // tile t covers query block qb0 + t; a tile past the last block does nothing
    const int qb0 = pr * QT;
    int nkb_t[QT];
#pragma unroll
    for (int t = 0; t < QT; ++t) nkb_t[t] = qb0 + t < a.nqb ? qb0 + t + 1 : 0;
    int n_kb = 0;
#pragma unroll
    for (int t = 0; t < QT; ++t) n_kb = max(n_kb, nkb_t[t]);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < 3; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
            mbar_init(&vfull[i], 1);
            mbar_init(&vempty[i], 1);
        }
        for (int t = 0; t < QT; ++t) {
            mbar_init(&sfull[t], 1);
            mbar_init(&pfull[t], 4);
            mbar_init(&oready[t], 1);
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

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_CONTROL));
      if (warp == 0) {
        if (lane == 0) {
            int ntiles = 0;
#pragma unroll
            for (int t = 0; t < QT; ++t) ntiles += nkb_t[t] > 0;
            mbar_arrive_expect_tx(bar_q, ntiles * C::Q_BYTES);
#pragma unroll
            for (int t = 0; t < QT; ++t) {
                if (nkb_t[t] == 0) continue;
                for (int at = 0; at < C::QA; ++at)
                    tma_load_2d(smem + C::OFF_Q + t * C::Q_BYTES + at * kAtom, &tq, bar_q,
                                h * a.q_hstride + 64 * at, row0 + (qb0 + t) * kBQ);
            }
            // block j: K into stage j % KS, V into stage j % VS; a stage is refilled once the
            // MMAs that read its previous block have completed
#pragma unroll 1
            for (int j = 0; j < n_kb; ++j) {
                const int sk = j % KS;
                if (!mbar_wait(&kempty[sk], ((j / KS) & 1) ^ 1, a.flags)) break;
                mbar_arrive_expect_tx(&kfull[sk], C::K_BYTES);
                for (int at = 0; at < C::QA; ++at)
                    tma_load_2d(smem + C::OFF_K + sk * C::K_BYTES + at * kAtom, &tk, &kfull[sk],
                                g * a.k_hstride + 64 * at, row0 + j * kBK);
                if (!SHARE_KV) {
                    const int sv = j % VS;
                    if (!mbar_wait(&vempty[sv], ((j / VS) & 1) ^ 1, a.flags)) break;
                    mbar_arrive_expect_tx(&vfull[sv], C::V_BYTES);
                    for (int at = 0; at < C::VA; ++at)
                        tma_load_2d(smem + C::OFF_V + sv * C::V_BYTES + at * kAtom, &tv, &vfull[sv],
                                    g * a.v_hstride + 64 * at, row0 + j * kBK);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(kBQ, kBK, 0);
            constexpr uint32_t id_o = idesc_bf16(kBQ, DV, 1);
            bool ok = mbar_wait(bar_q, 0, a.flags);
            int k_ready = -1;                 // K blocks 0 .. k_ready are known to be loaded
            // S_t(j) = Q_t K_j^T into score buffer `buf`; after the last tile that reads K_j,
            // K_j's stage is released (only if it is loaded again, so that no arrival is
            // pending when the CTA leaves; the shared latent K is released after its PVs)
            auto issue_s = [&](int t, int j, int buf) -> bool {
                for (; k_ready < j; ++k_ready)
                    if (!mbar_wait(&kfull[(k_ready + 1) % KS], ((k_ready + 1) / KS) & 1, a.flags)) return false;
                tc_fence_after();
                const uint32_t sk = smem_u32(smem + C::OFF_K + (j % KS) * C::K_BYTES);
                const uint32_t sq = smem_u32(smem + C::OFF_Q + t * C::Q_BYTES);
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    tc_mma_bf16(tmem + C::S_COL + buf * 128, sw128_kmajor_desc(sq + off),
                                sw128_kmajor_desc(sk + off), id_s, kk > 0);
                }
                tc_commit(&sfull[t]);
                if (!SHARE_KV) {
                    int last = 0;
#pragma unroll
                    for (int u = 0; u < QT; ++u)
                        if (j < nkb_t[u]) last = u;
                    if (t == last && j + KS < n_kb) tc_commit(&kempty[j % KS]);
                }
                return true;
            };
            // the first NSBUF scores, in order n = QT j + t
#pragma unroll 1
            for (int n = 0; n < C::NSBUF && ok; ++n) {
                const int t = n % QT, j = n / QT;
                if (j < nkb_t[t]) ok = issue_s(t, j, n);
            }
#pragma unroll 1
            for (int j = 0; j < n_kb && ok; ++j) {
                const int sv = SHARE_KV ? j % KS : j % VS;
                if (!SHARE_KV && !mbar_wait(&vfull[sv], (j / VS) & 1, a.flags)) { ok = false; break; }
                const uint32_t vaddr = SHARE_KV ? smem_u32(smem + C::OFF_K + sv * C::K_BYTES)
                                                : smem_u32(smem + C::OFF_V + sv * C::V_BYTES);
#pragma unroll 1
                for (int t = 0; t < QT && ok; ++t) {
                    if (j >= nkb_t[t]) continue;
                    if (!mbar_wait(&pfull[t], j & 1, a.flags)) { ok = false; break; }
                    tc_fence_after();
                    const int buf = (QT * j + t) % C::NSBUF;
                    // O_t += P_t(j) V_j: A = P (bf16 pairs in the first 64 columns of the buffer)
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma_bf16_ts(tmem + C::O_COL + t * DV, tmem + C::S_COL + buf * 128 + kk * 8,
                                       sw128_mnmajor_desc(vaddr + kk * 16 * 128, kAtom), id_o, (j > 0) || kk);
                    tc_commit(&oready[t]);
                    // the score NSBUF places later goes into the buffer PV_t(j) has just read
                    const int n2 = QT * j + t + C::NSBUF;
                    const int t2 = n2 % QT, j2 = n2 / QT;
                    if (j2 < nkb_t[t2]) ok = issue_s(t2, j2, buf);
                }
                if (!ok) break;
                // V_j (or the shared latent K_j, also the keys of block j) read by every PV of
                // block j: release its stage if it is loaded again
                if (SHARE_KV) {
                    if (j + KS < n_kb) tc_commit(&kempty[sv]);
                } else {
                    if (j + VS < n_kb) tc_commit(&vempty[sv]);
                }
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        // Softmax warpgroup 1 + t (warps 4 + 4t .. 7 + 4t): TMEM lane quadrant warp & 3, one
        // query row per thread.
        const int t = (warp - 4) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int qb = qb0 + t;
        const int qpos = qb * kBQ + r;
        const int nkb = nkb_t[t];
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t o_col = C::O_COL + t * DV;
        const float sl = a.scale_log2;
        float m_ref = -INFINITY, l = 0.0f;
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < nkb && ok; ++j) {
            if (!mbar_wait(&sfull[t], j & 1, a.flags)) { ok = false; break; }
            tc_fence_after();
            const uint32_t s_col = C::S_COL + ((QT * j + t) % C::NSBUF) * 128;
            uint32_t v[128];
            tmem_ld32(lane_base + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
            tmem_ld32(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            tmem_ld32(lane_base + s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
            tmem_ld32(lane_base + s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
            tmem_wait_ld();
            const int key0 = j * kBK;
            const bool need_mask = (j == qb) || (key0 + kBK > a.seq);
            if (need_mask) {
                const int kmax = min(qpos, a.seq - 1) - key0;      // last allowed key column
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i > kmax) v[i] = __float_as_uint(-INFINITY);
            }
            // row maximum, in four independent chains
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
#pragma unroll
                for (int u = 0; u < 4; ++u) m4[u] = fmaxf(m4[u], __uint_as_float(v[i + u]));
            }
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
            if (mx > m_ref + kRescaleThreshold) {
                const float corr = exp2_ftz(m_ref - mx);
                if (j > 0) {
                    // O_t holds blocks 0 .. j - 1 once PV_t(j - 1) has completed (PV_t(j - 2)
                    // has, since S_t(j) was issued after it: the phase is unambiguous)
                    if (!mbar_wait(&oready[t], (j - 1) & 1, a.flags)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < DV / 32; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(lane_base + o_col + c * 32, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
                        tmem_st32(lane_base + o_col + c * 32, ov);
                    }
                }
                l *= corr;
                m_ref = mx;
            }
            // P = 2^(S sl - m_ref) as bf16 pairs (key 2c in the low half of column c)
            const float2 slv = make_float2(sl, sl);
            const float2 mneg = make_float2(-m_ref, -m_ref);
            float2 rs2 = make_float2(0.0f, 0.0f);
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])),
                                            slv, mneg);
                const float p0 = exp2_ftz(x.x);
                const float p1 = exp2_ftz(x.y);
                rs2 = __fadd2_rn(rs2, make_float2(p0, p1));
                pk[c] = pack_bf16(p0, p1);
            }
            l += rs2.x + rs2.y;
            tmem_st32(lane_base + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(pk + 0));
            tmem_st32(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[t]);
        }
        if (nkb > 0) {
            if (ok) ok = mbar_wait(&oready[t], (nkb - 1) & 1, a.flags);   // the last PV_t
            tc_fence_after();
            const float inv = ok ? 1.0f / l : 0.0f;
            bf16* out = static_cast<bf16*>(a.o) + static_cast<size_t>(row0 + qpos) * a.ldo + h * a.dv_out;
#pragma unroll 1
            for (int c = 0; c < DV / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(lane_base + o_col + c * 32, ov);
                tmem_wait_ld();
                if (!ok || qpos >= a.seq) continue;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    w.x = pack_bf16(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
                    w.y = pack_bf16(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
                    w.z = pack_bf16(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
                    w.w = pack_bf16(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
                    *reinterpret_cast<uint4*>(out + c * 32 + 8 * q) = w;
                }
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

// ---------------------------------------------------------------------------------------
// Head width 64 (keys and values): blocks of 96 keys, QT query tiles of 128 rows per CTA and
// two score buffers per tile. Per tile t the TMEM holds S_t in two buffers of 96 fp32
// columns (P over the first 48 of its buffer as bf16 pairs) and O_t (64 columns): with
// QT = 2, 2 x (2 x 96 + 64) = 512 columns. Because a tile's next score block is computed in
// its other buffer while the softmax works on the current one, the softmax never waits for
// a round trip through the tensor cores; the exponentials (one thread per query row, 96
// per block) are the critical resource and the two tiles' exponentials alternate on the
// MUFU of each SM sub-partition.
//
// MMA order per block j: for each tile, PV_t(j) once P_t(j) is written, then S_t(j + 2) into
// the buffer that PV_t(j) has just read (the MMAs of one thread execute in issue order).
// The K and V of a block share one shared-memory stage, released after the block's last PV.

// Pairs of probabilities, out of the NV / 2 = 24 of a softmax thread's block, whose
// exponentials run on the FMA pipe instead of the MUFU (measured at 8192 positions with two
// softmax warps per row: 0 -> 369 us, 1 -> 360, 2 -> 358, 3 -> 361, 4 -> 363, 6 -> 374;
// with one warp per row, 24 of 96: 371 us against 413 with none).
constexpr int kPolyPairs = 2;


// Softmax warps per query row: 2 splits every block's 96 keys between two warps of the same
// TMEM lane quadrant (they exchange their row maxima through shared memory)
// (measured at 8192 positions: 381 us with one warp per row, 373 with two)
constexpr int kRowWarps = 2;

template <int QT>
struct K96Cfg {
    static constexpr int BK = 96;                       // keys per block
    static constexpr int RW = kRowWarps;                // softmax warps per query row
    static constexpr int NV = BK / RW;                  // scores per softmax thread and block
    static constexpr int KV_BYTES = BK * 128;           // 96 keys x 64 bf16
    static constexpr int STAGES = QT == 2 ? 4 : 3;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QT * kAtom;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
    static constexpr int OFF_X = OFF_BAR + 256;         // float [2 slots][QT][RW][128] row maxima, then [QT][RW][128] sums
    static constexpr int SMEM = OFF_X + 3 * QT * RW * 128 * 4 + 1024;   // + alignment slack
    static constexpr int O_COL = 2 * BK * QT;           // S buffers first, then O_t
    static constexpr int COLS_USED = O_COL + 64 * QT;
    static constexpr int TMEM_COLS = COLS_USED <= 256 ? 256 : 512;
    static constexpr int THREADS = 128 + 128 * QT * RW;
    static constexpr int BLOCKS_PER_SM = QT == 1 ? 2 : 1;
    static constexpr int REGS_LAUNCH = (65536 / (THREADS * BLOCKS_PER_SM)) / 8 * 8;
    static constexpr int REGS_CONTROL = RW == 2 ? 48 : 56;
    static constexpr int REGS_SOFTMAX = ((REGS_LAUNCH * THREADS - 128 * REGS_CONTROL) / (128 * QT * RW)) / 8 * 8;
    static_assert(RW == 1 || RW == 2, "one or two softmax warps per row");
    static_assert(128 * REGS_CONTROL + 128 * QT * RW * REGS_SOFTMAX <= REGS_LAUNCH * THREADS, "register split");
    static_assert(REGS_SOFTMAX <= 256, "setmaxnreg limit");
    static_assert(COLS_USED <= TMEM_COLS && TMEM_COLS * BLOCKS_PER_SM <= 512, "TMEM budget");
    static_assert(SMEM * BLOCKS_PER_SM <= 228 * 1024, "shared-memory budget");
};

// Warp-collective: lane i reads TMEM lane (base lane + i), 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// Warp-collective: lane i writes TMEM lane (base lane + i), 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Warp-collective: lane i writes TMEM lane (base lane + i), 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

template <int QT>
__global__ void __launch_bounds__(K96Cfg<QT>::THREADS, K96Cfg<QT>::BLOCKS_PER_SM)
    attn96_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const AttnTcArgs a) {
    using C = K96Cfg<QT>;
    constexpr int BK = C::BK;
    constexpr int NS = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q = bars + 0;
    uint64_t* full = bars + 1;      // [NS] K_j and V_j loaded into stage j % NS
    uint64_t* empty = bars + 5;     // [QT][NS] tile t's PV of the stage's block complete
    uint64_t* sfull = bars + 13;    // [QT][2] S_t(j) in buffer j % 2
    uint64_t* pfull = bars + 17;    // [QT][2] P_t(j) in buffer j % 2 (and O_t rescaled if needed)
    uint64_t* oready = bars + 21;   // [QT] PV_t(nkb - 2) complete (one phase)
    uint64_t* odone = bars + 23;    // [QT] the tile's last PV complete (one phase)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 25);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // work items heaviest first; with two CTAs per SM, when the grid needs more than one CTA
    // per SM but fits two, the CTA in position S + i takes the lightest item left
    const int W = a.npairs * a.hq * a.batch;
    const int L = blockIdx.x;
    const int rank = (C::BLOCKS_PER_SM == 2 && W > a.sms && W <= 2 * a.sms && L >= a.sms) ? W - 1 - (L - a.sms) : L;
    const int per_p = a.hq * a.batch;
    const int pr = a.npairs - 1 - rank / per_p;
    const int h = (rank % per_p) % a.hq;
    const int b = (rank % per_p) / a.hq;
    const int g = (h * a.hkv) / a.hq;
    const int row0 = b * a.seq;                 // first query row of this sequence
    const int kvrow0 = b * a.kv_seq;            // first key / value row of this sequence
    const int qb0 = pr * QT;
    // tile t (query block qb0 + t, positions from q_off + 128 (qb0 + t)) sees the key blocks
    // that start at or before its last position
    const int nkv = (a.kv_seq + BK - 1) / BK;
    const auto nkb_of = [&](int t) {
        return qb0 + t < a.nqb ? min((a.q_off + (qb0 + t + 1) * kBQ + BK - 1) / BK, nkv) : 0;
    };
    int n_kb = 0;
#pragma unroll
    for (int t = 0; t < QT; ++t) n_kb = max(n_kb, nkb_of(t));

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            for (int t = 0; t < QT; ++t) mbar_init(&empty[t * NS + i], 1);
        }
        for (int t = 0; t < QT; ++t) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(&sfull[2 * t + u], 1);
                mbar_init(&pfull[2 * t + u], 4 * C::RW);
            }
            mbar_init(&oready[t], 1);
            mbar_init(&odone[t], 1);
        }
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
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

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_CONTROL));
      if (warp == 0) {
        if (lane == 0) {
            int ntiles = 0;
#pragma unroll
            for (int t = 0; t < QT; ++t) ntiles += nkb_of(t) > 0;
            mbar_arrive_expect_tx(bar_q, ntiles * kAtom);
#pragma unroll
            for (int t = 0; t < QT; ++t)
                if (nkb_of(t) > 0)
                    tma_load_2d(smem + C::OFF_Q + t * kAtom, &tq, bar_q, h * a.q_hstride, row0 + (qb0 + t) * kBQ);
#pragma unroll 1
            bool ok = true;
            for (int j = 0; j < n_kb && ok; ++j) {
                const int s = j % NS;
                // the stage's previous block j - NS is free once every tile that reads it has
                // completed its PV of it
#pragma unroll
                for (int t = 0; t < QT; ++t)
                    if (ok && j >= NS && j - NS < nkb_of(t))
                        ok = mbar_wait(&empty[t * NS + s], ((j / NS) & 1) ^ 1, a.flags);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[s], 2 * C::KV_BYTES);
                tma_load_2d(smem + C::OFF_K + s * C::KV_BYTES, &tk, &full[s], g * a.k_hstride, kvrow0 + j * BK);
                tma_load_2d(smem + C::OFF_V + s * C::KV_BYTES, &tv, &full[s], g * a.v_hstride, kvrow0 + j * BK);
            }
        }
      } else if (warp <= QT) {
        // warp 1 + t issues the MMAs of tile t (one thread), so that one tile's waits overlap
        // the other tile's MMAs; the tensor core runs them in the order they arrive
        if (lane == 0) {
            const int t = warp - 1;
            const int nkb = nkb_of(t);
            constexpr uint32_t id_s = idesc_bf16(kBQ, BK, 0);
            constexpr uint32_t id_o = idesc_bf16(kBQ, 64, 1);
            // descriptors: start address in 16-byte units in the low bits, so a stage, a
            // 16-key step (V: 16 rows of 128 bytes) or a 16-element K step (32 bytes) is an add
            const uint64_t kdesc0 = sw128_kmajor_desc(smem_u32(smem + C::OFF_K));
            const uint64_t vdesc0 = sw128_mnmajor_desc(smem_u32(smem + C::OFF_V), kAtom);
            const uint64_t qdesc = sw128_kmajor_desc(smem_u32(smem + C::OFF_Q + t * kAtom));
            constexpr uint64_t kStage = C::KV_BYTES >> 4;
            const uint32_t sbase = tmem + 2 * BK * t;
            // S_t(j) = Q_t K_j^T into buffer j % 2 (K_j known to be loaded)
            auto issue_s = [&](int j) {
                const uint64_t kd = kdesc0 + (j % NS) * kStage;
                const uint32_t d = sbase + BK * (j & 1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) tc_mma_bf16(d, qdesc + 2 * kk, kd + 2 * kk, id_s, kk > 0);
                tc_commit(&sfull[2 * t + (j & 1)]);
            };
            bool ok = nkb > 0 && mbar_wait(bar_q, 0, a.flags);
#pragma unroll 1
            for (int j = 0; j < 2 && j < nkb && ok; ++j) {
                ok = mbar_wait(&full[j % NS], (j / NS) & 1, a.flags);
                tc_fence_after();
                if (ok) issue_s(j);
            }
#pragma unroll 1
            for (int j = 0; j < nkb && ok; ++j) {
                const int s = j % NS;
                if (!mbar_wait(&pfull[2 * t + (j & 1)], (j >> 1) & 1, a.flags)) break;
                tc_fence_after();
                // O_t += P_t(j) V_j: A = P (bf16 pairs in the first 48 columns of the buffer),
                // B = V (keys x 64, MN-major; 16 keys = 2048 bytes)
                const uint64_t vd = vdesc0 + s * kStage;
                const uint32_t pa = sbase + BK * (j & 1);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc_mma_bf16_ts(tmem + C::O_COL + 64 * t, pa + kk * 8, vd + kk * 128, id_o, (j > 0) || kk);
                // the last PV ends the tile; the one before it is what a rescale in the last
                // block waits for (earlier rescales wait for the next S, issued after it)
                if (j + 1 == nkb) tc_commit(&odone[t]);
                else if (j + 2 == nkb) tc_commit(&oready[t]);
                if (j + NS < n_kb) tc_commit(&empty[t * NS + s]);
                if (j + 2 < nkb) {
                    if (!mbar_wait(&full[(j + 2) % NS], ((j + 2) / NS) & 1, a.flags)) break;
                    tc_fence_after();
                    issue_s(j + 2);
                }
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        // softmax warps 4 + 4 RW t + 4 hf + quad: tile t, half hf of every block's keys (RW = 2),
        // TMEM lane quadrant quad, one query row per thread
        constexpr int RW = C::RW, NV = C::NV;
        const int sw = warp - 4;
        const int t = sw / (4 * RW);
        const int hf = RW == 2 ? (sw >> 2) & 1 : 0;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int qpos = (qb0 + t) * kBQ + r;
        const int nkb = nkb_of(t);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t o_col = C::O_COL + 64 * t;
        const float sl = a.scale_log2;
        const int kmax_row = min(a.q_off + qpos, a.kv_seq - 1);   // last key the row may see
        float* xmax = reinterpret_cast<float*>(smem + C::OFF_X);   // [2][QT][RW][128]
        float* xsum = xmax + 2 * QT * RW * 128;                   // [QT][RW][128]
        float m_ref = -INFINITY, l = 0.0f;
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < nkb; ++j) {
            const int u = j & 1;
            if (ok && !mbar_wait(&sfull[2 * t + u], (j >> 1) & 1, a.flags)) ok = false;
            tc_fence_after();
            const uint32_t s_col = 2 * BK * t + BK * u;
            uint32_t v[NV];
            if constexpr (RW == 1) {
                tmem_ld32(lane_base + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
                tmem_ld32(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                tmem_ld32(lane_base + s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
            } else {
                tmem_ld32(lane_base + s_col + NV * hf, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
                tmem_ld16(lane_base + s_col + NV * hf + 32, v + 32);
            }
            tmem_wait_ld();
            const int kmax = kmax_row - j * BK - NV * hf;
            if (kmax < NV - 1) {
#pragma unroll
                for (int i = 0; i < NV; ++i)
                    if (i > kmax) v[i] = __float_as_uint(-INFINITY);
            }
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < NV; i += 8) {
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    m4[w] = fmax3(m4[w], __uint_as_float(v[i + 2 * w]), __uint_as_float(v[i + 2 * w + 1]));
            }
            float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
            if constexpr (RW == 2) {
                // the two halves of the row agree on the maximum (so on m_ref): each writes its
                // own into this block's slot and reads the other's after the pair's barrier (the
                // slot alternates with the block, so a half a block ahead never overwrites a
                // value its partner has yet to read). The barrier also orders the partner's
                // score loads before this half's P overwrites its columns.
                float* slot = xmax + (u * QT + t) * RW * 128;
                slot[hf * 128 + r] = mx;
                named_barrier(1 + t * 4 + quad, 64);
                mx = fmaxf(mx, slot[(hf ^ 1) * 128 + r]);
            }
            float corr = 1.0f;
            if (mx > m_ref + kRescaleThreshold) {
                corr = exp2_ftz(m_ref - mx);
                l *= corr;
                m_ref = mx;
            }
            // a row that has seen no allowed key yet keeps m_ref = -inf: its P is 0
            const float mr = m_ref == -INFINITY ? 0.0f : m_ref;
            const float2 slv = make_float2(sl, sl);
            const float2 mneg = make_float2(-mr, -mr);
            float2 rs2 = make_float2(0.0f, 0.0f);
            uint32_t pk[NV / 2];
#pragma unroll
            for (int c = 0; c < NV / 2; ++c) {
                const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])),
                                            slv, mneg);
                // kPolyPairs of the NV / 2 pairs on the FMA pipe, evenly spaced; the rest on the MUFU
                float2 pp;
                if ((c * kPolyPairs) / (NV / 2) != ((c + 1) * kPolyPairs) / (NV / 2)) {
                    pp = exp2_poly2(x);
                } else {
                    pp = make_float2(exp2_ftz(x.x), exp2_ftz(x.y));
                }
                rs2 = __fadd2_rn(rs2, pp);
                pk[c] = pack_bf16(pp.x, pp.y);
            }
            l += rs2.x + rs2.y;
            // P over the first 48 score columns (keys 2c, 2c + 1 in column c)
            if constexpr (RW == 1) {
                tmem_st32(lane_base + s_col, *reinterpret_cast<uint32_t(*)[32]>(pk));
                tmem_st16(lane_base + s_col + 32, pk + 32);
            } else {
                tmem_st16(lane_base + s_col + (NV / 2) * hf, pk);
                tmem_st8(lane_base + s_col + (NV / 2) * hf + 16, pk + 16);
            }
            if (corr != 1.0f && j > 0) {
                // O_t holds blocks 0 .. j - 1 once PV_t(j - 1) has completed: S_t(j + 1) was
                // issued after it (its completion implies PV_t(j - 1)'s), and for the last
                // block the MMA thread commits oready after PV_t(j - 1). PV_t(j) waits for this
                // rescale (pfull). With two halves each rescales 32 of the 64 columns.
                const bool w = j + 1 < nkb ? mbar_wait(&sfull[2 * t + (u ^ 1)], ((j + 1) >> 1) & 1, a.flags)
                                           : mbar_wait(&oready[t], 0, a.flags);
                if (ok && !w) ok = false;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 2 / RW; ++c) {
                    uint32_t ov[32];
                    const uint32_t oc = o_col + (RW == 2 ? 32 * hf : 32 * c);
                    tmem_ld32(lane_base + oc, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
                    tmem_st32(lane_base + oc, ov);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[2 * t + u]);
        }
        if (nkb > 0) {
            if constexpr (RW == 2) {             // the row sum is the two halves' (same m_ref)
                xsum[(t * RW + hf) * 128 + r] = l;
                named_barrier(1 + t * 4 + quad, 64);
                l += xsum[(t * RW + (hf ^ 1)) * 128 + r];
            }
            if (ok) ok = mbar_wait(&odone[t], 0, a.flags);   // the tile's last PV
            tc_fence_after();
            const float inv = ok ? 1.0f / l : 0.0f;
            bf16* out = static_cast<bf16*>(a.o) + static_cast<size_t>(row0 + qpos) * a.ldo + h * a.dv_out;
#pragma unroll 1
            for (int c = 0; c < 2 / RW; ++c) {
                const int oc = RW == 2 ? 32 * hf : 32 * c;
                uint32_t ov[32];
                tmem_ld32(lane_base + o_col + oc, ov);
                tmem_wait_ld();
                if (!ok || qpos >= a.seq) continue;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w4[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        w4[w] = pack_bf16(__uint_as_float(ov[8 * q + 2 * w]) * inv,
                                          __uint_as_float(ov[8 * q + 2 * w + 1]) * inv);
                    *reinterpret_cast<uint4*>(out + oc + 8 * q) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
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

template <int QT>
rdt_status launch_k96(const AttnArgs& a, cudaStream_t st) {
    using C = K96Cfg<QT>;
    auto kern = attn96_kernel<QT>;
    static int configured[64] = {};
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        cudaFuncAttributes fa;
        RDT_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
        if (fa.numRegs != C::REGS_LAUNCH) {
            set_error("attention kernel: launch register count " + std::to_string(fa.numRegs) +
                      " differs from the " + std::to_string(C::REGS_LAUNCH) + " its register split assumes");
            return RDT_ERR_UNSUPPORTED;
        }
        RDT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
        RDT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    const long rows = static_cast<long>(a.batch) * a.seq;
    CUtensorMap tq, tk, tv;
    RDT_TRY(make_tmap_2d(&tq, a.q, true, a.ldq, rows, static_cast<uint64_t>(a.ldq) * 2, 64, 128));
    const int kv_seq = a.kv_seq > 0 ? a.kv_seq : a.seq;
    const long kv_rows = static_cast<long>(a.batch) * kv_seq;
    RDT_TRY(make_tmap_2d(&tk, a.k, true, a.ldk, kv_rows, static_cast<uint64_t>(a.ldk) * 2, 64, C::BK));
    RDT_TRY(make_tmap_2d(&tv, a.v, true, a.ldv, kv_rows, static_cast<uint64_t>(a.ldv) * 2, 64, C::BK));
    AttnTcArgs ta{};
    ta.seq = a.seq;
    ta.hq = a.hq;
    ta.hkv = a.hkv;
    ta.q_hstride = a.q_hstride;
    ta.k_hstride = a.k_hstride;
    ta.v_hstride = a.v_hstride;
    ta.ldo = a.ldo;
    ta.dv_out = a.dv;
    ta.q_off = a.q_off;
    ta.kv_seq = kv_seq;
    ta.scale_log2 = a.scale * 1.4426950408889634f;
    ta.o = a.o;
    ta.flags = a.flags;
    ta.nqb = (a.seq + kBQ - 1) / kBQ;
    ta.npairs = (ta.nqb + QT - 1) / QT;
    ta.batch = a.batch;
    ta.sms = num_sms();
    const dim3 grid(static_cast<unsigned>(ta.npairs) * a.hq * a.batch);
    RDT_CUDA_TRY(launch_pdl(kern, grid, dim3(C::THREADS), C::SMEM, st, tq, tk, tv, ta));
    return RDT_OK;
}

// Two query tiles per CTA (one CTA per SM) once their work items still give every SM at
// least two; otherwise one tile per CTA, two CTAs per SM.
rdt_status launch_k96_choose(const AttnArgs& a, cudaStream_t st) {
    const long nqb = (a.seq + kBQ - 1) / kBQ;
    const long items2 = (nqb + 1) / 2 * a.hq * a.batch;
    if (nqb >= 2 && items2 >= 2L * num_sms()) return launch_k96<2>(a, st);
    return launch_k96<1>(a, st);
}

template <int DQK, int DV, bool SHARE_KV, int QT>
rdt_status launch_tc(const AttnArgs& a, cudaStream_t st) {
    using C = AttnCfg<DQK, DV, SHARE_KV, QT>;
    auto kern = attn_tc_kernel<DQK, DV, SHARE_KV, QT>;
    static int configured[64] = {};        // per device: function attributes are set per device
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        // setmaxnreg moves registers within the block's launch allocation: the split is
        // computed for REGS_LAUNCH registers per thread and would wait forever on fewer
        cudaFuncAttributes fa;
        RDT_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
        if (fa.numRegs != C::REGS_LAUNCH) {
            set_error("attention kernel: launch register count " + std::to_string(fa.numRegs) +
                      " differs from the " + std::to_string(C::REGS_LAUNCH) + " its register split assumes");
            return RDT_ERR_UNSUPPORTED;
        }
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
    ta.npairs = (ta.nqb + QT - 1) / QT;
    ta.batch = a.batch;
    ta.sms = num_sms();
    const dim3 grid(static_cast<unsigned>(ta.npairs) * a.hq * a.batch);
    RDT_CUDA_TRY(launch_pdl(kern, grid, dim3(C::THREADS), C::SMEM, st, tq, tk, tv, ta));
    return RDT_OK;
}

// Two query tiles per CTA (one CTA per SM) once the work items of two tiles still give every
// SM at least two; otherwise one tile per CTA, two CTAs per SM.
template <int DQK, int DV, bool SHARE_KV>
rdt_status launch_choose(const AttnArgs& a, cudaStream_t st) {
    const long nqb = (a.seq + kBQ - 1) / kBQ;
    const long items2 = (nqb + 1) / 2 * a.hq * a.batch;
    if (nqb >= 2 && items2 >= 2L * num_sms()) return launch_tc<DQK, DV, SHARE_KV, 2>(a, st);
    return launch_tc<DQK, DV, SHARE_KV, 1>(a, st);
}

}  // namespace

rdt_status attention_tc(const AttnArgs& a, cudaStream_t st) {
    if (a.dqk == 64 && a.dv == 64) return launch_k96_choose(a, st);
    if (a.q_off != 0 || (a.kv_seq != 0 && a.kv_seq != a.seq)) {
        set_error("tensor-core attention: a query offset needs head width 64");
        return RDT_ERR_UNSUPPORTED;
    }
    if (a.dqk == 160 && a.dv == 128 && a.v == a.k) return launch_choose<160, 128, true>(a, st);
    // 160-wide keys with values of their own: one tile per CTA (two would not fit in shared memory)
    if (a.dqk == 160 && a.dv == 128) return launch_tc<160, 128, false, 1>(a, st);
    set_error("tensor-core attention: unsupported head dimensions");
    return RDT_ERR_UNSUPPORTED;
}

}  // namespace rdt
