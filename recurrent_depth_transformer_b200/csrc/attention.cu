// Causal self-attention forward, o = softmax(q k^T * scale, key > query masked) v, per
// (sequence, query head); query head h reads KV head floor(h * Hkv / Hq) (grouped-query
// attention, "Introducao ao OpenMythos" Passo 5; with Hkv = 1 it is the shared latent KV of
// absorbed MLA). The score is never materialised in memory: keys are consumed in blocks
// with a running row maximum and row sum (online softmax).
//
// bf16 head widths that the tcgen05 kernel (attention_tc.cu: 64/64, and the shared latent
// 160/128) does not cover run here: 64 query rows per CTA (16 per warp), 64-key blocks
// double-buffered in shared memory with cp.async, QK^T and PV on mma.sync m16n8k16 (bf16 in,
// fp32 accumulate).
// Causal blocks above the diagonal are skipped; CTAs with the most key blocks start first.
// fp32: one thread per query row (the tiny fp32 configuration only).
#include "rdt_internal.cuh"

namespace rdt {
namespace {

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
    const int n = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)),
                 "l"(gmem), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

constexpr int kBM = 64;   // query rows per CTA
constexpr int kBN = 64;   // keys per block

// Copy rows [row0, row0 + 64) x D columns (bf16) into shared memory with row stride SD;
// rows at or beyond `nrows` are zero-filled.
template <int D, int SD>
__device__ __forceinline__ void load_rows(bf16* dst, const bf16* src, int ld, int row0, int nrows) {
    constexpr int CPR = D / 8;   // 16-byte chunks per row
    for (int i = threadIdx.x; i < 64 * CPR; i += blockDim.x) {
        const int r = i / CPR, c = i % CPR;
        const bool ok = row0 + r < nrows;
        const bf16* g = src + static_cast<size_t>(ok ? row0 + r : 0) * ld + c * 8;
        cp_async16(dst + r * SD + c * 8, g, ok);
    }
}

template <int DQK, int DV>
__global__ void __launch_bounds__(128) attn_bf16_kernel(const AttnArgs a) {
    constexpr int SQ = DQK + 8;   // padded row strides: 16-byte shift per row, no bank conflicts
    constexpr int SV = DV + 8;
    extern __shared__ __align__(16) uint8_t smem_attn[];
    bf16* sQ = reinterpret_cast<bf16*>(smem_attn);
    bf16* sK = sQ + kBM * SQ;
    bf16* sV = sK + 2 * kBN * SQ;

    pdl_trigger();
    pdl_wait();
    const int qb = gridDim.x - 1 - blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int g = (h * a.hkv) / a.hq;
    const int q0 = qb * kBM;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const bf16* Q = static_cast<const bf16*>(a.q) + static_cast<size_t>(b) * a.seq * a.ldq + h * a.q_hstride;
    const bf16* K = static_cast<const bf16*>(a.k) + static_cast<size_t>(b) * a.seq * a.ldk + g * a.k_hstride;
    const bf16* V = static_cast<const bf16*>(a.v) + static_cast<size_t>(b) * a.seq * a.ldv + g * a.v_hstride;

    const int n_kb = qb + 1;   // key blocks 0..qb (kBM == kBN)
    load_rows<DQK, SQ>(sQ, Q, a.ldq, q0, a.seq);
    load_rows<DQK, SQ>(sK, K, a.ldk, 0, a.seq);
    load_rows<DV, SV>(sV, V, a.ldv, 0, a.seq);
    cp_async_commit();

    const float sc = a.scale * 1.4426950408889634f;   // exp(x) = exp2(x * log2 e)
    float o[DV / 8][4];
#pragma unroll
    for (int i = 0; i < DV / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    uint32_t qf[DQK / 16][4];

#pragma unroll 1
    for (int kb = 0; kb < n_kb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < n_kb) {
            load_rows<DQK, SQ>(sK + (buf ^ 1) * kBN * SQ, K, a.ldk, (kb + 1) * kBN, a.seq);
            load_rows<DV, SV>(sV + (buf ^ 1) * kBN * SV, V, a.ldv, (kb + 1) * kBN, a.seq);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (kb == 0) {
#pragma unroll
            for (int kk = 0; kk < DQK / 16; ++kk)
                ldsm_x4(qf[kk], sQ + (warp * 16 + (lane & 15)) * SQ + kk * 16 + (lane >> 4) * 8);
        }
        const bf16* sKb = sK + buf * kBN * SQ;
        const bf16* sVb = sV + buf * kBN * SV;

        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bfr[4];
                ldsm_x4(bfr, sKb + (np * 16 + (lane & 7) + ((lane >> 4) << 3)) * SQ + kk * 16 +
                                 ((lane >> 3) & 1) * 8);
                mma_bf16(s[2 * np], qf[kk], bfr[0], bfr[1]);
                mma_bf16(s[2 * np + 1], qf[kk], bfr[2], bfr[3]);
            }
        }

        // causal / length mask, then the online-softmax update of rows r0 and r0 + 8
        const int qrow0 = q0 + warp * 16 + (lane >> 2);
        const int key0 = kb * kBN + (lane & 3) * 2;
        const bool need_mask = (kb == qb) || ((kb + 1) * kBN > a.seq);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int qrow = qrow0 + half * 8;
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float& v = s[nt][half * 2 + i];
                    const int key = key0 + nt * 8 + i;
                    if (need_mask && (key > qrow || key >= a.seq)) v = -INFINITY;
                    mx = fmaxf(mx, v);
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[half], mx);
            const float corr = exp2f((m_run[half] - m_new) * sc);
            const float mb = m_new * sc;
            float rs = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float& v = s[nt][half * 2 + i];
                    v = exp2f(v * sc - mb);
                    rs += v;
                }
            }
            l_run[half] = l_run[half] * corr + rs;
            m_run[half] = m_new;
#pragma unroll
            for (int dt = 0; dt < DV / 8; ++dt) {
                o[dt][half * 2] *= corr;
                o[dt][half * 2 + 1] *= corr;
            }
        }

        // O += P V: the S accumulator layout is the A-fragment layout of the next MMA
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            uint32_t pa[4];
            pa[0] = pack_bf16(s[2 * kt][0], s[2 * kt][1]);
            pa[1] = pack_bf16(s[2 * kt][2], s[2 * kt][3]);
            pa[2] = pack_bf16(s[2 * kt + 1][0], s[2 * kt + 1][1]);
            pa[3] = pack_bf16(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
            for (int dp = 0; dp < DV / 16; ++dp) {
                uint32_t vb[4];
                ldsm_x4_t(vb, sVb + (kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * SV + dp * 16 +
                                  (lane >> 4) * 8);
                mma_bf16(o[2 * dp], pa, vb[0], vb[1]);
                mma_bf16(o[2 * dp + 1], pa, vb[2], vb[3]);
            }
        }
        __syncthreads();   // the buffer is refilled by the next iteration's prefetch
    }

#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float l = l_run[half];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const float inv = 1.0f / l;
        const int qrow = q0 + warp * 16 + (lane >> 2) + half * 8;
        if (qrow >= a.seq) continue;
        bf16* out = static_cast<bf16*>(a.o) + (static_cast<size_t>(b) * a.seq + qrow) * a.ldo +
                    h * a.dv + (lane & 3) * 2;
#pragma unroll
        for (int dt = 0; dt < DV / 8; ++dt) {
            *reinterpret_cast<__nv_bfloat162*>(out + dt * 8) =
                __floats2bfloat162_rn(o[dt][half * 2] * inv, o[dt][half * 2 + 1] * inv);
        }
    }
}

template <int DQK, int DV>
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnArgs a) {
    pdl_trigger();
    pdl_wait();
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    if (tid >= a.batch * a.hq * a.seq) return;
    const int s = tid % a.seq;
    const int h = (tid / a.seq) % a.hq;
    const int b = tid / (a.seq * a.hq);
    const int g = (h * a.hkv) / a.hq;
    const float* q = static_cast<const float*>(a.q) + (static_cast<size_t>(b) * a.seq + s) * a.ldq + h * a.q_hstride;
    const float* K = static_cast<const float*>(a.k) + static_cast<size_t>(b) * a.seq * a.ldk + g * a.k_hstride;
    const float* V = static_cast<const float*>(a.v) + static_cast<size_t>(b) * a.seq * a.ldv + g * a.v_hstride;
    float qr[DQK], o[DV];
#pragma unroll
    for (int i = 0; i < DQK; ++i) qr[i] = q[i];
#pragma unroll
    for (int i = 0; i < DV; ++i) o[i] = 0.0f;
    float m = -INFINITY, l = 0.0f;
    for (int j = 0; j <= s; ++j) {
        const float* kj = K + static_cast<size_t>(j) * a.ldk;
        float dot = 0.0f;
#pragma unroll
        for (int i = 0; i < DQK; ++i) dot = fmaf(qr[i], kj[i], dot);
        dot *= a.scale;
        const float m_new = fmaxf(m, dot);
        const float corr = expf(m - m_new);
        const float p = expf(dot - m_new);
        l = l * corr + p;
        const float* vj = V + static_cast<size_t>(j) * a.ldv;
#pragma unroll
        for (int i = 0; i < DV; ++i) o[i] = o[i] * corr + p * vj[i];
        m = m_new;
    }
    float* out = static_cast<float*>(a.o) + (static_cast<size_t>(b) * a.seq + s) * a.ldo + h * a.dv;
    const float inv = 1.0f / l;
#pragma unroll
    for (int i = 0; i < DV; ++i) out[i] = o[i] * inv;
}

template <int DQK, int DV>
rdt_status launch_bf16(const AttnArgs& a, cudaStream_t st) {
    constexpr int smem = (kBM * (DQK + 8) + 2 * kBN * (DQK + 8) + 2 * kBN * (DV + 8)) * 2;
    static int configured[64] = {};        // per device: function attributes are set per device
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        RDT_CUDA_TRY(cudaFuncSetAttribute(attn_bf16_kernel<DQK, DV>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    const dim3 grid((a.seq + kBM - 1) / kBM, a.hq, a.batch);
    RDT_CUDA_TRY(launch_pdl(attn_bf16_kernel<DQK, DV>, grid, dim3(128), smem, st, a));
    return RDT_OK;
}

template <int DQK, int DV>
rdt_status launch_f32(const AttnArgs& a, cudaStream_t st) {
    const int n = a.batch * a.hq * a.seq;
    RDT_CUDA_TRY(launch_pdl(attn_f32_kernel<DQK, DV>, dim3((n + 127) / 128), dim3(128), 0, st, a));
    return RDT_OK;
}

}  // namespace

rdt_status attention(bool bf16_elems, const AttnArgs& a, cudaStream_t st) {
    if (bf16_elems && ((a.dqk == 64 && a.dv == 64) || (a.dqk == 160 && a.dv == 128 && a.v == a.k)))
        return attention_tc(a, st);
    if (bf16_elems) {
        if (a.dqk == 64 && a.dv == 64) return launch_bf16<64, 64>(a, st);
        if (a.dqk == 160 && a.dv == 128) return launch_bf16<160, 128>(a, st);
    } else {
        if (a.dqk == 32 && a.dv == 32) return launch_f32<32, 32>(a, st);
        if (a.dqk == 64 && a.dv == 64) return launch_f32<64, 64>(a, st);
    }
    set_error("attention: unsupported head dimensions");
    return RDT_ERR_UNSUPPORTED;
}

}  // namespace rdt
