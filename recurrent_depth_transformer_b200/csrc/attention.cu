// Causal self-attention forward, o = softmax(q k^T * scale, key > query masked) v, per
// (sequence, query head); query head h reads KV head floor(h * Hkv / Hq) (grouped-query
// attention, "Introducao ao OpenMythos" Passo 5; with Hkv = 1 it is the shared latent KV of
// absorbed MLA). The score is never materialised in memory: keys are consumed one at a time
// with a running row maximum and row sum (online softmax).
//
// bf16 runs on the tensor cores (attention_tc.cu). The fp32 configuration (the tiny
// correctness configuration, head widths 32 and 64) runs here: one thread per query row on
// the CUDA cores.
#include "rdt_internal.cuh"

namespace rdt {
namespace {

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
rdt_status launch_f32(const AttnArgs& a, cudaStream_t st) {
    const int n = a.batch * a.hq * a.seq;
    RDT_CUDA_TRY(launch_pdl(attn_f32_kernel<DQK, DV>, dim3((n + 127) / 128), dim3(128), 0, st, a));
    return RDT_OK;
}

}  // namespace

rdt_status attention(bool bf16_elems, const AttnArgs& a, cudaStream_t st) {
    if (bf16_elems) return attention_tc(a, st);
    if (a.q_off != 0 || (a.kv_seq != 0 && a.kv_seq != a.seq)) {
        set_error("attention: a query offset needs bf16");
        return RDT_ERR_UNSUPPORTED;
    }
    {
        if (a.dqk == 32 && a.dv == 32) return launch_f32<32, 32>(a, st);
        if (a.dqk == 64 && a.dv == 64) return launch_f32<64, 64>(a, st);
    }
    set_error("attention: unsupported head dimensions");
    return RDT_ERR_UNSUPPORTED;
}

}  // namespace rdt
