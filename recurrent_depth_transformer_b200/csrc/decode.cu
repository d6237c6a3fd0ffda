// Decode with a per-loop KV cache: the kernels that differ from the prompt's path.
//
// The prompt (prefill) runs the loop as usual and keeps, for every loop t, the keys and
// values that loop t produced for every position; a decode step runs the T loops for one
// new token per sequence, and loop t of the new token attends over loop t's cache (the
// getting-started page "Introducao ao OpenMythos", Passo 4: the prompt once, then one token
// per call; troubleshooting item 1: every loop keeps K/V for all tokens). GQA caches its
// rotated keys and its values ([K | V] per row), absorbed MLA its normalised latent and
// rotated shared key ([c_kv | k_rope] per row), from which the heads' keys and values are
// the latent itself (Passo 5: K/V rebuilt from the latent at every step).
//
//   cache_append   copy the rows of the keys/values just projected into the cache of loop t
//                  at their positions (prompt rows, or the new token at the current length)
//   decode_attn    one new query per (sequence, head) against the cached keys 0 .. length,
//                  split over chunks of 256 keys: each CTA leaves a partial (max, sum, o)
//   decode_merge   the chunks' partials combined into o (bf16)
//   len_advance    the cache length grows by one after a decode step
// The current length lives in device memory so that a step's launch sequence does not
// depend on it and replays as one CUDA graph.
#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr int kDecChunk = 256;      // keys per CTA of the split decode attention
constexpr int kDecThreads = 128;    // four warps, 64 keys each

__global__ void __launch_bounds__(256) cache_append_kernel(const bf16* src, int src_ld, int src_col0,
                                                           int width, bf16* cache, int s_cap,
                                                           int rows_per_seq, const int* pos_dev, int ntok) {
    pdl_trigger();
    pdl_wait();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= ntok) return;
    const int b = row / rows_per_seq;
    const int s = row % rows_per_seq + (pos_dev ? *pos_dev : 0);
    const uint4* in = reinterpret_cast<const uint4*>(src + static_cast<size_t>(row) * src_ld + src_col0);
    uint4* out = reinterpret_cast<uint4*>(cache + (static_cast<size_t>(b) * s_cap + s) * width);
    const int nvec = width * 2 / 16;
    for (int i = lane; i < nvec; i += 32) out[i] = in[i];
}

struct DecAttnArgs {
    const bf16* q; int q_ld; int q_hstride;      // new queries: row b, head h at column h * q_hstride
    const bf16* cache; int cache_ld; int s_cap;  // loop t's cache: row (b * s_cap + s)
    int k_col0, k_hstride, v_col0, v_hstride;    // key / value columns of KV head g in a cache row
    int hq, hkv, n_chunks;
    const int* len_dev;                          // keys 0 .. *len_dev (the new token included)
    float scale_log2;
    float* part;                                 // [B, hq, n_chunks, DV + 2]: o, max, sum
};

// One CTA per (chunk, head, sequence). Scores are in log2 units (q is scaled on load). Each
// lane scores one key at a time against q held in shared memory; the warp then folds its 32
// probabilities into its running (max, sum, o) with the lanes spread over o's columns.
template <int DQK, int DV>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const DecAttnArgs a) {
    pdl_trigger();
    pdl_wait();
    __shared__ float qs[DQK];
    __shared__ float wm[4], wl[4];
    __shared__ float wo[4][DV];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = (h * a.hkv) / a.hq;
    const int n_keys = *a.len_dev + 1;
    const bf16* qrow = a.q + static_cast<size_t>(b) * a.q_ld + h * a.q_hstride;
    for (int i = threadIdx.x; i < DQK; i += kDecThreads) qs[i] = __bfloat162float(qrow[i]) * a.scale_log2;
    __syncthreads();
    constexpr int VPL = DV / 32;                 // o columns per lane
    float m = -INFINITY, l = 0.0f, o[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) o[i] = 0.0f;
    const bf16* base = a.cache + static_cast<size_t>(b) * a.s_cap * a.cache_ld;
    const int kbeg = c * kDecChunk + warp * (kDecChunk / 4);
#pragma unroll 1
    for (int r = 0; r < kDecChunk / 4 / 32; ++r) {
        const int key = kbeg + r * 32 + lane;
        float s = -INFINITY;
        if (key < n_keys) {
            const bf16* krow = base + static_cast<size_t>(key) * a.cache_ld + a.k_col0 + g * a.k_hstride;
            float acc = 0.0f;
#pragma unroll
            for (int d0 = 0; d0 < DQK; d0 += 8) {
                const uint4 u = *reinterpret_cast<const uint4*>(krow + d0);
                const bf16* kk = reinterpret_cast<const bf16*>(&u);
#pragma unroll
                for (int j = 0; j < 8; ++j) acc = fmaf(qs[d0 + j], __bfloat162float(kk[j]), acc);
            }
            s = acc;
        }
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (mx == -INFINITY) continue;           // no key of this group (warp-uniform)
        const float m_new = fmaxf(m, mx);
        const float corr = exp2f(m - m_new);     // 0 at the first group (m = -inf)
        const float p = exp2f(s - m_new);        // 0 for a key past the length
        float ps = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l = l * corr + ps;
#pragma unroll
        for (int i = 0; i < VPL; ++i) o[i] *= corr;
        const int kfirst = kbeg + r * 32;
        const int nk = min(32, n_keys - kfirst);
#pragma unroll 1
        for (int k = 0; k < nk; ++k) {
            const float pk = __shfl_sync(0xffffffffu, p, k);
            const bf16* vrow = base + static_cast<size_t>(kfirst + k) * a.cache_ld + a.v_col0 + g * a.v_hstride;
#pragma unroll
            for (int i = 0; i < VPL; ++i) o[i] = fmaf(pk, __bfloat162float(vrow[lane + 32 * i]), o[i]);
        }
        m = m_new;
    }
    // the four warps' partials, then the chunk's
    if (lane == 0) {
        wm[warp] = m;
        wl[warp] = l;
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) wo[warp][lane + 32 * i] = o[i];
    __syncthreads();
    if (warp == 0) {
        float mc = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
        float sc[4];
        float lc = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            sc[w] = mc == -INFINITY ? 0.0f : exp2f(wm[w] - mc);
            lc += wl[w] * sc[w];
        }
        float* part = a.part + ((static_cast<size_t>(b) * a.hq + h) * a.n_chunks + c) * (DV + 2);
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int col = lane + 32 * i;
            part[col] = wo[0][col] * sc[0] + wo[1][col] * sc[1] + wo[2][col] * sc[2] + wo[3][col] * sc[3];
        }
        if (lane == 0) {
            part[DV] = mc;
            part[DV + 1] = lc;
        }
    }
}

// One warp per (sequence, head): o = sum_c o_c 2^(m_c - m) / sum_c l_c 2^(m_c - m).
template <int DV>
__global__ void __launch_bounds__(256) decode_merge_kernel(const float* part, int hq, int n_chunks,
                                                           const int* len_dev, bf16* o, int ldo, int dv_out,
                                                           int nrows) {
    pdl_trigger();
    pdl_wait();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);      // b * hq + h
    const int lane = threadIdx.x & 31;
    if (row >= nrows) return;
    const int used = (*len_dev + 1 + kDecChunk - 1) / kDecChunk;
    const float* p = part + static_cast<size_t>(row) * n_chunks * (DV + 2);
    float m = -INFINITY;
    for (int c = 0; c < used; ++c) m = fmaxf(m, p[c * (DV + 2) + DV]);
    constexpr int VPL = DV / 32;
    float acc[VPL], l = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = 0.0f;
    for (int c = 0; c < used; ++c) {
        const float* pc = p + c * (DV + 2);
        const float s = pc[DV] == -INFINITY ? 0.0f : exp2f(pc[DV] - m);
        l += pc[DV + 1] * s;
#pragma unroll
        for (int i = 0; i < VPL; ++i) acc[i] = fmaf(pc[lane + 32 * i], s, acc[i]);
    }
    const float inv = 1.0f / l;
    const int b = row / hq, h = row % hq;
    bf16* out = o + static_cast<size_t>(b) * ldo + h * dv_out;
#pragma unroll
    for (int i = 0; i < VPL; ++i) out[lane + 32 * i] = __float2bfloat16_rn(acc[i] * inv);
}

__global__ void len_advance_kernel(int* len, int by) {
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x == 0 && blockIdx.x == 0) *len += by;
}

}  // namespace

rdt_status cache_append(const void* src, int src_ld, int src_col0, int width, void* cache, int s_cap,
                        int rows_per_seq, const int* pos_dev, int ntok, cudaStream_t st) {
    if ((width * 2) % 16 || (src_ld * 2) % 16 || (src_col0 * 2) % 16) {
        set_error("cache append: rows must be whole 16-byte vectors");
        return RDT_ERR_UNSUPPORTED;
    }
    RDT_CUDA_TRY(launch_pdl(cache_append_kernel, dim3((ntok + 7) / 8), dim3(256), 0, st,
                            static_cast<const bf16*>(src), src_ld, src_col0, width, static_cast<bf16*>(cache),
                            s_cap, rows_per_seq, pos_dev, ntok));
    return RDT_OK;
}

rdt_status decode_attention(const DecodeAttnArgs& d, cudaStream_t st) {
    DecAttnArgs a{};
    a.q = static_cast<const bf16*>(d.q);
    a.q_ld = d.q_ld;
    a.q_hstride = d.q_hstride;
    a.cache = static_cast<const bf16*>(d.cache);
    a.cache_ld = d.cache_ld;
    a.s_cap = d.s_cap;
    a.k_col0 = d.k_col0;
    a.k_hstride = d.k_hstride;
    a.v_col0 = d.v_col0;
    a.v_hstride = d.v_hstride;
    a.hq = d.hq;
    a.hkv = d.hkv;
    a.n_chunks = (d.s_cap + kDecChunk - 1) / kDecChunk;
    a.len_dev = d.len_dev;
    a.scale_log2 = d.scale * 1.4426950408889634f;
    a.part = d.part;
    const dim3 grid(a.n_chunks, d.hq, d.batch);
    const int nrows = d.batch * d.hq;
    if (d.dqk == 64 && d.dv == 64) {
        RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<64, 64>, grid, dim3(kDecThreads), 0, st, a));
        RDT_CUDA_TRY(launch_pdl(decode_merge_kernel<64>, dim3((nrows + 7) / 8), dim3(256), 0, st,
                                static_cast<const float*>(d.part), d.hq, a.n_chunks, d.len_dev,
                                static_cast<bf16*>(d.o), d.ldo, d.dv_out, nrows));
    } else if (d.dqk == 160 && d.dv == 128) {
        RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<160, 128>, grid, dim3(kDecThreads), 0, st, a));
        RDT_CUDA_TRY(launch_pdl(decode_merge_kernel<128>, dim3((nrows + 7) / 8), dim3(256), 0, st,
                                static_cast<const float*>(d.part), d.hq, a.n_chunks, d.len_dev,
                                static_cast<bf16*>(d.o), d.ldo, d.dv_out, nrows));
    } else {
        set_error("decode attention: unsupported head dimensions");
        return RDT_ERR_UNSUPPORTED;
    }
    return RDT_OK;
}

int decode_chunks(int s_cap) { return (s_cap + kDecChunk - 1) / kDecChunk; }

rdt_status len_advance(int* len, int by, cudaStream_t st) {
    RDT_CUDA_TRY(launch_pdl(len_advance_kernel, dim3(1), dim3(32), 0, st, len, by));
    return RDT_OK;
}

}  // namespace rdt
