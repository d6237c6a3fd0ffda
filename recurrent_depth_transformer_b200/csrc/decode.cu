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

// One CTA per (chunk, group of HG query heads, sequence); the HG heads share one KV head, so
// a key or value row is read once for all of them. Scores are in log2 units (q is scaled on
// load). Each lane scores one key at a time against the HG queries held in shared memory;
// the warp then folds its 32 probabilities into the heads' running (max, sum, o) with the
// lanes spread over o's columns (two adjacent columns per lane and pass: one coalesced
// 4-byte load per value row), eight keys' value loads in flight at a time.
template <int DQK, int DV, int HG>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const DecAttnArgs a) {
    pdl_trigger();
    pdl_wait();
    __shared__ float qs[HG][DQK];
    __shared__ float wm[4][HG], wl[4][HG];
    __shared__ float wo[4][HG][DV];
    const int c = blockIdx.x, hg0 = blockIdx.y * HG, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = (hg0 * a.hkv) / a.hq;
    const int n_keys = *a.len_dev + 1;
    for (int i = threadIdx.x; i < HG * DQK; i += kDecThreads) {
        const int hh = i / DQK, d = i % DQK;
        qs[hh][d] = __bfloat162float(a.q[static_cast<size_t>(b) * a.q_ld + (hg0 + hh) * a.q_hstride + d]) * a.scale_log2;
    }
    __syncthreads();
    constexpr int VP = DV / 64;                  // column pairs per lane
    float m[HG], l[HG], o[HG][VP][2];
#pragma unroll
    for (int hh = 0; hh < HG; ++hh) {
        m[hh] = -INFINITY;
        l[hh] = 0.0f;
#pragma unroll
        for (int i = 0; i < VP; ++i) o[hh][i][0] = o[hh][i][1] = 0.0f;
    }
    const bf16* base = a.cache + static_cast<size_t>(b) * a.s_cap * a.cache_ld;
    const int kbeg = c * kDecChunk + warp * (kDecChunk / 4);
#pragma unroll 1
    for (int r = 0; r < kDecChunk / 4 / 32; ++r) {
        const int kfirst = kbeg + r * 32;
        if (kfirst >= n_keys) break;                 // warp-uniform
        const int key = kfirst + lane;
        float sc[HG];
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) sc[hh] = -INFINITY;
        if (key < n_keys) {
            const bf16* krow = base + static_cast<size_t>(key) * a.cache_ld + a.k_col0 + g * a.k_hstride;
            float acc[HG];
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) acc[hh] = 0.0f;
#pragma unroll
            for (int d0 = 0; d0 < DQK; d0 += 8) {
                const uint4 u = *reinterpret_cast<const uint4*>(krow + d0);
                const bf16* kk = reinterpret_cast<const bf16*>(&u);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float kv = __bfloat162float(kk[j]);
#pragma unroll
                    for (int hh = 0; hh < HG; ++hh) acc[hh] = fmaf(qs[hh][d0 + j], kv, acc[hh]);
                }
            }
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) sc[hh] = acc[hh];
        }
        float p[HG];
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) {
            float mx = sc[hh];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m[hh], mx);        // finite: the group has a key
            const float corr = exp2f(m[hh] - m_new);     // 0 at the first group (m = -inf)
            p[hh] = exp2f(sc[hh] - m_new);               // 0 for a key past the length
            float ps = p[hh];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l[hh] = l[hh] * corr + ps;
#pragma unroll
            for (int i = 0; i < VP; ++i) {
                o[hh][i][0] *= corr;
                o[hh][i][1] *= corr;
            }
            m[hh] = m_new;
        }
        const int nk = min(32, n_keys - kfirst);
        const bf16* vbase = base + static_cast<size_t>(kfirst) * a.cache_ld + a.v_col0 + g * a.v_hstride + 2 * lane;
#pragma unroll 1
        for (int k0 = 0; k0 < nk; k0 += 8) {
            __nv_bfloat162 v[8][VP];
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int i = 0; i < VP; ++i)
                    v[u][i] = k0 + u < nk ? *reinterpret_cast<const __nv_bfloat162*>(
                                                vbase + static_cast<size_t>(k0 + u) * a.cache_ld + 64 * i)
                                          : __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) {
                    const float pk = __shfl_sync(0xffffffffu, p[hh], (k0 + u) & 31);
#pragma unroll
                    for (int i = 0; i < VP; ++i) {
                        const float2 vf = __bfloat1622float2(v[u][i]);
                        o[hh][i][0] = fmaf(pk, vf.x, o[hh][i][0]);
                        o[hh][i][1] = fmaf(pk, vf.y, o[hh][i][1]);
                    }
                }
            }
        }
    }
    // the four warps' partials, then the chunk's (warp hh % 4 merges head hh)
    if (lane == 0) {
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) {
            wm[warp][hh] = m[hh];
            wl[warp][hh] = l[hh];
        }
    }
#pragma unroll
    for (int hh = 0; hh < HG; ++hh)
#pragma unroll
        for (int i = 0; i < VP; ++i) {
            wo[warp][hh][64 * i + 2 * lane] = o[hh][i][0];
            wo[warp][hh][64 * i + 2 * lane + 1] = o[hh][i][1];
        }
    __syncthreads();
    for (int hh = warp; hh < HG; hh += 4) {
        const float mc = fmaxf(fmaxf(wm[0][hh], wm[1][hh]), fmaxf(wm[2][hh], wm[3][hh]));
        float sw[4];
        float lc = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            sw[w] = wm[w][hh] == -INFINITY ? 0.0f : exp2f(wm[w][hh] - mc);
            lc += wl[w][hh] * sw[w];
        }
        float* part = a.part + ((static_cast<size_t>(b) * a.hq + hg0 + hh) * a.n_chunks + c) * (DV + 2);
        for (int col = lane; col < DV; col += 32)
            part[col] = wo[0][hh][col] * sw[0] + wo[1][hh][col] * sw[1] + wo[2][hh][col] * sw[2] + wo[3][hh][col] * sw[3];
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
    // query heads per CTA: up to four of those that share a KV head
    const int G = d.hq / d.hkv;
    const int HG = G % 4 == 0 ? 4 : G % 2 == 0 ? 2 : 1;
    const dim3 grid(a.n_chunks, d.hq / HG, d.batch);
    const int nrows = d.batch * d.hq;
    if (d.dqk == 64 && d.dv == 64) {
        if (HG == 4) RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<64, 64, 4>, grid, dim3(kDecThreads), 0, st, a));
        else if (HG == 2) RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<64, 64, 2>, grid, dim3(kDecThreads), 0, st, a));
        else RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<64, 64, 1>, grid, dim3(kDecThreads), 0, st, a));
        RDT_CUDA_TRY(launch_pdl(decode_merge_kernel<64>, dim3((nrows + 7) / 8), dim3(256), 0, st,
                                static_cast<const float*>(d.part), d.hq, a.n_chunks, d.len_dev,
                                static_cast<bf16*>(d.o), d.ldo, d.dv_out, nrows));
    } else if (d.dqk == 160 && d.dv == 128) {
        if (HG == 4) RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<160, 128, 4>, grid, dim3(kDecThreads), 0, st, a));
        else if (HG == 2) RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<160, 128, 2>, grid, dim3(kDecThreads), 0, st, a));
        else RDT_CUDA_TRY(launch_pdl(decode_attn_kernel<160, 128, 1>, grid, dim3(kDecThreads), 0, st, a));
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
