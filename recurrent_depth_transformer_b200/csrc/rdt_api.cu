// The C ABI of librdt (include/rdt.h): argument validation, weight repacking, the
// library-owned workspace, TMA descriptors, and the per-loop launch sequence of the
// recurrent block
//
//   h_{t+1} = A (.) h_t + B.e + a_t + f_t       (techbriefly article, update equation)
//
// per loop t:  norm1 -> QKV(+RoPE, +LoRA) -> attention -> [LoRA-down] -> O-proj fused with
//              y = x + a and h_next = A h + B.e + a -> norm2 + router top-k -> dispatch ->
//              expert up (SwiGLU) -> expert down fused with gate weight and h_next += w E(yn).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "rdt_internal.cuh"

namespace rdt {

static thread_local std::string g_last_error;
void set_error(const std::string& msg) { g_last_error = msg; }

}  // namespace rdt

using namespace rdt;

struct rdt_handle {
    rdt_config cfg{};
    bool bf = true;
    size_t esz = 2;
    int ntok = 0;
    int G = 0;                     // expert groups = routed + shared
    float rho = 0.0f;
    cudaStream_t last_stream = nullptr;
    std::vector<void*> allocs;
    size_t bytes = 0;

    // weights (library-owned)
    float *A = nullptr, *Bw = nullptr, *g1 = nullptr, *g2 = nullptr, *rbias = nullptr;
    float *q_norm = nullptr, *kv_norm = nullptr;
    void *wqkv = nullptr, *wo = nullptr, *wr = nullptr, *w13 = nullptr, *w2 = nullptr;
    // depth-wise LoRA: loop t uses W_t = W + B_t A_t, merged at create for every adapter:
    // wqkv holds [W_q,l ; W_k ; W_v] for l = 0 .. n_lora - 1 (one block of nqkv rows each) and
    // wo holds W_o,l ([d, nq] each); without LoRA both hold the single base matrix
    int n_wsets = 1;
    void *wlat = nullptr, *wqabs = nullptr;
    float *rope_cos = nullptr, *rope_sin = nullptr;
    int rot = 0;

    // geometry
    int nq = 0, nkv = 0, nqkv = 0;  // GQA projection widths
    int owidth = 0;                 // width of the attention output o
    int qt_w = 0;                   // MLA: width of q~ (H * (kv_lat + rope))
    int lat_w = 0;                  // MLA: q_lat + kv_lat + rope

    // workspace
    float *hbuf[2] = {nullptr, nullptr}, *Be = nullptr, *y = nullptr, *lat = nullptr;
    void *xn = nullptr, *qkv = nullptr, *o = nullptr;
    void *cq = nullptr, *kvlat = nullptr, *xperm = nullptr, *U = nullptr, *yn_lo = nullptr;
    int bn_router = 64;
    int router_split = 1;          // K split of the router GEMM over CTAs
    int router_split_dec = 1;      // ... for a decode step's batch rows
    float* logits = nullptr;       // [N, E] partial-logit accumulator of the split router
    int* tile_count = nullptr;     // arrival counters of the split router, per 32 rows of a row tile
    // output tile widths of the projection and expert GEMMs (128, 192 on pairs, or 256), and
    // whether each runs on CTA pairs (256-row tiles) or single CTAs (128-row tiles)
    int bn_qkv = 128, bn_o = 128, bn_up = 128, bn_down = 128;
    int pair_qkv = 0, pair_o = 0, pair_up = 0, pair_down = 0;
    int split_down = 1;            // K split of the expert down-projection (linear epilogue)
    int32_t* idx = nullptr;
    float* wts = nullptr;
    int cap = 0;                   // rows reserved per expert group (tokens + padding)
    int *counts = nullptr, *row_token = nullptr, *slot_row = nullptr;
    float* row_w = nullptr;
    int max_tiles = 0;             // grouped GEMMs: bound on 128-row tiles
    int max_tiles_pair = 0;        // ... and on 256-row tiles
    int* flags = nullptr;
    float* det_rows = nullptr;     // deterministic mode: [cap * (S + E), dim] expert row outputs
    // decode with a per-loop KV cache (cfg.max_decode > 0): [max_loops][batch][s_cap][cache_w]
    int s_cap = 0;                 // positions a sequence may reach (seq + max_decode); RoPE rows
    int cache_w = 0;               // GQA: [K | V] = 2 n_kv_heads head_dim; MLA: kv_lat + rope
    void* kv_cache = nullptr;
    int* dec_len = nullptr;        // device: cached positions (the new token's position in a step)
    float* dec_part = nullptr;     // split decode attention partials
    int dec_T = 0;                 // loops of the prefill (decode steps run the same number)
    int dec_len_host = 0;          // the same length, tracked on the host for validation
    int mode = 0;                  // 0 plain loop, 1 prefill (fills the cache), 2 decode step
    // depth attention (cfg.da_heads > 0)
    int nq_d = 0, nkv_d = 0, nqkv_d = 0;
    float* g_da = nullptr;
    void *wqkv_d = nullptr, *wo_d = nullptr, *qkv_d = nullptr, *o_d = nullptr, *depth_cache = nullptr;
    float *dtab_cos = nullptr, *dtab_sin = nullptr;   // [max_loops * max_loops][head_dim / 2]
    int* didx = nullptr;           // device [max_loops]: 0, 1, .. (loop t's depth-cache row)
    CUtensorMap m_wqkv_d, m_od, m_wo_d;
    int cur_T = 0;                 // loops of the current call (the depth rotation's last depth)
    int cur_ntok = 0;              // tokens of the current call (batch in a decode step)
    void *stage_h0 = nullptr, *stage_e = nullptr;
    float* stage_out = nullptr;

    // context parallelism (cfg.cp_size > 1): this rank's gather buffer of every rank's rotated
    // keys and values ([batch][cp_size * seq][2 nkv]), its flag words, and the peers' (device
    // pointers valid in this process; the rank's own entries point to its own buffers)
    int cp_size = 1, cp_rank = 0;
    void* cp_kv = nullptr;
    unsigned* cp_flags = nullptr;
    void* cp_peer_kv[kMaxCp] = {};
    unsigned* cp_peer_flags[kMaxCp] = {};
    bool cp_connected = false;

    // ACT halting (rdt_set_act): head, and per-token running sum / loops run
    bool act_set = false;
    float* act_w = nullptr;
    float act_b = 0.0f, act_thr = 0.0f;
    float* act_cum = nullptr;
    int* act_loops = nullptr;

    // tensor maps
    CUtensorMap m_xn, m_o, m_xperm, m_w13, m_U, m_w2;
    std::vector<CUtensorMap> m_wqkv, m_wo;   // one per weight set (adapter)
    CUtensorMap m_wlat, m_cq, m_wqabs, m_ynlo, m_wr;

    // trace
    int32_t* tr_idx = nullptr;
    float* tr_w = nullptr;
    float* tr_h = nullptr;

    // launch accounting and optional per-kernel event timing
    int64_t launches = 0;
    bool prof_on = false;
    bool prof_graph = false;       // profiling inside graph replay (event-record nodes)
    bool capturing = false;        // the launch sequence is being captured into the graph
    std::vector<cudaEvent_t> ev_pool;       // events of eager calls, reused after every read
    size_t ev_used = 0;
    std::vector<cudaEvent_t> graph_events;  // events recorded by nodes of captured graphs
    // CUDA graph of the whole T-loop launch sequence, keyed by the call's pointers and T
    struct GraphKey {
        const void* h0 = nullptr;
        const void* e = nullptr;
        const float* out = nullptr;
        int T = 0;
        bool act = false;
        const int32_t* n_loops = nullptr;
        int mode = 0;
        bool operator==(const GraphKey& o) const {
            return h0 == o.h0 && e == o.e && out == o.out && T == o.T && act == o.act && n_loops == o.n_loops &&
                   mode == o.mode;
        }
    };
    cudaStream_t cap_stream = nullptr;
    cudaGraphExec_t gexec = nullptr;
    GraphKey gkey, seen_key;
    int64_t g_launches = 0;
    struct Pending { int kind; cudaEvent_t a, b; int n; };
    std::vector<Pending> pending;
    std::vector<Pending> graph_pending;   // event pairs recorded by every replay of the graph
    bool graph_ran = false;               // the graph ran since its events were last read
    std::vector<double> prof_ms;
    std::vector<int64_t> prof_n;
};

namespace {

// rows of filler after the grouped GEMMs' operand buffers (one pair tile)
constexpr int kFillerRows = 256;

// kernel classes reported by rdt_profile_read
enum Kind { K_HOIST, K_NORM1, K_GEMM_QKV, K_GEMM_LAT, K_MLA_NORM, K_GEMM_Q, K_ATTENTION,
            K_GEMM_O, K_NORM2, K_ROUTER, K_DISPATCH, K_GEMM_UP, K_GEMM_DOWN, K_CHECK, K_DENSE_B, K_ACT,
            K_COMBINE, K_CACHE, K_DEC_ATTN, K_DA_QKV, K_DA_ATTN, K_DA_O, K_CP_SYNC, K_COUNT };
const char* const kKindName[K_COUNT] = {"hoist", "norm1", "gemm_qkv", "gemm_latent", "mla_latent_norm",
                                         "gemm_q_absorbed", "attention", "gemm_o",
                                         "norm2", "router_topk", "moe_dispatch", "gemm_up", "gemm_down",
                                         "check_finite", "dense_injection", "act_halting", "moe_combine", "kv_cache_append",
                                         "decode_attention", "gemm_qkv_depth", "depth_attention",
                                         "gemm_o_depth", "cp_sync"};

// During graph capture the events become event-record nodes of the graph (external
// records), so that every replay records them again; they are then kept apart from the
// events of eager calls, which are reused after every read.
rdt_status prof_begin(rdt_handle* h, int kind, int nlaunch, cudaStream_t st) {
    h->launches += nlaunch;
    if (!h->prof_on) return RDT_OK;
    cudaEvent_t ev[2];
    for (cudaEvent_t& e : ev) {
        if (h->capturing) {
            RDT_CUDA_TRY(cudaEventCreate(&e));
            h->graph_events.push_back(e);  // destroyed with the handle
            continue;
        }
        while (h->ev_pool.size() <= h->ev_used) {
            cudaEvent_t x;
            RDT_CUDA_TRY(cudaEventCreate(&x));
            h->ev_pool.push_back(x);
        }
        e = h->ev_pool[h->ev_used++];
    }
    rdt_handle::Pending p{kind, ev[0], ev[1], nlaunch};
    if (h->capturing) {
        RDT_CUDA_TRY(cudaEventRecordWithFlags(p.a, st, cudaEventRecordExternal));
        h->graph_pending.push_back(p);
    } else {
        RDT_CUDA_TRY(cudaEventRecord(p.a, st));
        h->pending.push_back(p);
    }
    return RDT_OK;
}
rdt_status prof_end(rdt_handle* h, cudaStream_t st) {
    if (!h->prof_on) return RDT_OK;
    if (h->capturing)
        RDT_CUDA_TRY(cudaEventRecordWithFlags(h->graph_pending.back().b, st, cudaEventRecordExternal));
    else
        RDT_CUDA_TRY(cudaEventRecord(h->pending.back().b, st));
    return RDT_OK;
}
// Resolve recorded event pairs into the per-kind sums (the stream must have completed). The
// graph's pairs describe its last replay only: each replay records them anew.
rdt_status prof_flush(rdt_handle* h) {
    for (const auto& p : h->pending) {
        float ms = 0.0f;
        RDT_CUDA_TRY(cudaEventElapsedTime(&ms, p.a, p.b));
        h->prof_ms[p.kind] += ms;
        h->prof_n[p.kind] += p.n;
    }
    h->pending.clear();
    if (h->graph_ran) {
        for (const auto& p : h->graph_pending) {
            float ms = 0.0f;
            RDT_CUDA_TRY(cudaEventElapsedTime(&ms, p.a, p.b));
            h->prof_ms[p.kind] += ms;
            h->prof_n[p.kind] += p.n;
        }
        h->graph_ran = false;
    }
    // eager events are reused; the graph's belong to it (its nodes record them)
    h->ev_used = 0;
    return RDT_OK;
}

// Every launch of a kernel class is bracketed by an NVTX range named after the class (host
// side: visible to a timeline tool on eager calls and during graph capture) and, when
// profiling is on, by CUDA events.
struct NvtxRange {   // pushed for a scope, popped on every way out of it
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
#define TIMED(h, kind, n, st, expr)                \
    do {                                           \
        NvtxRange nvtx_range_(kKindName[(kind)]);  \
        RDT_TRY(prof_begin((h), (kind), (n), (st))); \
        RDT_TRY(expr);                             \
        RDT_TRY(prof_end((h), (st)));              \
    } while (0)

template <typename P>
rdt_status dev_alloc(rdt_handle* h, P** p, size_t bytes, bool zero = false, int fill_byte = 0) {
    void* q = nullptr;
    if (bytes == 0) bytes = 16;
    if (cudaMalloc(&q, bytes) != cudaSuccess) {
        cudaGetLastError();
        set_error("cudaMalloc of " + std::to_string(bytes) + " bytes failed");
        return RDT_ERR_OOM;
    }
    h->allocs.push_back(q);
    h->bytes += bytes;
    if (zero) RDT_CUDA_TRY(cudaMemset(q, fill_byte, bytes));
    *p = static_cast<P*>(q);
    return RDT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

rdt_status validate_config(const rdt_config* c) {
    auto bad = [](const char* m) { set_error(std::string("config: ") + m); return RDT_ERR_INVALID_ARG; };
    auto uns = [](const char* m) { set_error(std::string("config: ") + m); return RDT_ERR_UNSUPPORTED; };
    if (!c) return bad("NULL config");
    if (c->dtype != RDT_F32 && c->dtype != RDT_BF16) return bad("dtype");
    if (c->batch < 1 || c->seq < 1 || c->dim < 1) return bad("batch, seq and dim must be >= 1");
    if (static_cast<long long>(c->batch) * c->seq > (1 << 24)) return uns("too many tokens");
    const int nv = c->dim / 128;
    if (c->dim % 128 || (nv & (nv - 1)) || nv > 32) return uns("dim must be 128 * 2^k <= 4096");
    if (c->n_heads < 1) return bad("n_heads");
    if (c->n_experts < 1 || c->top_k < 1 || c->top_k > c->n_experts) return bad("n_experts / top_k");
    if (c->top_k > 16) return uns("top_k > 16");
    if (c->n_shared < 0 || c->n_experts + c->n_shared > 256) return uns("n_experts + n_shared > 256");
    if (c->dtype == RDT_F32 && c->n_experts > 64) return uns("f32: n_experts > 64");
    if (c->expert_hidden < 64 || c->expert_hidden % 64) return uns("expert_hidden % 64 != 0");
    if (c->dtype == RDT_F32 && c->expert_hidden % 128) return uns("f32: expert_hidden % 128 != 0");
    if (c->max_loops < 1 || c->max_loops > 64) return bad("max_loops must be in [1, 64]");
    if (c->gemm_tiles < 0 || c->gemm_tiles > 2) return bad("gemm_tiles must be 0, 1 or 2");
    if (c->deterministic != 0 && c->deterministic != 1) return bad("deterministic must be 0 or 1");
    if (c->max_decode < 0 || c->max_decode > (1 << 20)) return bad("max_decode");
    if (c->max_decode > 0 && c->dtype != RDT_BF16) return uns("decode with a KV cache is provided in bf16");
    if (static_cast<long long>(c->seq) + c->max_decode > (1 << 24)) return uns("seq + max_decode too large");
    if (c->cp_size < 0 || c->cp_size > kMaxCp) return bad("cp_size must be in [0, 8]");
    if (c->cp_size > 1) {
        if (c->cp_rank < 0 || c->cp_rank >= c->cp_size) return bad("cp_rank must be in [0, cp_size)");
        if (c->attn_type != RDT_GQA || c->dtype != RDT_BF16 || c->head_dim != 64)
            return uns("context parallelism is provided for bf16 GQA with head_dim 64");
        if (c->seq % 128) return uns("context parallelism: seq (this rank's share) must be a multiple of 128");
        if (c->max_decode > 0) return uns("context parallelism with a decode cache");
        if (static_cast<long long>(c->seq) * c->cp_size > (1 << 24)) return uns("cp_size * seq too large");
    } else if (c->cp_rank != 0) {
        return bad("cp_rank without cp_size > 1");
    }
    if (c->da_heads < 0 || c->da_kv_heads < 0) return bad("da_heads / da_kv_heads");
    if (c->da_heads > 0) {
        if (c->attn_type != RDT_GQA || c->dtype != RDT_BF16 || c->head_dim != 64)
            return uns("depth attention is provided for bf16 GQA with head_dim 64");
        if (c->da_kv_heads < 1 || c->da_heads % c->da_kv_heads) return bad("da_heads % da_kv_heads");
        if ((c->da_heads * 64) % 128 || ((c->da_heads + 2 * c->da_kv_heads) * 64) % 128)
            return uns("depth attention widths must be multiples of 128");
    }
    if (c->b_kind != RDT_B_DIAG && c->b_kind != RDT_B_DENSE) return bad("b_kind");
    if (!(c->norm_eps >= 0.0f) || !(c->rope_base > 1.0f)) return bad("norm_eps / rope_base");
    if (c->lora_rank < 0 || c->n_lora < 0) return bad("lora");
    if (c->n_lora > 0) {
        if (c->attn_type != RDT_GQA) return uns("LoRA is provided for the GQA projections");
        if (c->lora_rank < 1 || c->lora_rank > (c->dtype == RDT_BF16 ? 64 : 32)) return uns("lora_rank");
    }
    if (c->attn_type == RDT_GQA) {
        if (c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads) return bad("n_heads % n_kv_heads");
        if (c->dtype == RDT_BF16 ? c->head_dim != 64 : (c->head_dim != 32 && c->head_dim != 64))
            return uns("head_dim (bf16: 64; f32: 32 or 64)");
        if ((c->n_heads * c->head_dim) % 128) return uns("n_heads * head_dim % 128 != 0");
    } else if (c->attn_type == RDT_MLA) {
        if (c->dtype != RDT_BF16) return uns("MLA is provided in bf16");
        if (c->kv_lora_rank != 128 || c->qk_rope_dim != 32) return uns("MLA: kv_lora_rank 128, qk_rope_dim 32");
        if (c->q_lora_rank < 64 || c->q_lora_rank % 64) return uns("MLA: q_lora_rank % 64");
        if (c->qk_nope_dim < 1 || c->v_head_dim < 1 || c->v_head_dim % 32) return uns("MLA head dims");
    } else {
        return bad("attn_type");
    }
    return RDT_OK;
}

rdt_status need(const void* p, const char* name) {
    if (!p) {
        set_error(std::string("weights: ") + name + " is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (!aligned16(p)) {
        set_error(std::string("weights: ") + name + " is not 16-byte aligned");
        return RDT_ERR_MISALIGNED;
    }
    return RDT_OK;
}

rdt_status copy_d2d(void* dst, const void* src, size_t bytes, cudaStream_t st) {
    RDT_CUDA_TRY(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
    return RDT_OK;
}

// W1 || W3 interleaved in blocks of g rows (g = half the up-projection tile width):
// rows [2gj, 2gj+g) = W1 rows [gj, gj+g), rows [2gj+g, 2gj+2g) = W3 rows [gj, gj+g), so one
// output tile of the up GEMM holds matching gate and up columns.
rdt_status interleave_w13(void* dst, const void* w1, const void* w3, int hid, int dim, size_t esz, int g,
                          cudaStream_t st) {
    const size_t blk = static_cast<size_t>(g) * dim * esz;
    RDT_CUDA_TRY(cudaMemcpy2DAsync(dst, 2 * blk, w1, blk, blk, hid / g, cudaMemcpyDeviceToDevice, st));
    RDT_CUDA_TRY(cudaMemcpy2DAsync(static_cast<char*>(dst) + blk, 2 * blk, w3, blk, blk, hid / g,
                                   cudaMemcpyDeviceToDevice, st));
    return RDT_OK;
}

// Tile shape of a projection or expert GEMM: `rows` output rows (grouped: plus the partial
// last tile of each of `groups` groups, counted as half a tile), N columns, num_kb K blocks of
// 128 bytes. mode 0 chooses, 1 forces single CTAs, 2 forces CTA pairs where allowed.
//
// Measured on B200, these GEMMs are bound by what each SM ingests through TMA, so a tile's
// time is taken as proportional to the rows of A and B one CTA loads per K block (128 + BN
// single, 128 + BN/2 per CTA of a pair) times (its K blocks + 3 for pipeline fill and
// epilogue), scaled by the measured ingest of the shape (1 single 128-wide; 1.25 single
// 256-wide, which fits only 3 stages; 4/3 for a CTA of a pair); the persistent grid's time
// is that of its busiest CTA (pair). K splits (max_split > 1) are for epilogues that reduce
// into their output. Measured choices at batch 4 x seq 512 x dim 1024: QKV on 192-wide pairs,
// O single 128-wide, expert up on 256-wide pairs, expert down single 128-wide split 2.
struct TileChoice {
    int bn;
    int pair;
    int split;
};
TileChoice choose_tiles(long rows, long groups, int N, int num_kb, bool allow256, bool allow192,
                        bool allow_pair, int max_split, int mode) {
    const long sms = num_sms();
    TileChoice best{128, 0, 1};
    double best_cost = -1.0;
    for (int pair : {0, 1}) {
        if (pair && !allow_pair) continue;
        if (mode == 1 && pair) continue;
        if (mode == 2 && allow_pair && !pair) continue;
        const long tile_rows = pair ? 256 : 128;
        const long m_tiles = (rows + tile_rows - 1) / tile_rows + (groups + 1) / 2;
        const long slots = pair ? sms / 2 : sms;
        for (int bn : {256, 192, 128}) {
            if ((bn == 256 && !allow256) || (bn == 192 && !(allow192 && pair)) || N % bn) continue;
            const double rate = pair ? 4.0 / 3.0 : (bn == 256 ? 1.25 : 1.0);
            const double load_rows = 128.0 + (pair ? bn / 2 : bn);
            for (int sp = 1; sp <= max_split; ++sp) {
                if (num_kb % sp) continue;
                const long rounds = (m_tiles * (N / bn) * sp + slots - 1) / slots;
                const double cost = static_cast<double>(rounds) * (num_kb / sp + 3) * load_rows * rate;
                if (best_cost < 0 || cost < best_cost) {
                    best_cost = cost;
                    best = {bn, pair, sp};
                }
            }
        }
    }
    return best;
}

rdt_status build_maps(rdt_handle* h) {
    const rdt_config& c = h->cfg;
    const bool bf = h->bf;
    const uint32_t kbox = static_cast<uint32_t>(128 / h->esz);
    const size_t es = h->esz;
    const int N = h->ntok, d = c.dim;
    const int S = c.n_shared, E = c.n_experts, hid = c.expert_hidden;
    RDT_TRY(make_tmap_2d(&h->m_xn, h->xn, bf, d, N, d * es, kbox, 128));
    RDT_TRY(make_tmap_2d(&h->m_o, h->o, bf, h->owidth, N, h->owidth * es, kbox, 128));
    h->m_wo.resize(h->n_wsets);
    for (int l = 0; l < h->n_wsets; ++l)
        RDT_TRY(make_tmap_2d(&h->m_wo[l], static_cast<const char*>(h->wo) + static_cast<size_t>(l) * d * h->owidth * es,
                             bf, h->owidth, d, h->owidth * es, kbox, h->bn_o >> h->pair_o));
    if (c.attn_type == RDT_GQA) {
        h->m_wqkv.resize(h->n_wsets);
        for (int l = 0; l < h->n_wsets; ++l)
            RDT_TRY(make_tmap_2d(&h->m_wqkv[l], static_cast<const char*>(h->wqkv) + static_cast<size_t>(l) * h->nqkv * d * es,
                                 bf, d, h->nqkv, d * es, kbox, h->bn_qkv >> h->pair_qkv));
    } else {
        RDT_TRY(make_tmap_2d(&h->m_wlat, h->wlat, bf, d, h->lat_w, d * es, kbox, 128));
        RDT_TRY(make_tmap_2d(&h->m_cq, h->cq, bf, c.q_lora_rank, N, c.q_lora_rank * es, kbox, 128));
        RDT_TRY(make_tmap_2d(&h->m_wqabs, h->wqabs, bf, c.q_lora_rank, h->qt_w, c.q_lora_rank * es, kbox, 160));
    }
    // capacity layout, cap rows per group: xperm = [yn (N rows) | expert e: rows N + e cap ..
    // N + (e + 1) cap), U = [shared expert s: rows s cap .. | expert e: rows (S + e) cap ..],
    // and kFillerRows rows of filler after the last group of each
    const uint64_t xrows = static_cast<uint64_t>(N) + static_cast<uint64_t>(h->cap) * E + kFillerRows;
    const uint64_t urows = static_cast<uint64_t>(h->cap) * (S + E) + kFillerRows;
    RDT_TRY(make_tmap_2d(&h->m_xperm, h->xperm, bf, d, xrows, d * es, kbox, 128));
    RDT_TRY(make_tmap_2d(&h->m_w13, h->w13, bf, d, static_cast<uint64_t>(E + S) * 2 * hid, d * es, kbox, h->bn_up >> h->pair_up));
    RDT_TRY(make_tmap_2d(&h->m_U, h->U, bf, hid, urows, hid * es, kbox, 128));
    RDT_TRY(make_tmap_2d(&h->m_w2, h->w2, bf, hid, static_cast<uint64_t>(E + S) * d, hid * es, kbox, h->bn_down >> h->pair_down));
    RDT_TRY(make_tmap_2d(&h->m_ynlo, h->yn_lo, bf, d, N, d * es, kbox, 128));
    if (c.da_heads) {
        RDT_TRY(make_tmap_2d(&h->m_wqkv_d, h->wqkv_d, bf, d, h->nqkv_d, d * es, kbox, 128));
        RDT_TRY(make_tmap_2d(&h->m_od, h->o_d, bf, h->nq_d, N, h->nq_d * es, kbox, 128));
        RDT_TRY(make_tmap_2d(&h->m_wo_d, h->wo_d, bf, h->nq_d, d, h->nq_d * es, kbox, 128));
    }
    RDT_TRY(make_tmap_2d(&h->m_wr, h->wr, bf, d, E, d * es, kbox, h->bn_router));
    return RDT_OK;
}

rdt_status create_impl(const rdt_config* cfg, const rdt_weights* w, cudaStream_t st, rdt_handle* h) {
    const rdt_config& c = *cfg;
    h->cfg = c;
    h->bf = c.dtype == RDT_BF16;
    h->esz = h->bf ? 2 : 4;
    h->ntok = c.batch * c.seq;
    h->cur_ntok = h->ntok;
    h->G = c.n_experts + c.n_shared;
    h->prof_ms.assign(K_COUNT, 0.0);
    h->prof_n.assign(K_COUNT, 0);
    const size_t es = h->esz;
    const int N = h->ntok, d = c.dim, E = c.n_experts, S = c.n_shared, hid = c.expert_hidden;
    const int K = c.top_k;

    // ---- weights present and aligned
    RDT_TRY(need(w->A, "A"));
    RDT_TRY(need(w->B, "B"));
    RDT_TRY(need(w->norm1, "norm1"));
    RDT_TRY(need(w->norm2, "norm2"));
    RDT_TRY(need(w->w_router, "w_router"));
    RDT_TRY(need(w->w1, "w1"));
    RDT_TRY(need(w->w3, "w3"));
    RDT_TRY(need(w->w2, "w2"));
    if (w->router_bias) RDT_TRY(need(w->router_bias, "router_bias"));
    if (S) {
        RDT_TRY(need(w->ws1, "ws1"));
        RDT_TRY(need(w->ws3, "ws3"));
        RDT_TRY(need(w->ws2, "ws2"));
    }
    if (c.attn_type == RDT_GQA) {
        RDT_TRY(need(w->wq, "wq"));
        RDT_TRY(need(w->wk, "wk"));
        RDT_TRY(need(w->wv, "wv"));
        RDT_TRY(need(w->wo, "wo"));
    } else {
        RDT_TRY(need(w->w_dq, "w_dq"));
        RDT_TRY(need(w->q_norm, "q_norm"));
        RDT_TRY(need(w->w_uq, "w_uq"));
        RDT_TRY(need(w->w_dkv, "w_dkv"));
        RDT_TRY(need(w->kv_norm, "kv_norm"));
        RDT_TRY(need(w->w_kr, "w_kr"));
        RDT_TRY(need(w->w_uk, "w_uk"));
        RDT_TRY(need(w->w_uv, "w_uv"));
        RDT_TRY(need(w->wo, "wo"));
    }
    if (c.da_heads) {
        RDT_TRY(need(w->norm_da, "norm_da"));
        RDT_TRY(need(w->wq_d, "wq_d"));
        RDT_TRY(need(w->wk_d, "wk_d"));
        RDT_TRY(need(w->wv_d, "wv_d"));
        RDT_TRY(need(w->wo_d, "wo_d"));
    }
    if (c.n_lora) {
        RDT_TRY(need(w->lq_a, "lq_a"));
        RDT_TRY(need(w->lq_b, "lq_b"));
        RDT_TRY(need(w->lo_a, "lo_a"));
        RDT_TRY(need(w->lo_b, "lo_b"));
    }

    // ---- device and stability check (rho(A) = max |A_i| < 1, no clipping)
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    cudaDeviceProp prop;
    RDT_CUDA_TRY(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10) {
        set_error("an sm_100 (B200-class) device is required");
        return RDT_ERR_UNSUPPORTED;
    }
    {
        std::vector<float> a(d);
        RDT_CUDA_TRY(cudaMemcpy(a.data(), w->A, d * sizeof(float), cudaMemcpyDeviceToHost));
        float rho = 0.0f;
        for (float v : a) {
            if (!std::isfinite(v)) {
                set_error("A has a non-finite entry");
                return RDT_ERR_UNSTABLE_A;
            }
            rho = std::max(rho, std::fabs(v));
        }
        h->rho = rho;
        if (rho >= 1.0f) {
            set_error("rho(A) = " + std::to_string(rho) + " >= 1: the loop would not be stable");
            return RDT_ERR_UNSTABLE_A;
        }
    }

    // ---- weights
    RDT_TRY(dev_alloc(h, &h->A, d * 4));
    RDT_TRY(copy_d2d(h->A, w->A, d * 4, st));
    const size_t bsz = c.b_kind == RDT_B_DIAG ? d * 4 : static_cast<size_t>(d) * d * 4;
    RDT_TRY(dev_alloc(h, &h->Bw, bsz));
    RDT_TRY(copy_d2d(h->Bw, w->B, bsz, st));
    RDT_TRY(dev_alloc(h, &h->g1, d * 4));
    RDT_TRY(copy_d2d(h->g1, w->norm1, d * 4, st));
    RDT_TRY(dev_alloc(h, &h->g2, d * 4));
    RDT_TRY(copy_d2d(h->g2, w->norm2, d * 4, st));
    RDT_TRY(dev_alloc(h, &h->wr, static_cast<size_t>(E) * d * es));
    RDT_TRY(copy_d2d(h->wr, w->w_router, static_cast<size_t>(E) * d * es, st));
    if (w->router_bias) {
        RDT_TRY(dev_alloc(h, &h->rbias, E * 4));
        RDT_TRY(copy_d2d(h->rbias, w->router_bias, E * 4, st));
    }
    if (h->bf) {
        const long grows = static_cast<long>(N) * (K + S);
        const int mode = c.gemm_tiles;
        const int kb_d = static_cast<int>(d * es / 128), kb_h = static_cast<int>(hid * es / 128);
        const int ow = c.attn_type == RDT_GQA ? c.n_heads * c.head_dim : c.n_heads * c.kv_lora_rank;
        // SwiGLU tiles hold BN/2 gate and BN/2 up columns; W1/W3 are interleaved in blocks
        // of BN/2 rows, which must divide the hidden width
        TileChoice t = choose_tiles(grows, E + S, 2 * hid, kb_d, hid % 128 == 0, false, hid % 64 == 0, 1, mode);
        h->bn_up = t.bn;
        h->pair_up = t.pair;
        // the down-projection's epilogue reduces every output into h_next. CTA pairs load a
        // third less per SM (their B rows are split) and measured faster with many routed
        // rows (65536 rows: 191 -> 179 us; 36864: 116 -> 113 us), not with few (4096 rows:
        // the same), so pairs are allowed from 16384 rows on.
        // deterministic mode: no K split (its partial sums would meet in atomics)
        t = choose_tiles(grows, E + S, d, kb_h, true, false, mode == 2 || (mode == 0 && grows >= 16384),
                         c.deterministic ? 1 : 4, mode);
        h->bn_down = t.bn;
        h->pair_down = t.pair;
        h->split_down = t.split;
        t = choose_tiles(N, 0, d, static_cast<int>(ow * es / 128), true, false, true, 1, mode);
        h->bn_o = t.bn;
        h->pair_o = t.pair;
        if (c.attn_type == RDT_GQA) {
            const int nqkv = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
            t = choose_tiles(N, 0, nqkv, kb_d, nqkv % 256 == 0, 192 % c.head_dim == 0, true, 1, mode);
            h->bn_qkv = t.bn;
            h->pair_qkv = t.pair;
        }
    }
    const size_t wexp = static_cast<size_t>(hid) * d * es;   // one expert matrix
    RDT_TRY(dev_alloc(h, &h->w13, 2 * wexp * (E + S)));
    RDT_TRY(dev_alloc(h, &h->w2, wexp * (E + S)));
    for (int e = 0; e < E; ++e) {
        RDT_TRY(interleave_w13(static_cast<char*>(h->w13) + 2 * wexp * e,
                               static_cast<const char*>(w->w1) + wexp * e,
                               static_cast<const char*>(w->w3) + wexp * e, hid, d, es, h->bn_up / 2, st));
    }
    RDT_TRY(copy_d2d(h->w2, w->w2, wexp * E, st));
    for (int s = 0; s < S; ++s) {
        RDT_TRY(interleave_w13(static_cast<char*>(h->w13) + 2 * wexp * (E + s),
                               static_cast<const char*>(w->ws1) + wexp * s,
                               static_cast<const char*>(w->ws3) + wexp * s, hid, d, es, h->bn_up / 2, st));
    }
    if (S) RDT_TRY(copy_d2d(static_cast<char*>(h->w2) + wexp * E, w->ws2, wexp * S, st));

    if (c.attn_type == RDT_GQA) {
        h->nq = c.n_heads * c.head_dim;
        h->nkv = c.n_kv_heads * c.head_dim;
        h->nqkv = h->nq + 2 * h->nkv;
        h->owidth = h->nq;
        h->rot = c.head_dim;
        // one weight set per adapter: W_q,l = W_q + B_l A_l and W_o,l = W_o + B'_l A'_l, summed
        // in fp32 and rounded once to the element type
        const int L = c.n_lora ? c.n_lora : 1, r = c.lora_rank;
        h->n_wsets = L;
        const size_t qkv_set = static_cast<size_t>(h->nqkv) * d * es, o_set = static_cast<size_t>(d) * h->nq * es;
        RDT_TRY(dev_alloc(h, &h->wqkv, qkv_set * L));
        RDT_TRY(dev_alloc(h, &h->wo, o_set * L));
        for (int l = 0; l < L; ++l) {
            char* q = static_cast<char*>(h->wqkv) + qkv_set * l;
            char* o = static_cast<char*>(h->wo) + o_set * l;
            if (c.n_lora) {
                const char* qa = static_cast<const char*>(w->lq_a) + static_cast<size_t>(l) * r * d * es;
                const char* qb = static_cast<const char*>(w->lq_b) + static_cast<size_t>(l) * h->nq * r * es;
                const char* oa = static_cast<const char*>(w->lo_a) + static_cast<size_t>(l) * r * h->nq * es;
                const char* ob = static_cast<const char*>(w->lo_b) + static_cast<size_t>(l) * d * r * es;
                // C[m, n] = W[m, n] + sum_k B[m, k] A[k, n]
                RDT_TRY(prep_matmul(h->bf, qb, r, 1, qa, d, 1, q, d, h->nq, d, r, st, w->wq, d));
                RDT_TRY(prep_matmul(h->bf, ob, r, 1, oa, h->nq, 1, o, h->nq, d, h->nq, r, st, w->wo, h->nq));
            } else {
                RDT_TRY(copy_d2d(q, w->wq, static_cast<size_t>(h->nq) * d * es, st));
                RDT_TRY(copy_d2d(o, w->wo, o_set, st));
            }
            RDT_TRY(copy_d2d(q + static_cast<size_t>(h->nq) * d * es, w->wk, static_cast<size_t>(h->nkv) * d * es, st));
            RDT_TRY(copy_d2d(q + static_cast<size_t>(h->nq + h->nkv) * d * es, w->wv,
                             static_cast<size_t>(h->nkv) * d * es, st));
        }
    } else {
        const int H = c.n_heads, ql = c.q_lora_rank, kvl = c.kv_lora_rank, rp = c.qk_rope_dim;
        const int nope = c.qk_nope_dim, vd = c.v_head_dim;
        h->lat_w = ql + kvl + rp;
        h->qt_w = H * (kvl + rp);
        h->owidth = H * kvl;
        h->rot = rp;
        RDT_TRY(dev_alloc(h, &h->q_norm, ql * 4));
        RDT_TRY(copy_d2d(h->q_norm, w->q_norm, ql * 4, st));
        RDT_TRY(dev_alloc(h, &h->kv_norm, kvl * 4));
        RDT_TRY(copy_d2d(h->kv_norm, w->kv_norm, kvl * 4, st));
        // [W_dq; W_dkv; W_kr] -> one latent projection
        RDT_TRY(dev_alloc(h, &h->wlat, static_cast<size_t>(h->lat_w) * d * es));
        char* wl = static_cast<char*>(h->wlat);
        RDT_TRY(copy_d2d(wl, w->w_dq, static_cast<size_t>(ql) * d * es, st));
        RDT_TRY(copy_d2d(wl + static_cast<size_t>(ql) * d * es, w->w_dkv, static_cast<size_t>(kvl) * d * es, st));
        RDT_TRY(copy_d2d(wl + static_cast<size_t>(ql + kvl) * d * es, w->w_kr, static_cast<size_t>(rp) * d * es, st));
        // absorbed query projection, per head: rows [0, kvl) = W_uk,h^T W_uq_nope,h;
        // rows [kvl, kvl + rope) = W_uq_rope,h
        RDT_TRY(dev_alloc(h, &h->wqabs, static_cast<size_t>(h->qt_w) * ql * es));
        for (int hh = 0; hh < H; ++hh) {
            const char* uk = static_cast<const char*>(w->w_uk) + static_cast<size_t>(hh) * nope * kvl * es;
            const char* uq = static_cast<const char*>(w->w_uq) + static_cast<size_t>(hh) * (nope + rp) * ql * es;
            char* dst = static_cast<char*>(h->wqabs) + static_cast<size_t>(hh) * (kvl + rp) * ql * es;
            RDT_TRY(prep_matmul(h->bf, uk, 1, kvl, uq, ql, 1, dst, ql, kvl, ql, nope, st));
            RDT_TRY(copy_d2d(dst + static_cast<size_t>(kvl) * ql * es, uq + static_cast<size_t>(nope) * ql * es,
                             static_cast<size_t>(rp) * ql * es, st));
        }
        // absorbed output projection: W_o~[:, h*kvl + c] = sum_v W_o[:, h*vd + v] W_uv[h*vd + v, c]
        RDT_TRY(dev_alloc(h, &h->wo, static_cast<size_t>(d) * h->owidth * es));
        for (int hh = 0; hh < H; ++hh) {
            const char* wo = static_cast<const char*>(w->wo) + static_cast<size_t>(hh) * vd * es;
            const char* uv = static_cast<const char*>(w->w_uv) + static_cast<size_t>(hh) * vd * kvl * es;
            char* dst = static_cast<char*>(h->wo) + static_cast<size_t>(hh) * kvl * es;
            RDT_TRY(prep_matmul(h->bf, wo, static_cast<long>(H) * vd, 1, uv, kvl, 1, dst, h->owidth, d, kvl, vd, st));
        }
    }

    // RoPE tables [rot/2][s_cap] (frequency-major, so that consecutive positions are adjacent)
    // from double-precision angles, for every position a sequence may reach
    // (context parallelism: this rank's positions start at cp_rank * seq)
    h->cp_size = c.cp_size > 1 ? c.cp_size : 1;
    h->cp_rank = c.cp_size > 1 ? c.cp_rank : 0;
    h->s_cap = c.seq * h->cp_size + c.max_decode;
    {
        const int half = h->rot / 2;
        const int P = h->s_cap;
        std::vector<float> cs(static_cast<size_t>(P) * half), sn(cs.size());
        for (int i = 0; i < half; ++i)
            for (int p = 0; p < P; ++p) {
                const double ang = p * std::pow(static_cast<double>(c.rope_base), -2.0 * i / h->rot);
                cs[static_cast<size_t>(i) * P + p] = static_cast<float>(std::cos(ang));
                sn[static_cast<size_t>(i) * P + p] = static_cast<float>(std::sin(ang));
            }
        RDT_TRY(dev_alloc(h, &h->rope_cos, cs.size() * 4));
        RDT_TRY(dev_alloc(h, &h->rope_sin, sn.size() * 4));
        RDT_CUDA_TRY(cudaMemcpy(h->rope_cos, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice));
        RDT_CUDA_TRY(cudaMemcpy(h->rope_sin, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice));
    }

    // ---- workspace
    const size_t nd = static_cast<size_t>(N) * d;
    RDT_TRY(dev_alloc(h, &h->hbuf[0], nd * 4));
    RDT_TRY(dev_alloc(h, &h->hbuf[1], nd * 4));
    RDT_TRY(dev_alloc(h, &h->Be, nd * 4));
    RDT_TRY(dev_alloc(h, &h->y, nd * 4));
    RDT_TRY(dev_alloc(h, &h->xn, nd * es));
    if (c.attn_type == RDT_GQA) {
        RDT_TRY(dev_alloc(h, &h->qkv, static_cast<size_t>(N) * h->nqkv * es));
    } else {
        RDT_TRY(dev_alloc(h, &h->lat, static_cast<size_t>(N) * h->lat_w * 4));
        RDT_TRY(dev_alloc(h, &h->cq, static_cast<size_t>(N) * c.q_lora_rank * es));
        RDT_TRY(dev_alloc(h, &h->kvlat, static_cast<size_t>(N) * (c.kv_lora_rank + c.qk_rope_dim) * es));
        RDT_TRY(dev_alloc(h, &h->qkv, static_cast<size_t>(N) * h->qt_w * es));
    }
    RDT_TRY(dev_alloc(h, &h->o, static_cast<size_t>(N) * h->owidth * es));
    // groups are `cap` rows apart: the token count rounded up plus 64 rows, so that group
    // bases do not all fall on the same large power-of-two stride
    h->cap = (N + 63) / 64 * 64 + 64;
    // Rows of an expert group beyond its count are read by the group's last (partial) tile
    // and masked in its epilogue. They hold a non-zero filler (bytes 0x3F: 0.746 in bf16):
    // measured on B200, tiles whose padding rows are exact zeros run the grouped GEMMs
    // 1.6-1.8x slower than tiles padded with any non-zero value.
    // The last group's last tile may reach up to 255 rows past its group: kFillerRows more
    // rows of filler keep those reads inside the buffers (no zero fill from out-of-range TMA).
    RDT_TRY(dev_alloc(h, &h->xperm, (static_cast<size_t>(N) + static_cast<size_t>(h->cap) * E + kFillerRows) * d * es,
                      true, 0x3F));
    RDT_TRY(dev_alloc(h, &h->U, (static_cast<size_t>(h->cap) * (S + E) + kFillerRows) * hid * es, true, 0x3F));
    RDT_TRY(dev_alloc(h, &h->yn_lo, nd * es, true));
    h->bn_router = E <= 64 ? 64 : E <= 128 ? 128 : 256;
    if (h->bf) {
        // split the router's K blocks (2 d * 2 B / 128 B) so that the row tiles fill the GPU
        const int mt = (N + 127) / 128;
        const int kb = 2 * d * 2 / 128;
        int split = 1;
        // deterministic: logits in one CTA; the split's final read takes 16-byte row pieces,
        // so the expert count must be a multiple of 4
        for (int sp = 1; sp <= kb && !c.deterministic && E % 4 == 0; ++sp)
            if (kb % sp == 0 && static_cast<long>(mt) * sp <= num_sms()) split = sp;
        h->router_split = split;
        // a decode step routes batch rows: one row tile, so the K blocks spread over many CTAs
        int split_dec = 1;
        const int mt_dec = (c.batch + 127) / 128;
        for (int sp = 1; sp <= kb && c.max_decode > 0 && !c.deterministic && E % 4 == 0; ++sp)
            if (kb % sp == 0 && static_cast<long>(mt_dec) * sp <= num_sms()) split_dec = sp;
        h->router_split_dec = split_dec;
        RDT_TRY(dev_alloc(h, &h->logits, static_cast<size_t>(N) * E * 4, true));
        RDT_TRY(dev_alloc(h, &h->tile_count, static_cast<size_t>(mt) * 4 * 4, true));   // per 32 rows
    }
    RDT_TRY(dev_alloc(h, &h->idx, static_cast<size_t>(N) * K * 4));
    RDT_TRY(dev_alloc(h, &h->wts, static_cast<size_t>(N) * K * 4));
    RDT_TRY(dev_alloc(h, &h->counts, 256 * 4, true));
    RDT_TRY(dev_alloc(h, &h->row_token, static_cast<size_t>(h->cap) * E * 4, true));
    RDT_TRY(dev_alloc(h, &h->row_w, static_cast<size_t>(h->cap) * E * 4, true));
    RDT_TRY(dev_alloc(h, &h->slot_row, static_cast<size_t>(N) * K * 4, true));
    h->max_tiles = (N * K + 127) / 128 + E + S * ((N + 127) / 128);
    h->max_tiles_pair = (N * K + 255) / 256 + E + S * ((N + 255) / 256);
    RDT_TRY(dev_alloc(h, &h->flags, FLAG_COUNT * 4, true));
    if (c.deterministic)
        RDT_TRY(dev_alloc(h, &h->det_rows, static_cast<size_t>(h->cap) * (S + E) * d * 4));
    if (c.da_heads) {
        h->nq_d = c.da_heads * c.head_dim;
        h->nkv_d = c.da_kv_heads * c.head_dim;
        h->nqkv_d = h->nq_d + 2 * h->nkv_d;
        RDT_TRY(dev_alloc(h, &h->g_da, d * 4));
        RDT_TRY(copy_d2d(h->g_da, w->norm_da, d * 4, st));
        RDT_TRY(dev_alloc(h, &h->wqkv_d, static_cast<size_t>(h->nqkv_d) * d * es));
        char* q = static_cast<char*>(h->wqkv_d);
        RDT_TRY(copy_d2d(q, w->wq_d, static_cast<size_t>(h->nq_d) * d * es, st));
        RDT_TRY(copy_d2d(q + static_cast<size_t>(h->nq_d) * d * es, w->wk_d, static_cast<size_t>(h->nkv_d) * d * es, st));
        RDT_TRY(copy_d2d(q + static_cast<size_t>(h->nq_d + h->nkv_d) * d * es, w->wv_d,
                         static_cast<size_t>(h->nkv_d) * d * es, st));
        RDT_TRY(dev_alloc(h, &h->wo_d, static_cast<size_t>(d) * h->nq_d * es));
        RDT_TRY(copy_d2d(h->wo_d, w->wo_d, static_cast<size_t>(d) * h->nq_d * es, st));
        RDT_TRY(dev_alloc(h, &h->qkv_d, static_cast<size_t>(N) * h->nqkv_d * es));
        RDT_TRY(dev_alloc(h, &h->o_d, static_cast<size_t>(N) * h->nq_d * es));
        RDT_TRY(dev_alloc(h, &h->depth_cache, static_cast<size_t>(N) * c.max_loops * 2 * h->nkv_d * es));
        // rotation of loop t of T: pairs i < head_dim/4 at t, the others at T - 1 - t
        const int half = c.head_dim / 2, L = c.max_loops;
        std::vector<float> dc(static_cast<size_t>(L) * L * half, 0.0f), ds(dc.size(), 0.0f);
        for (int T = 1; T <= L; ++T)
            for (int t = 0; t < T; ++t)
                for (int i = 0; i < half; ++i) {
                    const double pos = i < c.head_dim / 4 ? t : T - 1 - t;
                    const double ang = pos * std::pow(static_cast<double>(c.rope_base), -2.0 * i / c.head_dim);
                    const size_t o = (static_cast<size_t>(T - 1) * L + t) * half + i;
                    dc[o] = static_cast<float>(std::cos(ang));
                    ds[o] = static_cast<float>(std::sin(ang));
                }
        RDT_TRY(dev_alloc(h, &h->dtab_cos, dc.size() * 4));
        RDT_TRY(dev_alloc(h, &h->dtab_sin, ds.size() * 4));
        RDT_CUDA_TRY(cudaMemcpy(h->dtab_cos, dc.data(), dc.size() * 4, cudaMemcpyHostToDevice));
        RDT_CUDA_TRY(cudaMemcpy(h->dtab_sin, ds.data(), ds.size() * 4, cudaMemcpyHostToDevice));
        std::vector<int> idx(L);
        for (int t = 0; t < L; ++t) idx[t] = t;
        RDT_TRY(dev_alloc(h, &h->didx, L * 4));
        RDT_CUDA_TRY(cudaMemcpy(h->didx, idx.data(), L * 4, cudaMemcpyHostToDevice));
    }
    if (c.max_decode > 0) {
        h->cache_w = c.attn_type == RDT_GQA ? 2 * c.n_kv_heads * c.head_dim : c.kv_lora_rank + c.qk_rope_dim;
        RDT_TRY(dev_alloc(h, &h->kv_cache,
                          static_cast<size_t>(c.max_loops) * c.batch * h->s_cap * h->cache_w * es));
        RDT_TRY(dev_alloc(h, &h->dec_len, 16, true));
        const int dv = c.attn_type == RDT_GQA ? c.head_dim : c.kv_lora_rank;
        RDT_TRY(dev_alloc(h, &h->dec_part, static_cast<size_t>(c.batch) * c.n_heads * decode_chunks(h->s_cap) *
                                               (dv + 2) * 4));
    }
    if (h->cp_size > 1) {
        // zeroed: rows no rank writes here (later ranks' positions) meet P = 0 in the PV
        // product, and 0 * garbage could be NaN
        RDT_TRY(dev_alloc(h, &h->cp_kv, static_cast<size_t>(c.batch) * h->s_cap * 2 * c.n_kv_heads * c.head_dim * es,
                          true));
        RDT_TRY(dev_alloc(h, &h->cp_flags, 256, true));
        h->cp_peer_kv[h->cp_rank] = h->cp_kv;
        h->cp_peer_flags[h->cp_rank] = h->cp_flags;
    }
    RDT_TRY(dev_alloc(h, &h->stage_h0, nd * es));
    RDT_TRY(dev_alloc(h, &h->stage_e, nd * es));
    RDT_TRY(dev_alloc(h, &h->stage_out, nd * 4));

    RDT_TRY(build_maps(h));
    RDT_CUDA_TRY(cudaStreamSynchronize(st));
    return RDT_OK;
}

int lora_index(const rdt_handle* h, int t) { return std::min(t, h->cfg.n_lora - 1); }

// The O-projection epilogue's inputs for y = x + acc and h_next = A (.) h + B.e + acc, x = h
// (+ e when the block input includes it): a diagonal B is applied to e there, a dense B's
// product (or B.e when the block input leaves e out) comes from the hoisted Be.
void set_residual(const rdt_handle* h, const float* hin, const void* e, EpiParams& eo) {
    eo.h_in = hin;
    eo.e_in = e;
    eo.a_diag = h->A;
    eo.b_diag = h->cfg.b_kind == RDT_B_DIAG && e ? h->Bw : nullptr;
    eo.be = h->Be;
}

// ---- depth attention of loop t: RMSNorm_da(x) -> [q; k; v] with the depth rotation -> loop
// t's keys and values into the token's depth cache -> attention over loops 0 .. t -> output
// projection forming y = x + d and h_next = A h + B e + d
rdt_status depth_block(rdt_handle* h, const float* hin, const void* e, int t, float* h_next, cudaStream_t st) {
    const rdt_config& c = h->cfg;
    const int N = h->cur_ntok, d = c.dim;
    Norm1Args n1{};
    n1.h = hin;
    n1.e = e;
    n1.gamma = h->g_da;
    n1.xn = h->xn;
    n1.ntok = N;
    n1.dim = d;
    n1.eps = c.norm_eps;
    n1.zero_counts = h->counts;
    n1.n_zero = h->G;
    TIMED(h, K_NORM1, 1, st, norm1(h->bf, n1, st));

    GemmArgs ga{};
    ga.M = N;
    ga.N = h->nqkv_d;
    ga.kb_main = static_cast<int>(d * h->esz / 128);
    ga.flags = h->flags;
    EpiParams ep{};
    ep.flags = h->flags;
    ep.kind = EPI_ROPE;
    ep.out = h->qkv_d;
    ep.ldo = h->nqkv_d;
    ep.ncols_valid = h->nqkv_d;
    const size_t tab = (static_cast<size_t>(h->cur_T - 1) * c.max_loops + t) * (c.head_dim / 2);
    ep.rope_cos = h->dtab_cos + tab;   // one row: every token of loop t at the same depth
    ep.rope_sin = h->dtab_sin + tab;
    ep.seq = 1;
    ep.rope_ld = 1;
    ep.head_w = c.head_dim;
    ep.rot_off = 0;
    ep.rot_dim = c.head_dim;
    ep.rope_limit = h->nq_d + h->nkv_d;
    TIMED(h, K_DA_QKV, 1, st, gemm_tc(h->bf, 128, h->m_xn, h->m_wqkv_d, nullptr, nullptr, ga, ep, st));
    // loop t's keys and values: row (token, t) of the depth cache
    TIMED(h, K_CACHE, 1, st, cache_append(h->qkv_d, h->nqkv_d, h->nq_d, 2 * h->nkv_d, h->depth_cache, c.max_loops,
                                          1, h->didx + t, N, st));
    DepthAttnArgs da{};
    da.q = static_cast<const bf16*>(h->qkv_d);
    da.q_ld = h->nqkv_d;
    da.cache = static_cast<const bf16*>(h->depth_cache);
    da.cache_w = 2 * h->nkv_d;
    da.max_depth = c.max_loops;
    da.v_col0 = h->nkv_d;
    da.t = t;
    da.ntok = N;
    da.hq = c.da_heads;
    da.hkv = c.da_kv_heads;
    da.scale_log2 = 1.4426950408889634f / std::sqrt(static_cast<float>(c.head_dim));
    da.o = static_cast<bf16*>(h->o_d);
    da.o_ld = h->nq_d;
    TIMED(h, K_DA_ATTN, 1, st, depth_attention(da, st));

    GemmArgs go{};
    go.M = N;
    go.N = d;
    go.kb_main = static_cast<int>(h->nq_d * h->esz / 128);
    go.flags = h->flags;
    EpiParams eo{};
    eo.flags = h->flags;
    eo.kind = EPI_OPROJ_LOOP;
    eo.ncols_valid = d;
    eo.y = h->y;
    eo.h_next = h_next;
    eo.ld = d;
    set_residual(h, hin, e, eo);   // y = x + d, h_next = A h + B.e + d
    TIMED(h, K_DA_O, 1, st, gemm_tc(h->bf, 128, h->m_od, h->m_wo_d, nullptr, nullptr, go, eo, st));
    return RDT_OK;
}

// ---- the attention sublayer: norm1 -> projections -> attention -> O projection
rdt_status attention_block(rdt_handle* h, const float* hin, const void* e, int t, bool loop_mode,
                           float* a_out, float* h_next, cudaStream_t st) {
    const rdt_config& c = h->cfg;
    const int N = h->cur_ntok, d = c.dim;
    const bool lora = c.n_lora > 0;
    const int li = lora ? lora_index(h, t) : 0;
    const bool step = h->mode == 2;
    // positions: a prompt row r sits at r % seq; a decode step's row b at the cached length
    const int pos_seq = step ? 1 : c.seq;
    const int* pos_dev = step ? h->dec_len : nullptr;
    void* cache_t = h->mode ? static_cast<char*>(h->kv_cache) +
                                  static_cast<size_t>(t) * c.batch * h->s_cap * h->cache_w * h->esz
                            : nullptr;

    const bool depth = c.da_heads > 0 && loop_mode;
    if (depth) RDT_TRY(depth_block(h, hin, e, t, h_next, st));
    Norm1Args n1{};
    n1.h = depth ? h->y : hin;          // with depth attention: x' = x + d, complete in y
    n1.e = depth ? nullptr : e;
    n1.gamma = h->g1;
    n1.xn = h->xn;
    n1.ntok = N;
    n1.dim = d;
    n1.eps = c.norm_eps;
    if (loop_mode && !depth) {          // (the depth block's RMSNorm did this)
        n1.zero_counts = h->counts;
        n1.n_zero = h->G;
    }
    TIMED(h, K_NORM1, 1, st, norm1(h->bf, n1, st));

    GemmArgs ga{};
    ga.M = N;
    ga.flags = h->flags;
    EpiParams ep{};
    ep.flags = h->flags;
    AttnArgs at{};
    at.batch = c.batch;
    at.seq = c.seq;
    at.hq = c.n_heads;
    at.o = h->o;
    at.ldo = h->owidth;
    if (c.attn_type == RDT_GQA) {
        ga.N = h->nqkv;
        ga.kb_main = static_cast<int>(d * h->esz / 128);
        ga.pair = h->pair_qkv;
        ep.kind = EPI_ROPE;
        ep.out = h->qkv;
        ep.ldo = h->nqkv;
        ep.ncols_valid = h->nqkv;
        ep.rope_cos = h->rope_cos;
        ep.rope_sin = h->rope_sin;
        ep.seq = pos_seq;
        ep.pos_dev = pos_dev;
        ep.rope_ld = h->s_cap;
        ep.head_w = c.head_dim;
        ep.rot_off = 0;
        ep.rot_dim = c.head_dim;
        ep.rope_limit = h->nq + h->nkv;
        const bool cp = h->cp_size > 1;
        CpSyncArgs cs{};
        if (cp) {
            // this rank's positions start at cp_rank * seq; its rotated keys and values also go
            // to the gather buffers of this rank and the later ones (the causal mask gives rank
            // q the keys of ranks 0 .. q), once those have finished with the previous loop's
            cs.flags = h->cp_flags;
            for (int q = 0; q < h->cp_size; ++q) cs.peer_flags[q] = h->cp_peer_flags[q];
            cs.rank = h->cp_rank;
            cs.size = h->cp_size;
            cs.status = h->flags;
            TIMED(h, K_CP_SYNC, 1, st, cp_wait_consumed(cs, st));
            ep.pos_off = h->cp_rank * c.seq;
            ep.cp_n = h->cp_size - h->cp_rank;
            for (int q = h->cp_rank; q < h->cp_size; ++q) ep.cp_dst[q - h->cp_rank] = h->cp_peer_kv[q];
            ep.cp_col0 = h->nq;
            ep.cp_w = 2 * h->nkv;
            ep.cp_seq_tot = h->cp_size * c.seq;
            ep.cp_row_off = h->cp_rank * c.seq;
        }
        TIMED(h, K_GEMM_QKV, 1, st, gemm_tc(h->bf, h->bn_qkv, h->m_xn, h->m_wqkv[li], nullptr, nullptr, ga, ep, st));
        if (cp) TIMED(h, K_CP_SYNC, 1, st, cp_ready(cs, st));
        if (cache_t)   // loop t's rotated keys and values of these positions: [K | V] per row
            TIMED(h, K_CACHE, 1, st, cache_append(h->qkv, h->nqkv, h->nq, h->cache_w, cache_t, h->s_cap, pos_seq,
                                                  pos_dev, N, st));
        at.q = h->qkv;
        at.ldq = h->nqkv;
        at.q_hstride = c.head_dim;
        at.k = static_cast<const char*>(h->qkv) + static_cast<size_t>(h->nq) * h->esz;
        at.ldk = h->nqkv;
        at.k_hstride = c.head_dim;
        at.v = static_cast<const char*>(h->qkv) + static_cast<size_t>(h->nq + h->nkv) * h->esz;
        at.ldv = h->nqkv;
        at.v_hstride = c.head_dim;
        at.hkv = c.n_kv_heads;
        at.dqk = c.head_dim;
        at.dv = c.head_dim;
        at.scale = 1.0f / std::sqrt(static_cast<float>(c.head_dim));
        if (cp) {   // every rank's keys and values up to this rank's positions, from the gather buffer
            at.k = h->cp_kv;
            at.ldk = 2 * h->nkv;
            at.v = static_cast<const char*>(h->cp_kv) + static_cast<size_t>(h->nkv) * h->esz;
            at.ldv = 2 * h->nkv;
            at.q_off = h->cp_rank * c.seq;
            at.kv_seq = h->cp_size * c.seq;
        }
    } else {
        const int ql = c.q_lora_rank, kvl = c.kv_lora_rank, rp = c.qk_rope_dim;
        // latent projection -> fp32 [N, ql + kvl + rope]
        ga.N = h->lat_w;
        ga.kb_main = static_cast<int>(d * h->esz / 128);
        ep.kind = EPI_STORE_F32;
        ep.out = h->lat;
        ep.ldo = h->lat_w;
        ep.ncols_valid = h->lat_w;
        TIMED(h, K_GEMM_LAT, 1, st, gemm_tc(h->bf, 128, h->m_xn, h->m_wlat, nullptr, nullptr, ga, ep, st));
        MlaNormArgs mn{};
        mn.lat = h->lat;
        mn.ld_lat = h->lat_w;
        mn.q_norm = h->q_norm;
        mn.kv_norm = h->kv_norm;
        mn.cq = h->cq;
        mn.kv = h->kvlat;
        mn.rope_cos = h->rope_cos;
        mn.rope_sin = h->rope_sin;
        mn.ntok = N;
        mn.seq = pos_seq;
        mn.pos_dev = pos_dev;
        mn.rope_ld = h->s_cap;
        mn.q_lat = ql;
        mn.kv_lat = kvl;
        mn.rope = rp;
        mn.eps = c.norm_eps;
        TIMED(h, K_MLA_NORM, 1, st, mla_latent_norm(h->bf, mn, st));
        if (cache_t)   // loop t's normalised latent and rotated shared key: [c_kv | k_rope] per row
            TIMED(h, K_CACHE, 1, st, cache_append(h->kvlat, kvl + rp, 0, h->cache_w, cache_t, h->s_cap, pos_seq,
                                                  pos_dev, N, st));
        // absorbed query projection with RoPE on the last rope columns of each head
        GemmArgs gq{};
        gq.M = N;
        gq.N = h->qt_w;
        gq.kb_main = static_cast<int>(ql * h->esz / 128);
        gq.flags = h->flags;
        EpiParams eq{};
        eq.flags = h->flags;
        eq.kind = EPI_ROPE;
        eq.out = h->qkv;
        eq.ldo = h->qt_w;
        eq.ncols_valid = h->qt_w;
        eq.rope_cos = h->rope_cos;
        eq.rope_sin = h->rope_sin;
        eq.seq = pos_seq;
        eq.pos_dev = pos_dev;
        eq.rope_ld = h->s_cap;
        eq.head_w = kvl + rp;
        eq.rot_off = kvl;
        eq.rot_dim = rp;
        eq.rope_limit = h->qt_w;
        TIMED(h, K_GEMM_Q, 1, st, gemm_tc(h->bf, 160, h->m_cq, h->m_wqabs, nullptr, nullptr, gq, eq, st));
        at.q = h->qkv;
        at.ldq = h->qt_w;
        at.q_hstride = kvl + rp;
        at.k = h->kvlat;
        at.ldk = kvl + rp;
        at.k_hstride = 0;
        at.v = h->kvlat;
        at.ldv = kvl + rp;
        at.v_hstride = 0;
        at.hkv = 1;
        at.dqk = kvl + rp;
        at.dv = kvl;
        at.scale = 1.0f / std::sqrt(static_cast<float>(c.qk_nope_dim + rp));
    }
    at.flags = h->flags;
    if (step) {
        // one new query per sequence against loop t's cache (positions 0 .. length)
        DecodeAttnArgs da{};
        da.q = at.q;
        da.q_ld = at.ldq;
        da.q_hstride = at.q_hstride;
        da.cache = cache_t;
        da.cache_ld = h->cache_w;
        da.s_cap = h->s_cap;
        if (c.attn_type == RDT_GQA) {
            da.k_col0 = 0;
            da.k_hstride = c.head_dim;
            da.v_col0 = h->nkv;
            da.v_hstride = c.head_dim;
        } else {          // the shared latent: keys the whole row, values its first kv_lat columns
            da.k_col0 = 0;
            da.k_hstride = 0;
            da.v_col0 = 0;
            da.v_hstride = 0;
        }
        da.batch = c.batch;
        da.hq = c.n_heads;
        da.hkv = at.hkv;
        da.dqk = at.dqk;
        da.dv = at.dv;
        da.len_dev = h->dec_len;
        da.scale = at.scale;
        da.part = h->dec_part;
        da.o = h->o;
        da.ldo = h->owidth;
        da.dv_out = at.dv;
        TIMED(h, K_DEC_ATTN, 2, st, decode_attention(da, st));
    } else {
        TIMED(h, K_ATTENTION, 1, st, attention(h->bf, at, st));
        if (h->cp_size > 1) {
            CpSyncArgs cs{};
            cs.flags = h->cp_flags;
            for (int q = 0; q < h->cp_size; ++q) cs.peer_flags[q] = h->cp_peer_flags[q];
            cs.rank = h->cp_rank;
            cs.size = h->cp_size;
            cs.status = h->flags;
            TIMED(h, K_CP_SYNC, 1, st, cp_consumed(cs, st));
        }
    }

    GemmArgs go{};
    go.M = N;
    go.N = d;
    go.kb_main = static_cast<int>(h->owidth * h->esz / 128);
    go.pair = h->pair_o;
    go.flags = h->flags;
    EpiParams eo{};
    eo.flags = h->flags;
    eo.ncols_valid = d;
    if (loop_mode) {
        eo.kind = EPI_OPROJ_LOOP;
        eo.y = h->y;
        eo.h_next = h_next;
        eo.ld = d;
        // without depth attention the O projection forms y and h_next from h and e; after
        // it, both already hold x + d and A h + B.e + d, and a is added in
        if (!depth) set_residual(h, hin, e, eo);
    } else {
        eo.kind = EPI_OPROJ_PLAIN;
        eo.out = a_out;
        eo.ldo = d;
    }
    TIMED(h, K_GEMM_O, 1, st, gemm_tc(h->bf, h->bn_o, h->m_o, h->m_wo[li], nullptr, nullptr, go, eo, st));
    return RDT_OK;
}

// ---- the MoE sublayer: norm2 + router (the fused shared-memory router, or RMSNorm2 and the
// tensor-core router with its top-k epilogue, or the fp32 FMA router) -> dispatch -> experts;
// adds into dst. With `halted` (ACT), tokens whose entry is nonzero are routed nowhere.
rdt_status moe_block(rdt_handle* h, const float* yin, float* dst, int32_t* idx_out, float* w_out,
                     int32_t* tr_idx, float* tr_w, const int* halted, cudaStream_t st) {
    const rdt_config& c = h->cfg;
    // N: tokens of this call; NL: the capacity layout's row base (expert rows start after it)
    const int N = h->cur_ntok, NL = h->ntok, d = c.dim, hid = c.expert_hidden;
    int32_t* idx = idx_out ? idx_out : h->idx;
    float* wts = w_out ? w_out : h->wts;
    bool copies_written = false;
    if (router_fits_smem(h->bf, c.n_experts, c.top_k, d)) {
        // small router: RMSNorm2, fp32 logits, top-k and the experts' row copies in one
        // kernel, W_r staged in shared memory
        RouterArgs ra{};
        ra.y = yin;
        ra.gamma = h->g2;
        ra.yn = h->xperm;
        ra.ntok = N;
        ra.dim = d;
        ra.eps = c.norm_eps;
        ra.w_router = h->wr;
        ra.bias = h->rbias;
        ra.n_exp = c.n_experts;
        ra.top_k = c.top_k;
        ra.idx = idx;
        ra.w = wts;
        ra.counts = h->counts;
        ra.trace_idx = tr_idx;
        ra.trace_w = tr_w;
        ra.row_token = h->row_token;
        ra.row_w = h->row_w;
        ra.cap = h->cap;
        ra.xperm = h->xperm;
        ra.a_routed_base = NL;
        ra.store_yn = c.n_shared > 0;          // shared experts read yn itself
        if (h->det_rows) ra.slot_row = h->slot_row;   // the combine finds each slot's row
        ra.weights_static = 1;                 // the library's own copy, written at create
        ra.halted = halted;
        TIMED(h, K_ROUTER, 1, st, norm2_router_smem(h->bf, ra, st));
        copies_written = true;
    } else if (!h->bf) {
        // fp32: the tensor cores would read W_r as tf32, so the router stays in fp32 FMA
        RouterArgs ra{};
        ra.y = yin;
        ra.gamma = h->g2;
        ra.yn = h->xperm;
        ra.ntok = N;
        ra.dim = d;
        ra.eps = c.norm_eps;
        ra.w_router = h->wr;
        ra.bias = h->rbias;
        ra.n_exp = c.n_experts;
        ra.top_k = c.top_k;
        ra.idx = idx;
        ra.w = wts;
        ra.counts = h->counts;
        ra.trace_idx = tr_idx;
        ra.trace_w = tr_w;
        ra.row_token = h->row_token;
        ra.row_w = h->row_w;
        ra.slot_row = h->slot_row;
        ra.cap = h->cap;
        ra.halted = halted;
        TIMED(h, K_ROUTER, 1, st, norm2_router(false, ra, st));
    } else {
        Norm2Args n2{};
        n2.y = yin;
        n2.gamma = h->g2;
        n2.yn = h->xperm;
        n2.yn_lo = h->yn_lo;
        n2.ntok = N;
        n2.dim = d;
        n2.eps = c.norm_eps;
        const int rsplit = h->mode == 2 ? h->router_split_dec : h->router_split;
        if (rsplit > 1) {
            n2.zero_rows = h->logits;
            n2.zero_width = c.n_experts;
        }
        TIMED(h, K_NORM2, 1, st, norm2_split(h->bf, n2, st));

        GemmArgs gr{};
        gr.M = N;
        gr.N = c.n_experts;
        gr.kb_main = static_cast<int>(d * h->esz / 128);
        gr.kb_ext = gr.kb_main;
        gr.b2_row0 = 0;
        gr.split_k = rsplit;
        gr.flags = h->flags;
        EpiParams er{};
        er.kind = EPI_TOPK;
        er.n_exp = c.n_experts;
        er.top_k = c.top_k;
        er.bias = h->rbias;
        er.idx_out = idx;
        er.w_out = wts;
        er.counts = h->counts;
        er.trace_idx = tr_idx;
        er.trace_w = tr_w;
        er.logits = h->logits;
        er.tile_count = h->tile_count;
        er.route_token = h->row_token;
        er.route_w = h->row_w;
        er.slot_row = h->slot_row;
        er.cap = h->cap;
        er.halted = halted;
        er.flags = h->flags;
        TIMED(h, K_ROUTER, 1, st, gemm_tc(h->bf, h->bn_router, h->m_xperm, h->m_wr, &h->m_ynlo, &h->m_wr, gr, er, st));
    }
    if (!copies_written)
        TIMED(h, K_DISPATCH, 1, st, moe_copy(h->bf, h->xperm, h->slot_row, N, c.top_k, d, NL, st));

    GemmArgs gu{};
    gu.M = N;
    gu.N = 2 * hid;
    gu.kb_main = static_cast<int>(d * h->esz / 128);
    gu.counts = h->counts;
    gu.n_routed = c.n_experts;
    gu.n_shared = c.n_shared;
    gu.cap = h->cap;
    gu.a_routed_base = NL;
    gu.pair = h->pair_up;
    gu.max_tiles = h->pair_up ? h->max_tiles_pair : h->max_tiles;
    gu.flags = h->flags;
    EpiParams eu{};
    eu.kind = EPI_SWIGLU;
    eu.out = h->U;
    eu.ldo = hid;
    eu.ncols_valid = 2 * hid;
    eu.flags = h->flags;
    TIMED(h, K_GEMM_UP, 1, st, gemm_tc(h->bf, h->bn_up, h->m_xperm, h->m_w13, nullptr, nullptr, gu, eu, st));

    GemmArgs gd{};
    gd.M = N;
    gd.N = d;
    gd.kb_main = static_cast<int>(hid * h->esz / 128);
    gd.counts = h->counts;
    gd.n_routed = c.n_experts;
    gd.n_shared = c.n_shared;
    gd.cap = h->cap;
    gd.a_routed_base = NL;
    gd.pair = h->pair_down;
    gd.split_k = h->split_down;
    gd.max_tiles = h->pair_down ? h->max_tiles_pair : h->max_tiles;
    gd.a_from_c = 1;
    gd.flags = h->flags;
    EpiParams ed{};
    ed.kind = EPI_SCATTER;
    ed.ncols_valid = d;
    ed.row_token = h->row_token;
    ed.row_w = h->row_w;
    ed.shared_rows = c.n_shared * h->cap;
    ed.ntok = h->cap;
    ed.dst = dst;
    ed.ld = d;
    ed.rows_out = h->det_rows;
    ed.flags = h->flags;
    TIMED(h, K_GEMM_DOWN, 1, st, gemm_tc(h->bf, h->bn_down, h->m_U, h->m_w2, nullptr, nullptr, gd, ed, st));
    if (h->det_rows)
        TIMED(h, K_COMBINE, 1, st, moe_combine(h->det_rows, h->slot_row, N, c.top_k, c.n_shared, h->cap, dst, d, st));
    return RDT_OK;
}

// With act, every loop ends with the ACT step: h_{t+1} stays in the workspace, `out`
// collects the weighted states, halted tokens keep their state and are routed nowhere.
rdt_status loop_impl(rdt_handle* h, const void* h0, const void* e, int T, float* out, bool act,
                     int32_t* n_loops, cudaStream_t st) {
    const rdt_config& c = h->cfg;
    const int N = h->cur_ntok, d = c.dim;
    const size_t nd = static_cast<size_t>(N) * d;
    h->cur_T = T;
    // B.e is only kept for dense B or when the block input leaves e out (the O projection
    // forms a diagonal B's product from the e it reads)
    const bool keep_be = c.b_kind == RDT_B_DIAG && !c.inject_e;
    TIMED(h, K_HOIST, 1, st, hoist(h->bf, h0, e, keep_be ? h->Bw : nullptr, h->hbuf[0], h->Be, nd, d, st));
    if (c.b_kind == RDT_B_DENSE) TIMED(h, K_DENSE_B, 1, st, matmul_nt_simt(h->bf, e, h->Bw, h->Be, N, d, d, st));
    if (h->tr_h) RDT_CUDA_TRY(cudaMemcpyAsync(h->tr_h, h->hbuf[0], nd * 4, cudaMemcpyDeviceToDevice, st));
    for (int t = 0; t < T; ++t) {
        NvtxRange loop_range("rdt loop");
        float* hcur = h->hbuf[t & 1];
        float* hnext = (t == T - 1 && !act) ? out : h->hbuf[(t + 1) & 1];
        RDT_TRY(attention_block(h, hcur, c.inject_e ? e : nullptr, t, true, nullptr, hnext, st));
        const size_t tk = static_cast<size_t>(t) * h->ntok * c.top_k;   // trace layout [loops, batch * seq, k]
        RDT_TRY(moe_block(h, h->y, hnext, nullptr, nullptr, h->tr_idx ? h->tr_idx + tk : nullptr,
                          h->tr_w ? h->tr_w + tk : nullptr, act && t > 0 ? h->act_loops : nullptr, st));
        if (act) {
            ActArgs aa{};
            aa.h_cur = hcur;
            aa.h_next = hnext;
            aa.out = out;
            aa.w_halt = h->act_w;
            aa.b_halt = h->act_b;
            aa.threshold = h->act_thr;
            aa.cum = h->act_cum;
            aa.loops = h->act_loops;
            aa.ntok = N;
            aa.dim = d;
            aa.t = t;
            aa.last = t == T - 1;
            TIMED(h, K_ACT, 1, st, act_step(aa, st));
        }
        if (h->tr_h)
            RDT_CUDA_TRY(cudaMemcpyAsync(h->tr_h + (t + 1) * nd, hnext, nd * 4, cudaMemcpyDeviceToDevice, st));
    }
    if (act && n_loops)
        RDT_CUDA_TRY(cudaMemcpyAsync(n_loops, h->act_loops, static_cast<size_t>(N) * 4, cudaMemcpyDeviceToDevice, st));
    TIMED(h, K_CHECK, 1, st, check_finite(out, nd, h->flags, st));
    if (h->mode == 1) {            // the cache now holds the prompt's positions
        RDT_CUDA_TRY(cudaMemsetAsync(h->dec_len, 0, 4, st));
        RDT_TRY(len_advance(h->dec_len, c.seq, st));
    } else if (h->mode == 2) {     // and one more after a step
        RDT_TRY(len_advance(h->dec_len, 1, st));
    }
    return RDT_OK;
}

void drop_graph(rdt_handle* h) {
    if (h->gexec) cudaGraphExecDestroy(h->gexec);
    h->gexec = nullptr;
    h->gkey = rdt_handle::GraphKey{};
    h->seen_key = rdt_handle::GraphKey{};
}

// Runs the loop, replaying a captured CUDA graph when the same pointers and T come back:
// the first call with a key runs eagerly, the second captures (on the handle's own stream)
// and launches the graph, later ones only launch it. Tracing or profiling runs eagerly.
rdt_status run_loop(rdt_handle* h, const void* h0, const void* e, int T, float* out, cudaStream_t st,
                    bool act = false, int32_t* n_loops = nullptr) {
    if (h->cp_size > 1 && !h->cp_connected) {
        set_error("context parallelism: rdt_cp_connect has not been called on this handle");
        return RDT_ERR_INVALID_ARG;
    }
    if (h->cp_size > 1 && act) {
        // ranks that stop at different loops would leave their peers waiting
        set_error("context parallelism with ACT halting is not provided");
        return RDT_ERR_UNSUPPORTED;
    }
    const bool graphable = (!h->prof_on || h->prof_graph) && !h->tr_idx && !h->tr_w && !h->tr_h;
    if (!graphable) return loop_impl(h, h0, e, T, out, act, n_loops, st);
    rdt_handle::GraphKey key;
    key.h0 = h0;
    key.e = e;
    key.out = out;
    key.T = T;
    key.act = act;
    key.n_loops = n_loops;
    key.mode = h->mode;
    if (h->gexec && h->gkey == key) {
        RDT_CUDA_TRY(cudaGraphLaunch(h->gexec, st));
        h->launches += h->g_launches;
        h->graph_ran = true;
        return RDT_OK;
    }
    if (!(h->seen_key == key)) {
        h->seen_key = key;
        return loop_impl(h, h0, e, T, out, act, n_loops, st);
    }
    if (h->gexec) {
        cudaGraphExecDestroy(h->gexec);
        h->gexec = nullptr;
    }
    if (!h->cap_stream) RDT_CUDA_TRY(cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
    const int64_t l0 = h->launches;
    h->graph_pending.clear();
    RDT_CUDA_TRY(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal));
    h->capturing = true;
    const rdt_status s = loop_impl(h, h0, e, T, out, act, n_loops, h->cap_stream);
    h->capturing = false;
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->cap_stream, &g);
    if (s != RDT_OK) {
        if (g) cudaGraphDestroy(g);
        h->launches = l0;
        return s;
    }
    if (ce != cudaSuccess) {
        set_error(std::string("stream capture failed: ") + cudaGetErrorString(ce));
        return RDT_ERR_CUDA;
    }
    const cudaError_t ie = cudaGraphInstantiate(&h->gexec, g, 0);
    cudaGraphDestroy(g);
    if (ie != cudaSuccess) {
        h->gexec = nullptr;
        set_error(std::string("graph instantiation failed: ") + cudaGetErrorString(ie));
        return RDT_ERR_CUDA;
    }
    h->g_launches = h->launches - l0;
    h->launches = l0;
    h->gkey = key;
    RDT_CUDA_TRY(cudaGraphLaunch(h->gexec, st));
    h->launches += h->g_launches;
    h->graph_ran = true;
    return RDT_OK;
}

}  // namespace

// =====================================================================================
// C ABI
// =====================================================================================

extern "C" {

const char* rdt_status_string(rdt_status s) {
    switch (s) {
        case RDT_OK: return "ok";
        case RDT_ERR_INVALID_ARG: return "invalid argument";
        case RDT_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case RDT_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case RDT_ERR_UNSTABLE_A: return "rho(A) >= 1";
        case RDT_ERR_OOM: return "out of device memory";
        case RDT_ERR_CUDA: return "CUDA error";
        case RDT_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case RDT_ERR_NONFINITE: return "non-finite value in the state";
    }
    return "unknown status";
}

const char* rdt_last_error(void) { return g_last_error.c_str(); }

rdt_status rdt_create(const rdt_config* cfg, const rdt_weights* w, void* stream, rdt_handle** out) {
    if (!out) {
        set_error("out is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    *out = nullptr;
    RDT_TRY(validate_config(cfg));
    if (!w) {
        set_error("weights is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    rdt_handle* h = new (std::nothrow) rdt_handle();
    if (!h) {
        set_error("host allocation of the handle failed");
        return RDT_ERR_OOM;
    }
    rdt_status s = RDT_ERR_OOM;
    try {          // std::vector growth inside may throw: no exception crosses the C ABI
        s = create_impl(cfg, w, static_cast<cudaStream_t>(stream), h);
    } catch (const std::bad_alloc&) {
        set_error("host allocation failed during create");
        s = RDT_ERR_OOM;
    } catch (...) {
        set_error("unexpected host exception during create");
        s = RDT_ERR_CUDA;
    }
    if (s != RDT_OK) {
        rdt_destroy(h);
        return s;
    }
    *out = h;
    return RDT_OK;
}

static rdt_status check_ptr(const void* p, const char* name) {
    if (!p) {
        set_error(std::string(name) + " is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (!aligned16(p)) {
        set_error(std::string(name) + " is not 16-byte aligned");
        return RDT_ERR_MISALIGNED;
    }
    return RDT_OK;
}

// Every entry point names the tokens its call processes: all batch * seq positions, or one
// new position per sequence in a decode step.
static void set_mode(rdt_handle* h, int mode) {
    h->mode = mode;
    h->cur_ntok = mode == 2 ? h->cfg.batch : h->ntok;
}

rdt_status rdt_attn_forward(rdt_handle* h, const void* x, int loop, float* a_out, void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (h->cp_size > 1) {
        set_error("context parallelism runs through rdt_loop_forward only");
        return RDT_ERR_UNSUPPORTED;
    }
    set_mode(h, 0);
    RDT_TRY(check_ptr(x, "x"));
    RDT_TRY(check_ptr(a_out, "a_out"));
    if (loop < 0) {
        set_error("loop must be >= 0");
        return RDT_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    // x in the configuration's element type enters RMSNorm1 through its injection operand
    // (block input = e alone when the state operand is absent)
    return attention_block(h, nullptr, x, loop, false, a_out, nullptr, st);
}

rdt_status rdt_moe_forward(rdt_handle* h, const float* y, float* f_out, int32_t* topk_idx, float* topk_w,
                           void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(y, "y"));
    RDT_TRY(check_ptr(f_out, "f_out"));
    if (topk_idx) RDT_TRY(check_ptr(topk_idx, "topk_idx"));
    if (topk_w) RDT_TRY(check_ptr(topk_w, "topk_w"));
    set_mode(h, 0);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    const size_t nd = static_cast<size_t>(h->ntok) * h->cfg.dim;
    RDT_CUDA_TRY(cudaMemsetAsync(f_out, 0, nd * 4, st));
    RDT_CUDA_TRY(cudaMemsetAsync(h->counts, 0, 256 * 4, st));
    return moe_block(h, y, f_out, topk_idx, topk_w, nullptr, nullptr, nullptr, st);
}

rdt_status rdt_loop_forward(rdt_handle* h, const void* h0, const void* e, int T, float* out, void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(h0, "h0"));
    RDT_TRY(check_ptr(e, "e"));
    RDT_TRY(check_ptr(out, "out"));
    if (T < 1 || T > h->cfg.max_loops) {
        set_error("T must be in [1, max_loops]");
        return RDT_ERR_INVALID_ARG;
    }
    if (out == e) {
        set_error("out must not alias e (e is read in every loop)");
        return RDT_ERR_INVALID_ARG;
    }
    set_mode(h, 0);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    return run_loop(h, h0, e, T, out, st);
}

rdt_status rdt_decode_prefill(rdt_handle* h, const void* h0, const void* e, int T, float* out, void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (!h->kv_cache) {
        set_error("the handle has no KV cache: create it with max_decode > 0");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(h0, "h0"));
    RDT_TRY(check_ptr(e, "e"));
    RDT_TRY(check_ptr(out, "out"));
    if (T < 1 || T > h->cfg.max_loops) {
        set_error("T must be in [1, max_loops]");
        return RDT_ERR_INVALID_ARG;
    }
    if (out == e) {
        set_error("out must not alias e (e is read in every loop)");
        return RDT_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    h->dec_T = 0;
    set_mode(h, 1);
    const rdt_status s = run_loop(h, h0, e, T, out, st);
    set_mode(h, 0);
    if (s == RDT_OK) {
        h->dec_T = T;
        h->dec_len_host = h->cfg.seq;
    }
    return s;
}

rdt_status rdt_decode_step(rdt_handle* h, const void* h0, const void* e, int T, float* out, void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(h0, "h0"));
    RDT_TRY(check_ptr(e, "e"));
    RDT_TRY(check_ptr(out, "out"));
    if (h->dec_T == 0) {
        set_error("no prefill: call rdt_decode_prefill first");
        return RDT_ERR_INVALID_ARG;
    }
    if (T != h->dec_T) {
        set_error("a decode step runs the prefill's number of loops (every loop needs its cache)");
        return RDT_ERR_INVALID_ARG;
    }
    if (h->dec_len_host >= h->s_cap) {
        set_error("the KV cache is full (seq + max_decode positions)");
        return RDT_ERR_INVALID_ARG;
    }
    if (out == e) {
        set_error("out must not alias e (e is read in every loop)");
        return RDT_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    set_mode(h, 2);
    const rdt_status s = run_loop(h, h0, e, T, out, st);
    set_mode(h, 0);
    if (s == RDT_OK) h->dec_len_host += 1;
    return s;
}

rdt_status rdt_loop_forward_host(rdt_handle* h, const void* h0_host, const void* e_host, int T, float* out_host,
                                 void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (!h0_host || !e_host || !out_host) {
        set_error("host buffers must be non-NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (T < 1 || T > h->cfg.max_loops) {
        set_error("T must be in [1, max_loops]");
        return RDT_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    const size_t nd = static_cast<size_t>(h->ntok) * h->cfg.dim;
    RDT_CUDA_TRY(cudaMemcpyAsync(h->stage_e, e_host, nd * h->esz, cudaMemcpyHostToDevice, st));
    const void* h0d = h->stage_e;
    if (h0_host != e_host) {
        RDT_CUDA_TRY(cudaMemcpyAsync(h->stage_h0, h0_host, nd * h->esz, cudaMemcpyHostToDevice, st));
        h0d = h->stage_h0;
    }
    set_mode(h, 0);
    RDT_TRY(run_loop(h, h0d, h->stage_e, T, h->stage_out, st));
    RDT_CUDA_TRY(cudaMemcpyAsync(out_host, h->stage_out, nd * 4, cudaMemcpyDeviceToHost, st));
    RDT_CUDA_TRY(cudaStreamSynchronize(st));
    return RDT_OK;
}

rdt_status rdt_set_act(rdt_handle* h, const float* w_halt, float b_halt, float threshold, void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(w_halt, "w_halt"));
    if (!std::isfinite(b_halt) || !(threshold > 0.0f && threshold <= 1.0f)) {
        set_error("b_halt must be finite and threshold in (0, 1]");
        return RDT_ERR_INVALID_ARG;
    }
    const int N = h->ntok, d = h->cfg.dim;
    if (d % 128 != 0) {
        set_error("ACT halting needs dim to be a multiple of 128");
        return RDT_ERR_UNSUPPORTED;
    }
    if (!h->act_w) {
        // all three or none: the handle keeps them only once every allocation succeeded
        // (a failed one leaves the others in the handle's list, freed by rdt_destroy)
        float *w = nullptr, *cum = nullptr;
        int* loops = nullptr;
        RDT_TRY(dev_alloc(h, &w, static_cast<size_t>(d) * 4));
        RDT_TRY(dev_alloc(h, &cum, static_cast<size_t>(N) * 4, true));
        RDT_TRY(dev_alloc(h, &loops, static_cast<size_t>(N) * 4, true));
        h->act_w = w;
        h->act_cum = cum;
        h->act_loops = loops;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    RDT_CUDA_TRY(cudaMemcpyAsync(h->act_w, w_halt, static_cast<size_t>(d) * 4, cudaMemcpyDeviceToDevice, st));
    RDT_CUDA_TRY(cudaStreamSynchronize(st));
    h->act_b = b_halt;
    h->act_thr = threshold;
    h->act_set = true;
    drop_graph(h);                    // a captured loop holds the old head's scalars
    return RDT_OK;
}

rdt_status rdt_loop_forward_act(rdt_handle* h, const void* h0, const void* e, int T, float* out,
                                int32_t* n_loops, void* stream) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (!h->act_set) {
        set_error("rdt_set_act has not been called on this handle");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(h0, "h0"));
    RDT_TRY(check_ptr(e, "e"));
    RDT_TRY(check_ptr(out, "out"));
    if (n_loops) RDT_TRY(check_ptr(n_loops, "n_loops"));
    if (T < 1 || T > h->cfg.max_loops) {
        set_error("T must be in [1, max_loops]");
        return RDT_ERR_INVALID_ARG;
    }
    if (out == e) {
        set_error("out must not alias e (e is read in every loop)");
        return RDT_ERR_INVALID_ARG;
    }
    set_mode(h, 0);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    return run_loop(h, h0, e, T, out, st, true, n_loops);
}

rdt_status rdt_matmul(int32_t dtype, const void* A, const void* B, float* C, int M, int N, int K,
                      void* stream) {
    if (dtype != RDT_BF16 && dtype != RDT_F32) {
        set_error("dtype must be RDT_BF16 or RDT_F32");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(A, "A"));
    RDT_TRY(check_ptr(B, "B"));
    RDT_TRY(check_ptr(C, "C"));
    const bool bf = dtype == RDT_BF16;
    const int es = bf ? 2 : 4;
    if (M < 1 || N < 32 || K < 1 || N % 32 || (static_cast<long>(K) * es) % 128) {
        set_error("matmul: need M >= 1, N % 32 == 0, K * element size % 128 == 0");
        return RDT_ERR_UNSUPPORTED;
    }
    CUtensorMap ta, tb;
    const uint32_t kbox = 128 / es;
    RDT_TRY(make_tmap_2d(&ta, A, bf, K, M, static_cast<uint64_t>(K) * es, kbox, 128));
    RDT_TRY(make_tmap_2d(&tb, B, bf, K, N, static_cast<uint64_t>(K) * es, kbox, 128));
    GemmArgs ga{};
    ga.M = M;
    ga.N = N;
    ga.kb_main = static_cast<int>(static_cast<long>(K) * es / 128);
    EpiParams ep{};
    ep.kind = EPI_STORE_F32;
    ep.out = C;
    ep.ldo = N;
    ep.ncols_valid = N;
    return gemm_tc(bf, 128, ta, tb, nullptr, nullptr, ga, ep, static_cast<cudaStream_t>(stream));
}

rdt_status rdt_attention(int32_t dtype, const void* q, const void* k, const void* v, void* o,
                         int batch, int seq, int n_heads, int n_kv_heads, int dqk, int dv,
                         float scale, void* stream) {
    if (dtype != RDT_BF16 && dtype != RDT_F32) {
        set_error("dtype must be RDT_BF16 or RDT_F32");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_TRY(check_ptr(q, "q"));
    RDT_TRY(check_ptr(k, "k"));
    RDT_TRY(check_ptr(v, "v"));
    RDT_TRY(check_ptr(o, "o"));
    if (batch < 1 || seq < 1 || n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads) {
        set_error("attention: bad sizes");
        return RDT_ERR_INVALID_ARG;
    }
    AttnArgs a{};
    a.q = q; a.ldq = n_heads * dqk; a.q_hstride = dqk;
    a.k = k; a.ldk = n_kv_heads * dqk; a.k_hstride = dqk;
    a.v = v; a.ldv = n_kv_heads * dv; a.v_hstride = dv;
    if (v == k && dv <= dqk) {          // values are the first dv columns of the keys
        a.ldv = a.ldk;
        a.v_hstride = a.k_hstride;
    }
    a.o = o; a.ldo = n_heads * dv;
    a.batch = batch; a.seq = seq; a.hq = n_heads; a.hkv = n_kv_heads; a.dqk = dqk; a.dv = dv;
    a.scale = scale;
    return attention(dtype == RDT_BF16, a, static_cast<cudaStream_t>(stream));
}

rdt_status rdt_set_trace(rdt_handle* h, int32_t* idx, float* w, float* h_traj) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if ((idx && !aligned16(idx)) || (w && !aligned16(w)) || (h_traj && !aligned16(h_traj))) {
        set_error("trace buffers must be 16-byte aligned");
        return RDT_ERR_MISALIGNED;
    }
    h->tr_idx = idx;
    h->tr_w = w;
    h->tr_h = h_traj;
    drop_graph(h);
    return RDT_OK;
}

rdt_status rdt_get_diagnostics(rdt_handle* h, rdt_diag* out) {
    if (!h || !out) {
        set_error("handle or out is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    int flags[FLAG_COUNT];
    RDT_CUDA_TRY(cudaMemcpy(flags, h->flags, sizeof(flags), cudaMemcpyDeviceToHost));
    std::memset(out, 0, sizeof(*out));
    out->rho_A = h->rho;
    out->nonfinite = flags[FLAG_NONFINITE];
    out->timeout = flags[FLAG_TIMEOUT];
    int counts[256];
    RDT_CUDA_TRY(cudaMemcpy(counts, h->counts, sizeof(counts), cudaMemcpyDeviceToHost));
    int tot = 0;
    for (int i = 0; i < h->cfg.n_experts; ++i) {
        out->expert_counts[i] = counts[i];
        tot += counts[i];
    }
    for (int s = 0; s < h->cfg.n_shared; ++s) out->expert_counts[h->cfg.n_experts + s] = h->ntok;
    out->last_routed_rows = tot;
    return RDT_OK;
}

rdt_status rdt_profile(rdt_handle* h, int enable) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (enable < 0 || enable > 2) {
        set_error("enable must be 0, 1 or 2");
        return RDT_ERR_INVALID_ARG;
    }
    if (enable) {
        RDT_CUDA_TRY(cudaStreamSynchronize(h->last_stream));
        h->pending.clear();
        h->ev_used = 0;
        h->graph_ran = false;
        std::fill(h->prof_ms.begin(), h->prof_ms.end(), 0.0);
        std::fill(h->prof_n.begin(), h->prof_n.end(), 0);
        if (h->prof_on && h->prof_graph == (enable == 2)) return RDT_OK;   // statistics restarted
    }
    h->prof_on = enable != 0;
    h->prof_graph = enable == 2;
    drop_graph(h);
    h->graph_pending.clear();
    return RDT_OK;
}

rdt_status rdt_profile_read(rdt_handle* h, rdt_kernel_stat* out, int max_entries, int* n_entries,
                            int64_t* total_launches) {
    if (!h) {
        set_error("handle is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    RDT_CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    RDT_TRY(prof_flush(h));
    int n = 0;
    for (int k = 0; k < K_COUNT; ++k) {
        if (h->prof_n[k] == 0) continue;
        if (out && n < max_entries) {
            std::memset(out[n].name, 0, sizeof(out[n].name));
            std::strncpy(out[n].name, kKindName[k], sizeof(out[n].name) - 1);
            out[n].launches = h->prof_n[k];
            out[n].total_ms = h->prof_ms[k];
        }
        ++n;
    }
    if (n_entries) *n_entries = std::min(n, max_entries);
    if (total_launches) *total_launches = h->launches;
    return RDT_OK;
}

rdt_status rdt_memory_bytes(const rdt_handle* h, size_t* bytes) {
    if (!h || !bytes) {
        set_error("handle or bytes is NULL");
        return RDT_ERR_INVALID_ARG;
    }
    *bytes = h->bytes;
    return RDT_OK;
}

rdt_status rdt_cp_buffers(rdt_handle* h, void** kv, size_t* kv_bytes, void** flags, size_t* flag_bytes) {
    if (!h || !kv || !kv_bytes || !flags || !flag_bytes) {
        set_error("rdt_cp_buffers: NULL argument");
        return RDT_ERR_INVALID_ARG;
    }
    if (h->cp_size < 2) {
        set_error("rdt_cp_buffers: the handle was created without cp_size > 1");
        return RDT_ERR_INVALID_ARG;
    }
    const rdt_config& c = h->cfg;
    *kv = h->cp_kv;
    *kv_bytes = static_cast<size_t>(c.batch) * h->s_cap * 2 * h->nkv * h->esz;
    *flags = h->cp_flags;
    *flag_bytes = 256;
    return RDT_OK;
}

rdt_status rdt_cp_connect(rdt_handle* h, void* const* peer_kv, void* const* peer_flags) {
    if (!h || !peer_kv || !peer_flags) {
        set_error("rdt_cp_connect: NULL argument");
        return RDT_ERR_INVALID_ARG;
    }
    if (h->cp_size < 2) {
        set_error("rdt_cp_connect: the handle was created without cp_size > 1");
        return RDT_ERR_INVALID_ARG;
    }
    for (int q = 0; q < h->cp_size; ++q) {
        if (q == h->cp_rank) continue;
        if (!peer_kv[q] || !peer_flags[q] || (reinterpret_cast<uintptr_t>(peer_kv[q]) & 15) ||
            (reinterpret_cast<uintptr_t>(peer_flags[q]) & 15)) {
            set_error("rdt_cp_connect: rank " + std::to_string(q) + "'s buffers are NULL or not 16-byte aligned");
            return RDT_ERR_INVALID_ARG;
        }
    }
    for (int q = 0; q < h->cp_size; ++q) {
        if (q == h->cp_rank) continue;
        h->cp_peer_kv[q] = peer_kv[q];
        h->cp_peer_flags[q] = static_cast<unsigned*>(peer_flags[q]);
    }
    drop_graph(h);              // captured graphs hold the previous peers
    h->cp_connected = true;
    return RDT_OK;
}

void rdt_destroy(rdt_handle* h) {
    if (!h) return;
    cudaDeviceSynchronize();
    for (cudaEvent_t ev : h->ev_pool) cudaEventDestroy(ev);
    for (cudaEvent_t ev : h->graph_events) cudaEventDestroy(ev);
    if (h->gexec) cudaGraphExecDestroy(h->gexec);
    if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
    for (void* p : h->allocs) cudaFree(p);
    delete h;
}

}  // extern "C"
