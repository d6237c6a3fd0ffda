/*
 * rdt.h - C ABI of the B200 (sm_100a) recurrent-depth block library, librdt.so.
 *
 * The library runs the looped recurrent block of a recurrent-depth transformer:
 *
 *     h_{t+1} = A (.) h_t + B.e + Block(h_t, e),      t = 0 .. T-1,
 *
 * (the update equation of the techbriefly article on the OpenMythos project,
 * whose transformer term is Block here; e is the prelude encoding, injected
 * again in every loop, and rho(A) < 1). Block is a pre-RMSNorm causal
 * attention sublayer (GQA, or MLA with a latent KV) followed by a top-k sparse
 * mixture of SwiGLU experts, with optional per-loop (depth-wise) LoRA on the Q
 * and O projections (getting-started page "Introducao ao OpenMythos",
 * Passo 2 and Passo 5; techbriefly article, MoE and LoRA paragraphs).
 *
 * Readings fixed by this library where the pages are silent:
 *   x = h + e (inject_e = 1) or x = h;  a = Attn(RMSNorm1(x));  y = x + a;
 *   f = MoE(RMSNorm2(y));  Block(h, e) = a + f  (the residual increment).
 *   A is diagonal (fp32 [dim]); B is diagonal [dim] or dense [dim, dim] (fp32).
 *
 * Conventions for every call:
 *   - Pointers named *device* are CUDA device pointers on the current device;
 *     *host* pointers are ordinary host memory. Tensors are row-major and
 *     token-major: a [N, dim] tensor holds token n = b * seq + s in row n.
 *     Every device tensor must be 16-byte aligned (RDT_ERR_MISALIGNED).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls enqueue work and return without synchronising, except where noted;
 *     caller buffers must stay valid until that work has completed.
 *   - Arguments are validated before anything is enqueued; a non-OK status
 *     means nothing was launched (except RDT_ERR_CUDA, raised by a failing
 *     CUDA call). rdt_last_error() gives the message of the calling thread's
 *     last failure.
 *   - A handle must not be used from two host threads or two streams at once:
 *     its workspace is shared by all its calls.
 */
#ifndef RDT_H
#define RDT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RDT_OK = 0,
    RDT_ERR_INVALID_ARG = 1,    /* null pointer, size or loop count out of range      */
    RDT_ERR_UNSUPPORTED = 2,    /* no sm_100 device, or a shape the kernels do not tile */
    RDT_ERR_MISALIGNED = 3,     /* a tensor pointer not 16-byte aligned                 */
    RDT_ERR_UNSTABLE_A = 4,     /* rho(A) = max |A_i| >= 1 at create                    */
    RDT_ERR_OOM = 5,            /* device allocation failed                             */
    RDT_ERR_CUDA = 6,           /* a CUDA runtime or driver call failed                 */
    RDT_ERR_DEVICE_TIMEOUT = 7, /* a bounded device-side wait gave up (diagnostics)     */
    RDT_ERR_NONFINITE = 8       /* a NaN or Inf reached the state (diagnostics)          */
} rdt_status;

enum { RDT_F32 = 0, RDT_BF16 = 1 };        /* rdt_config.dtype        */
enum { RDT_GQA = 0, RDT_MLA = 1 };         /* rdt_config.attn_type    */
enum { RDT_B_DIAG = 0, RDT_B_DENSE = 1 };  /* rdt_config.b_kind       */

/* Block hyper-parameters (the block-level fields of MythosConfig, getting-started
 * page Passo 2 and Passo 5). `batch` and `seq` are the sizes every forward call
 * uses; the workspace is allocated for them at create.
 * Tiling limits checked at create (RDT_ERR_UNSUPPORTED otherwise): dim = 128 * 2^k
 * <= 4096; GQA head_dim 64 (bf16) or 32 / 64 (fp32), n_heads % n_kv_heads == 0,
 * n_heads * head_dim % 128 == 0; expert_hidden % 64 == 0 (fp32: % 128);
 * n_experts + n_shared <= 256; top_k <= min(n_experts, 16); LoRA on GQA only with
 * lora_rank <= 64 (bf16) / 32 (fp32); MLA in bf16 only with kv_lora_rank 128,
 * qk_rope_dim 32, q_lora_rank % 64 == 0, v_head_dim % 32 == 0. */
typedef struct {
    int32_t dtype;                  /* RDT_F32 or RDT_BF16: storage of h0, e, weights   */
    int32_t batch, seq, dim;
    int32_t attn_type;              /* RDT_GQA or RDT_MLA                               */
    int32_t n_heads, n_kv_heads, head_dim;                            /* GQA           */
    int32_t q_lora_rank, kv_lora_rank, qk_nope_dim, qk_rope_dim, v_head_dim; /* MLA    */
    float rope_base;                /* RoPE base (1e4)                                  */
    float norm_eps;                 /* RMSNorm epsilon (1e-6)                           */
    int32_t n_experts, top_k, n_shared, expert_hidden;
    int32_t lora_rank, n_lora;      /* depth-wise LoRA on Q and O; n_lora = 0: none     */
    int32_t b_kind;                 /* RDT_B_DIAG or RDT_B_DENSE                        */
    int32_t inject_e;               /* 1: block input x = h + e; 0: x = h               */
    int32_t max_loops;              /* largest T accepted (<= 64; the pages loop <= 16) */
    int32_t gemm_tiles;             /* projection / expert GEMM tiles: 0 chosen per GEMM
                                     * from its shape (and a K split for the expert
                                     * down-projection), 1 one CTA per 128-row tile, 2 CTA
                                     * pairs per 256-row tile (bf16 only; fp32 uses 1).
                                     * Results agree up to fp32 summation order.        */
    int32_t deterministic;          /* 1: bit-identical results from run to run: each
                                     * expert row's weighted output is stored in its own
                                     * row and the rows of a token are added in a fixed
                                     * order (shared experts, then slots 0 .. top_k - 1)
                                     * by a combine kernel; no K splits that reduce with
                                     * atomics. Costs N * top_k * dim * 8 bytes of extra
                                     * traffic per loop. 0: reductions by fp32 atomics,
                                     * whose order (and so the last bits) may vary.      */
    int32_t max_decode;             /* > 0: a per-loop KV cache of seq + max_decode positions
                                     * per sequence for rdt_decode_prefill / _step (bf16
                                     * only): max_loops * batch * (seq + max_decode) rows of
                                     * 2 n_kv_heads head_dim (GQA) or kv_lora_rank +
                                     * qk_rope_dim (MLA) elements. 0: no cache.         */
    int32_t da_heads;               /* depth attention: query heads (0: none); GQA, bf16,
                                     * head width head_dim = 64                          */
    int32_t da_kv_heads;            /* depth attention: KV heads (divides da_heads)     */
    int32_t cp_size;                /* context parallelism: ranks (GPUs) one sequence is
                                     * split over, 0 or 1: none, <= 8. Rank r holds
                                     * positions [r * seq, (r + 1) * seq) of sequences of
                                     * cp_size * seq positions (seq, batch as above: this
                                     * rank's share). GQA, bf16, head_dim 64, seq % 128 ==
                                     * 0, no decode cache, no ACT; rdt_cp_connect before the
                                     * first rdt_loop_forward.                             */
    int32_t cp_rank;                /* this rank, 0 .. cp_size - 1                       */
} rdt_config;

/* Weights, all DEVICE pointers, row-major [out, in]; element type = cfg.dtype
 * unless marked fp32. rdt_create copies and repacks them into library-owned
 * memory, so the caller may free them once rdt_create has returned.
 * Fields a configuration does not use must be NULL. */
typedef struct {
    const float* A;            /* [dim] fp32, diagonal of A; rho(A) < 1 required         */
    const float* B;            /* [dim] (RDT_B_DIAG) or [dim, dim] (RDT_B_DENSE), fp32   */
    const float* norm1;        /* [dim] fp32 RMSNorm gain before attention               */
    const float* norm2;        /* [dim] fp32 RMSNorm gain before the MoE                 */
    /* GQA */
    const void* wq;            /* [n_heads * head_dim, dim]                              */
    const void* wk;            /* [n_kv_heads * head_dim, dim]                           */
    const void* wv;            /* [n_kv_heads * head_dim, dim]                           */
    const void* wo;            /* [dim, n_heads * head_dim] (MLA: [dim, n_heads * v_head_dim]) */
    /* MLA */
    const void* w_dq;          /* [q_lora_rank, dim]                                     */
    const float* q_norm;       /* [q_lora_rank] fp32                                     */
    const void* w_uq;          /* [n_heads * (qk_nope_dim + qk_rope_dim), q_lora_rank]   */
    const void* w_dkv;         /* [kv_lora_rank, dim]                                    */
    const float* kv_norm;      /* [kv_lora_rank] fp32                                    */
    const void* w_kr;          /* [qk_rope_dim, dim]                                     */
    const void* w_uk;          /* [n_heads * qk_nope_dim, kv_lora_rank]                  */
    const void* w_uv;          /* [n_heads * v_head_dim, kv_lora_rank]                   */
    /* MoE */
    const void* w_router;      /* [n_experts, dim]                                       */
    const float* router_bias;  /* [n_experts] fp32 or NULL: added for selection only     */
    const void* w1;            /* [n_experts, expert_hidden, dim] (gate)                 */
    const void* w3;            /* [n_experts, expert_hidden, dim] (up)                   */
    const void* w2;            /* [n_experts, dim, expert_hidden] (down)                 */
    const void* ws1;           /* [n_shared, expert_hidden, dim] or NULL                 */
    const void* ws3;           /* [n_shared, expert_hidden, dim] or NULL                 */
    const void* ws2;           /* [n_shared, dim, expert_hidden] or NULL                 */
    /* depth-wise LoRA (GQA): W_t = W + B_t A_t, adapter min(t, n_lora - 1) at loop t */
    const void* lq_a;          /* [n_lora, lora_rank, dim]                               */
    const void* lq_b;          /* [n_lora, n_heads * head_dim, lora_rank]                */
    const void* lo_a;          /* [n_lora, lora_rank, n_heads * head_dim]                */
    const void* lo_b;          /* [n_lora, dim, lora_rank]                               */
    /* depth attention (cfg.da_heads > 0): before the sequence attention of loop t of T,
     * x' = x + DA(RMSNorm_da(x)); a token's query attends over its own keys and values of
     * loops 0 .. t (RoPE over the loop index: rotation pairs i < head_dim/4 at t, the rest
     * at T - 1 - t); the sequence attention takes x' and the increment is d + a + f
     * (gist.science summary of "Dreamer", depth attention) */
    const float* norm_da;      /* [dim] fp32 RMSNorm gain of the depth attention        */
    const void* wq_d;          /* [da_heads * head_dim, dim]                             */
    const void* wk_d;          /* [da_kv_heads * head_dim, dim]                          */
    const void* wv_d;          /* [da_kv_heads * head_dim, dim]                          */
    const void* wo_d;          /* [dim, da_heads * head_dim]                             */
} rdt_weights;

typedef struct rdt_handle rdt_handle;

typedef struct {
    float rho_A;                   /* max |A_i| of the weights given at create             */
    int32_t nonfinite;             /* 1 if a non-finite value reached the state            */
    int32_t timeout;               /* 1 if a bounded device wait gave up                   */
    int32_t last_routed_rows;      /* sum of the per-expert counts of the last MoE         */
    int32_t expert_counts[256];    /* tokens per expert in the last MoE (routed, then shared) */
} rdt_diag;

/* Validates cfg and weights, allocates the workspace for cfg.batch * cfg.seq
 * tokens, copies and repacks the weights (on `stream`, then synchronises it) and
 * returns a handle in *out. Errors: INVALID_ARG (bad sizes or NULL weights),
 * UNSUPPORTED (not an sm_100 device, or a shape outside the tiling limits),
 * UNSTABLE_A (max |A_i| >= 1: the parameterisation, not a clip, must keep
 * rho(A) < 1 - getting-started page, Passo 6 and troubleshooting item 3), OOM, CUDA. */
rdt_status rdt_create(const rdt_config* cfg, const rdt_weights* w, void* stream,
                      rdt_handle** out);

/* Attention sublayer alone: a = Attn(RMSNorm1(x)) including the output
 * projection and the LoRA adapter of loop `loop` (ignored without LoRA).
 *   x     : device [N, dim] block input in cfg.dtype (N = batch * seq)
 *   a_out : device fp32 [N, dim]                                              */
rdt_status rdt_attn_forward(rdt_handle* h, const void* x, int loop, float* a_out,
                            void* stream);

/* MoE sublayer alone: f = MoE(RMSNorm2(y)), routed top-k experts weighted by the
 * softmax of their logits renormalised over the k chosen, plus every shared
 * expert with weight 1.
 *   y        : device fp32 [N, dim]
 *   f_out    : device fp32 [N, dim]
 *   topk_idx : device int32 [N, top_k] or NULL: chosen experts, by (logit + bias)
 *              descending, ties to the lower index
 *   topk_w   : device fp32 [N, top_k] or NULL: their gate weights             */
rdt_status rdt_moe_forward(rdt_handle* h, const float* y, float* f_out, int32_t* topk_idx,
                           float* topk_w, void* stream);

/* The looped block: out = h_T after T loops of the update equation.
 *   h0, e : device [N, dim] in cfg.dtype (h0 may alias e)
 *   T     : 1 .. cfg.max_loops (INVALID_ARG otherwise)
 *   out   : device fp32 [N, dim]; the state is kept in fp32 throughout; must
 *           not alias e, which every loop reads (INVALID_ARG)                 */
rdt_status rdt_loop_forward(rdt_handle* h, const void* h0, const void* e, int T, float* out,
                            void* stream);

/* The same call for callers holding HOST buffers: copies h0 and e (cfg.dtype,
 * [N, dim]) to the device, runs rdt_loop_forward, copies h_T (fp32 [N, dim])
 * back to `out_host` and synchronises `stream` before returning. Page-locked
 * host memory gives asynchronous copies; pageable memory also works. */
rdt_status rdt_loop_forward_host(rdt_handle* h, const void* h0_host, const void* e_host, int T,
                                 float* out_host, void* stream);

/* Decode with a per-loop KV cache (getting-started page "Introducao ao OpenMythos", Passo 4:
 * the prompt is run once, then one token per call; troubleshooting item 1: every loop keeps
 * the keys and values of all tokens; Passo 5: MLA caches its compressed latent and rebuilds
 * K and V from it). Loop t of a new token attends over the keys and values that loop t
 * produced for the earlier positions and for itself. GQA caches its rotated keys and its
 * values; MLA its normalised latent and rotated shared key. Needs cfg.max_decode > 0.
 *
 * rdt_decode_prefill runs the loop over the prompt (h0, e: device [batch, seq, dim] in
 * cfg.dtype; out: device fp32 [batch, seq, dim] = h_T) exactly as rdt_loop_forward and fills
 * the cache of loops 0 .. T - 1 with positions 0 .. seq - 1 (a new prefill starts over).
 * rdt_decode_step runs T loops (T must be the prefill's) for one new token per sequence at
 * the next position (h0, e: device [batch, dim] in cfg.dtype; out: device fp32 [batch, dim]
 * = h_T of the new tokens) and appends it to every loop's cache. INVALID_ARG without a
 * prefill, for another T or when the cache is full (seq + max_decode positions). The
 * position advances on the device, so a step's launch sequence replays as one CUDA graph.
 * A trace set by rdt_set_trace records a step's loops in its first batch rows: loop t's
 * routing at offset t * batch * seq * top_k, its states packed as [T + 1, batch, dim]. */
rdt_status rdt_decode_prefill(rdt_handle* h, const void* h0, const void* e, int T, float* out,
                              void* stream);
rdt_status rdt_decode_step(rdt_handle* h, const void* h0, const void* e, int T, float* out,
                           void* stream);

/* ACT halting ("Dynamic Adaptive Computation Time" halting, techbriefly article on
 * the OpenMythos project; act_threshold = 0.99, getting-started page
 * "Introducao ao OpenMythos", troubleshooting item 4: a position leaves the
 * loop once its accumulated halting probability reaches the threshold). The
 * pages give no halting head; this one is a linear map of the state to one
 * logit: p_t = sigmoid(w_halt . h_{t+1} + b_halt).
 *
 * rdt_set_act sets the head of a handle: copies w_halt (device fp32 [dim],
 * 16-byte aligned; the caller may free it on return), keeps b_halt and the
 * threshold. Synchronises `stream`. INVALID_ARG for a NULL w_halt, a
 * non-finite b_halt or a threshold outside (0, 1]; UNSUPPORTED when dim is
 * not a multiple of 128; OOM if its small workspace (dim + 2 N words) cannot
 * be allocated. */
rdt_status rdt_set_act(rdt_handle* h, const float* w_halt, float b_halt, float threshold,
                       void* stream);

/* The looped block with ACT halting per position. Each loop runs the block for
 * every position (attention sees every position's current state); positions
 * still running are routed through the MoE and updated as in rdt_loop_forward,
 * halted positions keep their state and are routed to no expert. After loop t
 * a running position with earlier halting probabilities summing to c takes
 * p_t; it halts at loop t if c + p_t >= threshold or t = T - 1, and h_{t+1}
 * enters the output with weight 1 - c; otherwise with weight p_t.
 *   h0, e   : device [N, dim] in cfg.dtype (h0 may alias e)
 *   T       : 1 .. cfg.max_loops (INVALID_ARG otherwise)
 *   out     : device fp32 [N, dim] = sum over t of weight_t * h_{t+1}; must not
 *             alias e (INVALID_ARG)
 *   n_loops : device int32 [N] (16-byte aligned) or NULL: loops each position ran
 * INVALID_ARG if rdt_set_act has not been called on the handle. */
rdt_status rdt_loop_forward_act(rdt_handle* h, const void* h0, const void* e, int T, float* out,
                                int32_t* n_loops, void* stream);

/* Per-loop trace for parity checks (all device pointers, or NULL to disable):
 *   idx    : int32 [max_loops, N, top_k] routing of every loop
 *   w      : fp32  [max_loops, N, top_k] gate weights of every loop
 *   h_traj : fp32  [max_loops + 1, N, dim] the state h_0 .. h_T
 * Later rdt_loop_forward and rdt_loop_forward_act calls write loop t at offset t (a
 * token halted by ACT has index -1 and weight 0 there). Pass all NULL to stop. */
rdt_status rdt_set_trace(rdt_handle* h, int32_t* idx, float* w, float* h_traj);

/* Synchronises the handle's last stream and fills *out (see rdt_diag). */
rdt_status rdt_get_diagnostics(rdt_handle* h, rdt_diag* out);

/* Bytes of device memory the handle owns (weights + workspace). */
rdt_status rdt_memory_bytes(const rdt_handle* h, size_t* bytes);

/* ---- kernel-level calls: the tensor-core GEMM and the attention kernel alone, on
 * caller buffers (unit parity and per-kernel measurement). */

/* C = A B^T on the 5th-generation tensor cores (bf16 operands, or fp32 operands read as
 * tf32), fp32 accumulation and output.
 *   dtype : RDT_BF16 or RDT_F32, element type of A and B
 *   A     : device [M, K] row-major;  B : device [N, K] row-major;  C : device fp32 [M, N]
 * Limits: K * element size a multiple of 128 bytes; N a multiple of 32; M >= 1. */
rdt_status rdt_matmul(int32_t dtype, const void* A, const void* B, float* C, int M, int N, int K,
                      void* stream);

/* Causal attention o = softmax(q k^T * scale, keys after the query masked) v per sequence
 * and query head; query head h reads KV head floor(h * n_kv_heads / n_heads).
 *   q : device [batch * seq, n_heads * dqk]    k : device [batch * seq, n_kv_heads * dqk]
 *   v : device [batch * seq, n_kv_heads * dv]  o : device [batch * seq, n_heads * dv]
 * bf16: (dqk, dv) = (64, 64) or (160, 128); fp32: (32, 32) or (64, 64). v may equal k
 * with dv <= dqk: the values are then the first dv columns of each key row (absorbed MLA's
 * shared latent), read with the keys' row stride. */
rdt_status rdt_attention(int32_t dtype, const void* q, const void* k, const void* v, void* o,
                         int batch, int seq, int n_heads, int n_kv_heads, int dqk, int dv,
                         float scale, void* stream);

/* ---- MoE router without allocation (the pages have no counterpart: this is a library
 * convenience). For callers that cannot call cudaMalloc - code running inside another
 * framework's memory pool that owns all device memory, serving loops that forbid
 * allocation after start-up, or hosts that capture the work into their own CUDA graphs -
 * and so cannot create a handle. Runs the router kernels of rdt_moe_forward: RMSNorm2 of y
 * with gain norm2, fp32 logits against w_router, top-k of logits + bias (ties to the lower
 * expert index), softmax over the k chosen logits, per-expert token counts.
 *   dtype         : RDT_BF16 or RDT_F32, element type of w_router
 *   y             : device fp32 [ntok, dim];  norm2 : device fp32 [dim]
 *   w_router      : device [n_experts, dim];  router_bias : device fp32 [n_experts] or NULL
 *   topk_idx      : device int32 [ntok, top_k];  topk_w : device fp32 [ntok, top_k]
 *   expert_counts : device int32 [n_experts] or NULL
 * No allocation: the kernels' scratch (counters, status words and, where the path needs
 * them, normalised rows) is one static device array of 8 MiB that every process loading
 * librdt holds on every GPU it uses until exit. Row scratch by path: none when w_router
 * takes at most 64 KB with n_experts <= 64, top_k <= 8 and dim 128, 1024 or 2048 (the fused
 * router); otherwise 2 * ntok * dim * 2 bytes (bf16: rows and their residuals) or
 * ntok * dim * 4 bytes (fp32), which must not exceed 8 MiB - 4 KiB (RDT_ERR_UNSUPPORTED
 * otherwise); dim = 128 * 2^k <= 4096, n_experts <= 256, top_k <= min(n_experts, 16).
 * The first call on a device (and the first after its context was re-created) looks up
 * the array's device address (a runtime call, no allocation); make that first call before
 * any stream capture. All calls share the array, and the counters and status words are
 * cleared at the start of each call, so calls that overlap on the GPU (other streams,
 * other threads) race: serialise them. */
rdt_status rdt_moe_route_noalloc(int32_t dtype, const float* y, const float* norm2,
                                 const void* w_router, const float* router_bias, int ntok, int dim,
                                 int n_experts, int top_k, float eps, int32_t* topk_idx,
                                 float* topk_w, int32_t* expert_counts, void* stream);

/* Status of the last rdt_moe_route_noalloc call on the current device: synchronises
 * `stream` (the one that call used) and reads the router's device status word from the
 * static array (no allocation). RDT_ERR_DEVICE_TIMEOUT if a bounded device-side wait of
 * the tensor-core router gave up (its top-k outputs are then incomplete), else RDT_OK. */
rdt_status rdt_moe_route_noalloc_status(void* stream);

/* ---- per-kernel timing (CUDA events recorded around every launch of the handle) */
typedef struct {
    char name[32];          /* kernel class, e.g. "gemm_up", "attention", "router_topk"  */
    int64_t launches;       /* launches timed since profiling was enabled               */
    double total_ms;        /* summed event time of those launches                      */
} rdt_kernel_stat;

/* enable = 1 times eager launches (the loop is not replayed from its CUDA graph while on);
 * enable = 2 times inside graph replay: the events become event-record nodes of the loop's
 * captured graph, so the timing describes the replayed sequence (the records sit between the
 * kernels, so each launch waits for its predecessor to finish); 0 stops timing. Switching
 * mode clears the statistics and drops a captured graph; enabling the current mode again
 * only clears the statistics. Timing adds two event records per launch on the launch
 * stream. In mode 2 a replay records the graph's events anew: rdt_profile_read counts the
 * last replay before it, so read after every replayed call. */
rdt_status rdt_profile(rdt_handle* h, int enable);

/* Synchronises the handle's last stream and returns up to max_entries statistics
 * (*n_entries set to their number) and, in *total_launches, the number of kernels
 * the handle has launched since create (counted whether or not timing is on). */
rdt_status rdt_profile_read(rdt_handle* h, rdt_kernel_stat* out, int max_entries, int* n_entries,
                            int64_t* total_launches);

/* Failure-detection probe of the bounded device-side waits (library diagnostics; the pages
 * have no counterpart). Launches one kernel that waits, with the same bounded mbarrier wait
 * every pipeline kernel uses but a limit of limit_ns (1 .. 2e9), on a barrier that nothing
 * arrives on; the wait gives up, the kernel records the timeout in its status word and
 * returns. Synchronises `stream`. Returns RDT_ERR_DEVICE_TIMEOUT, the expected outcome
 * (the device context stays usable); INVALID_ARG for a limit out of range. */
rdt_status rdt_wait_probe(int64_t limit_ns, void* stream);

/* Context parallelism (cfg.cp_size > 1; the pages run several GPUs only through torchrun,
 * "Introducao ao OpenMythos" Passo 8, so the split of one long sequence over GPUs is this
 * library's own). Per loop the QKV projection of rank r writes its rotated keys and values
 * into its own gather buffer and, over peer memory (NVLink), into those of ranks r + 1 ..
 * cp_size - 1, which attend over them; ranks signal one another through flag words in each
 * other's memory with bounded waits (a wait that gives up records a timeout in the
 * diagnostics). Everything else in the block is token-local.
 *
 * rdt_cp_buffers: this handle's gather buffer ([batch][cp_size * seq][2 n_kv_heads head_dim]
 * bf16) and flag words, both device memory owned by the handle, for the caller to share
 * with the other ranks (rdt_ipc_get_handle). INVALID_ARG without cp_size > 1.
 * rdt_cp_connect: peer_kv[q] and peer_flags[q] (q = 0 .. cp_size - 1) are rank q's two
 * buffers as device pointers valid in this process (rdt_ipc_open_handle, or the buffers of
 * another handle on the same device); entry cp_rank is ignored. The pointers must stay
 * valid while the handle runs loops; every rank must connect before any rank's first
 * rdt_loop_forward, and every rank must run the same loop counts in the same order (their
 * calls wait for one another). */
rdt_status rdt_cp_buffers(rdt_handle* h, void** kv, size_t* kv_bytes, void** flags, size_t* flag_bytes);
rdt_status rdt_cp_connect(rdt_handle* h, void* const* peer_kv, void* const* peer_flags);

/* CUDA inter-process handles of device memory for sharing the buffers above between
 * processes (64 bytes, opaque). rdt_ipc_open_handle maps another process's allocation into
 * this one (peer access enabled on demand); rdt_ipc_close_handle unmaps it. */
rdt_status rdt_ipc_get_handle(const void* dev_ptr, void* handle64);
rdt_status rdt_ipc_open_handle(const void* handle64, void** dev_ptr);
rdt_status rdt_ipc_close_handle(void* dev_ptr);

const char* rdt_status_string(rdt_status s);
const char* rdt_last_error(void);

/* Frees everything the handle owns (after synchronising the device). NULL is a no-op. */
void rdt_destroy(rdt_handle* h);

#ifdef __cplusplus
}
#endif
#endif /* RDT_H */
