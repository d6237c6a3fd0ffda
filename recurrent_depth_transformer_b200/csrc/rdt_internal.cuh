// Internal declarations of librdt: device helpers (mbarrier, TMA, tcgen05 wrappers in
// inline PTX for sm_100a) and the host launchers each .cu file provides.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/rdt.h"

namespace rdt {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ error plumbing (host)

void set_error(const std::string& msg);
#define RDT_CUDA_TRY(expr)                                                                   \
    do {                                                                                     \
        cudaError_t _e = (expr);                                                             \
        if (_e != cudaSuccess) {                                                             \
            ::rdt::set_error(std::string(#expr) + ": " + cudaGetErrorString(_e));            \
            return RDT_ERR_CUDA;                                                             \
        }                                                                                    \
    } while (0)
#define RDT_TRY(expr)                                                                        \
    do {                                                                                     \
        rdt_status _s = (expr);                                                              \
        if (_s != RDT_OK) return _s;                                                         \
    } while (0)

// Device-side status words (one int each, in a small device buffer).
enum DevFlag { FLAG_NONFINITE = 0, FLAG_TIMEOUT = 1, FLAG_COUNT = 8 };

// Bound on any single device-side wait before the kernel records a timeout and bails out.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

// ------------------------------------------------------------------ small device helpers

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Load 4 consecutive elements as fp32.
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load4(const bf16* p, float (&v)[4]) {
    uint2 x = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&x.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&x.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}
__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(bf16* p, const float (&v)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 x;
    x.x = *reinterpret_cast<uint32_t*>(&a);
    x.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = x;
}

// ------------------------------------------------------------------ programmatic dependent launch

// Every kernel of the library is launched with programmatic stream serialisation: it may
// start while its predecessor finishes, runs only its prologue (shared memory, barriers,
// TMEM, descriptor prefetch) before pdl_wait(), and touches global memory only after it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// cluster_x > 1 launches clusters of that many consecutive CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    return launch_pdl_cluster(kern, grid, block, smem, st, 1, std::forward<Args>(args)...);
}

int num_sms();   // SM count of the current device (cached)

// ------------------------------------------------------------------ mbarrier (sm_90+)

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase of parity `parity` to complete, at most limit_ns (kWaitLimitNs in
// every pipeline kernel). On timeout sets flags[FLAG_TIMEOUT] and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* flags,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) {
            if (flags) atomicExch(flags + FLAG_TIMEOUT, 1);
            return false;
        }
    }
}

// ------------------------------------------------------------------ TMA (bulk tensor copies)

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 2-D tiled load global -> this CTA's shared memory, completion counted on `bar`.
// x is the innermost (contiguous) coordinate in elements; it is always a multiple of the
// 128-byte box width here, so the 16-byte alignment rule of tiled copies holds.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* m, uint64_t* bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// ------------------------------------------------------------------ clusters (CTA pairs)

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared-window address of the same variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// All threads of every CTA in the cluster; release/acquire orders shared-memory traffic.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// Arrive on a barrier given by its cluster address (default semantics: release, CTA scope;
// the arrivals here only order tcgen05 reads already waited for, not memory traffic).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
// 2-D tiled load into this CTA's shared memory whose completion is counted on a barrier of
// either CTA of the pair (given by its cluster address). Not a multicast: one destination.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* m, uint32_t bar,
                                                 int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// ------------------------------------------------------------------ tcgen05 (5th-gen tensor cores)

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}
// CTA-pair forms (cta_group::2): allocation and release are issued by the same warp of both
// CTAs of the pair; the MMA by one thread of the even CTA, reading A and B from both CTAs'
// shared memory at the same offsets and accumulating into both CTAs' TMEM.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// Arrive on the barrier at this shared offset in every CTA of `cta_mask` once the pair's
// prior tcgen05 operations issued by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0), "r"(0),
        "r"(0), "r"(0), "r"(0)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
// Same with kind::tf32 (fp32 operands read as tf32, fp32 accumulate).
__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
// Warp-collective: lane i reads TMEM lane (base lane + i), 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
// Warp-collective: lane i reads TMEM lane (base lane + i), 4 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Warp-collective: lane i writes TMEM lane (base lane + i), 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with the 128-byte
// swizzle: rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart (stride byte offset),
// leading byte offset unused for this layout, descriptor version 1 (sm_100), layout
// code 2 (128-byte swizzle) in bits 61-63.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor: fp32 accumulator, A/B format (1 = bf16, 2 = tf32), both K-major,
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t make_idesc(int ab_format, int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(ab_format) << 7) |
           (static_cast<uint32_t>(ab_format) << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------------ host-side launchers

// Tensor maps (driver entry point resolved once through the runtime).
rdt_status make_tmap_2d(CUtensorMap* map, const void* base, bool bf16_elems, uint64_t inner,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                        uint32_t box_rows);

// Grouped (per-expert) operands use a capacity layout: group g's rows start at a fixed
// offset (routed expert e: e * cap, cap = tokens, since a token picks an expert at most once;
// shared expert s: all tokens), and a row inside a group is claimed with one atomic on the
// group's counter. The grouped GEMM decodes its 128-row tiles from those counters on the
// device; the host never sees them.
enum EpiKind {
    EPI_STORE = 0,      // C[row, col] = acc                     (OutT)
    EPI_ROPE = 1,       // C = acc with RoPE on the rotary part of rotated heads (OutT)
    EPI_OPROJ_LOOP = 2, // given h_in: y = x + acc, h_next = A h + B.e + acc (stores); without:
                        // y += acc, h_next += acc (fp32 vector atomics, into an earlier O
                        // projection's y and h_next: after depth attention)
    EPI_OPROJ_PLAIN = 3,// a_out = acc                             (fp32)
    EPI_SWIGLU = 4,     // U[row, j] = silu(acc_gate) * acc_up    (OutT)
    EPI_SCATTER = 5,    // dst[token, col] += w * acc             (fp32, vector atomics)
    EPI_STORE_F32 = 6,  // C[row, col] = acc                     (fp32)
    EPI_TOPK = 7        // router: top-k of the row's logits, gate weights, histogram
};

constexpr int kMaxCp = 8;   // context-parallel ranks at most

struct EpiParams {
    int kind;
    void* out;             // EPI_STORE / ROPE / SWIGLU: output base; OPROJ_PLAIN: a_out
    int ldo;               // row stride (elements) of `out`
    int ncols_valid;       // N (columns beyond are not stored)
    // RoPE
    const float* rope_cos; // [seq, rot/2]
    const float* rope_sin;
    int seq;               // positions per sequence: row r sits at r % seq (+ *pos_dev)
    const int* pos_dev;    // decode: the device-resident position of every row, or NULL
    int rope_ld;           // row stride of the angle tables ([rot/2][rope_ld])
    int head_w;            // width of one head's columns (64 or 160)
    int rot_off;           // rotary part starts at this column inside a head
    int rot_dim;           // rotary width
    int rope_limit;        // columns >= rope_limit are not rotated (V heads)
    int pos_off;           // context parallelism: position of this rank's first row of a sequence
    // context parallelism: the rotated K and V columns [cp_col0, cp_col0 + cp_w) of every row
    // are also stored into cp_n gather buffers (this rank's and its peers': [batch][cp_seq_tot]
    // [cp_w]), row (r / seq) * cp_seq_tot + cp_row_off + r % seq
    void* cp_dst[kMaxCp];
    int cp_n, cp_col0, cp_w, cp_seq_tot, cp_row_off;
    // O-projection loop epilogue. With h_in (no K split): the epilogue reads h (and e) itself
    // and stores y = x + a, h_next = A (.) h + B.e + a. Without h_in: y and h_next already
    // hold x + d and A (.) h + B.e + d (the depth-attention O projection formed them) and a
    // is added into both.
    float* y;              // x + a (stored, or += a)
    float* h_next;         // A*h + Be + a (stored, or += a); the MoE adds its share later
    int ld;                // row stride of y and h_next (= dim)
    const float* h_in;     // h_t [rows, ld] fp32, or NULL
    const void* e_in;      // e [rows, ld] (element type) when the block input is h + e, else NULL
    const float* a_diag;   // A [ld]
    const float* b_diag;   // diagonal B [ld] (B.e formed from e_in), or NULL: be is read
    const float* be;       // B.e [rows, ld] fp32 (dense B, or no e in the block input)
    // scatter
    const int* row_token;  // routed rows: token of each output row
    const float* row_w;    // routed rows: gate weight
    int shared_rows;       // rows [0, shared_rows) are shared-expert rows: token = row % ntok
    int ntok;              // scatter: row stride of the shared groups in U
    float* dst;            // scatter destination [ntok, ld]
    float* rows_out;       // scatter, deterministic mode: w * acc stored at its own row
                           // ([rows, ld], the tile's output row index) instead of reduced
    // router top-k (and dispatch: claim a row of each chosen expert)
    int n_exp, top_k;
    int* route_token;      // [n_exp * cap] token of each claimed row (or NULL: no dispatch)
    float* route_w;        // [n_exp * cap] gate weight of each claimed row
    int* slot_row;         // [ntok, top_k] claimed row of each (token, slot)
    int cap;
    const float* bias;     // selection bias [n_exp] or NULL
    int32_t* idx_out;      // [ntok, top_k]
    float* w_out;          // [ntok, top_k]
    int* counts;           // [n_exp] histogram (atomics)
    int32_t* trace_idx;    // optional copies
    float* trace_w;
    float* logits;         // split-K router: [ntok, n_exp] fp32 partial sums (zeroed beforehand)
    int* tile_count;       // split-K router: arrival counters per (row tile, 32-row quadrant)
                           // (zero, reset after use)
    const int* halted;     // ACT: [ntok] loops run by a halted token, 0 while running (or NULL):
                           // a halted token is routed to no expert (index -1, weight 0)
    int* flags;            // device status words
};

struct GemmArgs {
    int M;                 // rows of A / C (dense); grouped: rows of each shared group (tokens)
    int N;                 // columns of C (= rows of B per group)
    int kb_main;           // K blocks (128 bytes each) of A/B
    int kb_ext;            // extra K blocks from (A2, B2), at K offsets 0, 1, .. blocks
    int b2_row0;           // row offset into B2 for the extension blocks
    const int* counts;     // grouped: rows of each routed group [n_routed] (NULL = dense)
    int n_routed, n_shared;// grouped: routed groups, then shared groups (n_rows = cap each)
    int cap;               // grouped: rows reserved per group (>= tokens; the group stride)
    int a_routed_base;     // grouped: first A row of routed group 0 (shared groups read rows 0..cap)
    int max_tiles;         // grouped: upper bound on the row tiles (128 or 256 rows; grid sizing)
    int a_from_c;          // grouped: read A at the tile's output row (down projection)
    int split_k;           // > 1: K blocks split over that many CTAs per output tile (router)
    int pair;              // 1: CTA-pair tiles of 256 rows (cta_group::2); 0: one CTA, 128 rows
    int* flags;
};

// C = A B^T (+ extension) with the chosen epilogue, on tcgen05 tensor cores.
// tA: [rows, K] box (128 B x 128 rows); tB: [Nrows, K] box (128 B x BN rows, or BN/2 rows
// for pair tiles, where each CTA of the pair loads half of the tile's B rows).
rdt_status gemm_tc(bool bf16_elems, int bn, const CUtensorMap& tA, const CUtensorMap& tB,
                   const CUtensorMap* tA2, const CUtensorMap* tB2, const GemmArgs& args,
                   const EpiParams& epi, cudaStream_t st);
// The pair-tile instantiations (bf16, BN 128, 192 or 256, every epilogue but the router's).
rdt_status gemm_tc_pair(int bn, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                        const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                        cudaStream_t st);

// Causal attention. q rows [N, ldq], head h at column h*q_hstride; k/v similarly with
// Hkv heads; o [N, ldo] head h at column h*dv.
struct AttnArgs {
    const void* q; int ldq; int q_hstride;
    const void* k; int ldk; int k_hstride;
    const void* v; int ldv; int v_hstride;
    void* o; int ldo;
    int batch, seq, hq, hkv, dqk, dv;
    float scale;
    int* flags;
    // context parallelism (head width 64 only): the queries are positions q_off .. q_off +
    // seq - 1 of sequences whose keys and values have kv_seq rows each (0: kv_seq = seq,
    // q_off = 0)
    int q_off, kv_seq;
};
rdt_status attention(bool bf16_elems, const AttnArgs& a, cudaStream_t st);
// tcgen05 kernel: (dqk, dv) = (64, 64), or (160, 128) with v == k (absorbed MLA)
rdt_status attention_tc(const AttnArgs& a, cudaStream_t st);

// Context-parallel synchronisation (cp.cu). flags: this rank's words [READY 0..7 | CONS
// 0..7 | epoch]; peer_flags[q]: rank q's (this rank's own at q == rank). A loop's epoch is
// the handle's epoch + 1.
constexpr int kCpReady = 0, kCpCons = kMaxCp, kCpEpoch = 2 * kMaxCp, kCpFlagWords = 2 * kMaxCp + 1;
struct CpSyncArgs {
    unsigned* flags;
    unsigned* peer_flags[kMaxCp];
    int rank, size;
    int* status;
};
// before the push of loop e: ranks q > rank have consumed loop e - 1's keys
rdt_status cp_wait_consumed(const CpSyncArgs& a, cudaStream_t st);
// after the push: tell ranks q > rank that loop e's keys are there, wait for ranks s < rank
rdt_status cp_ready(const CpSyncArgs& a, cudaStream_t st);
// after the attention: tell ranks s < rank that loop e's keys are consumed; epoch = e
rdt_status cp_consumed(const CpSyncArgs& a, cudaStream_t st);

// Row kernels (rowops.cu).
struct Norm1Args {
    const float* h;    // fp32 state (NULL: none, the block input x is e alone)
    const void* e;     // cfg-dtype injection (x = h + e) or NULL
    const float* gamma;
    void* xn;          // [N, dim] cfg dtype
    int ntok, dim; float eps;
    int* zero_counts; int n_zero;   // counts to clear (next MoE), or NULL
};
rdt_status norm1(bool bf16_elems, const Norm1Args& a, cudaStream_t st);

// RMSNorm2 for the tensor-core router: yn (element type, also the experts' input) and
// the residual yn - yn_hi in the same type, so that [yn | yn_lo] . [W_r | W_r]^T gives the
// logits of the fp32 normalised row to ~2^-17 relative.
struct Norm2Args {
    const float* y; const float* gamma; void* yn; void* yn_lo; int ntok, dim; float eps;
    float* zero_rows; int zero_width;   // optional: rows of a [ntok, zero_width] fp32 buffer to clear
};
rdt_status norm2_split(bool bf16_elems, const Norm2Args& a, cudaStream_t st);

struct RouterArgs {
    const float* y; const float* gamma; void* yn; int ntok, dim; float eps;
    const void* w_router; const float* bias; int n_exp, top_k;
    int32_t* idx; float* w; int* counts;
    int32_t* trace_idx; float* trace_w;
    // dispatch (optional): counts double as the claim counters of the capacity layout
    int* row_token; float* row_w; int* slot_row; int cap;
    void* xperm; int a_routed_base;   // fused router: write yn into the claimed rows here
    int store_yn;                      // fused router: also write yn at row `row` of yn
    int weights_static;                // fused router: w_router is not written by the previous
                                       // kernel in the stream (staged before waiting on it)
    const int* halted;                 // ACT: [ntok], nonzero = halted token, routed to no
                                       // expert (index -1, weight 0); NULL = all route
};
rdt_status norm2_router(bool bf16_elems, const RouterArgs& a, cudaStream_t st);
// RMSNorm2 fused with the fp32 router when W_r (n_exp x dim, element type) takes at most
// 64 KB (staged in shared memory in its element type), n_exp <= 64, top_k <= 8 and dim is
// 128, 1024 or 2048
bool router_fits_smem(bool bf16_elems, int n_exp, int top_k, int dim);
rdt_status norm2_router_smem(bool bf16_elems, const RouterArgs& a, cudaStream_t st);

// Copy yn[token] into the claimed row of every (token, slot) (routers that do not write
// the copies themselves): xperm[a_routed_base + slot_row[token * k + j]] = xperm[token];
// a slot whose claimed row is negative (a halted token) is skipped.
rdt_status moe_copy(bool bf16_elems, void* xperm, const int* slot_row, int ntok, int top_k, int dim,
                    int a_routed_base, cudaStream_t st);

// Deterministic combine of the expert outputs: for each token n, in this order,
// dst[n] += rows[s * cap + n] for every shared expert s, then dst[n] += rows[n_shared * cap
// + slot_row[n * top_k + j]] for j = 0 .. top_k - 1 (slots with a negative row are skipped).
rdt_status moe_combine(const float* rows, const int* slot_row, int ntok, int top_k, int n_shared, int cap,
                       float* dst, int dim, cudaStream_t st);


rdt_status hoist(bool bf16_elems, const void* h0, const void* e, const float* Bdiag, float* h,
                 float* Be, size_t n, int dim, cudaStream_t st);
rdt_status matmul_nt_simt(bool a_bf16, const void* A, const float* B, float* C, int M, int N,
                          int K, cudaStream_t st);

struct MlaNormArgs {
    const float* lat; int ld_lat;   // [N, q_lat + kv_lat + rope] fp32
    const float* q_norm; const float* kv_norm;
    void* cq;   // [N, q_lat]
    void* kv;   // [N, kv_lat + rope]
    const float* rope_cos; const float* rope_sin;
    int ntok, seq, q_lat, kv_lat, rope; float eps;
    const int* pos_dev;    // decode: added to every row's position (NULL: 0)
    int rope_ld;           // row stride of the angle tables
};
rdt_status mla_latent_norm(bool bf16_elems, const MlaNormArgs& a, cudaStream_t st);

// One loop's ACT halting step over the fp32 state (one warp per token):
//   a token halted in an earlier loop (t > 0 and loops[n] > 0) keeps its state:
//     h_next[n] <- h_cur[n];
//   a running token takes p = sigmoid(w_halt . h_next[n] + b_halt); with c = cum[n] (0 at
//     t = 0) it halts if c + p >= threshold or last: out[n] (+)= (1 - c) h_next[n] and
//     loops[n] = t + 1; else out[n] (+)= p h_next[n] and loops[n] = 0; cum[n] = c + p.
//   At t = 0 out, cum and loops are written, not read.
struct ActArgs {
    const float* h_cur; float* h_next; float* out;   // [ntok, dim] fp32
    const float* w_halt; float b_halt, threshold;     // head [dim] fp32
    float* cum; int* loops;                           // [ntok]
    int ntok, dim, t, last;
};
rdt_status act_step(const ActArgs& a, cudaStream_t st);

// Weight preparation: C[m, n] = add[m, n] + sum_k A(m, k) B(k, n) with A(m, k) = A[m*sam + k*sak]
// and B(k, n) = B[k*sbk + n*sbn] (element type of the configuration; add [M, ld_add] or NULL),
// fp32 sums rounded once.
rdt_status prep_matmul(bool bf16_elems, const void* A, long sam, long sak, const void* B, long sbk,
                       long sbn, void* C, int ldc, int M, int N, int K, cudaStream_t st,
                       const void* add = nullptr, int ld_add = 0);
rdt_status check_finite(const float* x, size_t n, int* flags, cudaStream_t st);

// ---- decode with a per-loop KV cache (decode.cu). Caches hold bf16 rows; the current length
// (the new token's position during a step) lives in device memory.

// Copy columns [src_col0, src_col0 + width) of ntok rows into a loop's cache: row r belongs to
// sequence r / rows_per_seq at position r % rows_per_seq (+ *pos_dev), cache row
// (sequence * s_cap + position), width elements per cache row.
rdt_status cache_append(const void* src, int src_ld, int src_col0, int width, void* cache, int s_cap,
                        int rows_per_seq, const int* pos_dev, int ntok, cudaStream_t st);

struct DecodeAttnArgs {
    const void* q; int q_ld, q_hstride;      // new queries: row b, head h at column h * q_hstride
    const void* cache; int cache_ld, s_cap;  // loop t's cache, row (b * s_cap + position)
    int k_col0, k_hstride, v_col0, v_hstride;// key / value columns of KV head g in a cache row
    int batch, hq, hkv, dqk, dv;
    const int* len_dev;                      // keys 0 .. *len_dev
    float scale;
    float* part;                             // [batch, hq, decode_chunks(s_cap), dv + 2] scratch
    void* o; int ldo, dv_out;                // o [batch, ldo] bf16, head h at column h * dv_out
};
// softmax(q k^T * scale) v over the cached keys 0 .. length of each sequence, split over
// chunks of keys, then merged (two launches).
rdt_status decode_attention(const DecodeAttnArgs& a, cudaStream_t st);
int decode_chunks(int s_cap);
rdt_status len_advance(int* len, int by, cudaStream_t st);

// ---- depth attention (depth.cu): a token's query at loop t against its own keys and values
// of loops 0 .. t, kept in a per-token depth cache [ntok][max_depth][cache_w] (bf16).
struct DepthAttnArgs {
    const bf16* q; int q_ld;               // queries: row n, head h at column h * 64
    const bf16* cache; int cache_w, max_depth, v_col0;   // keys at column g * 64, values at v_col0 + g * 64
    int t, ntok, hq, hkv;
    float scale_log2;
    bf16* o; int o_ld;                     // o: row n, head h at column h * 64
};
rdt_status depth_attention(const DepthAttnArgs& a, cudaStream_t st);

}  // namespace rdt
