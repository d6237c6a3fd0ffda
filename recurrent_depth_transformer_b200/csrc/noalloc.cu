// MoE router for callers that cannot allocate device memory.
//
// rdt_moe_route_noalloc runs the router of rdt_moe_forward (RMSNorm2 of y, logits of the
// fp32 normalised row, top-k, softmax over the chosen logits, per-expert histogram) without
// a handle and without any allocation, choosing its kernels exactly as the handle does:
// routers whose weight fits in shared memory run the fused RMSNorm2 + fp32-logit kernel,
// larger bf16 routers the RMSNorm2 split kernel and the tensor-core router GEMM, larger fp32
// routers the fp32 FMA kernel. Their scratch - the per-expert counters, a status word and,
// for the two larger-router paths, the normalised rows (bf16: also their residuals) - lives
// in the file-scope array below, which every process that loads librdt holds on every GPU
// it uses until exit.
#include <mutex>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr size_t kCountsBytes = 4096;               // 256 int32 counters, then the status words
constexpr size_t kFlagsOffset = 1024;               // FLAG_COUNT int32 device status words
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

// Device address of g_route_scratch, resolved once per (device, context): host code cannot
// use the symbol's name as a device address, and a context created anew (after a device
// reset) may load the module at another address, so the cached address is keyed on the
// context current when it was looked up.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};
CUcontext g_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}

rdt_status scratch_address(void** out) {
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device index out of range for the router scratch table");
        return RDT_ERR_UNSUPPORTED;
    }
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    CUcontext ctx = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) {
        set_error("cuCtxGetCurrent is unavailable");
        return RDT_ERR_CUDA;
    }
    if (!ctx) {                                 // nothing initialised yet on this thread:
        RDT_CUDA_TRY(cudaSetDevice(dev));       // make the device's primary context current
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) {
            set_error("no CUDA context is current");
            return RDT_ERR_CUDA;
        }
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev] || g_ctx[dev] != ctx) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || p == nullptr) {
            set_error(std::string("cudaGetSymbolAddress(router scratch): ") + cudaGetErrorString(e));
            return RDT_ERR_CUDA;
        }
        g_addr[dev] = p;
        g_ctx[dev] = ctx;
    }
    *out = g_addr[dev];
    return RDT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace rdt

using namespace rdt;

extern "C" rdt_status rdt_moe_route_noalloc(int32_t dtype, const float* y, const float* norm2,
                                            const void* w_router, const float* router_bias, int ntok,
                                            int dim, int n_experts, int top_k, float eps,
                                            int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                                            void* stream) {
    if (dtype != RDT_BF16 && dtype != RDT_F32) {
        set_error("dtype must be RDT_BF16 or RDT_F32");
        return RDT_ERR_INVALID_ARG;
    }
    if (!y || !norm2 || !w_router || !topk_idx || !topk_w) {
        set_error("y, norm2, w_router, topk_idx and topk_w must be non-NULL");
        return RDT_ERR_INVALID_ARG;
    }
    if (!aligned16(y) || !aligned16(norm2) || !aligned16(w_router) || !aligned16(topk_idx) ||
        !aligned16(topk_w) || (router_bias && !aligned16(router_bias)) ||
        (expert_counts && !aligned16(expert_counts))) {
        set_error("every pointer must be 16-byte aligned");
        return RDT_ERR_MISALIGNED;
    }
    const int nv = dim / 128;
    if (ntok < 1 || dim < 128 || dim % 128 || (nv & (nv - 1)) || nv > 32) {
        set_error("ntok >= 1 and dim = 128 * 2^k <= 4096 required");
        return RDT_ERR_UNSUPPORTED;
    }
    if (n_experts < 1 || n_experts > 256 || top_k < 1 || top_k > n_experts || top_k > 16) {
        set_error("need 1 <= top_k <= min(n_experts, 16) and n_experts <= 256");
        return RDT_ERR_UNSUPPORTED;
    }
    const bool bf = dtype == RDT_BF16;
    const size_t esz = bf ? 2 : 4;
    const size_t row_bytes = static_cast<size_t>(ntok) * dim * esz;
    // Row scratch per path: the fused shared-memory router keeps its normalised rows in
    // registers (none); the bf16 tensor-core router needs yn and its residual yn_lo; the
    // fp32 FMA router writes yn.
    const bool fused = router_fits_smem(bf, n_experts, top_k, dim);
    const size_t need = fused ? 0 : bf ? 2 * row_bytes : row_bytes;
    if (need > kScratchBytes - kCountsBytes) {
        set_error("the router needs " + std::to_string(need) + " bytes of scratch for ntok = " +
                  std::to_string(ntok) + ", dim = " + std::to_string(dim) + "; the array holds " +
                  std::to_string(kScratchBytes - kCountsBytes));
        return RDT_ERR_UNSUPPORTED;
    }
    void* base = nullptr;
    RDT_TRY(scratch_address(&base));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* counts = static_cast<int*>(base);
    int* flags = reinterpret_cast<int*>(static_cast<unsigned char*>(base) + kFlagsOffset);
    void* yn = static_cast<unsigned char*>(base) + kCountsBytes;
    void* yn_lo = static_cast<unsigned char*>(yn) + row_bytes;
    // the counters and the status words start at zero
    RDT_CUDA_TRY(cudaMemsetAsync(counts, 0, kCountsBytes, st));

    if (fused) {
        // the same kernel as rdt_moe_forward for routers whose weight fits in shared memory
        RouterArgs ra{};
        ra.y = y;
        ra.gamma = norm2;
        ra.yn = nullptr;             // no normalised copy: nothing here reads one
        ra.ntok = ntok;
        ra.dim = dim;
        ra.eps = eps;
        ra.w_router = w_router;
        ra.bias = router_bias;
        ra.n_exp = n_experts;
        ra.top_k = top_k;
        ra.idx = topk_idx;
        ra.w = topk_w;
        ra.counts = counts;
        ra.store_yn = 0;
        RDT_TRY(norm2_router_smem(bf, ra, st));
    } else if (bf) {
        // the same two steps as rdt_moe_forward: RMSNorm2 split into yn + yn_lo, then the
        // tensor-core router GEMM [yn | yn_lo] . [W_r | W_r]^T with the top-k epilogue
        Norm2Args n2{};
        n2.y = y;
        n2.gamma = norm2;
        n2.yn = yn;
        n2.yn_lo = yn_lo;
        n2.ntok = ntok;
        n2.dim = dim;
        n2.eps = eps;
        RDT_TRY(norm2_split(true, n2, st));
        const int bn = n_experts <= 64 ? 64 : n_experts <= 128 ? 128 : 256;
        CUtensorMap m_yn, m_lo, m_wr;   // host-side descriptors: encoding allocates nothing
        RDT_TRY(make_tmap_2d(&m_yn, yn, true, dim, ntok, static_cast<uint64_t>(dim) * 2, 64, 128));
        RDT_TRY(make_tmap_2d(&m_lo, yn_lo, true, dim, ntok, static_cast<uint64_t>(dim) * 2, 64, 128));
        RDT_TRY(make_tmap_2d(&m_wr, w_router, true, dim, n_experts, static_cast<uint64_t>(dim) * 2, 64, bn));
        GemmArgs gr{};
        gr.M = ntok;
        gr.N = n_experts;
        gr.kb_main = dim * 2 / 128;
        gr.kb_ext = gr.kb_main;
        gr.flags = flags;           // a bounded wait that gives up is recorded here
        EpiParams er{};
        er.flags = flags;
        er.kind = EPI_TOPK;
        er.n_exp = n_experts;
        er.top_k = top_k;
        er.bias = router_bias;
        er.idx_out = topk_idx;
        er.w_out = topk_w;
        er.counts = counts;
        RDT_TRY(gemm_tc(true, bn, m_yn, m_wr, &m_lo, &m_wr, gr, er, st));
    } else {
        RouterArgs ra{};
        ra.y = y;
        ra.gamma = norm2;
        ra.yn = yn;
        ra.ntok = ntok;
        ra.dim = dim;
        ra.eps = eps;
        ra.w_router = w_router;
        ra.bias = router_bias;
        ra.n_exp = n_experts;
        ra.top_k = top_k;
        ra.idx = topk_idx;
        ra.w = topk_w;
        ra.counts = counts;
        RDT_TRY(norm2_router(false, ra, st));
    }
    if (expert_counts)
        RDT_CUDA_TRY(cudaMemcpyAsync(expert_counts, counts, static_cast<size_t>(n_experts) * 4,
                                     cudaMemcpyDeviceToDevice, st));
    return RDT_OK;
}

extern "C" rdt_status rdt_moe_route_noalloc_status(void* stream) {
    void* base = nullptr;
    RDT_TRY(scratch_address(&base));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    RDT_CUDA_TRY(cudaStreamSynchronize(st));
    int flags[FLAG_COUNT];
    RDT_CUDA_TRY(cudaMemcpy(flags, static_cast<unsigned char*>(base) + kFlagsOffset, sizeof(flags),
                            cudaMemcpyDeviceToHost));
    if (flags[FLAG_TIMEOUT]) {
        set_error("a bounded device-side wait of the router gave up: its outputs are incomplete");
        return RDT_ERR_DEVICE_TIMEOUT;
    }
    return RDT_OK;
}
