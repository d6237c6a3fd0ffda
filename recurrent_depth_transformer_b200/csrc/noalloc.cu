// MoE router for callers that cannot allocate device memory.
//
// rdt_moe_route_noalloc runs the same router kernel as rdt_moe_forward (RMSNorm2 of y,
// fp32 logits, top-k, softmax over the chosen logits, per-expert histogram) without a
// handle and without any allocation. The kernel's scratch - the normalised rows it writes
// for the experts and the per-expert counters - lives in the file-scope array below,
// which every process that loads librdt holds on every GPU it uses until exit.
#include <mutex>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr size_t kCountsBytes = 4096;               // 256 int32 counters, padded
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

// Device address of g_route_scratch, resolved once per device (host code cannot use the
// symbol's name as a device address).
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

rdt_status scratch_address(void** out) {
    int dev = 0;
    RDT_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device index out of range for the router scratch table");
        return RDT_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || p == nullptr) {
            set_error(std::string("cudaGetSymbolAddress(router scratch): ") + cudaGetErrorString(e));
            return RDT_ERR_CUDA;
        }
        g_addr[dev] = p;
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
    const size_t esz = dtype == RDT_BF16 ? 2 : 4;
    const size_t rows_bytes = static_cast<size_t>(ntok) * dim * esz;
    if (rows_bytes > kScratchBytes - kCountsBytes) {
        set_error("ntok * dim * element size = " + std::to_string(rows_bytes) +
                  " bytes exceeds the router scratch of " +
                  std::to_string(kScratchBytes - kCountsBytes) + " bytes");
        return RDT_ERR_UNSUPPORTED;
    }
    void* base = nullptr;
    RDT_TRY(scratch_address(&base));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* counts = static_cast<int*>(base);
    void* yn = static_cast<unsigned char*>(base) + kCountsBytes;
    RDT_CUDA_TRY(cudaMemsetAsync(counts, 0, kCountsBytes, st));   // the counters start at zero

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
    RDT_TRY(norm2_router(dtype == RDT_BF16, ra, st));
    if (expert_counts)
        RDT_CUDA_TRY(cudaMemcpyAsync(expert_counts, counts, static_cast<size_t>(n_experts) * 4,
                                     cudaMemcpyDeviceToDevice, st));
    return RDT_OK;
}
