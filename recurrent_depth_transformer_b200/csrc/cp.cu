// Context parallelism: the flag protocol between the ranks that share one sequence, and the
// inter-process handles that let them map one another's buffers.
//
// Rank r of `size` holds positions [r S, (r + 1) S) of each sequence. In loop e (the
// handle's epoch + 1) the QKV projection of rank r writes its rotated keys and values into
// the gather buffers of ranks r .. size - 1 (the causal mask lets rank q see the keys of
// ranks 0 .. q only), so:
//   before the push   rank r waits until every q > r has consumed loop e - 1 (CONS[q] of
//                     rank r's words >= e - 1): the push must not overwrite keys in use;
//   after the push    rank r sets READY[r] = e in the words of every q > r, then waits
//                     until READY[s] >= e for every s < r;
//   after attention   rank r sets CONS[r] = e in the words of every s < r, and epoch = e.
// Flags are written with system-scope release stores (after a system-scope fence, so that
// the preceding kernels' stores to peer memory are visible first) and read with
// system-scope acquire loads; every wait is bounded (kWaitLimitNs), and one that gives up
// records a timeout in the status words and returns.
#include <cstring>

#include "rdt_internal.cuh"

namespace rdt {
namespace {

__device__ __forceinline__ unsigned ld_acquire_sys(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_sys(unsigned* p, unsigned v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// until *p >= want (wrap-safe), at most kWaitLimitNs
__device__ bool wait_at_least(const unsigned* p, unsigned want, int* status) {
    if (static_cast<int>(ld_acquire_sys(p) - want) >= 0) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i) {
            if (static_cast<int>(ld_acquire_sys(p) - want) >= 0) return true;
            __nanosleep(100);
        }
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            if (status) atomicExch(status + FLAG_TIMEOUT, 1);
            return false;
        }
    }
}

// One warp; lane q speaks for rank q.
__global__ void cp_wait_consumed_kernel(const CpSyncArgs a) {
    const int q = threadIdx.x;
    const unsigned e = a.flags[kCpEpoch] + 1;
    if (q > a.rank && q < a.size) wait_at_least(a.flags + kCpCons + q, e - 1, a.status);
}

__global__ void cp_ready_kernel(const CpSyncArgs a) {
    const int q = threadIdx.x;
    const unsigned e = a.flags[kCpEpoch] + 1;
    __threadfence_system();   // this rank's keys (written by the projection) before the flag
    if (q > a.rank && q < a.size) st_release_sys(a.peer_flags[q] + kCpReady + a.rank, e);
    if (q < a.rank) wait_at_least(a.flags + kCpReady + q, e, a.status);
}

__global__ void cp_consumed_kernel(const CpSyncArgs a) {
    const int q = threadIdx.x;
    const unsigned e = a.flags[kCpEpoch] + 1;
    __threadfence_system();   // the attention's reads of the gathered keys are done
    if (q < a.rank) st_release_sys(a.peer_flags[q] + kCpCons + a.rank, e);
    __syncwarp();
    if (q == 0) a.flags[kCpEpoch] = e;
}

rdt_status launch_sync(void (*k)(CpSyncArgs), const CpSyncArgs& a, cudaStream_t st) {
    if (a.size < 2 || a.size > kMaxCp || a.rank < 0 || a.rank >= a.size) {
        set_error("context parallelism: rank / size out of range");
        return RDT_ERR_INVALID_ARG;
    }
    k<<<1, 32, 0, st>>>(a);
    RDT_CUDA_TRY(cudaGetLastError());
    return RDT_OK;
}

}  // namespace

rdt_status cp_wait_consumed(const CpSyncArgs& a, cudaStream_t st) { return launch_sync(cp_wait_consumed_kernel, a, st); }
rdt_status cp_ready(const CpSyncArgs& a, cudaStream_t st) { return launch_sync(cp_ready_kernel, a, st); }
rdt_status cp_consumed(const CpSyncArgs& a, cudaStream_t st) { return launch_sync(cp_consumed_kernel, a, st); }

}  // namespace rdt

extern "C" {

rdt_status rdt_ipc_get_handle(const void* dev_ptr, void* handle64) {
    static_assert(sizeof(cudaIpcMemHandle_t) == 64, "handle size");
    if (!dev_ptr || !handle64) return RDT_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hd;
    const cudaError_t err = cudaIpcGetMemHandle(&hd, const_cast<void*>(dev_ptr));
    if (err != cudaSuccess) {
        rdt::set_error(std::string("cudaIpcGetMemHandle: ") + cudaGetErrorString(err));
        return RDT_ERR_CUDA;
    }
    std::memcpy(handle64, &hd, sizeof(hd));
    return RDT_OK;
}

rdt_status rdt_ipc_open_handle(const void* handle64, void** dev_ptr) {
    if (!handle64 || !dev_ptr) return RDT_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hd;
    std::memcpy(&hd, handle64, sizeof(hd));
    const cudaError_t err = cudaIpcOpenMemHandle(dev_ptr, hd, cudaIpcMemLazyEnablePeerAccess);
    if (err != cudaSuccess) {
        rdt::set_error(std::string("cudaIpcOpenMemHandle: ") + cudaGetErrorString(err));
        return RDT_ERR_CUDA;
    }
    return RDT_OK;
}

rdt_status rdt_ipc_close_handle(void* dev_ptr) {
    if (!dev_ptr) return RDT_ERR_INVALID_ARG;
    const cudaError_t err = cudaIpcCloseMemHandle(dev_ptr);
    if (err != cudaSuccess) {
        rdt::set_error(std::string("cudaIpcCloseMemHandle: ") + cudaGetErrorString(err));
        return RDT_ERR_CUDA;
    }
    return RDT_OK;
}

}  // extern "C"
