// Failure-detection probe of the bounded device-side waits.
//
// Every pipeline kernel of the library (the tensor-core GEMMs and attention) waits on
// mbarrier phases with mbar_wait, which gives up after a time limit, records the timeout in
// a device status word and lets the kernel leave. rdt_wait_probe exercises exactly that wait
// on a barrier that nothing ever arrives on (no copy, MMA or other CTA is involved), with a
// caller-chosen limit, so that a test can see the wait run out, the kernel return and the
// status reach the host, with the context still usable afterwards.
#include "rdt_internal.cuh"

namespace rdt {
namespace {

static __device__ int g_probe_flags[FLAG_COUNT];

__global__ void wait_probe_kernel(unsigned long long limit_ns, int* flags) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 of a barrier expecting one arrival that never comes
        const bool done = mbar_wait(&bar, 0, flags, limit_ns);
        if (done) atomicExch(flags + FLAG_NONFINITE, 1);   // cannot happen: nothing arrives
    }
}

}  // namespace
}  // namespace rdt

using namespace rdt;

extern "C" rdt_status rdt_wait_probe(int64_t limit_ns, void* stream) {
    if (limit_ns < 1 || limit_ns > 2000000000LL) {
        set_error("limit_ns must be in [1, 2e9]");
        return RDT_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* flags = nullptr;
    RDT_CUDA_TRY(cudaGetSymbolAddress(reinterpret_cast<void**>(&flags), g_probe_flags));
    RDT_CUDA_TRY(cudaMemsetAsync(flags, 0, FLAG_COUNT * sizeof(int), st));
    wait_probe_kernel<<<1, 32, 0, st>>>(static_cast<unsigned long long>(limit_ns), flags);
    RDT_CUDA_TRY(cudaGetLastError());
    RDT_CUDA_TRY(cudaStreamSynchronize(st));
    int host[FLAG_COUNT];
    RDT_CUDA_TRY(cudaMemcpy(host, flags, sizeof(host), cudaMemcpyDeviceToHost));
    if (host[FLAG_TIMEOUT]) {
        set_error("the probe's bounded wait gave up, as it should");
        return RDT_ERR_DEVICE_TIMEOUT;
    }
    set_error("the probe's wait completed although nothing arrived");
    return RDT_ERR_CUDA;
}
