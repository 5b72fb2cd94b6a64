// Diagnostics of the device-side failure path: a bounded mbarrier wait that nothing
// completes, so that a test can watch the timeout reach the device status word without
// faulting, trapping or hanging the GPU.
#include "gla_common.cuh"
#include "sm100.cuh"

namespace gla {
namespace {

__global__ void __launch_bounds__(32) k_wait_timeout(int* status, uint32_t polls) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::mbar_fence_init();
    }
    __syncthreads();
    // phase 0 of the barrier never completes (nothing arrives): the wait gives up after `polls`
    // polls, as every wait in the library's kernels does, and records the timeout
    if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, polls)) atomicOr(status, kDevStatusTimeout);
}

}  // namespace
}  // namespace gla

extern "C" gla_status gla_debug_wait_timeout(void* ws, unsigned polls, void* stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return GLA_ERR_INVALID_ARG;
    if (polls == 0 || polls > gla::sm100::kWaitPolls) return GLA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = cudaMemsetAsync(ws, 0, gla::kStatusBytes, st);
    if (e != cudaSuccess) return gla::record_cuda(e, "status word reset");
    GLA_LAUNCH("debug_wait_timeout", st, gla::k_wait_timeout<<<1, 32, 0, st>>>(static_cast<int*>(ws), polls));
    return gla::record_cuda(cudaGetLastError(), "wait-timeout kernel launch");
}
