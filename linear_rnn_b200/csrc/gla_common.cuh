// Shared device/host helpers of the CUDA library (not of the oracle).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/gla.h"

namespace gla {

// Kernel-side view of one problem. Pointers are device pointers.
struct Dims {
    int B, H, L, Dk, Dv, C, N;  // N = number of chunks = ceil(L / C)
    int gate;                    // gla_gate_mode
    float scale;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device status word at the start of every workspace (first 256 bytes).
constexpr size_t kStatusBytes = 256;
constexpr int kDevStatusOk = 0;
constexpr int kDevStatusTimeout = 1;   // bits of the device status word
constexpr int kDevStatusRange = 2;
// Most negative in-tile total log-decay the tensor-core plans evaluate. They factor the in-tile
// decay e^(b_t - b_s) as e^(b_t) e^(-b_s) with one reference row per 64-token tile, so their
// operands and accumulators carry factors up to e^|Gamma| (k e^-b, sums of up to 64 such terms
// times O(Dk) products) and down to e^-|Gamma| (q e^b): at |Gamma| = 70 the largest stays about
// 1e4 below the fp32 / bf16 maximum and the smallest above the smallest normal.
constexpr float kMinTileLogDecay = -70.f;

// Devices a process may drive, for the per-device host state (launch attributes, streams).
constexpr int kMaxDevices = 64;

// Raises the dynamic shared-memory limit of `kern` to `bytes` on the current device, once per
// device and call site (`seen`, one flag per device): the attribute belongs to the device's
// context, so a process that launches on several devices sets it on each.
template <typename K>
inline cudaError_t smem_attr_once(K kern, size_t bytes, std::atomic<bool> (&seen)[kMaxDevices]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (seen[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) seen[dev].store(true, std::memory_order_release);
    return e;
}

// Launch accounting (gla_api.cu): every kernel launch of the library goes through
// GLA_LAUNCH, which counts it and, while the profiler is enabled, brackets it with CUDA
// events recorded on the launching stream.
void prof_begin(const char* name, cudaStream_t st);
void prof_end(cudaStream_t st);
// Whether launches are being timed (gla_profiler_enable): plans then keep every kernel on the
// caller's stream, so that each launch's events time that kernel alone.
bool prof_enabled();

// Maps a CUDA error to the C ABI's status: GLA_OK for cudaSuccess, otherwise GLA_ERR_CUDA after
// recording where it happened and the CUDA error's name and text for gla_last_error_detail
// (gla_api.cu; one record per host thread).
gla_status record_cuda(cudaError_t e, const char* where);

}  // namespace gla

#define GLA_LAUNCH(name, stream, ...)      \
    do {                                   \
        ::gla::prof_begin(name, stream);   \
        __VA_ARGS__;                       \
        ::gla::prof_end(stream);           \
    } while (0)
