// Forward pass that allocates nothing: the CUDA-core (SIMT) forward of this library, with
// its scratch memory (the 256-byte device status word, the in-chunk cumulative log-gates
// and the chunk-boundary states) taken from one fixed array compiled into the library
// instead of from a caller-provided workspace.
//
// Who needs this: callers that cannot allocate device memory themselves, for instance a
// host that runs under a fixed device-memory budget owned by another allocator, or code
// that must not call cudaMalloc because it synchronises the device and would stall
// latency-critical work. They still pass their inputs and outputs; only the scratch is
// provided here.
//
// Limits and sharing: the array holds GLA_STATIC_SCRATCH_BYTES bytes on every GPU that
// loads the library, for the life of the process. Every call uses the same array and it
// keeps the last call's contents; two calls whose work overlaps on the GPU (different
// streams, or different host threads) race on it. Problems whose scratch need exceeds the
// array are rejected with GLA_ERR_WORKSPACE before any launch.
#include <mutex>

#include "gla_common.cuh"
#include "gla_plans.h"

#define GLA_STATIC_SCRATCH_BYTES (16u << 20)

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[GLA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device. In host code the array's name is
// only a host-side stand-in, so the address must come from cudaGetSymbolAddress, once per
// device, with that device current.
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d == 64 || d == 128 || d == 256; }

}  // namespace

extern "C" {

gla_status gla_fwd_static_scratch(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                                  const float* igate, const float* h0, void* o, float* hT, void* stream) {
    using namespace gla;
    if (!p) return GLA_ERR_INVALID_ARG;
    if (p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE && p->gate != GLA_GATE_PER_KEY && p->gate != GLA_GATE_PER_HEAD)
        return GLA_ERR_INVALID_ARG;
    if (p->chunk < 16 || p->chunk > 1024 || p->chunk % 16 != 0) return GLA_ERR_UNSUPPORTED;
    if (!dim_ok(p->Dk) || !dim_ok(p->Dv)) return GLA_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 65535LL) return GLA_ERR_UNSUPPORTED;
    Dims P;
    P.B = p->B; P.H = p->H; P.L = p->L; P.Dk = p->Dk; P.Dv = p->Dv; P.C = p->chunk;
    P.N = cdiv(p->L, p->chunk);
    P.gate = p->gate;
    P.scale = p->scale;
    const bool empty = (size_t)P.B * P.H * P.L == 0;
    if (!empty && (!q || !k || !v || !o)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, igate, h0, o, hT};
    for (const void* x : ptrs)
        if (!aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (simt::workspace_bytes(P, false) > GLA_STATIC_SCRATCH_BYTES) return GLA_ERR_WORKSPACE;
    void* ws = nullptr;
    if (scratch_on_current_device(&ws) != cudaSuccess) return GLA_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    // the status word must start at zero; everything else is written before it is read
    if (cudaMemsetAsync(ws, 0, kStatusBytes, st) != cudaSuccess) return GLA_ERR_CUDA;
    if ((size_t)P.B * P.H == 0) return GLA_OK;
    const cudaError_t e = simt::fwd(P, p->io, q, k, v, g, igate, h0, o, hT, ws, st);
    return e == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

}  // extern "C"
