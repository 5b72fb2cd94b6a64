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
#include <cudaTypedefs.h>

#include <mutex>

#include "gla_common.cuh"
#include "gla_plans.h"

#define GLA_STATIC_SCRATCH_BYTES (16u << 20)

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[GLA_STATIC_SCRATCH_BYTES];

using gla::kMaxDevices;
std::mutex g_mu;
// Per device: the array's device address and the id of the CUDA context it was looked up in.
// A device reset (cudaDeviceReset) ends that context and the next one loads the array anew, so
// the address is looked up again whenever the current context's id differs.
void* g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};

// Id of the calling thread's current CUDA context (unique for the process's lifetime), or 0
// when there is none or the driver cannot say.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the array on the current device. In host code the array's name is only a
// host-side stand-in, so the address comes from cudaGetSymbolAddress, with the device current:
// once per device and CUDA context, then from the cache.
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);   // also makes the device's context current
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = current_context_id();
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
    cudaError_t e = scratch_on_current_device(&ws);
    if (e != cudaSuccess) return record_cuda(e, "static scratch address lookup");
    cudaStream_t st = (cudaStream_t)stream;
    // the status word must start at zero; everything else is written before it is read
    e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
    if (e != cudaSuccess) return record_cuda(e, "status word reset");
    if ((size_t)P.B * P.H == 0) return GLA_OK;
    e = simt::fwd(P, p->io, q, k, v, g, igate, h0, o, hT, ws, st);
    return record_cuda(e, "launch");
}

}  // extern "C"
