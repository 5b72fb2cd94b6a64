// Internal interface between the C-ABI layer (gla_api.cu) and the kernel plans.
#pragma once
#include <cuda_runtime.h>

#include "gla_common.cuh"

namespace gla {
namespace simt {
size_t workspace_bytes(const Dims& P, bool bwd);
cudaError_t fwd(const Dims& P, gla_dtype io, const void* q, const void* k, const void* v, const float* g,
                const float* ig, const float* h0, void* o, float* hT, void* ws, cudaStream_t st);
cudaError_t bwd(const Dims& P, gla_dtype io, const void* q, const void* k, const void* v, const float* g,
                const float* ig, const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                float* dg, float* di, float* dh0, void* ws, cudaStream_t st);
}  // namespace simt

namespace tc {
struct FwdPlan {
    int dvt;            // Dv columns per CTA
    int nseg;           // sequence segments processed in parallel (1 = single pass)
    int tiles_per_seg;  // 64-token tiles per segment
};
FwdPlan plan_fwd(const Dims& P);
bool supports(const Dims& P);
size_t fwd_workspace_bytes(const Dims& P);
cudaError_t fwd(const Dims& P, const void* q, const void* k, const void* v, const float* g, const float* ig,
                const float* h0, void* o, float* hT, void* ws, cudaStream_t st);
}  // namespace tc
}  // namespace gla
