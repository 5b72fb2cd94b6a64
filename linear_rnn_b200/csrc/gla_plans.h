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
// saved (nullable): [BH, nseg_b, Dk, Dv] states entering the backward plan's segments
// z = 1 .. nseg_b-1 (bwd_plan_info), written on the way
cudaError_t fwd(const Dims& P, const void* q, const void* k, const void* v, const float* g, const float* ig,
                const float* h0, void* o, float* hT, float* saved, void* ws, cudaStream_t st);
// Segment state passes and scans shared by the forward and the backward.
//   mode 1: forward local end states of segments 0..nseg-2 (a = k, b = v)
//   mode 2: reverse local state gradients of segments 1..nseg-1 (a = q, b = dO)
//   mode 3: forward local end states of all segments 0..nseg-1 (a = k, b = v)
//   mode 4: reverse local state gradients of all segments 0..nseg-1 (a = q, b = dO)
cudaError_t state_pass(const Dims& P, int mode, const void* a_src, const void* b_src, const float* g,
                       const float* ig, int nseg, int tiles_per_seg, float* seg_state, float* seg_gamma, int* status,
                       cudaStream_t st);
cudaError_t seg_scan(const Dims& P, int nseg, const float* seg_state, const float* seg_gamma, const float* h0,
                     float* sinit, cudaStream_t st);
cudaError_t seg_rscan(const Dims& P, int nseg, const float* seg_state, const float* seg_gamma, const float* dhT,
                      float* gend, cudaStream_t st);
int num_sms();
// DeltaNet on the tensor cores (gla_deltanet_tc.cu): bf16 I/O, Dk 64 or 128, Dv a multiple of
// 64, chunk 64. Forward walk; o null: the state walk only (the backward's recompute). saved
// (nullable): [BH, ceil(L/64), Dk, Dv] bf16, the state entering every chunk; status (nullable):
// device status word for a wait that gave up.
cudaError_t deltanet_fwd(int B, int H, int L, int Dk, int Dv, float scale, const void* q, const void* k,
                         const void* v, const float* beta, const float* h0, void* o, float* hT, void* saved,
                         int* status, cudaStream_t st);
// The backward's reverse walk: dR ([BH*L, Dv] fp32), dv (bf16), dh0, and the gradient at every
// chunk's end (bf16, laid out as saved).
cudaError_t deltanet_walk(int B, int H, int L, int Dk, int Dv, float scale, const void* q, const void* k,
                          const float* beta, const void* dO, const float* dhT, float* drw, void* dsend, void* dv,
                          float* dh0, cudaStream_t st);
// The backward's per-chunk gradients: dq, dk (bf16) and dbeta from the saved states, the end
// gradients and dR, one CTA per (chunk, batch*head).
cudaError_t deltanet_grads(int B, int H, int L, int Dk, int Dv, float scale, const void* q, const void* k,
                           const void* v, const float* beta, const void* dO, const void* saved, const float* drw,
                           const void* dsend, void* dq, void* dk, float* dbeta, cudaStream_t st);
// Backward (gla_tc_bwd.cu)
bool bwd_supports(const Dims& P);
size_t bwd_workspace_bytes(const Dims& P);
void bwd_plan_info(const Dims& P, int* nseg, int* tiles_per_seg);
// saved (nullable): the states a forward wrote for this problem; skips the forward state pass
cudaError_t bwd(const Dims& P, const void* q, const void* k, const void* v, const float* g, const float* ig,
                const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dg, float* di,
                float* dh0, const float* saved, void* ws, cudaStream_t st);
}  // namespace tc
}  // namespace gla
