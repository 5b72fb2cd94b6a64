// Sequence sharding: the per-shard pieces of the chunkwise forward when a sequence is cut
// into contiguous shards (one per rank). The chunkwise algorithm of the talk summary
// "Hardware-Efficient Training of Linear Attention Models" (section 11:58) carries a state
// across chunk boundaries; across shard boundaries the same holds with the shard as the
// chunk: shard p's initial state is
//   S_in(p) = fold over p' < p of  S <- diag(e^{Gamma_p'}) S + S_loc(p'),   S <- h0 first,
// where S_loc(p') is shard p''s end state from a zero initial state and Gamma_p' its total
// log-decay (the state-passing form of the Tiled Flash Linear Attention abstract, with the
// shards as the tiles). gla_shard_state gives (S_loc, Gamma) of a shard, gla_state_fold the
// fold; one all-gather of the (S_loc, Gamma) pairs between them is the only exchange. The
// backward mirrors it: gla_shard_state_grad gives a shard's state gradient at its start from a
// zero gradient at its end, G_loc, and the same fold run over the later shards in reverse
// order, from the upstream dhT, gives the gradient flowing into the shard's end.
#include "gla_common.cuh"
#include "gla_plans.h"
#include "gla_tc_common.cuh"

namespace gla {
namespace {

// One thread per four consecutive state elements of one (bh, key dim) row.
__global__ void __launch_bounds__(256) k_state_fold(const float* __restrict__ states, const float* __restrict__ gammas,
                                                    const float* __restrict__ h0, float* __restrict__ out, int count,
                                                    int BH, int Dk, int Dv) {
    const long per4 = (long)Dk * Dv / 4;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)BH * per4) return;
    const int bh = (int)(idx / per4);
    const int d = (int)(4 * (idx - (long)bh * per4) / Dv);
    float4 S = h0 ? reinterpret_cast<const float4*>(h0)[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < count; ++p) {
        const float e = __expf(gammas[((long)p * BH + bh) * Dk + d]);
        const float4 x = reinterpret_cast<const float4*>(states)[(long)p * BH * per4 + idx];
        S = make_float4(fmaf(e, S.x, x.x), fmaf(e, S.y, x.y), fmaf(e, S.z, x.z), fmaf(e, S.w, x.w));
    }
    reinterpret_cast<float4*>(out)[idx] = S;
}

bool aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }
bool dims_ok(const gla_problem* p) {
    return (p->Dk == 64 || p->Dk == 128 || p->Dk == 256) && (p->Dv == 64 || p->Dv == 128 || p->Dv == 256);
}

}  // namespace
}  // namespace gla

extern "C" gla_status gla_shard_state(const gla_problem* p, const void* k, const void* v, const float* g,
                                      const float* igate, float* state, float* gamma, void* ws, size_t ws_bytes,
                                      void* stream) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE && p->gate != GLA_GATE_PER_KEY && p->gate != GLA_GATE_PER_HEAD)
        return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_BF16 || !gla::dims_ok(p) || p->chunk < 64 || p->chunk > 1024 || p->chunk % 64 != 0)
        return GLA_ERR_UNSUPPORTED;   // the tensor-core state pass: bf16 I/O, whole 64-token tiles
    if ((long long)p->B * p->H > 65535LL) return GLA_ERR_UNSUPPORTED;
    if (!state || !gamma || !ws) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < gla::kStatusBytes) return GLA_ERR_WORKSPACE;
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!k || !v)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {k, v, g, igate, state, gamma, ws};
    for (const void* x : ptrs)
        if (!gla::aligned16(x)) return GLA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, gla::kStatusBytes, st);
    if (e != cudaSuccess) return gla::record_cuda(e, "status word reset");
    const size_t BH = (size_t)p->B * p->H;
    if (BH == 0) return GLA_OK;
    if (p->L == 0) {   // an empty shard passes the state through: zero state, zero log-decay
        e = cudaMemsetAsync(state, 0, 4 * BH * p->Dk * p->Dv, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gamma, 0, 4 * BH * p->Dk, st);
        return gla::record_cuda(e, "empty shard");
    }
    gla::Dims P;
    P.B = p->B; P.H = p->H; P.L = p->L; P.Dk = p->Dk; P.Dv = p->Dv; P.C = p->chunk;
    P.N = gla::cdiv(p->L, p->chunk);
    P.gate = p->gate;
    P.scale = p->scale;
    // the whole shard as the one segment of the state-only pass: one CTA per (head, Dv tile)
    // walks it (the shards themselves are the sequence parallelism)
    const int ntiles = gla::cdiv(p->L, gla::tc::TR);
    e = gla::tc::state_pass(P, 3, k, v, g, igate, 1, ntiles, state, gamma, static_cast<int*>(ws), st);
    return gla::record_cuda(e, "shard state pass");
}

extern "C" gla_status gla_shard_state_grad(const gla_problem* p, const void* q, const void* dO, const float* g,
                                           float* state_grad, float* gamma, void* ws, size_t ws_bytes, void* stream) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE && p->gate != GLA_GATE_PER_KEY && p->gate != GLA_GATE_PER_HEAD)
        return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_BF16 || !gla::dims_ok(p) || p->chunk < 64 || p->chunk > 1024 || p->chunk % 64 != 0)
        return GLA_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 65535LL) return GLA_ERR_UNSUPPORTED;
    if (!state_grad || !gamma || !ws) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < gla::kStatusBytes) return GLA_ERR_WORKSPACE;
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!q || !dO)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, dO, g, state_grad, gamma, ws};
    for (const void* x : ptrs)
        if (!gla::aligned16(x)) return GLA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, gla::kStatusBytes, st);
    if (e != cudaSuccess) return gla::record_cuda(e, "status word reset");
    const size_t BH = (size_t)p->B * p->H;
    if (BH == 0) return GLA_OK;
    if (p->L == 0) {
        e = cudaMemsetAsync(state_grad, 0, 4 * BH * p->Dk * p->Dv, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gamma, 0, 4 * BH * p->Dk, st);
        return gla::record_cuda(e, "empty shard");
    }
    gla::Dims P;
    P.B = p->B; P.H = p->H; P.L = p->L; P.Dk = p->Dk; P.Dv = p->Dv; P.C = p->chunk;
    P.N = gla::cdiv(p->L, p->chunk);
    P.gate = p->gate;
    P.scale = p->scale;
    const int ntiles = gla::cdiv(p->L, gla::tc::TR);
    e = gla::tc::state_pass(P, 4, q, dO, g, nullptr, 1, ntiles, state_grad, gamma, static_cast<int*>(ws), st);
    return gla::record_cuda(e, "shard state-gradient pass");
}

extern "C" gla_status gla_state_fold(const gla_problem* p, int count, const float* states, const float* gammas,
                                     const float* h0, float* out, void* stream) {
    if (!p || p->B < 0 || p->H < 0 || count < 0) return GLA_ERR_INVALID_ARG;
    if (!gla::dims_ok(p)) return GLA_ERR_UNSUPPORTED;
    if (!out || (count > 0 && (!states || !gammas))) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {states, gammas, h0, out};
    for (const void* x : ptrs)
        if (!gla::aligned16(x)) return GLA_ERR_INVALID_ARG;
    const long BH = (long)p->B * p->H;
    if (BH == 0) return GLA_OK;
    const long n = BH * p->Dk * p->Dv / 4;
    cudaStream_t st = (cudaStream_t)stream;
    GLA_LAUNCH("state_fold", st,
               gla::k_state_fold<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(states, gammas, h0, out, count, (int)BH,
                                                                             p->Dk, p->Dv));
    return gla::record_cuda(cudaGetLastError(), "state fold launch");
}
