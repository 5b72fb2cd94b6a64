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

// A shard's state (or state gradient) from the pairs of its segments, laid out [BH][nseg][Dk][Dv]
// and [BH][nseg][Dk] by the state pass: S <- diag(e^{Gamma_z}) S + S_z over z = 0 .. nseg-1 from
// zero (reverse = 1: z = nseg-1 .. 0, the gradient at the shard's start from zero at its end);
// gamma_out = sum_z Gamma_z. One thread per four consecutive elements of one (bh, key dim) row.
__global__ void __launch_bounds__(256) k_seg_reduce(const float* __restrict__ seg_state,
                                                    const float* __restrict__ seg_gamma, float* __restrict__ out,
                                                    float* __restrict__ gamma_out, int BH, int Dk, int Dv, int nseg,
                                                    int reverse) {
    const int per4 = Dk * Dv / 4;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)BH * per4) return;
    const int bh = (int)(idx / per4), de4 = (int)(idx - (long)bh * per4), d = 4 * de4 / Dv;
    const float4* src = reinterpret_cast<const float4*>(seg_state) + (size_t)bh * nseg * per4 + de4;
    const float* gam = seg_gamma + (size_t)bh * nseg * Dk + d;
    float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
    float gsum = 0.f;
    for (int j = 0; j < nseg; ++j) {
        const int z = reverse ? nseg - 1 - j : j;
        const float gz = __ldg(gam + (size_t)z * Dk);
        const float e = __expf(gz);
        const float4 x = __ldg(src + (size_t)z * per4);
        S = make_float4(fmaf(e, S.x, x.x), fmaf(e, S.y, x.y), fmaf(e, S.z, x.z), fmaf(e, S.w, x.w));
        gsum += gz;
    }
    reinterpret_cast<float4*>(out)[idx] = S;
    if (4 * de4 % Dv == 0) gamma_out[(size_t)bh * Dk + d] = gsum;
}

bool aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }
bool dims_ok(const gla_problem* p) {
    return (p->Dk == 64 || p->Dk == 128 || p->Dk == 256) && (p->Dv == 64 || p->Dv == 128 || p->Dv == 256);
}

// Segments of a shard's state pass: as many as keep its CTAs (one per head, Dv tile and
// segment) within one wave of the GPU, in whole 64-token tiles.
struct ShardPlan {
    int nseg, tps;
    size_t ws;   // workspace bytes: the status word, then the segments' states and log-decays
};
ShardPlan shard_plan(const gla_problem* p) {
    ShardPlan pl{1, 0, kStatusBytes};
    const int ntiles = cdiv(p->L, tc::TR);
    pl.tps = ntiles;
    // the state-only pass's Dv tile (the rule of the tensor-core forward's state passes)
    const int sdvt = p->Dv % 128 != 0 ? 64 : p->Dk == 256 ? (p->gate == GLA_GATE_PER_KEY ? 64 : 128)
                                                           : (p->Dv == 256 ? 256 : 128);
    const long base = (long)p->B * p->H * (p->Dv / sdvt);
    if (ntiles <= 1 || base <= 0) return pl;
    int nseg = (int)(tc::num_sms() / base);
    if (nseg > ntiles) nseg = ntiles;
    if (nseg <= 1) return pl;
    pl.tps = cdiv(ntiles, nseg);
    pl.nseg = cdiv(ntiles, pl.tps);
    if (pl.nseg <= 1) {
        pl.nseg = 1;
        pl.tps = ntiles;
        return pl;
    }
    const size_t BH = (size_t)p->B * p->H;
    pl.ws = align_up(kStatusBytes + 4 * BH * pl.nseg * p->Dk * p->Dv, 256) + 4 * BH * pl.nseg * p->Dk;
    return pl;
}

// The state-only pass over the shard (mode 3: end states from zero, mode 4: start-state
// gradients from zero), in segments reduced by k_seg_reduce when the plan has several.
cudaError_t shard_pass(const gla_problem* p, int mode, const void* a, const void* b, const float* g,
                       const float* ig, float* out, float* gamma, void* ws, cudaStream_t st) {
    Dims P;
    P.B = p->B; P.H = p->H; P.L = p->L; P.Dk = p->Dk; P.Dv = p->Dv; P.C = p->chunk;
    P.N = cdiv(p->L, p->chunk);
    P.gate = p->gate;
    P.scale = p->scale;
    const ShardPlan pl = shard_plan(p);
    int* status = static_cast<int*>(ws);
    if (pl.nseg <= 1) return tc::state_pass(P, mode, a, b, g, ig, 1, pl.tps, out, gamma, status, st);
    const size_t BH = (size_t)p->B * p->H;
    float* ss = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
    float* sg = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                         align_up(kStatusBytes + 4 * BH * pl.nseg * p->Dk * p->Dv, 256));
    cudaError_t e = tc::state_pass(P, mode, a, b, g, ig, pl.nseg, pl.tps, ss, sg, status, st);
    if (e != cudaSuccess) return e;
    const long n = (long)BH * p->Dk * p->Dv / 4;
    GLA_LAUNCH("seg_reduce", st,
               k_seg_reduce<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(ss, sg, out, gamma, (int)BH, p->Dk, p->Dv,
                                                                          pl.nseg, mode == 4 ? 1 : 0));
    return cudaGetLastError();
}

}  // namespace
}  // namespace gla

extern "C" size_t gla_shard_workspace_bytes(const gla_problem* p) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0 || !gla::dims_ok(p)) return 0;
    if (p->chunk < 64 || p->chunk > 1024 || p->chunk % 64 != 0) return 0;
    return gla::shard_plan(p).ws;
}

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
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!k || !v)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {k, v, g, igate, state, gamma, ws};
    for (const void* x : ptrs)
        if (!gla::aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < gla::shard_plan(p).ws) return GLA_ERR_WORKSPACE;
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
    e = gla::shard_pass(p, 3, k, v, g, igate, state, gamma, ws, st);
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
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!q || !dO)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, dO, g, state_grad, gamma, ws};
    for (const void* x : ptrs)
        if (!gla::aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < gla::shard_plan(p).ws) return GLA_ERR_WORKSPACE;
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
    e = gla::shard_pass(p, 4, q, dO, g, nullptr, state_grad, gamma, ws, st);
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
