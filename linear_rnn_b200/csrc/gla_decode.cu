// Recurrent single-token step of gated linear attention from a given state (the recurrent
// form of the talk summary "Hardware-Efficient Training of Linear Attention Models", sections
// 4:04 and 7:36, with the GLA abstract's data-dependent gates):
//   S <- diag(alpha) S + k'^T v,   o = scale * q S   (alpha = e^g, k' = i k),
// the state updated in place. Per (b, h) the step reads and writes the Dk x Dv fp32 state once
// and touches only Dk + Dv values otherwise, so it is bound by HBM bandwidth: a mat-vec on CUDA
// cores, no tensor-core shape fits one token.
#include "gla_common.cuh"

namespace gla {
namespace {

constexpr int NT_D = 256;

// CTA = (b*h, block of CB value columns). Thread = (4 consecutive columns, group of rows):
// it updates its rows' 16-byte pieces of the state (coalesced: a warp covers 512 contiguous
// bytes of a row) and accumulates q S for its columns; the row groups' partial sums are added
// in shared memory.
template <typename T, int GATE, int CB>
__global__ void __launch_bounds__(NT_D) k_decode(const T* __restrict__ q, const T* __restrict__ k,
                                                 const T* __restrict__ v, const float* __restrict__ g,
                                                 const float* __restrict__ ig, float* __restrict__ S,
                                                 T* __restrict__ o, int Dk, int Dv, float scale) {
    constexpr int NC4 = CB / 4, NRG = NT_D / NC4;
    __shared__ float sq[256], sk[256], sa[256];
    __shared__ float4 red[NRG][NC4];
    const int bh = blockIdx.x, tid = threadIdx.x;
    const int c4 = tid % NC4, rg = tid / NC4;
    const float iv = ig ? ig[bh] : 1.f;
    for (int d = tid; d < Dk; d += NT_D) {
        sq[d] = scale * to_f(q[(size_t)bh * Dk + d]);
        sk[d] = iv * to_f(k[(size_t)bh * Dk + d]);
        sa[d] = GATE == 1 ? __expf(g[(size_t)bh * Dk + d]) : GATE == 2 ? __expf(g[bh]) : 1.f;
    }
    __syncthreads();
    const int col = blockIdx.y * CB + 4 * c4;
    const T* vp = v + (size_t)bh * Dv + col;
    const float4 vv = make_float4(to_f(vp[0]), to_f(vp[1]), to_f(vp[2]), to_f(vp[3]));
    float* Sp = S + (size_t)bh * Dk * Dv + col;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // rows in batches of RB: all RB loads are issued before the first store, so that each thread
    // keeps RB 16-byte reads in flight (the walk is a read-modify-write of the state)
    constexpr int RB = 8;
    for (int d0 = rg; d0 < Dk; d0 += RB * NRG) {
        float4 s[RB];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int d = d0 + u * NRG;
            if (d < Dk) s[u] = *reinterpret_cast<const float4*>(Sp + (size_t)d * Dv);
        }
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int d = d0 + u * NRG;
            if (d < Dk) {
                const float a = sa[d], kd = sk[d], qd = sq[d];
                s[u].x = fmaf(a, s[u].x, kd * vv.x);
                s[u].y = fmaf(a, s[u].y, kd * vv.y);
                s[u].z = fmaf(a, s[u].z, kd * vv.z);
                s[u].w = fmaf(a, s[u].w, kd * vv.w);
                *reinterpret_cast<float4*>(Sp + (size_t)d * Dv) = s[u];
                acc.x = fmaf(qd, s[u].x, acc.x);
                acc.y = fmaf(qd, s[u].y, acc.y);
                acc.z = fmaf(qd, s[u].z, acc.z);
                acc.w = fmaf(qd, s[u].w, acc.w);
            }
        }
    }
    red[rg][c4] = acc;
    __syncthreads();
    if (rg == 0) {
        float4 r = red[0][c4];
#pragma unroll
        for (int j = 1; j < NRG; ++j) {
            const float4 x = red[j][c4];
            r.x += x.x;
            r.y += x.y;
            r.z += x.z;
            r.w += x.w;
        }
        T* op = o + (size_t)bh * Dv + col;
        op[0] = from_f<T>(r.x);
        op[1] = from_f<T>(r.y);
        op[2] = from_f<T>(r.z);
        op[3] = from_f<T>(r.w);
    }
}

template <typename T, int GATE>
cudaError_t launch(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                   const float* ig, float* S, void* o, cudaStream_t st) {
    const int BH = p->B * p->H;
    const T* tq = static_cast<const T*>(q);
    const T* tk = static_cast<const T*>(k);
    const T* tv = static_cast<const T*>(v);
    T* to = static_cast<T*>(o);
    if (p->Dv >= 128) {
        dim3 grid(BH, p->Dv / 128);
        GLA_LAUNCH("decode", st, (k_decode<T, GATE, 128><<<grid, NT_D, 0, st>>>(tq, tk, tv, g, ig, S, to, p->Dk, p->Dv, p->scale)));
    } else {
        dim3 grid(BH, 1);
        GLA_LAUNCH("decode", st, (k_decode<T, GATE, 64><<<grid, NT_D, 0, st>>>(tq, tk, tv, g, ig, S, to, p->Dk, p->Dv, p->scale)));
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gate(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                        const float* ig, float* S, void* o, cudaStream_t st) {
    switch (p->gate) {
        case GLA_GATE_NONE: return launch<T, 0>(p, q, k, v, g, ig, S, o, st);
        case GLA_GATE_PER_KEY: return launch<T, 1>(p, q, k, v, g, ig, S, o, st);
        default: return launch<T, 2>(p, q, k, v, g, ig, S, o, st);
    }
}

bool aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

}  // namespace
}  // namespace gla

extern "C" gla_status gla_decode(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                                 const float* igate, float* state, void* o, void* stream) {
    if (!p || p->B < 0 || p->H < 0 || p->L != 1) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE && p->gate != GLA_GATE_PER_KEY && p->gate != GLA_GATE_PER_HEAD)
        return GLA_ERR_INVALID_ARG;
    const bool dim_ok = (p->Dk == 64 || p->Dk == 128 || p->Dk == 256) && (p->Dv == 64 || p->Dv == 128 || p->Dv == 256);
    if (!dim_ok) return GLA_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 2147483647LL) return GLA_ERR_UNSUPPORTED;
    if ((size_t)p->B * p->H == 0) return GLA_OK;
    if (!q || !k || !v || !state || !o) return GLA_ERR_INVALID_ARG;
    if ((p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, igate, state, o};
    for (const void* x : ptrs)
        if (!gla::aligned16(x)) return GLA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = p->io == GLA_BF16 ? gla::launch_gate<__nv_bfloat16>(p, q, k, v, g, igate, state, o, st)
                                      : gla::launch_gate<float>(p, q, k, v, g, igate, state, o, st);
    return gla::record_cuda(e, "decode launch");
}
