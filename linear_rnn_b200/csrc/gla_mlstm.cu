// mLSTM cell (matrix memory with an exponential input gate, a normaliser and a max-stabiliser),
// forward and backward, on top of the library's chunkwise gated linear attention.
//
// The Tiled Flash Linear Attention abstract names mLSTM, the matrix-memory cell of the xLSTM
// family, as what its kernels speed up; the cell is taken as published for xLSTM. Per (batch,
// head), with g_t the log forget gate and i~_t the log of the exponential input gate:
//     C_t = e^{g_t} C_{t-1} + e^{i~_t} k_t^T v_t,   n_t = e^{g_t} n_{t-1} + e^{i~_t} k_t,
//     h_t = num_t / max(|den_t|, 1),   num_t = (scale q_t) C_t,   den_t = (scale q_t) . n_t,
// from zero states. The recurrent form keeps C, n and a running max m_t of the log weights
// (the stabiliser) so that no exp(i~) leaves the floating-point range; the states it keeps
// are exp(-m_t) times C_t and n_t and its bound exp(-m_t) times 1, so h_t is unchanged.
//
// Here num and den are two passes of the gated linear attention kernels (per-head log-decay g,
// input gate e^{i~ - c}; values v, and a tile of ones whose every output column is den), with
// c the largest i~ of the head: the same kind of constant shift as the stabiliser, it keeps every
// input gate <= 1 and turns the bound into e^{-c}. Small kernels then form h, and in the backward
// the upstream gradients of the two passes,
//     dnum = dh / N,   dden = -(dh . h) / N * sign(den) where |den| > e^{-c} (else 0),
// and, after the two backward passes, the sums of their dq, dk, dg and the chain rule through
// the input gate, d i~ = (di_num + di_den) e^{i~ - c} (h does not depend on c).
#include <math.h>
#include <stdint.h>

#include "gla_common.cuh"

namespace gla {
namespace {

constexpr int ML_NT = 256;

template <typename T>
__device__ __forceinline__ float ld_f(const T* p) { return to_f(*p); }

// Per head: c = max_t i~_t, and the input gate e^{i~_t - c} (<= 1) for the two passes.
__global__ void __launch_bounds__(ML_NT) k_mlstm_prep(const float* __restrict__ itil, int L, float* __restrict__ ig,
                                                      float* __restrict__ cst) {
    __shared__ float red[ML_NT / 32];
    const long bh = blockIdx.x;
    const float* x = itil + bh * L;
    float m = -INFINITY;
    for (int t = threadIdx.x; t < L; t += ML_NT) m = fmaxf(m, x[t]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float c = red[0];
#pragma unroll
    for (int w = 1; w < ML_NT / 32; ++w) c = fmaxf(c, red[w]);
    if (threadIdx.x == 0) cst[bh] = c;
    for (int t = threadIdx.x; t < L; t += ML_NT) ig[bh * L + t] = expf(x[t] - c);
}

template <typename T>
__global__ void k_fill_ones(T* __restrict__ p, long n) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
        p[i] = from_f<T>(1.f);
}

template <typename Tin, typename Tout>
__global__ void k_cast(const Tin* __restrict__ a, Tout* __restrict__ b, long n) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
        b[i] = from_f<Tout>(to_f(a[i]));
}

// One warp per token row: N = max(|den|, e^{-c}), h = num / N.
template <typename Ti, typename To>
__global__ void __launch_bounds__(ML_NT) k_mlstm_norm(const Ti* __restrict__ num, const Ti* __restrict__ den,
                                                      const float* __restrict__ cst, To* __restrict__ h, long rows,
                                                      int L, int Dv, int Dvn) {
    const long row = blockIdx.x * (long)(ML_NT / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float N = fmaxf(fabsf(ld_f(den + row * Dvn)), expf(-cst[row / L]));
    const float inv = 1.f / N;
    for (int e = lane; e < Dv; e += 32) h[row * Dv + e] = from_f<To>(ld_f(num + row * Dv + e) * inv);
}

// One warp per token row: the upstream gradients of the two passes.
template <typename Ti, typename To>
__global__ void __launch_bounds__(ML_NT) k_mlstm_bwd_prep(const Ti* __restrict__ num, const Ti* __restrict__ den,
                                                          const float* __restrict__ cst, const To* __restrict__ dh,
                                                          Ti* __restrict__ dnum, Ti* __restrict__ dden, long rows, int L,
                                                          int Dv, int Dvn) {
    const long row = blockIdx.x * (long)(ML_NT / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float dn = ld_f(den + row * Dvn);
    const float bound = expf(-cst[row / L]);
    const float N = fmaxf(fabsf(dn), bound);
    const float inv = 1.f / N;
    float s = 0.f;   // dh . h
    for (int e = lane; e < Dv; e += 32) {
        const float d = ld_f(dh + row * Dv + e);
        s += d * ld_f(num + row * Dv + e) * inv;
        dnum[row * Dv + e] = from_f<Ti>(d * inv);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float dd = fabsf(dn) > bound ? -s * inv * (dn > 0.f ? 1.f : -1.f) : 0.f;
    for (int e = lane; e < Dvn; e += 32) dden[row * Dvn + e] = from_f<Ti>(e == 0 ? dd : 0.f);
}

// dq = dq1 + dq2 and dk = dk1 + dk2 (n_qk elements), dv = dv1 (n_v elements, only when the passes
// ran in another type than the outputs), dg = dg1 + dg2 and d i~ = (di1 + di2) * e^{i~ - c}
// (n_t tokens). dq1 / dk1 / dv1 may be the outputs themselves.
template <typename Ti, typename To>
__global__ void k_mlstm_bwd_final(To* dq, To* dk, To* dv, const Ti* dq1, const Ti* dk1, const Ti* dv1,
                                  const Ti* __restrict__ dq2, const Ti* __restrict__ dk2, long n_qk, long n_v,
                                  float* __restrict__ dg, const float* __restrict__ dg2, const float* __restrict__ di1,
                                  const float* __restrict__ di2, const float* __restrict__ ig,
                                  float* __restrict__ ditil, long n_t) {
    const long stride = (long)gridDim.x * blockDim.x;
    const long i0 = blockIdx.x * (long)blockDim.x + threadIdx.x;
    for (long i = i0; i < n_qk; i += stride) {
        dq[i] = from_f<To>(to_f(dq1[i]) + to_f(dq2[i]));
        dk[i] = from_f<To>(to_f(dk1[i]) + to_f(dk2[i]));
    }
    for (long i = i0; i < n_v; i += stride) dv[i] = from_f<To>(to_f(dv1[i]));
    for (long i = i0; i < n_t; i += stride) {
        dg[i] += dg2[i];
        ditil[i] = (di1[i] + di2[i]) * ig[i];
    }
}

// The device status word of the second pass joins the first (the one at the workspace start).
__global__ void k_status_or(int* a, const int* b) { atomicOr(a, *b); }

bool ml_aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

struct MlLayout {
    gla_problem pa, pb;   // value pass, normaliser pass (a tile of Dvn ones)
    bool f32;             // the passes run with fp32 I/O (converted copies of bf16 inputs)
    bool cast;            // ... and the I/O is bf16: inputs are converted, gradients cast back
    size_t wsa, wsb;      // the passes' workspace bytes
    size_t o_wsb, o_ig, o_c, o_qf, o_kf, o_vf, o_num, o_den, o_ones;
    size_t o_dnum, o_dden, o_dq1, o_dk1, o_dv1, o_dq2, o_dk2, o_dv2, o_dg2, o_di1, o_di2;
    size_t total;
};

// Width of the normaliser pass's value tile: the smallest head dim whose tensor-core backward
// runs with this key dim (key dim 256 needs 128).
int ml_dvn(const gla_problem* p) { return p->Dk > 128 ? 128 : 64; }

gla_status ml_layout(const gla_problem* p, bool bwd, MlLayout* w) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_PER_HEAD) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->plan < GLA_PLAN_AUTO || p->plan > GLA_PLAN_TC) return GLA_ERR_INVALID_ARG;
    w->pa = *p;
    w->pb = *p;
    w->pb.Dv = ml_dvn(p);
    // The automatic plan (and GLA_PLAN_SIMT) runs both passes on the CUDA cores with fp32 I/O:
    // h divides by |den| wherever |den| exceeds the bound, den is a sum of terms of both signs,
    // and the gradients add the two passes' parts, which can nearly cancel. An error proportional
    // to the terms (bf16 operands and bf16-rounded partial results) then becomes a large relative
    // error where |den| sits just above the bound. GLA_PLAN_TC runs the tensor-core passes in the
    // I/O dtype instead (faster, less accurate there).
    w->f32 = p->plan != GLA_PLAN_TC;
    w->cast = w->f32 && p->io == GLA_BF16;
    if (w->f32) {
        w->pa.plan = w->pb.plan = GLA_PLAN_SIMT;
        w->pa.io = w->pb.io = GLA_F32;
    }
    auto need = [&](const gla_problem* q) {
        const size_t f = gla_workspace_bytes(q, 0);
        const size_t b = bwd ? gla_workspace_bytes(q, 1) : 0;
        return (f == 0 || (bwd && b == 0)) ? (size_t)0 : (f > b ? f : b);
    };
    w->wsa = need(&w->pa);
    w->wsb = need(&w->pb);
    if (w->wsa == 0 || w->wsb == 0) return GLA_ERR_UNSUPPORTED;   // the verdict gla_fwd / gla_bwd give
    const size_t BHL = (size_t)p->B * p->H * p->L, BH = (size_t)p->B * p->H;
    const size_t e = w->f32 ? 4 : 2;   // bytes of the passes' elements
    const int Dvn = w->pb.Dv;
    size_t off = align_up(w->wsa, 256);
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    w->o_wsb = take(w->wsb);
    w->o_ig = take(4 * BHL);
    w->o_c = take(4 * BH);
    if (w->cast) {
        w->o_qf = take(4 * BHL * p->Dk);
        w->o_kf = take(4 * BHL * p->Dk);
        w->o_vf = take(4 * BHL * p->Dv);
    }
    w->o_num = take(e * BHL * p->Dv);
    w->o_den = take(e * BHL * Dvn);
    w->o_ones = take(e * BHL * Dvn);
    if (bwd) {
        w->o_dnum = take(e * BHL * p->Dv);
        w->o_dden = take(e * BHL * Dvn);
        if (w->cast) {
            w->o_dq1 = take(4 * BHL * p->Dk);
            w->o_dk1 = take(4 * BHL * p->Dk);
            w->o_dv1 = take(4 * BHL * p->Dv);
        }
        w->o_dq2 = take(e * BHL * p->Dk);
        w->o_dk2 = take(e * BHL * p->Dk);
        w->o_dv2 = take(e * BHL * Dvn);
        w->o_dg2 = take(4 * BHL);
        w->o_di1 = take(4 * BHL);
        w->o_di2 = take(4 * BHL);
    }
    w->total = off;
    return GLA_OK;
}

unsigned ml_grid(long n, int nt) {
    const long b = (n + nt - 1) / nt;
    return (unsigned)(b < 1 ? 1 : b > 148L * 16 ? 148L * 16 : b);
}

// Shared by the forward and the backward: the input gate, fp32 copies of bf16 inputs where the
// passes run in fp32, the ones tile, and the two forward passes (num, den) in the workspace.
// q, k, v are replaced by the pointers the passes read.
template <typename Ti, typename To>
gla_status ml_forward_passes(const gla_problem* p, const MlLayout& w, const void*& q, const void*& k, const void*& v,
                             const float* g, const float* itil, char* ws, cudaStream_t st) {
    const long BH = (long)p->B * p->H, BHL = BH * p->L;
    float* ig = reinterpret_cast<float*>(ws + w.o_ig);
    float* cst = reinterpret_cast<float*>(ws + w.o_c);
    Ti* ones = reinterpret_cast<Ti*>(ws + w.o_ones);
    GLA_LAUNCH("mlstm_prep", st, k_mlstm_prep<<<(unsigned)BH, ML_NT, 0, st>>>(itil, p->L, ig, cst));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e, "mLSTM gate launch");
    if (w.cast) {
        const long nq = BHL * p->Dk, nv = BHL * p->Dv;
        float* qf = reinterpret_cast<float*>(ws + w.o_qf);
        float* kf = reinterpret_cast<float*>(ws + w.o_kf);
        float* vf = reinterpret_cast<float*>(ws + w.o_vf);
        GLA_LAUNCH("mlstm_cast", st, (k_cast<To, float><<<ml_grid(nq, 256), 256, 0, st>>>(static_cast<const To*>(q), qf, nq)));
        GLA_LAUNCH("mlstm_cast", st, (k_cast<To, float><<<ml_grid(nq, 256), 256, 0, st>>>(static_cast<const To*>(k), kf, nq)));
        GLA_LAUNCH("mlstm_cast", st, (k_cast<To, float><<<ml_grid(nv, 256), 256, 0, st>>>(static_cast<const To*>(v), vf, nv)));
        if ((e = cudaGetLastError()) != cudaSuccess) return record_cuda(e, "mLSTM input conversion launch");
        q = qf;
        k = kf;
        v = vf;
    }
    const long nones = BHL * w.pb.Dv;
    GLA_LAUNCH("mlstm_ones", st, k_fill_ones<Ti><<<ml_grid(nones, 256), 256, 0, st>>>(ones, nones));
    if ((e = cudaGetLastError()) != cudaSuccess) return record_cuda(e, "mLSTM ones launch");
    gla_status s = gla_fwd(&w.pa, q, k, v, g, ig, nullptr, ws + w.o_num, nullptr, ws, w.wsa, st);
    if (s != GLA_OK) return s;
    return gla_fwd(&w.pb, q, k, ones, g, ig, nullptr, ws + w.o_den, nullptr, ws + w.o_wsb, w.wsb, st);
}

template <typename Ti, typename To>
gla_status ml_fwd(const gla_problem* p, const MlLayout& w, const void* q, const void* k, const void* v,
                  const float* g, const float* itil, void* h, char* ws, cudaStream_t st) {
    gla_status s = ml_forward_passes<Ti, To>(p, w, q, k, v, g, itil, ws, st);
    if (s != GLA_OK) return s;
    const long rows = (long)p->B * p->H * p->L;
    GLA_LAUNCH("mlstm_norm", st,
               (k_mlstm_norm<Ti, To><<<(unsigned)((rows + ML_NT / 32 - 1) / (ML_NT / 32)), ML_NT, 0, st>>>(
                   reinterpret_cast<const Ti*>(ws + w.o_num), reinterpret_cast<const Ti*>(ws + w.o_den),
                   reinterpret_cast<const float*>(ws + w.o_c), static_cast<To*>(h), rows, p->L, p->Dv, w.pb.Dv)));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e, "mLSTM normalise launch");
    GLA_LAUNCH("mlstm_status", st,
               k_status_or<<<1, 1, 0, st>>>(reinterpret_cast<int*>(ws), reinterpret_cast<const int*>(ws + w.o_wsb)));
    return record_cuda(cudaGetLastError(), "mLSTM status launch");
}

template <typename Ti, typename To>
gla_status ml_bwd(const gla_problem* p, const MlLayout& w, const void* q, const void* k, const void* v,
                  const float* g, const float* itil, const void* dh, void* dq, void* dk, void* dv, float* dg,
                  float* ditil, char* ws, cudaStream_t st) {
    gla_status s = ml_forward_passes<Ti, To>(p, w, q, k, v, g, itil, ws, st);
    if (s != GLA_OK) return s;
    const long rows = (long)p->B * p->H * p->L;
    const int Dvn = w.pb.Dv;
    Ti* dnum = reinterpret_cast<Ti*>(ws + w.o_dnum);
    Ti* dden = reinterpret_cast<Ti*>(ws + w.o_dden);
    GLA_LAUNCH("mlstm_bwd_prep", st,
               (k_mlstm_bwd_prep<Ti, To><<<(unsigned)((rows + ML_NT / 32 - 1) / (ML_NT / 32)), ML_NT, 0, st>>>(
                   reinterpret_cast<const Ti*>(ws + w.o_num), reinterpret_cast<const Ti*>(ws + w.o_den),
                   reinterpret_cast<const float*>(ws + w.o_c), static_cast<const To*>(dh), dnum, dden, rows, p->L,
                   p->Dv, Dvn)));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e, "mLSTM backward prep launch");
    const float* ig = reinterpret_cast<const float*>(ws + w.o_ig);
    float* di1 = reinterpret_cast<float*>(ws + w.o_di1);
    float* di2 = reinterpret_cast<float*>(ws + w.o_di2);
    float* dg2 = reinterpret_cast<float*>(ws + w.o_dg2);
    // the value pass writes its gradients straight into the outputs unless they are cast back
    void* dq1 = w.cast ? ws + w.o_dq1 : dq;
    void* dk1 = w.cast ? ws + w.o_dk1 : dk;
    void* dv1 = w.cast ? ws + w.o_dv1 : dv;
    s = gla_bwd(&w.pa, q, k, v, g, ig, nullptr, dnum, nullptr, dq1, dk1, dv1, dg, di1, nullptr, ws, w.wsa, st);
    if (s != GLA_OK) return s;
    s = gla_bwd(&w.pb, q, k, ws + w.o_ones, g, ig, nullptr, dden, nullptr, ws + w.o_dq2, ws + w.o_dk2,
                ws + w.o_dv2, dg2, di2, nullptr, ws + w.o_wsb, w.wsb, st);
    if (s != GLA_OK) return s;
    const long nqk = rows * p->Dk, nv = w.cast ? rows * p->Dv : 0;
    GLA_LAUNCH("mlstm_bwd_final", st,
               (k_mlstm_bwd_final<Ti, To><<<ml_grid(nqk, 256), 256, 0, st>>>(
                   static_cast<To*>(dq), static_cast<To*>(dk), static_cast<To*>(dv), static_cast<const Ti*>(dq1),
                   static_cast<const Ti*>(dk1), static_cast<const Ti*>(dv1), reinterpret_cast<const Ti*>(ws + w.o_dq2),
                   reinterpret_cast<const Ti*>(ws + w.o_dk2), nqk, nv, dg, dg2, di1, di2, ig, ditil, rows)));
    if ((e = cudaGetLastError()) != cudaSuccess) return record_cuda(e, "mLSTM backward final launch");
    GLA_LAUNCH("mlstm_status", st,
               k_status_or<<<1, 1, 0, st>>>(reinterpret_cast<int*>(ws), reinterpret_cast<const int*>(ws + w.o_wsb)));
    return record_cuda(cudaGetLastError(), "mLSTM status launch");
}

}  // namespace
}  // namespace gla

extern "C" {

size_t gla_mlstm_workspace_bytes(const gla_problem* p, int for_backward) {
    gla::MlLayout w;
    if (gla::ml_layout(p, for_backward != 0, &w) != GLA_OK) return 0;
    return w.total;
}

gla_status gla_mlstm_fwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                         const float* itil, void* h, void* ws, size_t ws_bytes, void* stream) {
    gla::MlLayout w;
    const gla_status s = gla::ml_layout(p, false, &w);
    if (s != GLA_OK) return s;
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!q || !k || !v || !g || !itil || !h)) return GLA_ERR_INVALID_ARG;
    if (!ws) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, itil, h, ws};
    for (const void* x : ptrs)
        if (!gla::ml_aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return GLA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = cudaMemsetAsync(ws, 0, gla::kStatusBytes, st);
    if (e != cudaSuccess) return gla::record_cuda(e, "status word reset");
    if (empty) return GLA_OK;
    char* wsb = static_cast<char*>(ws);
    if (p->io == GLA_F32) return gla::ml_fwd<float, float>(p, w, q, k, v, g, itil, h, wsb, st);
    return w.f32 ? gla::ml_fwd<float, __nv_bfloat16>(p, w, q, k, v, g, itil, h, wsb, st)
                 : gla::ml_fwd<__nv_bfloat16, __nv_bfloat16>(p, w, q, k, v, g, itil, h, wsb, st);
}

gla_status gla_mlstm_bwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                         const float* itil, const void* dh, void* dq, void* dk, void* dv, float* dg, float* ditil,
                         void* ws, size_t ws_bytes, void* stream) {
    gla::MlLayout w;
    const gla_status s = gla::ml_layout(p, true, &w);
    if (s != GLA_OK) return s;
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!q || !k || !v || !g || !itil || !dh || !dq || !dk || !dv || !dg || !ditil))
        return GLA_ERR_INVALID_ARG;
    if (!ws) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, ws};
    for (const void* x : ptrs)
        if (!gla::ml_aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return GLA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = cudaMemsetAsync(ws, 0, gla::kStatusBytes, st);
    if (e != cudaSuccess) return gla::record_cuda(e, "status word reset");
    if (empty) return GLA_OK;
    char* wsb = static_cast<char*>(ws);
    if (p->io == GLA_F32) return gla::ml_bwd<float, float>(p, w, q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, wsb, st);
    return w.f32 ? gla::ml_bwd<float, __nv_bfloat16>(p, w, q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, wsb, st)
                 : gla::ml_bwd<__nv_bfloat16, __nv_bfloat16>(p, w, q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, wsb,
                                                             st);
}

}  // extern "C"
