// CUDA-core (FFMA) chunk-parallel plan of chunkwise gated linear attention.
//
// The plan follows the chunkwise ("trunk-wise") algorithm of the talk summary
// "Hardware-Efficient Training of Linear Attention Models", section 11:58, one kernel
// per step so each step can be checked on its own:
//   k_cumsum  in-chunk inclusive log-cumsum of the gate, b (relative to chunk start)
//   k_state   inter-chunk state pass: S_c = diag(e^Gamma) S_{c-1} + (k' e^(Gamma-b))^T V,
//             writing the state before every chunk (states only at chunk boundaries)
//   k_out     o = scale [ (q e^b) S_{c-1} + masked intra-chunk product ] with the
//             intra-chunk part tiled into 64-row sub-tiles, each tile pair factorised
//             around a reference row in log space so no exponential exceeds the tile span
//   k_dstate  reverse state-gradient pass G_{c-1} = diag(e^Gamma) G_c + scale (q e^b)^T dO
//   k_dq, k_dk, k_dv   per-chunk gradients from S_{c-1}, G_c and the intra-chunk tiles
//   k_dg_*    reverse cumulative sum over the whole sequence of q*dq - k'*dk' (+ the
//             final-state term), the closed form of the decay gradient
// Every product is fp32 FFMA on 64x64 tiles (256 threads, 4x4 outputs each), so this
// plan meets fp32 I/O accuracy; it also runs bf16 I/O (converted on load). Large chunks
// (up to 1024) are tiled within the chunk as in the Tiled Flash Linear Attention
// abstract: only the states at chunk boundaries are materialised.
#include "gla_common.cuh"
#include "gla_plans.h"

namespace gla {
namespace simt {

constexpr int TT = 64;   // tile edge
constexpr int KS = 32;   // contraction slice
constexpr int NT = 256;  // threads: 16 x 16, each a 4 x 4 micro-tile
constexpr int LD = KS + 1;
constexpr int LT = TT + 1;

// b (in-chunk cumulative log-decay) at flat row `row` (= bh*L + t) and key dim d.
__device__ __forceinline__ float bval(const float* b, int gate, long row, int d, int Dk) {
    if (gate == GLA_GATE_PER_KEY) return b[row * Dk + d];
    if (gate == GLA_GATE_PER_HEAD) return b[row];
    return 0.f;
}

__device__ __forceinline__ float igv(const float* ig, long row) { return ig ? ig[row] : 1.f; }

// acc[i][j] += sum_k A[(r0+i)*lda + k] * B[k*ldb + c0+j]
__device__ __forceinline__ void mm_AB(float acc[4][4], const float* A, int lda, const float* B, int ldb,
                                      int K, int r0, int c0) {
    for (int kk = 0; kk < K; ++kk) {
        float a[4], bb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = A[(r0 + i) * lda + kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) bb[j] = B[kk * ldb + c0 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
}
// acc[i][j] += sum_k A[(r0+i)*lda + k] * B[(c0+j)*ldb + k]
__device__ __forceinline__ void mm_ABt(float acc[4][4], const float* A, int lda, const float* B, int ldb,
                                       int K, int r0, int c0) {
    for (int kk = 0; kk < K; ++kk) {
        float a[4], bb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = A[(r0 + i) * lda + kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) bb[j] = B[(c0 + j) * ldb + kk];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
}
// acc[i][j] += sum_k A[k*lda + r0+i] * B[k*ldb + c0+j]
__device__ __forceinline__ void mm_AtB(float acc[4][4], const float* A, int lda, const float* B, int ldb,
                                       int K, int r0, int c0) {
    for (int kk = 0; kk < K; ++kk) {
        float a[4], bb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = A[kk * lda + r0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bb[j] = B[kk * ldb + c0 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
}

__device__ __forceinline__ void zero(float a[4][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) a[i][j] = 0.f;
}

// ---------------------------------------------------------------- A1: in-chunk cumsum
__global__ void k_cumsum(const float* __restrict__ g, float* __restrict__ b, Dims P) {
    const int c = blockIdx.x;
    const long bh = blockIdx.y;
    const int t0 = c * P.C, t1 = min(t0 + P.C, P.L);
    const int width = (P.gate == GLA_GATE_PER_KEY) ? P.Dk : 1;
    for (int d = threadIdx.x; d < width; d += blockDim.x) {
        float acc = 0.f;
        for (int t = t0; t < t1; ++t) {
            const long idx = (bh * P.L + t) * width + d;
            acc += g[idx];
            b[idx] = acc;
        }
    }
}

// ------------------------------------------------------------- A2: inter-chunk states
// grid (Dv/64, Dk/64, B*H); Sprev[bh][c] = state before chunk c.
template <typename T>
__global__ void __launch_bounds__(NT) k_state(const T* __restrict__ k, const T* __restrict__ v,
                                              const float* __restrict__ ig, const float* __restrict__ b,
                                              const float* __restrict__ h0, float* __restrict__ Sprev,
                                              float* __restrict__ hT, Dims P) {
    const int e0 = blockIdx.x * TT, d0 = blockIdx.y * TT;
    const long bh = blockIdx.z;
    const int tid = threadIdx.x, r0 = (tid / 16) * 4, c0 = (tid % 16) * 4;
    __shared__ float Ks[KS][LT];
    __shared__ float Vs[KS][LT];
    __shared__ float gam[TT];
    float S[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            S[i][j] = h0 ? h0[(bh * P.Dk + d0 + r0 + i) * P.Dv + e0 + c0 + j] : 0.f;
    for (int c = 0; c < P.N; ++c) {
        const int t0 = c * P.C, t1 = min(t0 + P.C, P.L), last = t1 - 1;
        float* dst = Sprev + ((bh * P.N + c) * P.Dk) * (long)P.Dv;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[(long)(d0 + r0 + i) * P.Dv + e0 + c0 + j] = S[i][j];
        if (tid < TT) gam[tid] = bval(b, P.gate, bh * P.L + last, d0 + tid, P.Dk);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float eg = __expf(gam[r0 + i]);
#pragma unroll
            for (int j = 0; j < 4; ++j) S[i][j] *= eg;
        }
        for (int s0 = t0; s0 < t1; s0 += KS) {
            for (int idx = tid; idx < KS * TT; idx += NT) {
                const int s = idx / TT, dd = idx % TT, t = s0 + s;
                float kv = 0.f, vv = 0.f;
                if (t < t1) {
                    const long row = bh * P.L + t;
                    kv = to_f(k[row * P.Dk + d0 + dd]) * igv(ig, row) *
                         __expf(gam[dd] - bval(b, P.gate, row, d0 + dd, P.Dk));
                    vv = to_f(v[row * P.Dv + e0 + dd]);
                }
                Ks[s][dd] = kv;
                Vs[s][dd] = vv;
            }
            __syncthreads();
            mm_AtB(S, &Ks[0][0], LT, &Vs[0][0], LT, KS, r0, c0);
            __syncthreads();
        }
    }
    if (hT) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) hT[(bh * P.Dk + d0 + r0 + i) * P.Dv + e0 + c0 + j] = S[i][j];
    }
}

// Compute the 64x64 intra-chunk score tile A[t][s] = sum_d q_td k'_sd e^(b_td - b_sd)
// (unmasked) for query rows [tq0, tq0+nq) and key rows [ts0, ts0+ns) around reference
// row `rrow`, into registers acc (rows = t, cols = s).
template <typename T>
__device__ __forceinline__ void score_tile(float acc[4][4], const T* __restrict__ q, const T* __restrict__ k,
                                           const float* __restrict__ ig, const float* __restrict__ b,
                                           const Dims& P, long bh, int tq0, int nq, int ts0, int ns, int rrow,
                                           float (*Qh)[LD], float (*Kh)[LD], float* rref, int r0, int c0) {
    const int tid = threadIdx.x;
    zero(acc);
    for (int d0 = 0; d0 < P.Dk; d0 += KS) {
        if (tid < KS) rref[tid] = bval(b, P.gate, bh * P.L + rrow, d0 + tid, P.Dk);
        __syncthreads();
        for (int idx = tid; idx < TT * KS; idx += NT) {
            const int r = idx / KS, dd = idx % KS;
            float qv = 0.f, kv = 0.f;
            if (r < nq) {
                const long row = bh * P.L + tq0 + r;
                qv = to_f(q[row * P.Dk + d0 + dd]) * __expf(bval(b, P.gate, row, d0 + dd, P.Dk) - rref[dd]);
            }
            if (r < ns) {
                const long row = bh * P.L + ts0 + r;
                kv = to_f(k[row * P.Dk + d0 + dd]) * igv(ig, row) *
                     __expf(rref[dd] - bval(b, P.gate, row, d0 + dd, P.Dk));
            }
            Qh[r][dd] = qv;
            Kh[r][dd] = kv;
        }
        __syncthreads();
        mm_ABt(acc, &Qh[0][0], LD, &Kh[0][0], LD, KS, r0, c0);
        __syncthreads();
    }
}

// ------------------------------------------------------------------ A3: output
// grid (Dv/64, ceil(L/TQ), B*H)
template <typename T>
__global__ void __launch_bounds__(NT) k_out(const T* __restrict__ q, const T* __restrict__ k,
                                            const T* __restrict__ v, const float* __restrict__ ig,
                                            const float* __restrict__ b, const float* __restrict__ Sprev,
                                            T* __restrict__ o, Dims P, int TQ) {
    const int e0 = blockIdx.x * TT;
    const int t0 = blockIdx.y * TQ;
    const long bh = blockIdx.z;
    const int c = t0 / P.C, cs = c * P.C, ce = min(cs + P.C, P.L);
    const int nq = min(TQ, P.L - t0);
    const int tid = threadIdx.x, r0 = (tid / 16) * 4, c0 = (tid % 16) * 4;
    __shared__ float Qh[TT][LD];
    __shared__ float Kh[TT][LD];
    __shared__ float As[TT][LT];
    __shared__ float Xs[KS][LT];  // state slice, then value slice
    __shared__ float rref[KS];
    float acc[4][4];
    zero(acc);
    // inter-chunk term: (q e^b) S_{c-1}
    const float* Sc = Sprev + ((bh * P.N + c) * P.Dk) * (long)P.Dv;
    for (int d0 = 0; d0 < P.Dk; d0 += KS) {
        for (int idx = tid; idx < TT * KS; idx += NT) {
            const int r = idx / KS, dd = idx % KS;
            float qv = 0.f;
            if (r < nq) {
                const long row = bh * P.L + t0 + r;
                qv = to_f(q[row * P.Dk + d0 + dd]) * __expf(bval(b, P.gate, row, d0 + dd, P.Dk));
            }
            Qh[r][dd] = qv;
        }
        for (int idx = tid; idx < KS * TT; idx += NT) {
            const int dd = idx / TT, ee = idx % TT;
            Xs[dd][ee] = Sc[(long)(d0 + dd) * P.Dv + e0 + ee];
        }
        __syncthreads();
        mm_AB(acc, &Qh[0][0], LD, &Xs[0][0], LT, KS, r0, c0);
        __syncthreads();
    }
    // intra-chunk term, key tiles from the chunk start up to the diagonal tile
    for (int s0 = cs; s0 <= t0; s0 += TQ) {
        const bool diag = (s0 == t0);
        const int ns = min(TQ, ce - s0);
        const int rrow = diag ? t0 : s0 + TQ - 1;
        float a[4][4];
        score_tile(a, q, k, ig, b, P, bh, t0, nq, s0, ns, rrow, Qh, Kh, rref, r0, c0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int tt = r0 + i, ss = c0 + j;
                const bool ok = (tt < nq) && (ss < ns) && (s0 + ss <= t0 + tt);
                As[tt][ss] = ok ? a[i][j] : 0.f;
            }
        for (int sl = 0; sl < TT; sl += KS) {
            __syncthreads();
            for (int idx = tid; idx < KS * TT; idx += NT) {
                const int s = idx / TT, ee = idx % TT;
                Xs[s][ee] = (sl + s < ns) ? to_f(v[(bh * P.L + s0 + sl + s) * P.Dv + e0 + ee]) : 0.f;
            }
            __syncthreads();
            mm_AB(acc, &As[0][sl], LT, &Xs[0][0], LT, KS, r0, c0);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (r0 + i >= nq) continue;
        const long row = bh * P.L + t0 + r0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) o[row * P.Dv + e0 + c0 + j] = from_f<T>(P.scale * acc[i][j]);
    }
}

// ------------------------------------------------- A6: reverse state-gradient pass
// grid (Dv/64, Dk/64, B*H); Gst[bh][c] = dL/dS_c (state at the end of chunk c).
template <typename T>
__global__ void __launch_bounds__(NT) k_dstate(const T* __restrict__ q, const T* __restrict__ dO,
                                               const float* __restrict__ b, const float* __restrict__ dhT,
                                               float* __restrict__ Gst, float* __restrict__ dh0, Dims P) {
    const int e0 = blockIdx.x * TT, d0 = blockIdx.y * TT;
    const long bh = blockIdx.z;
    const int tid = threadIdx.x, r0 = (tid / 16) * 4, c0 = (tid % 16) * 4;
    __shared__ float Qs[KS][LT];
    __shared__ float Os[KS][LT];
    __shared__ float gam[TT];
    float G[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) G[i][j] = dhT ? dhT[(bh * P.Dk + d0 + r0 + i) * P.Dv + e0 + c0 + j] : 0.f;
    for (int c = P.N - 1; c >= 0; --c) {
        const int t0 = c * P.C, t1 = min(t0 + P.C, P.L), last = t1 - 1;
        float* dst = Gst + ((bh * P.N + c) * P.Dk) * (long)P.Dv;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[(long)(d0 + r0 + i) * P.Dv + e0 + c0 + j] = G[i][j];
        if (tid < TT) gam[tid] = bval(b, P.gate, bh * P.L + last, d0 + tid, P.Dk);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float eg = __expf(gam[r0 + i]);
#pragma unroll
            for (int j = 0; j < 4; ++j) G[i][j] *= eg;
        }
        for (int s0 = t0; s0 < t1; s0 += KS) {
            for (int idx = tid; idx < KS * TT; idx += NT) {
                const int s = idx / TT, xx = idx % TT, t = s0 + s;
                float qv = 0.f, ov = 0.f;
                if (t < t1) {
                    const long row = bh * P.L + t;
                    qv = P.scale * to_f(q[row * P.Dk + d0 + xx]) * __expf(bval(b, P.gate, row, d0 + xx, P.Dk));
                    ov = to_f(dO[row * P.Dv + e0 + xx]);
                }
                Qs[s][xx] = qv;
                Os[s][xx] = ov;
            }
            __syncthreads();
            mm_AtB(G, &Qs[0][0], LT, &Os[0][0], LT, KS, r0, c0);
            __syncthreads();
        }
    }
    if (dh0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) dh0[(bh * P.Dk + d0 + r0 + i) * P.Dv + e0 + c0 + j] = G[i][j];
    }
}

// dA tile [t][s] = sum_e dO_te v_se for query rows [tq0,+nq), key rows [ts0,+ns).
template <typename T>
__device__ __forceinline__ void dscore_tile(float acc[4][4], const T* __restrict__ dO, const T* __restrict__ v,
                                            const Dims& P, long bh, int tq0, int nq, int ts0, int ns,
                                            float (*Os)[LD], float (*Vs)[LD], int r0, int c0) {
    const int tid = threadIdx.x;
    zero(acc);
    for (int e0 = 0; e0 < P.Dv; e0 += KS) {
        for (int idx = tid; idx < TT * KS; idx += NT) {
            const int r = idx / KS, ee = idx % KS;
            Os[r][ee] = (r < nq) ? to_f(dO[(bh * P.L + tq0 + r) * P.Dv + e0 + ee]) : 0.f;
            Vs[r][ee] = (r < ns) ? to_f(v[(bh * P.L + ts0 + r) * P.Dv + e0 + ee]) : 0.f;
        }
        __syncthreads();
        mm_ABt(acc, &Os[0][0], LD, &Vs[0][0], LD, KS, r0, c0);
        __syncthreads();
    }
}

// ----------------------------------------------------------------- A7: dq
// grid (Dk/64, ceil(L/TQ), B*H). Writes dq and dB = q*dq (fp32 workspace).
template <typename T>
__global__ void __launch_bounds__(NT) k_dq(const T* __restrict__ q, const T* __restrict__ k,
                                           const T* __restrict__ v, const float* __restrict__ ig,
                                           const float* __restrict__ b, const float* __restrict__ Sprev,
                                           const T* __restrict__ dO, T* __restrict__ dq, float* __restrict__ dB,
                                           Dims P, int TQ) {
    const int d0 = blockIdx.x * TT;
    const int t0 = blockIdx.y * TQ;
    const long bh = blockIdx.z;
    const int c = t0 / P.C, cs = c * P.C, ce = min(cs + P.C, P.L);
    const int nq = min(TQ, P.L - t0);
    const int tid = threadIdx.x, r0 = (tid / 16) * 4, c0 = (tid % 16) * 4;
    __shared__ float Os[TT][LD];
    __shared__ float Vs[TT][LD];
    __shared__ float As[TT][LT];
    __shared__ float Xs[KS][LT];
    __shared__ float rref[TT];
    float acc1[4][4], acc2[4][4];
    zero(acc1);
    zero(acc2);
    // dO S_{c-1}^T : acc1[t][d] = sum_e dO_te S[d][e]
    const float* Sc = Sprev + ((bh * P.N + c) * P.Dk) * (long)P.Dv;
    for (int e0 = 0; e0 < P.Dv; e0 += KS) {
        for (int idx = tid; idx < TT * KS; idx += NT) {
            const int r = idx / KS, ee = idx % KS;
            Os[r][ee] = (r < nq) ? to_f(dO[(bh * P.L + t0 + r) * P.Dv + e0 + ee]) : 0.f;
        }
        for (int idx = tid; idx < KS * TT; idx += NT) {
            const int ee = idx / TT, dd = idx % TT;
            Xs[ee][dd] = Sc[(long)(d0 + dd) * P.Dv + e0 + ee];
        }
        __syncthreads();
        mm_AB(acc1, &Os[0][0], LD, &Xs[0][0], LT, KS, r0, c0);
        __syncthreads();
    }
    for (int s0 = cs; s0 <= t0; s0 += TQ) {
        const bool diag = (s0 == t0);
        const int ns = min(TQ, ce - s0);
        const int rrow = diag ? t0 : s0 + TQ - 1;
        float a[4][4];
        dscore_tile(a, dO, v, P, bh, t0, nq, s0, ns, Os, Vs, r0, c0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int tt = r0 + i, ss = c0 + j;
                const bool ok = (tt < nq) && (ss < ns) && (s0 + ss <= t0 + tt);
                As[tt][ss] = ok ? P.scale * a[i][j] : 0.f;
            }
        if (tid < TT) rref[tid] = bval(b, P.gate, bh * P.L + rrow, d0 + tid, P.Dk);
        float pp[4][4];
        zero(pp);
        for (int sl = 0; sl < TT; sl += KS) {
            __syncthreads();
            for (int idx = tid; idx < KS * TT; idx += NT) {
                const int s = idx / TT, dd = idx % TT;
                float kv = 0.f;
                if (sl + s < ns) {
                    const long row = bh * P.L + s0 + sl + s;
                    kv = to_f(k[row * P.Dk + d0 + dd]) * igv(ig, row) *
                         __expf(rref[dd] - bval(b, P.gate, row, d0 + dd, P.Dk));
                }
                Xs[s][dd] = kv;
            }
            __syncthreads();
            mm_AB(pp, &As[0][sl], LT, &Xs[0][0], LT, KS, r0, c0);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (r0 + i >= nq) continue;
            const long row = bh * P.L + t0 + r0 + i;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc2[i][j] += __expf(bval(b, P.gate, row, d0 + c0 + j, P.Dk) - rref[c0 + j]) * pp[i][j];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (r0 + i >= nq) continue;
        const long row = bh * P.L + t0 + r0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int d = d0 + c0 + j;
            const float val = P.scale * __expf(bval(b, P.gate, row, d, P.Dk)) * acc1[i][j] + acc2[i][j];
            dq[row * P.Dk + d] = from_f<T>(val);
            dB[row * P.Dk + d] = to_f(q[row * P.Dk + d]) * val;
        }
    }
}

// ----------------------------------------------------------------- A7: dk
// grid (Dk/64, ceil(L/TQ), B*H). Writes dk (= i dk'), dB -= k' dk', and per-tile
// partial sums of k . dk' for the input-gate gradient.
template <typename T>
__global__ void __launch_bounds__(NT) k_dk(const T* __restrict__ q, const T* __restrict__ k,
                                           const T* __restrict__ v, const float* __restrict__ ig,
                                           const float* __restrict__ b, const float* __restrict__ Gst,
                                           const T* __restrict__ dO, T* __restrict__ dk, float* __restrict__ dB,
                                           float* __restrict__ dipart, Dims P, int TQ) {
    const int d0 = blockIdx.x * TT;
    const int s0 = blockIdx.y * TQ;
    const long bh = blockIdx.z;
    const int c = s0 / P.C, cs = c * P.C, ce = min(cs + P.C, P.L);
    const int ns = min(TQ, P.L - s0);
    const int tid = threadIdx.x, r0 = (tid / 16) * 4, c0 = (tid % 16) * 4;
    __shared__ float Os[TT][LD];
    __shared__ float Vs[TT][LD];
    __shared__ float As[TT][LT];
    __shared__ float Xs[KS][LT];
    __shared__ float rref[TT];
    __shared__ float gam[TT];
    float acc1[4][4], acc2[4][4];
    zero(acc1);
    zero(acc2);
    (void)cs;
    // acc1[s][d] = sum_e v_se G_c[d][e]
    const float* Gc = Gst + ((bh * P.N + c) * P.Dk) * (long)P.Dv;
    for (int e0 = 0; e0 < P.Dv; e0 += KS) {
        for (int idx = tid; idx < TT * KS; idx += NT) {
            const int r = idx / KS, ee = idx % KS;
            Vs[r][ee] = (r < ns) ? to_f(v[(bh * P.L + s0 + r) * P.Dv + e0 + ee]) : 0.f;
        }
        for (int idx = tid; idx < KS * TT; idx += NT) {
            const int ee = idx / TT, dd = idx % TT;
            Xs[ee][dd] = Gc[(long)(d0 + dd) * P.Dv + e0 + ee];
        }
        __syncthreads();
        mm_AB(acc1, &Vs[0][0], LD, &Xs[0][0], LT, KS, r0, c0);
        __syncthreads();
    }
    if (tid < TT) gam[tid] = bval(b, P.gate, bh * P.L + ce - 1, d0 + tid, P.Dk);
    for (int t0 = s0; t0 < ce; t0 += TQ) {
        const bool diag = (t0 == s0);
        const int nq = min(TQ, ce - t0);
        const int rrow = diag ? s0 : s0 + TQ - 1;
        float a[4][4];
        dscore_tile(a, dO, v, P, bh, t0, nq, s0, ns, Os, Vs, r0, c0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int tt = r0 + i, ss = c0 + j;
                const bool ok = (tt < nq) && (ss < ns) && (s0 + ss <= t0 + tt);
                As[tt][ss] = ok ? P.scale * a[i][j] : 0.f;
            }
        if (tid < TT) rref[tid] = bval(b, P.gate, bh * P.L + rrow, d0 + tid, P.Dk);
        float pp[4][4];
        zero(pp);
        for (int tl = 0; tl < TT; tl += KS) {
            __syncthreads();
            for (int idx = tid; idx < KS * TT; idx += NT) {
                const int t = idx / TT, dd = idx % TT;
                float qv = 0.f;
                if (tl + t < nq) {
                    const long row = bh * P.L + t0 + tl + t;
                    qv = to_f(q[row * P.Dk + d0 + dd]) * __expf(bval(b, P.gate, row, d0 + dd, P.Dk) - rref[dd]);
                }
                Xs[t][dd] = qv;
            }
            __syncthreads();
            // pp[s][d] += sum_t As[t][s] Qh[t][d]
            mm_AtB(pp, &As[tl][0], LT, &Xs[0][0], LT, KS, r0, c0);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (r0 + i >= ns) continue;
            const long row = bh * P.L + s0 + r0 + i;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc2[i][j] += __expf(rref[c0 + j] - bval(b, P.gate, row, d0 + c0 + j, P.Dk)) * pp[i][j];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool valid = (r0 + i < ns);
        float dsum = 0.f;
        if (valid) {
            const long row = bh * P.L + s0 + r0 + i;
            const float iv = igv(ig, row);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int d = d0 + c0 + j;
                const float bd = bval(b, P.gate, row, d, P.Dk);
                const float dkp = __expf(gam[c0 + j] - bd) * acc1[i][j] + acc2[i][j];
                const float kr = to_f(k[row * P.Dk + d]);
                dk[row * P.Dk + d] = from_f<T>(iv * dkp);
                dB[row * P.Dk + d] -= iv * kr * dkp;
                dsum += kr * dkp;
            }
        }
        // reduce over the 16 threads (c0) that share this row
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
        if (dipart && valid && (tid % 16) == 0)
            dipart[((long)blockIdx.x * gridDim.z + bh) * P.L + s0 + r0 + i] = dsum;
    }
}

// ----------------------------------------------------------------- A7: dv
// grid (Dv/64, ceil(L/TQ), B*H)
template <typename T>
__global__ void __launch_bounds__(NT) k_dv(const T* __restrict__ q, const T* __restrict__ k,
                                           const float* __restrict__ ig, const float* __restrict__ b,
                                           const float* __restrict__ Gst, const T* __restrict__ dO,
                                           T* __restrict__ dv, Dims P, int TQ) {
    const int e0 = blockIdx.x * TT;
    const int s0 = blockIdx.y * TQ;
    const long bh = blockIdx.z;
    const int c = s0 / P.C, cs = c * P.C, ce = min(cs + P.C, P.L);
    const int ns = min(TQ, P.L - s0);
    const int tid = threadIdx.x, r0 = (tid / 16) * 4, c0 = (tid % 16) * 4;
    __shared__ float Qh[TT][LD];
    __shared__ float Kh[TT][LD];
    __shared__ float As[TT][LT];
    __shared__ float Xs[KS][LT];
    __shared__ float rref[KS];
    float acc[4][4];
    zero(acc);
    (void)cs;
    // acc[s][e] = sum_d k'_sd e^(Gamma_d - b_sd) G_c[d][e]
    const float* Gc = Gst + ((bh * P.N + c) * P.Dk) * (long)P.Dv;
    for (int d0 = 0; d0 < P.Dk; d0 += KS) {
        if (tid < KS) rref[tid] = bval(b, P.gate, bh * P.L + ce - 1, d0 + tid, P.Dk);
        __syncthreads();
        for (int idx = tid; idx < TT * KS; idx += NT) {
            const int r = idx / KS, dd = idx % KS;
            float kv = 0.f;
            if (r < ns) {
                const long row = bh * P.L + s0 + r;
                kv = to_f(k[row * P.Dk + d0 + dd]) * igv(ig, row) *
                     __expf(rref[dd] - bval(b, P.gate, row, d0 + dd, P.Dk));
            }
            Kh[r][dd] = kv;
        }
        for (int idx = tid; idx < KS * TT; idx += NT) {
            const int dd = idx / TT, ee = idx % TT;
            Xs[dd][ee] = Gc[(long)(d0 + dd) * P.Dv + e0 + ee];
        }
        __syncthreads();
        mm_AB(acc, &Kh[0][0], LD, &Xs[0][0], LT, KS, r0, c0);
        __syncthreads();
    }
    for (int t0 = s0; t0 < ce; t0 += TQ) {
        const bool diag = (t0 == s0);
        const int nq = min(TQ, ce - t0);
        const int rrow = diag ? s0 : s0 + TQ - 1;
        float a[4][4];
        score_tile(a, q, k, ig, b, P, bh, t0, nq, s0, ns, rrow, Qh, Kh, rref, r0, c0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int tt = r0 + i, ss = c0 + j;
                const bool ok = (tt < nq) && (ss < ns) && (s0 + ss <= t0 + tt);
                As[tt][ss] = ok ? P.scale * a[i][j] : 0.f;
            }
        for (int tl = 0; tl < TT; tl += KS) {
            __syncthreads();
            for (int idx = tid; idx < KS * TT; idx += NT) {
                const int t = idx / TT, ee = idx % TT;
                Xs[t][ee] = (tl + t < nq) ? to_f(dO[(bh * P.L + t0 + tl + t) * P.Dv + e0 + ee]) : 0.f;
            }
            __syncthreads();
            mm_AtB(acc, &As[tl][0], LT, &Xs[0][0], LT, KS, r0, c0);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (r0 + i >= ns) continue;
        const long row = bh * P.L + s0 + r0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) dv[row * P.Dv + e0 + c0 + j] = from_f<T>(acc[i][j]);
    }
}

// ------------------------------------------------ A8: reverse cumsum for dg (+ di)
// Per-key gates: grid (B*H), block Dk threads; thread d scans its column backwards.
__global__ void k_dg_key(const float* __restrict__ dB, const float* __restrict__ dhT,
                         const float* __restrict__ hT, float* __restrict__ dg, Dims P) {
    const long bh = blockIdx.x;
    const int d = threadIdx.x;
    if (d >= P.Dk) return;
    float carry = 0.f;
    if (dhT) {
        const float* a = dhT + (bh * P.Dk + d) * (long)P.Dv;
        const float* h = hT + (bh * P.Dk + d) * (long)P.Dv;
        for (int e = 0; e < P.Dv; ++e) carry += a[e] * h[e];
    }
    for (int t = P.L - 1; t >= 0; --t) {
        const long idx = (bh * P.L + t) * P.Dk + d;
        carry += dB[idx];
        dg[idx] = carry;
    }
}

// Row sums over key dims: tok[bh*L+t] = sum_d dB[t][d]; also the input-gate gradient
// di[t] = sum over key tiles of dipart. One warp per token row.
__global__ void k_rowsum(const float* __restrict__ dB, float* __restrict__ tok, const float* __restrict__ dipart,
                         float* __restrict__ di, int ntiles, long rows, int Dk) {
    const long w = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (w >= rows) return;
    if (tok) {
        float s = 0.f;
        for (int d = lane; d < Dk; d += 32) s += dB[w * Dk + d];
        for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) tok[w] = s;
    }
    if (di && lane == 0) {
        float s = 0.f;
        for (int j = 0; j < ntiles; ++j) s += dipart[(long)j * rows + w];
        di[w] = s;
    }
}

// Per-head gates: grid (B*H), one thread scans the token sums backwards.
__global__ void k_dg_head(const float* __restrict__ tok, const float* __restrict__ dhT,
                          const float* __restrict__ hT, float* __restrict__ dg, Dims P) {
    const long bh = blockIdx.x;
    __shared__ float red[256];
    float part = 0.f;
    if (dhT) {
        const long n = (long)P.Dk * P.Dv;
        for (long i = threadIdx.x; i < n; i += blockDim.x) part += dhT[bh * n + i] * hT[bh * n + i];
    }
    red[threadIdx.x] = part;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x != 0) return;
    float carry = red[0];
    for (int t = P.L - 1; t >= 0; --t) {
        carry += tok[bh * P.L + t];
        dg[bh * P.L + t] = carry;
    }
}

// ------------------------------------------------------------------ host side
static int pick_tq(int C) { return (C % 64 == 0) ? 64 : (C % 32 == 0) ? 32 : 16; }

struct WsLayout {
    size_t b, S, G, dB, hT, dipart, tok, total;
};

static WsLayout layout(const Dims& P, bool bwd) {
    WsLayout w{};
    const size_t BH = (size_t)P.B * P.H;
    size_t off = kStatusBytes;
    const size_t bw = (P.gate == GLA_GATE_PER_KEY) ? (size_t)P.Dk : (P.gate == GLA_GATE_PER_HEAD ? 1 : 0);
    w.b = off;
    off = align_up(off + 4 * BH * P.L * bw, 256);
    w.S = off;
    off = align_up(off + 4 * BH * (size_t)P.N * P.Dk * P.Dv, 256);
    if (bwd) {
        w.G = off;
        off = align_up(off + 4 * BH * (size_t)P.N * P.Dk * P.Dv, 256);
        w.dB = off;
        off = align_up(off + 4 * BH * (size_t)P.L * P.Dk, 256);
        w.hT = off;
        off = align_up(off + 4 * BH * (size_t)P.Dk * P.Dv, 256);
        w.dipart = off;
        off = align_up(off + 4 * (size_t)(P.Dk / TT) * BH * P.L, 256);
        w.tok = off;
        off = align_up(off + 4 * BH * (size_t)P.L, 256);
    }
    w.total = off;
    return w;
}

size_t workspace_bytes(const Dims& P, bool bwd) { return layout(P, bwd).total; }

template <typename T>
static cudaError_t fwd_t(const Dims& P, const T* q, const T* k, const T* v, const float* g, const float* ig,
                         const float* h0, T* o, float* hT, char* ws, cudaStream_t st) {
    const WsLayout w = layout(P, false);
    float* b = P.gate != GLA_GATE_NONE ? (float*)(ws + w.b) : nullptr;
    float* S = (float*)(ws + w.S);
    const int BH = P.B * P.H;
    if (P.L == 0) {
        if (hT) {
            const size_t n = (size_t)BH * P.Dk * P.Dv * sizeof(float);
            return h0 ? cudaMemcpyAsync(hT, h0, n, cudaMemcpyDeviceToDevice, st) : cudaMemsetAsync(hT, 0, n, st);
        }
        return cudaSuccess;
    }
    if (b) GLA_LAUNCH("simt_cumsum", st, k_cumsum<<<dim3(P.N, BH), 128, 0, st>>>(g, b, P));
    GLA_LAUNCH("simt_state", st, k_state<T><<<dim3(P.Dv / TT, P.Dk / TT, BH), NT, 0, st>>>(k, v, ig, b, h0, S, hT, P));
    const int TQ = pick_tq(P.C);
    GLA_LAUNCH("simt_out", st, k_out<T><<<dim3(P.Dv / TT, cdiv(P.L, TQ), BH), NT, 0, st>>>(q, k, v, ig, b, S, o, P, TQ));
    return cudaGetLastError();
}

template <typename T>
static cudaError_t bwd_t(const Dims& P, const T* q, const T* k, const T* v, const float* g, const float* ig,
                         const float* h0, const T* dO, const float* dhT, T* dq, T* dk, T* dv, float* dg,
                         float* di, float* dh0, char* ws, cudaStream_t st) {
    const WsLayout w = layout(P, true);
    float* b = P.gate != GLA_GATE_NONE ? (float*)(ws + w.b) : nullptr;
    float* S = (float*)(ws + w.S);
    float* G = (float*)(ws + w.G);
    float* dB = (float*)(ws + w.dB);
    float* hTw = (float*)(ws + w.hT);
    float* dip = (float*)(ws + w.dipart);
    float* tok = (float*)(ws + w.tok);
    const int BH = P.B * P.H;
    if (P.L == 0) {
        if (dh0) {
            const size_t n = (size_t)BH * P.Dk * P.Dv * sizeof(float);
            return dhT ? cudaMemcpyAsync(dh0, dhT, n, cudaMemcpyDeviceToDevice, st) : cudaMemsetAsync(dh0, 0, n, st);
        }
        return cudaSuccess;
    }
    if (b) GLA_LAUNCH("simt_cumsum", st, k_cumsum<<<dim3(P.N, BH), 128, 0, st>>>(g, b, P));
    GLA_LAUNCH("simt_state", st, k_state<T><<<dim3(P.Dv / TT, P.Dk / TT, BH), NT, 0, st>>>(k, v, ig, b, h0, S, hTw, P));
    GLA_LAUNCH("simt_dstate", st, k_dstate<T><<<dim3(P.Dv / TT, P.Dk / TT, BH), NT, 0, st>>>(q, dO, b, dhT, G, dh0, P));
    const int TQ = pick_tq(P.C);
    const int nt = cdiv(P.L, TQ);
    GLA_LAUNCH("simt_dq", st, k_dq<T><<<dim3(P.Dk / TT, nt, BH), NT, 0, st>>>(q, k, v, ig, b, S, dO, dq, dB, P, TQ));
    GLA_LAUNCH("simt_dk", st, k_dk<T><<<dim3(P.Dk / TT, nt, BH), NT, 0, st>>>(q, k, v, ig, b, G, dO, dk, dB, ig ? dip : nullptr, P, TQ));
    GLA_LAUNCH("simt_dv", st, k_dv<T><<<dim3(P.Dv / TT, nt, BH), NT, 0, st>>>(q, k, ig, b, G, dO, dv, P, TQ));
    const long rows = (long)BH * P.L;
    if (P.gate == GLA_GATE_PER_KEY) {
        GLA_LAUNCH("simt_dg_key", st, k_dg_key<<<BH, P.Dk, 0, st>>>(dB, dhT, hTw, dg, P));
    }
    if (P.gate == GLA_GATE_PER_HEAD || di) {
        GLA_LAUNCH("simt_rowsum", st, k_rowsum<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
            dB, P.gate == GLA_GATE_PER_HEAD ? tok : nullptr, dip, di, P.Dk / TT, rows, P.Dk));
    }
    if (P.gate == GLA_GATE_PER_HEAD) GLA_LAUNCH("simt_dg_head", st, k_dg_head<<<BH, 256, 0, st>>>(tok, dhT, hTw, dg, P));
    return cudaGetLastError();
}

cudaError_t fwd(const Dims& P, gla_dtype io, const void* q, const void* k, const void* v, const float* g,
                const float* ig, const float* h0, void* o, float* hT, void* ws, cudaStream_t st) {
    if (io == GLA_BF16)
        return fwd_t<__nv_bfloat16>(P, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                    g, ig, h0, (__nv_bfloat16*)o, hT, (char*)ws, st);
    return fwd_t<float>(P, (const float*)q, (const float*)k, (const float*)v, g, ig, h0, (float*)o, hT,
                        (char*)ws, st);
}

cudaError_t bwd(const Dims& P, gla_dtype io, const void* q, const void* k, const void* v, const float* g,
                const float* ig, const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                float* dg, float* di, float* dh0, void* ws, cudaStream_t st) {
    typedef __nv_bfloat16 bf;
    if (io == GLA_BF16)
        return bwd_t<bf>(P, (const bf*)q, (const bf*)k, (const bf*)v, g, ig, h0, (const bf*)dO, dhT, (bf*)dq,
                         (bf*)dk, (bf*)dv, dg, di, dh0, (char*)ws, st);
    return bwd_t<float>(P, (const float*)q, (const float*)k, (const float*)v, g, ig, h0, (const float*)dO, dhT,
                        (float*)dq, (float*)dk, (float*)dv, dg, di, dh0, (char*)ws, st);
}

}  // namespace simt
}  // namespace gla
