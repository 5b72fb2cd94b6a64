// Chunkwise DeltaNet (delta rule) forward, after the talk summary "Hardware-Efficient Training
// of Linear Attention Models", sections 22:36 and 31:16: a writing strength beta_t, one gradient
// step per token on the key-to-value regression loss, an identity-plus-rank-one transition
// whose product over a chunk the WY representation turns into matrix products. In the row form
// (state S [Dk, Dv], keys and queries rows):
//   S_t = (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t,   o_t = scale q_t S_t.
//
// Chunk form used here. For a chunk of n tokens that starts from S, let x_t be what token t
// adds to the state beyond the transitions, so that S_t = (product of transitions) S + sum
// k_i^T x_i. Unrolling the recurrence gives the triangular system
//   x_t = beta_t (v_t - k_t S - sum_{i<t} (k_t . k_i) x_i),
// i.e. X = T diag(beta) (V - K S) with T = (I + strict_lower(diag(beta) K K^T))^{-1}, unit lower
// triangular. Then
//   O = scale (Q S + lower(Q K^T) X)   (lower keeps the diagonal),   S <- S + K^T X.
// This is the WY form with its two factors (W for the transition product, U for the writes)
// folded into one right-hand side per chunk, so the chunk needs no Dk-wide W.
//
// Plan: CUDA cores, fp32 throughout. One CTA per (b*h, 64-column slice of the values): the
// value columns of the state are independent, so every CTA walks all chunks of its (b, h) in
// order with its [Dk, 64] state slice resident (registers, copied to shared memory for the
// next chunk's products). Per 64-token chunk:
//   1. one pass over Dk computes K K^T, Q K^T, K S and Q S in 4x4 register tiles;
//   2. T by forward substitution, one column per group of 4 lanes (columns are independent,
//      rows sequential; the group splits each dot product and reduces by shuffles);
//   3. X = T R with R = diag(beta)(V - K S);
//   4. O = scale (Q S + lower(Q K^T) X) to global memory, and S += K^T X.
#include <type_traits>

#include "gla_common.cuh"
#include "gla_plans.h"

namespace gla {
namespace {

constexpr int DN_C = 64;     // tokens per chunk
constexpr int DN_VT = 64;    // value columns per CTA
constexpr int DN_NT = 256;   // threads per CTA
constexpr int DN_TS = 68;    // row stride of the token-minor tiles (16-byte rows, spread banks)

template <int DK>
struct DnSmem {
    static constexpr int KT = 0;                       // K^T  [DK][DN_TS]   (sKt[i][t] = k_t[i])
    static constexpr int QT = KT + DK * DN_TS;         // Q^T  [DK][DN_TS]
    static constexpr int R = QT + DK * DN_TS;          // V, then diag(beta)(V - K S)  [C][VT]
    static constexpr int S = R + DN_C * DN_VT;         // state slice [DK][VT]
    static constexpr int A = S + DK * DN_VT;           // beta_t k_t . k_s for s < t, else 0  [C][C]
    static constexpr int QKT = A + DN_C * DN_C;        // (Q K^T)^T masked to s <= t  [C][DN_TS]
    static constexpr int TT = QKT + DN_C * DN_TS;      // T^T  [C][DN_TS]  (sT[c][t] = T[t][c])
    static constexpr int X = TT + DN_C * DN_TS;        // X  [C][VT]
    static constexpr int QS = X + DN_C * DN_VT;        // Q S  [C][VT]
    static constexpr int BETA = QS + DN_C * DN_VT;     // beta  [C]
    static constexpr int FLOATS = BETA + DN_C;
    static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ float f4at(const float4& v, int e) { return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w; }

template <typename T, int DK>
__global__ void __launch_bounds__(DN_NT, 1) k_deltanet_fwd(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, const float* __restrict__ beta,
                                                          const float* __restrict__ h0, T* __restrict__ o,
                                                          float* __restrict__ hT, float* __restrict__ saved, int L,
                                                          int Dv, float scale) {
    using SM = DnSmem<DK>;
    constexpr int RI = DK / 16;                // state rows per thread
    extern __shared__ __align__(16) float sm[];
    float* sKt = sm + SM::KT;
    float* sQt = sm + SM::QT;
    float* sR = sm + SM::R;
    float* sS = sm + SM::S;
    float* sA = sm + SM::A;
    float* sQKt = sm + SM::QKT;
    float* sT = sm + SM::TT;
    float* sX = sm + SM::X;
    float* sQS = sm + SM::QS;
    float* sB = sm + SM::BETA;

    const int bh = blockIdx.x, col0 = blockIdx.y * DN_VT, tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    const int t0 = 4 * ty, j0 = 4 * tx;        // the thread's 4x4 tile of a [C][C] or [C][VT] product
    const int ri0 = RI * ty;                   // the thread's RI x 4 tile of the [DK][VT] state

    // state slice: registers (the thread's tile) and shared memory (the whole slice)
    float Sr[RI][4];
#pragma unroll
    for (int r = 0; r < RI; ++r) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (h0) x = ld4(h0 + ((size_t)bh * DK + ri0 + r) * Dv + col0 + j0);
        Sr[r][0] = x.x;
        Sr[r][1] = x.y;
        Sr[r][2] = x.z;
        Sr[r][3] = x.w;
        st4(sS + (ri0 + r) * DN_VT + j0, x.x, x.y, x.z, x.w);
    }

    const int warp = tid >> 5, lane = tid & 31;
    const int sc = warp * 8 + (lane >> 2), sp = lane & 3;   // solve: column, lane within its group

    for (int c0 = 0; c0 < L; c0 += DN_C) {
        if (saved) {   // the state at this chunk's start, for the backward
            const size_t base = (size_t)bh * ((L + DN_C - 1) / DN_C) + c0 / DN_C;
#pragma unroll
            for (int r = 0; r < RI; ++r)
                st4(saved + (base * DK + ri0 + r) * Dv + col0 + j0, Sr[r][0], Sr[r][1], Sr[r][2], Sr[r][3]);
        }
        __syncthreads();   // the previous chunk is done with every tile below
        // ---- load the chunk (rows past the end read as zero: they add nothing)
        for (int e = tid; e < DN_C * DK; e += DN_NT) {
            const int t = e / DK, i = e - t * DK, gt = c0 + t;
            float kv = 0.f, qv = 0.f;
            if (gt < L) {
                const size_t off = ((size_t)bh * L + gt) * DK + i;
                kv = to_f(k[off]);
                qv = to_f(q[off]);
            }
            sKt[i * DN_TS + t] = kv;
            sQt[i * DN_TS + t] = qv;
        }
        for (int e = tid; e < DN_C * DN_VT; e += DN_NT) {
            const int t = e / DN_VT, j = e - t * DN_VT, gt = c0 + t;
            sR[e] = gt < L ? to_f(v[((size_t)bh * L + gt) * Dv + col0 + j]) : 0.f;
        }
        if (tid < DN_C) sB[tid] = c0 + tid < L ? beta[(size_t)bh * L + c0 + tid] : 0.f;
        __syncthreads();

        // ---- 1. K K^T, Q K^T (rows t0.., columns j0.. as key index s), K S and Q S (columns j0..)
        {
            float kk[4][4] = {}, qk[4][4] = {}, ks[4][4] = {}, qs[4][4] = {};
#pragma unroll 4
            for (int i = 0; i < DK; ++i) {
                const float4 ak = ld4(sKt + i * DN_TS + t0), aq = ld4(sQt + i * DN_TS + t0);
                const float4 bk = ld4(sKt + i * DN_TS + j0), bs = ld4(sS + i * DN_VT + j0);
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float ka = f4at(ak, a), qa = f4at(aq, a);
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const float kb = f4at(bk, b), sb = f4at(bs, b);
                        kk[a][b] = fmaf(ka, kb, kk[a][b]);
                        qk[a][b] = fmaf(qa, kb, qk[a][b]);
                        ks[a][b] = fmaf(ka, sb, ks[a][b]);
                        qs[a][b] = fmaf(qa, sb, qs[a][b]);
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int t = t0 + a;
                const float bt = sB[t];
                float av[4], rv[4];
                const float4 vv = ld4(sR + t * DN_VT + j0);
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    av[b] = j0 + b < t ? bt * kk[a][b] : 0.f;
                    rv[b] = bt * (f4at(vv, b) - ks[a][b]);
                }
                st4(sA + t * DN_C + j0, av[0], av[1], av[2], av[3]);
                st4(sR + t * DN_VT + j0, rv[0], rv[1], rv[2], rv[3]);
                st4(sQS + t * DN_VT + j0, qs[a][0], qs[a][1], qs[a][2], qs[a][3]);
            }
            // (Q K^T)^T: column s = j0 + b holds rows t0..t0+3, kept where s <= t
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int s = j0 + b;
                st4(sQKt + s * DN_TS + t0, s <= t0 ? qk[0][b] : 0.f, s <= t0 + 1 ? qk[1][b] : 0.f,
                    s <= t0 + 2 ? qk[2][b] : 0.f, s <= t0 + 3 ? qk[3][b] : 0.f);
            }
        }
        __syncthreads();

        // ---- 2. T = (I + A)^{-1}: T[t][c] = [t == c] - sum_{c <= i < t} A[t][i] T[i][c], row by row
        for (int t = 0; t < DN_C; ++t) {
            float part = 0.f;
            for (int i = sc + sp; i < t; i += 4) part = fmaf(sA[t * DN_C + i], sT[sc * DN_TS + i], part);
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (sp == 0) sT[sc * DN_TS + t] = t < sc ? 0.f : t == sc ? 1.f : -part;
            __syncwarp();
        }
        __syncthreads();

        // ---- 3. X = T R (T[t][i] = 0 for i > t)
        {
            float x[4][4] = {};
            for (int i = 0; i < t0 + 4; ++i) {
                const float4 a4 = ld4(sT + i * DN_TS + t0), b4 = ld4(sR + i * DN_VT + j0);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) x[a][b] = fmaf(f4at(a4, a), f4at(b4, b), x[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) st4(sX + (t0 + a) * DN_VT + j0, x[a][0], x[a][1], x[a][2], x[a][3]);
        }
        __syncthreads();

        // ---- 4. O = scale (Q S + lower(Q K^T) X) (skipped when only states are wanted), and S += K^T X
        if (o) {
            float y[4][4] = {};
            for (int i = 0; i < t0 + 4; ++i) {
                const float4 a4 = ld4(sQKt + i * DN_TS + t0), b4 = ld4(sX + i * DN_VT + j0);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) y[a][b] = fmaf(f4at(a4, a), f4at(b4, b), y[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int gt = c0 + t0 + a;
                if (gt < L) {
                    const float4 qs4 = ld4(sQS + (t0 + a) * DN_VT + j0);
                    T* op = o + ((size_t)bh * L + gt) * Dv + col0 + j0;
                    op[0] = from_f<T>(scale * (qs4.x + y[a][0]));
                    op[1] = from_f<T>(scale * (qs4.y + y[a][1]));
                    op[2] = from_f<T>(scale * (qs4.z + y[a][2]));
                    op[3] = from_f<T>(scale * (qs4.w + y[a][3]));
                }
            }
        }
        {
#pragma unroll 4
            for (int t = 0; t < DN_C; ++t) {
                const float4 b4 = ld4(sX + t * DN_VT + j0);
#pragma unroll
                for (int r = 0; r < RI; ++r) {
                    const float kr = sKt[(ri0 + r) * DN_TS + t];
                    Sr[r][0] = fmaf(kr, b4.x, Sr[r][0]);
                    Sr[r][1] = fmaf(kr, b4.y, Sr[r][1]);
                    Sr[r][2] = fmaf(kr, b4.z, Sr[r][2]);
                    Sr[r][3] = fmaf(kr, b4.w, Sr[r][3]);
                }
            }
            // sS is read only in step 1, behind the next chunk's barriers
#pragma unroll
            for (int r = 0; r < RI; ++r) st4(sS + (ri0 + r) * DN_VT + j0, Sr[r][0], Sr[r][1], Sr[r][2], Sr[r][3]);
        }
    }

    if (hT) {
#pragma unroll
        for (int r = 0; r < RI; ++r)
            st4(hT + ((size_t)bh * DK + ri0 + r) * Dv + col0 + j0, Sr[r][0], Sr[r][1], Sr[r][2], Sr[r][3]);
    }
}

template <typename T, int DK>
cudaError_t dn_launch(const gla_problem* p, const void* q, const void* k, const void* v, const float* beta,
                      const float* h0, void* o, float* hT, float* saved, cudaStream_t st) {
    auto kern = k_deltanet_fwd<T, DK>;
    const size_t smem = DnSmem<DK>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p->B * p->H, p->Dv / DN_VT);
    // without an output it is the backward's state pass: timed under its own name
    GLA_LAUNCH(o ? "deltanet_fwd" : "deltanet_state", st,
               (kern<<<grid, DN_NT, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                static_cast<const T*>(v), beta, h0, static_cast<T*>(o), hT, saved,
                                                p->L, p->Dv, p->scale)));
    return cudaGetLastError();
}

// bf16 I/O runs the tensor-core forward (gla_deltanet_tc.cu); fp32 I/O the CUDA-core one above.
template <typename T>
cudaError_t dn_launch_dk(const gla_problem* p, const void* q, const void* k, const void* v, const float* beta,
                         const float* h0, void* o, float* hT, float* saved, cudaStream_t st) {
    if (std::is_same<T, __nv_bfloat16>::value)
        return tc::deltanet_fwd(p->B, p->H, p->L, p->Dk, p->Dv, p->scale, q, k, v, beta, h0, o, hT, saved, nullptr, st);
    return p->Dk == 64 ? dn_launch<T, 64>(p, q, k, v, beta, h0, o, hT, saved, st)
                       : dn_launch<T, 128>(p, q, k, v, beta, h0, o, hT, saved, st);
}

// ------------------------------------------------------------------ backward
// With R = diag(beta) U, U = V - K S, X = T R, P = lower(Q K^T) and the gradient dS' reaching
// the chunk's end state, the chunk's gradients are (G a strict-lower n x n matrix):
//   dX = scale P^T dO + K dS'          dR = T^T dX          dV = diag(beta) dR
//   dS = dS' + scale Q^T dO - K^T diag(beta) dR            (the gradient at the chunk's start)
//   dP = scale lower(dO X^T)           G = -strict_lower(dR X^T)
//   dbeta_t = sum_j dR_tj U_tj + sum_{s<t} G_ts (k_t . k_s)
//   dQ = scale dO S^T + dP K
//   dK = dP^T Q + X dS'^T - diag(beta) dR S^T + diag(beta) G K + G^T diag(beta) K.
// Only dS carries across chunks, and its value columns are independent, so a reverse walk per
// (b*h, 64-column slice) (k_deltanet_bwd_walk) produces X, dR, dV, the end gradients dS' and
// each slice's part of sum_j dR U; then one CTA per (b*h, chunk) (k_deltanet_bwd_grads) sums
// the products over every value slice and forms dQ, dK, dbeta, all chunks in parallel. The
// chunks' start states come from the forward kernel (its `saved` output).
template <int DK>
struct DnWalkSmem {
    static constexpr int KT = 0;                       // K^T [DK][DN_TS]
    static constexpr int QT = KT + DK * DN_TS;         // Q^T [DK][DN_TS]
    static constexpr int DS = QT + DK * DN_TS;         // dS' slice [DK][VT]
    static constexpr int U = DS + DK * DN_VT;          // V, then U = V - K S  [C][VT]
    static constexpr int DO = U + DN_C * DN_VT;        // dO [C][VT]
    static constexpr int KK = DO + DN_C * DN_VT;       // k_t . k_s for s < t, else 0  [C][C]
    static constexpr int PR = KK + DN_C * DN_C;        // P = lower(Q K^T) [C][C], then dR [C][VT]
    static constexpr int DX = PR + DN_C * DN_C;        // K dS', then dX  [C][VT]
    static constexpr int TT = DX + DN_C * DN_VT;       // T^T [C][DN_TS]
    static constexpr int BETA = TT + DN_C * DN_TS;     // beta [C]
    static constexpr int FLOATS = BETA + DN_C;
    static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

template <typename T, int DK>
__global__ void __launch_bounds__(DN_NT, 1) k_deltanet_bwd_walk(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ beta,
    const T* __restrict__ dO, const float* __restrict__ dhT, const float* __restrict__ saved, float* __restrict__ xw,
    float* __restrict__ drw, float* __restrict__ dsend, float* __restrict__ db1, T* __restrict__ dv,
    float* __restrict__ dh0, int BH, int L, int Dv, float scale) {
    using SM = DnWalkSmem<DK>;
    constexpr int RI = DK / 16;
    extern __shared__ __align__(16) float sm[];
    float* sKt = sm + SM::KT;
    float* sQt = sm + SM::QT;
    float* sdS = sm + SM::DS;
    float* sU = sm + SM::U;
    float* sdO = sm + SM::DO;
    float* sKK = sm + SM::KK;
    float* sPR = sm + SM::PR;
    float* sdX = sm + SM::DX;
    float* sT = sm + SM::TT;
    float* sB = sm + SM::BETA;

    const int bh = blockIdx.x, slice = blockIdx.y, col0 = slice * DN_VT, tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    const int t0 = 4 * ty, j0 = 4 * tx, ri0 = RI * ty;
    const int NC = (L + DN_C - 1) / DN_C;

    float Gr[RI][4];   // dS' slice tile
#pragma unroll
    for (int r = 0; r < RI; ++r) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (dhT) x = ld4(dhT + ((size_t)bh * DK + ri0 + r) * Dv + col0 + j0);
        Gr[r][0] = x.x;
        Gr[r][1] = x.y;
        Gr[r][2] = x.z;
        Gr[r][3] = x.w;
        st4(sdS + (ri0 + r) * DN_VT + j0, x.x, x.y, x.z, x.w);
    }
    const int warp = tid >> 5, lane = tid & 31;
    const int sc = warp * 8 + (lane >> 2), sp = lane & 3;

    for (int ci = NC - 1; ci >= 0; --ci) {
        const int c0 = ci * DN_C;
        const size_t sbase = (size_t)bh * NC + ci;   // chunk's row of the per-chunk state arrays
        __syncthreads();
        for (int e = tid; e < DN_C * DK; e += DN_NT) {
            const int t = e / DK, i = e - t * DK, gt = c0 + t;
            float kv = 0.f, qv = 0.f;
            if (gt < L) {
                const size_t off = ((size_t)bh * L + gt) * DK + i;
                kv = to_f(k[off]);
                qv = to_f(q[off]);
            }
            sKt[i * DN_TS + t] = kv;
            sQt[i * DN_TS + t] = qv;
        }
        for (int e = tid; e < DN_C * DN_VT; e += DN_NT) {
            const int t = e / DN_VT, j = e - t * DN_VT, gt = c0 + t;
            const size_t off = ((size_t)bh * L + gt) * Dv + col0 + j;
            sU[e] = gt < L ? to_f(v[off]) : 0.f;
            sdO[e] = gt < L ? to_f(dO[off]) : 0.f;
        }
        if (tid < DN_C) sB[tid] = c0 + tid < L ? beta[(size_t)bh * L + c0 + tid] : 0.f;
        __syncthreads();

        // ---- 1. K K^T, Q K^T, K S (S: the chunk's start state, from global) and K dS'
        {
            float kk[4][4] = {}, qk[4][4] = {}, ks[4][4] = {}, kd[4][4] = {};
            const float* Sg = saved + (sbase * DK) * Dv + col0 + j0;
#pragma unroll 4
            for (int i = 0; i < DK; ++i) {
                const float4 ak = ld4(sKt + i * DN_TS + t0), aq = ld4(sQt + i * DN_TS + t0);
                const float4 bk = ld4(sKt + i * DN_TS + j0), bd = ld4(sdS + i * DN_VT + j0);
                const float4 bs = __ldg(reinterpret_cast<const float4*>(Sg + (size_t)i * Dv));
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float ka = f4at(ak, a), qa = f4at(aq, a);
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        kk[a][b] = fmaf(ka, f4at(bk, b), kk[a][b]);
                        qk[a][b] = fmaf(qa, f4at(bk, b), qk[a][b]);
                        ks[a][b] = fmaf(ka, f4at(bs, b), ks[a][b]);
                        kd[a][b] = fmaf(ka, f4at(bd, b), kd[a][b]);
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int t = t0 + a;
                const float4 vv = ld4(sU + t * DN_VT + j0);
                st4(sKK + t * DN_C + j0, j0 < t ? kk[a][0] : 0.f, j0 + 1 < t ? kk[a][1] : 0.f,
                    j0 + 2 < t ? kk[a][2] : 0.f, j0 + 3 < t ? kk[a][3] : 0.f);
                st4(sPR + t * DN_C + j0, j0 <= t ? qk[a][0] : 0.f, j0 + 1 <= t ? qk[a][1] : 0.f,
                    j0 + 2 <= t ? qk[a][2] : 0.f, j0 + 3 <= t ? qk[a][3] : 0.f);
                st4(sU + t * DN_VT + j0, vv.x - ks[a][0], vv.y - ks[a][1], vv.z - ks[a][2], vv.w - ks[a][3]);
                st4(sdX + t * DN_VT + j0, kd[a][0], kd[a][1], kd[a][2], kd[a][3]);
            }
        }
        __syncthreads();

        // ---- 2. T = (I + diag(beta) strict_lower(K K^T))^{-1}, as in the forward
        for (int t = 0; t < DN_C; ++t) {
            float part = 0.f;
            for (int i = sc + sp; i < t; i += 4) part = fmaf(sKK[t * DN_C + i], sT[sc * DN_TS + i], part);
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (sp == 0) sT[sc * DN_TS + t] = t < sc ? 0.f : t == sc ? 1.f : -sB[t] * part;
            __syncwarp();
        }
        __syncthreads();

        // ---- 3. dX = K dS' + scale P^T dO (own tile, in place), and X = T diag(beta) U to global
        {
            float y[4][4] = {};
            for (int s2 = t0; s2 < DN_C; ++s2) {   // P[s][t] = 0 for s < t
                const float4 a4 = ld4(sPR + s2 * DN_C + t0), b4 = ld4(sdO + s2 * DN_VT + j0);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) y[a][b] = fmaf(f4at(a4, a), f4at(b4, b), y[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                float* d = sdX + (t0 + a) * DN_VT + j0;
                const float4 x = ld4(d);
                st4(d, fmaf(scale, y[a][0], x.x), fmaf(scale, y[a][1], x.y), fmaf(scale, y[a][2], x.z),
                    fmaf(scale, y[a][3], x.w));
            }
            float x[4][4] = {};
            for (int i = 0; i < t0 + 4; ++i) {
                const float4 a4 = ld4(sT + i * DN_TS + t0), u4 = ld4(sU + i * DN_VT + j0);
                const float bi = sB[i];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) x[a][b] = fmaf(f4at(a4, a), bi * f4at(u4, b), x[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int gt = c0 + t0 + a;
                if (gt < L) st4(xw + ((size_t)bh * L + gt) * Dv + col0 + j0, x[a][0], x[a][1], x[a][2], x[a][3]);
            }
        }
        __syncthreads();

        // ---- 4. dR = T^T dX (T[s][t] = 0 for s < t), over P's tile
        {
            float y[4][4] = {};
            for (int s2 = t0; s2 < DN_C; ++s2) {
                const float4 b4 = ld4(sdX + s2 * DN_VT + j0);
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float tv = sT[(t0 + a) * DN_TS + s2];
#pragma unroll
                    for (int b = 0; b < 4; ++b) y[a][b] = fmaf(tv, f4at(b4, b), y[a][b]);
                }
            }
            // P's last reads were in step 3, behind the barrier above
#pragma unroll
            for (int a = 0; a < 4; ++a) st4(sPR + (t0 + a) * DN_VT + j0, y[a][0], y[a][1], y[a][2], y[a][3]);
        }
        __syncthreads();

        // ---- 5. dV, dR, the slice's part of sum_j dR U, the end gradient dS', and dS
        {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int t = t0 + a, gt = c0 + t;
                if (gt < L) {
                    const float4 r4 = ld4(sPR + t * DN_VT + j0);
                    const float bt = sB[t];
                    const size_t off = ((size_t)bh * L + gt) * Dv + col0 + j0;
                    st4(drw + off, r4.x, r4.y, r4.z, r4.w);
                    dv[off] = from_f<T>(bt * r4.x);
                    dv[off + 1] = from_f<T>(bt * r4.y);
                    dv[off + 2] = from_f<T>(bt * r4.z);
                    dv[off + 3] = from_f<T>(bt * r4.w);
                }
            }
            {   // 4 threads per token row, 16 columns each
                const int t = tid >> 2, part = tid & 3;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) acc = fmaf(sPR[t * DN_VT + part * 16 + j], sU[t * DN_VT + part * 16 + j], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (part == 0 && c0 + t < L) db1[((size_t)slice * BH + bh) * L + c0 + t] = acc;
            }
#pragma unroll
            for (int r = 0; r < RI; ++r)
                st4(dsend + (sbase * DK + ri0 + r) * Dv + col0 + j0, Gr[r][0], Gr[r][1], Gr[r][2], Gr[r][3]);
#pragma unroll 4
            for (int t = 0; t < DN_C; ++t) {
                const float4 o4 = ld4(sdO + t * DN_VT + j0), r4 = ld4(sPR + t * DN_VT + j0);
                const float bt = sB[t];
#pragma unroll
                for (int r = 0; r < RI; ++r) {
                    const float qv = scale * sQt[(ri0 + r) * DN_TS + t], kv = bt * sKt[(ri0 + r) * DN_TS + t];
                    Gr[r][0] = fmaf(qv, o4.x, fmaf(-kv, r4.x, Gr[r][0]));
                    Gr[r][1] = fmaf(qv, o4.y, fmaf(-kv, r4.y, Gr[r][1]));
                    Gr[r][2] = fmaf(qv, o4.z, fmaf(-kv, r4.z, Gr[r][2]));
                    Gr[r][3] = fmaf(qv, o4.w, fmaf(-kv, r4.w, Gr[r][3]));
                }
            }
            // sdS is read only in step 1, behind the next chunk's barriers
#pragma unroll
            for (int r = 0; r < RI; ++r) st4(sdS + (ri0 + r) * DN_VT + j0, Gr[r][0], Gr[r][1], Gr[r][2], Gr[r][3]);
        }
    }
    if (dh0) {
#pragma unroll
        for (int r = 0; r < RI; ++r)
            st4(dh0 + ((size_t)bh * DK + ri0 + r) * Dv + col0 + j0, Gr[r][0], Gr[r][1], Gr[r][2], Gr[r][3]);
    }
}

template <int DK>
struct DnGradSmem {
    static constexpr int KS = DK + 4;                  // row stride of the [C][DK] and [VT][DK] tiles
    static constexpr int K = 0;                        // K [C][KS]
    static constexpr int Q = K + DN_C * KS;            // Q [C][KS]
    static constexpr int DOT = Q + DN_C * KS;          // dO^T [VT][DN_TS], later dP [C][DN_TS]
    static constexpr int XT = DOT + DN_VT * DN_TS;     // X^T, later dP^T
    static constexpr int DRT = XT + DN_VT * DN_TS;     // dR^T, later G
    static constexpr int ST = DRT + DN_VT * DN_TS;     // S^T [VT][KS], later G^T
    static constexpr int DST = ST + DN_VT * KS;        // dS'^T [VT][KS]
    static constexpr int BETA = DST + DN_VT * KS;      // beta [C]
    static constexpr int FLOATS = BETA + DN_C;
    static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

template <typename T, int DK>
__global__ void __launch_bounds__(DN_NT, 1) k_deltanet_bwd_grads(
    const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ beta, const T* __restrict__ dO,
    const float* __restrict__ saved, const float* __restrict__ xw, const float* __restrict__ drw,
    const float* __restrict__ dsend, const float* __restrict__ db1, T* __restrict__ dq, T* __restrict__ dk,
    float* __restrict__ dbeta, int BH, int L, int Dv, float scale) {
    using SM = DnGradSmem<DK>;
    constexpr int KS = SM::KS, IC = DK / 16;   // IC: key columns per thread
    extern __shared__ __align__(16) float sm[];
    float* sK = sm + SM::K;
    float* sQ = sm + SM::Q;
    float* sdOt = sm + SM::DOT;
    float* sXt = sm + SM::XT;
    float* sdRt = sm + SM::DRT;
    float* sSt = sm + SM::ST;
    float* sdSt = sm + SM::DST;
    float* sB = sm + SM::BETA;

    const int ci = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int NC = (L + DN_C - 1) / DN_C, c0 = ci * DN_C;
    const size_t sbase = (size_t)bh * NC + ci;
    const int ty = tid >> 4, tx = tid & 15;
    const int t0 = 4 * ty, s0 = 4 * tx, i0 = IC * tx;

    for (int e = tid; e < DN_C * DK; e += DN_NT) {
        const int t = e / DK, i = e - t * DK, gt = c0 + t;
        float kv = 0.f, qv = 0.f;
        if (gt < L) {
            const size_t off = ((size_t)bh * L + gt) * DK + i;
            kv = to_f(k[off]);
            qv = to_f(q[off]);
        }
        sK[t * KS + i] = kv;
        sQ[t * KS + i] = qv;
    }
    if (tid < DN_C) sB[tid] = c0 + tid < L ? beta[(size_t)bh * L + c0 + tid] : 0.f;

    float dP[4][4] = {}, Gm[4][4] = {}, dQa[4][IC] = {}, dKa[4][IC] = {};
    const int nsl = Dv / DN_VT;
    for (int sl = 0; sl < nsl; ++sl) {
        const int col0 = sl * DN_VT;
        __syncthreads();   // the previous slice's tiles are consumed
        for (int e = tid; e < DN_C * DN_VT; e += DN_NT) {
            const int t = e / DN_VT, j = e - t * DN_VT, gt = c0 + t;
            const size_t off = ((size_t)bh * L + gt) * Dv + col0 + j;
            const bool in = gt < L;
            sdOt[j * DN_TS + t] = in ? to_f(dO[off]) : 0.f;
            sXt[j * DN_TS + t] = in ? xw[off] : 0.f;
            sdRt[j * DN_TS + t] = in ? drw[off] : 0.f;
        }
        for (int e = tid; e < DK * DN_VT; e += DN_NT) {
            const int i = e / DN_VT, j = e - i * DN_VT;
            const size_t off = (sbase * DK + i) * Dv + col0 + j;
            sSt[j * KS + i] = saved[off];
            sdSt[j * KS + i] = dsend[off];
        }
        __syncthreads();
        for (int j = 0; j < DN_VT; ++j) {
            const float4 ao = ld4(sdOt + j * DN_TS + t0), ar = ld4(sdRt + j * DN_TS + t0);
            const float4 ax = ld4(sXt + j * DN_TS + t0), bx = ld4(sXt + j * DN_TS + s0);
            float br[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) br[a] = sB[t0 + a] * f4at(ar, a);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    dP[a][b] = fmaf(f4at(ao, a), f4at(bx, b), dP[a][b]);
                    Gm[a][b] = fmaf(f4at(ar, a), f4at(bx, b), Gm[a][b]);
                }
#pragma unroll
            for (int c4 = 0; c4 < IC; c4 += 4) {
                const float4 bs = ld4(sSt + j * KS + i0 + c4), bd = ld4(sdSt + j * KS + i0 + c4);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        // dO S^T, and X dS'^T - diag(beta) dR S^T
                        dQa[a][c4 + c] = fmaf(f4at(ao, a), f4at(bs, c), dQa[a][c4 + c]);
                        dKa[a][c4 + c] = fmaf(f4at(ax, a), f4at(bd, c), fmaf(-br[a], f4at(bs, c), dKa[a][c4 + c]));
                    }
            }
        }
    }
    __syncthreads();   // all slices consumed: the transposed tiles become dP, dP^T, G, G^T
    float* sdP = sdOt;    // dP [t][s], s <= t
    float* sdPt = sXt;    // dP^T [s][t]
    float* sG = sdRt;     // G [t][s], s < t
    float* sGt = sSt;     // G^T [s][t]
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int t = t0 + a;
        float pv[4], gv[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            pv[b] = s0 + b <= t ? scale * dP[a][b] : 0.f;
            gv[b] = s0 + b < t ? -Gm[a][b] : 0.f;
        }
        st4(sdP + t * DN_TS + s0, pv[0], pv[1], pv[2], pv[3]);
        st4(sG + t * DN_TS + s0, gv[0], gv[1], gv[2], gv[3]);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            sdPt[(s0 + b) * DN_TS + t] = pv[b];
            sGt[(s0 + b) * DN_TS + t] = gv[b];
        }
    }
    __syncthreads();

    // dQ = scale dO S^T + dP K;  dK = (X dS'^T - diag(beta) dR S^T) + dP^T Q + diag(beta) G K + G^T diag(beta) K
    float GK[4][IC] = {};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < IC; ++c) dQa[a][c] *= scale;
    for (int s2 = 0; s2 < DN_C; ++s2) {
        const float4 pT = ld4(sdPt + s2 * DN_TS + t0);   // dP[t0+a][s2]
        const float4 pr = ld4(sdP + s2 * DN_TS + t0);    // dP[s2][t0+a]
        const float4 gT = ld4(sGt + s2 * DN_TS + t0);    // G[t0+a][s2]
        const float4 gr = ld4(sG + s2 * DN_TS + t0);     // G[s2][t0+a]
        const float bs = sB[s2];
#pragma unroll
        for (int c4 = 0; c4 < IC; c4 += 4) {
            const float4 kv = ld4(sK + s2 * KS + i0 + c4), qv = ld4(sQ + s2 * KS + i0 + c4);
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float gb = f4at(gr, a) * bs;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    dQa[a][c4 + c] = fmaf(f4at(pT, a), f4at(kv, c), dQa[a][c4 + c]);
                    dKa[a][c4 + c] = fmaf(f4at(pr, a), f4at(qv, c), fmaf(gb, f4at(kv, c), dKa[a][c4 + c]));
                    GK[a][c4 + c] = fmaf(f4at(gT, a), f4at(kv, c), GK[a][c4 + c]);
                }
            }
        }
    }
    float dbp[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int t = t0 + a, gt = c0 + t;
        const float bt = sB[t];
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < IC; ++c) {
            dKa[a][c] = fmaf(bt, GK[a][c], dKa[a][c]);
            acc = fmaf(sK[t * KS + i0 + c], GK[a][c], acc);   // sum_s G_ts (k_t . k_s), this thread's keys
        }
        dbp[a] = acc;
        if (gt < L) {
            const size_t off = ((size_t)bh * L + gt) * DK + i0;
#pragma unroll
            for (int c = 0; c < IC; ++c) {
                dq[off + c] = from_f<T>(dQa[a][c]);
                dk[off + c] = from_f<T>(dKa[a][c]);
            }
        }
    }
    // the 16 threads of a row group (one half-warp) hold the row's key columns
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        float x = dbp[a];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        const int gt = c0 + t0 + a;
        if (tx == 0 && gt < L) {
            for (int sl = 0; sl < nsl; ++sl) x += db1[((size_t)sl * BH + bh) * L + gt];
            dbeta[(size_t)bh * L + gt] = x;
        }
    }
}

struct DnBwdWs {
    float *saved, *xw, *drw, *dsend, *db1;
    size_t bytes;
};

// Backward workspace. fp32 I/O (CUDA-core kernels): the chunk start states and end gradients in
// fp32, X and dR, and each value slice's sum_j dR U. bf16 I/O (tensor-core kernels): the chunk
// start states and end gradients in bf16 (the precision the products read them in) and dR; the
// gradient kernel forms X and sum_j dR U itself.
DnBwdWs dn_bwd_ws(const gla_problem* p, void* base) {
    const size_t BH = (size_t)p->B * p->H, NC = (size_t)((p->L + DN_C - 1) / DN_C);
    const size_t st = BH * NC * p->Dk * p->Dv, tok = BH * p->L * p->Dv, nsl = p->Dv / DN_VT;
    const bool tc = p->io == GLA_BF16;
    const size_t bytes[5] = {st * (tc ? 2 : 4), tc ? 0 : tok * 4, tok * 4, st * (tc ? 2 : 4), tc ? 0 : nsl * BH * p->L * 4};
    DnBwdWs w{};
    float** dst[5] = {&w.saved, &w.xw, &w.drw, &w.dsend, &w.db1};
    size_t off = 0;
    for (int i = 0; i < 5; ++i) {
        *dst[i] = (base && bytes[i]) ? reinterpret_cast<float*>(static_cast<char*>(base) + off) : nullptr;
        off += (bytes[i] + 255) / 256 * 256;
    }
    w.bytes = off > 0 ? off : 256;   // never 0, which the size query reserves for "unsupported"
    return w;
}

// states_given: w.saved already holds the chunk start states (left by the forward of a training
// pair), so the forward's state walk is not run again.
template <typename T, int DK>
cudaError_t dn_bwd_launch(const gla_problem* p, const void* q, const void* k, const void* v, const float* beta,
                          const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                          float* dbeta, float* dh0, const DnBwdWs& w, bool states_given, cudaStream_t st) {
    cudaError_t e = states_given ? cudaSuccess : dn_launch_dk<T>(p, q, k, v, beta, h0, nullptr, nullptr, w.saved, st);
    if (e != cudaSuccess) return e;
    const int BH = p->B * p->H, NC = (p->L + DN_C - 1) / DN_C;
    auto walk = k_deltanet_bwd_walk<T, DK>;
    auto grads = k_deltanet_bwd_grads<T, DK>;
    const size_t sw = DnWalkSmem<DK>::BYTES, sg = DnGradSmem<DK>::BYTES;
    if ((e = cudaFuncSetAttribute(walk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sw)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(grads, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg)) != cudaSuccess)
        return e;
    const T* tq = static_cast<const T*>(q);
    const T* tk = static_cast<const T*>(k);
    const T* tdo = static_cast<const T*>(dO);
    if (std::is_same<T, __nv_bfloat16>::value) {   // bf16 I/O: the tensor-core walk
        e = tc::deltanet_walk(p->B, p->H, p->L, DK, p->Dv, p->scale, q, k, beta, dO, dhT, w.drw, w.dsend, dv, dh0,
                              st);
    } else {
        GLA_LAUNCH("deltanet_bwd_walk", st,
                   (walk<<<dim3(BH, p->Dv / DN_VT), DN_NT, sw, st>>>(tq, tk, static_cast<const T*>(v), beta, tdo, dhT,
                                                                     w.saved, w.xw, w.drw, w.dsend, w.db1,
                                                                     static_cast<T*>(dv), dh0, BH, p->L, p->Dv,
                                                                     p->scale)));
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    if (std::is_same<T, __nv_bfloat16>::value)   // bf16 I/O: the tensor-core gradients
        return tc::deltanet_grads(p->B, p->H, p->L, DK, p->Dv, p->scale, q, k, v, beta, dO, w.saved, w.drw,
                                  w.dsend, dq, dk, dbeta, st);
    if (NC > 0)
        GLA_LAUNCH("deltanet_bwd_grads", st,
                   (grads<<<dim3(NC, BH), DN_NT, sg, st>>>(tq, tk, beta, tdo, w.saved, w.xw, w.drw, w.dsend, w.db1,
                                                           static_cast<T*>(dq), static_cast<T*>(dk), dbeta, BH, p->L,
                                                           p->Dv, p->scale)));
    return cudaGetLastError();
}

static_assert(DnWalkSmem<128>::BYTES <= 227 * 1024, "shared memory of the Dk = 128 backward walk");
static_assert(DnGradSmem<128>::BYTES <= 227 * 1024, "shared memory of the Dk = 128 backward gradients");

bool dn_aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

static_assert(DnSmem<128>::BYTES <= 227 * 1024, "shared memory of the Dk = 128 plan");

// Validation shared by the forward and the backward, so that a problem one accepts the other
// accepts too. B*H is at most 65535: the backward's per-chunk gradient kernel puts the heads on
// the grid's y extent.
gla_status dn_check(const gla_problem* p) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE) return GLA_ERR_INVALID_ARG;
    if ((p->Dk != 64 && p->Dk != 128) || p->Dv <= 0 || p->Dv % DN_VT != 0 || p->Dv > 4096 || p->chunk != DN_C)
        return GLA_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 65535LL) return GLA_ERR_UNSUPPORTED;
    return GLA_OK;
}

}  // namespace
}  // namespace gla

namespace gla {
namespace {

// Bytes of the chunk start states the backward reads: [B*H][chunks][Dk][Dv] in bf16 for bf16 I/O
// (the precision the tensor-core products read them in), fp32 for fp32 I/O.
size_t dn_saved_bytes(const gla_problem* p) {
    const size_t BH = (size_t)p->B * p->H, NC = (size_t)((p->L + DN_C - 1) / DN_C);
    return BH * NC * p->Dk * p->Dv * (p->io == GLA_BF16 ? 2 : 4);
}

gla_status dn_fwd_entry(const gla_problem* p, const void* q, const void* k, const void* v, const float* beta,
                        const float* h0, void* o, float* hT, void* saved, void* stream) {
    const gla_status c = dn_check(p);
    if (c != GLA_OK) return c;
    if ((size_t)p->B * p->H == 0) return GLA_OK;
    if (p->L > 0 && (!q || !k || !v || !beta || !o)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, h0, o, hT, saved};
    for (const void* x : ptrs)
        if (!dn_aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (dn_saved_bytes(p) == 0) saved = nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    float* sv = static_cast<float*>(saved);
    const cudaError_t e = p->io == GLA_BF16 ? dn_launch_dk<__nv_bfloat16>(p, q, k, v, beta, h0, o, hT, sv, st)
                                            : dn_launch_dk<float>(p, q, k, v, beta, h0, o, hT, sv, st);
    return record_cuda(e, "DeltaNet forward launch");
}

gla_status dn_bwd_entry(const gla_problem* p, const void* q, const void* k, const void* v, const float* beta,
                        const float* h0, const void* dO, const float* dhT, const void* saved, void* dq, void* dk,
                        void* dv, float* dbeta, float* dh0, void* ws, size_t ws_bytes, void* stream) {
    const gla_status c = dn_check(p);
    if (c != GLA_OK) return c;
    if ((size_t)p->B * p->H == 0) return GLA_OK;
    if (p->L > 0 && (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, h0, dO, dhT, saved, dq, dk, dv, dbeta, dh0, ws};
    for (const void* x : ptrs)
        if (!dn_aligned16(x)) return GLA_ERR_INVALID_ARG;
    DnBwdWs w = dn_bwd_ws(p, ws);
    if (!ws || ws_bytes < w.bytes) return GLA_ERR_WORKSPACE;
    const bool given = saved != nullptr && dn_saved_bytes(p) > 0;
    if (given) w.saved = const_cast<float*>(static_cast<const float*>(saved));   // read only
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (p->io == GLA_BF16)
        e = p->Dk == 64 ? dn_bwd_launch<__nv_bfloat16, 64>(p, q, k, v, beta, h0, dO, dhT, dq, dk, dv, dbeta, dh0, w, given, st)
                        : dn_bwd_launch<__nv_bfloat16, 128>(p, q, k, v, beta, h0, dO, dhT, dq, dk, dv, dbeta, dh0, w, given, st);
    else
        e = p->Dk == 64 ? dn_bwd_launch<float, 64>(p, q, k, v, beta, h0, dO, dhT, dq, dk, dv, dbeta, dh0, w, given, st)
                        : dn_bwd_launch<float, 128>(p, q, k, v, beta, h0, dO, dhT, dq, dk, dv, dbeta, dh0, w, given, st);
    return record_cuda(e, "DeltaNet backward launch");
}

}  // namespace
}  // namespace gla

extern "C" gla_status gla_deltanet_fwd(const gla_problem* p, const void* q, const void* k, const void* v,
                                       const float* beta, const float* h0, void* o, float* hT, void* stream) {
    return gla::dn_fwd_entry(p, q, k, v, beta, h0, o, hT, nullptr, stream);
}

extern "C" size_t gla_deltanet_saved_bytes(const gla_problem* p) {
    if (gla::dn_check(p) != GLA_OK) return 0;
    return gla::dn_saved_bytes(p);
}

extern "C" gla_status gla_deltanet_fwd_save(const gla_problem* p, const void* q, const void* k, const void* v,
                                            const float* beta, const float* h0, void* o, float* hT, void* saved,
                                            void* stream) {
    return gla::dn_fwd_entry(p, q, k, v, beta, h0, o, hT, saved, stream);
}

extern "C" size_t gla_deltanet_bwd_workspace_bytes(const gla_problem* p) {
    if (gla::dn_check(p) != GLA_OK) return 0;
    return gla::dn_bwd_ws(p, nullptr).bytes;
}

extern "C" gla_status gla_deltanet_bwd(const gla_problem* p, const void* q, const void* k, const void* v,
                                       const float* beta, const float* h0, const void* dO, const float* dhT,
                                       void* dq, void* dk, void* dv, float* dbeta, float* dh0, void* ws,
                                       size_t ws_bytes, void* stream) {
    return gla::dn_bwd_entry(p, q, k, v, beta, h0, dO, dhT, nullptr, dq, dk, dv, dbeta, dh0, ws, ws_bytes, stream);
}

extern "C" gla_status gla_deltanet_bwd_saved(const gla_problem* p, const void* q, const void* k, const void* v,
                                             const float* beta, const float* h0, const void* dO, const float* dhT,
                                             const void* saved, void* dq, void* dk, void* dv, float* dbeta,
                                             float* dh0, void* ws, size_t ws_bytes, void* stream) {
    return gla::dn_bwd_entry(p, q, k, v, beta, h0, dO, dhT, saved, dq, dk, dv, dbeta, dh0, ws, ws_bytes, stream);
}
