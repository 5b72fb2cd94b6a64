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
#include "gla_common.cuh"

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
                                                          float* __restrict__ hT, int L, int Dv, float scale) {
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

        // ---- 4. O = scale (Q S + lower(Q K^T) X), and S += K^T X
        {
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
                      const float* h0, void* o, float* hT, cudaStream_t st) {
    auto kern = k_deltanet_fwd<T, DK>;
    const size_t smem = DnSmem<DK>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p->B * p->H, p->Dv / DN_VT);
    GLA_LAUNCH("deltanet_fwd", st,
               (kern<<<grid, DN_NT, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                static_cast<const T*>(v), beta, h0, static_cast<T*>(o), hT, p->L,
                                                p->Dv, p->scale)));
    return cudaGetLastError();
}

template <typename T>
cudaError_t dn_launch_dk(const gla_problem* p, const void* q, const void* k, const void* v, const float* beta,
                         const float* h0, void* o, float* hT, cudaStream_t st) {
    return p->Dk == 64 ? dn_launch<T, 64>(p, q, k, v, beta, h0, o, hT, st)
                       : dn_launch<T, 128>(p, q, k, v, beta, h0, o, hT, st);
}

bool dn_aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

static_assert(DnSmem<128>::BYTES <= 227 * 1024, "shared memory of the Dk = 128 plan");

}  // namespace
}  // namespace gla

extern "C" gla_status gla_deltanet_fwd(const gla_problem* p, const void* q, const void* k, const void* v,
                                       const float* beta, const float* h0, void* o, float* hT, void* stream) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE) return GLA_ERR_INVALID_ARG;
    if ((p->Dk != 64 && p->Dk != 128) || p->Dv <= 0 || p->Dv % gla::DN_VT != 0 || p->Dv > 4096 ||
        p->chunk != gla::DN_C)
        return GLA_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 2147483647LL) return GLA_ERR_UNSUPPORTED;
    if ((size_t)p->B * p->H == 0) return GLA_OK;
    if (p->L > 0 && (!q || !k || !v || !beta || !o)) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, h0, o, hT};
    for (const void* x : ptrs)
        if (!gla::dn_aligned16(x)) return GLA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = p->io == GLA_BF16 ? gla::dn_launch_dk<__nv_bfloat16>(p, q, k, v, beta, h0, o, hT, st)
                                            : gla::dn_launch_dk<float>(p, q, k, v, beta, h0, o, hT, st);
    return e == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}
