// Chunkwise DeltaNet forward on the tensor cores (tcgen05 / TMEM / TMA), bf16 I/O.
//
// The chunk form of the talk summary "Hardware-Efficient Training of Linear Attention Models",
// sections 22:36 and 31:16 (delta rule with writing strength beta; the WY representation turns
// the product of a chunk's identity-plus-rank-one transitions into matrix products). In the row
// form (state S [Dk, Dv], keys and queries rows), for a 64-token chunk entered with S:
//   T = (I + strict_lower(diag(beta) K K^T))^{-1}      (unit lower triangular)
//   R = diag(beta) (V - K S),   X = T R
//   O = scale (Q S + lower(Q K^T) X)                    (lower keeps the diagonal)
//   S <- S + K^T X
// One CTA per (batch*head, 64-column value slice): the value columns of the state are
// independent, so a CTA walks its head's chunks in order with its [Dk, 64] state slice in tensor
// memory (fp32; the state product accumulates onto it) and a bf16 copy in shared memory as the
// B operand of K S and Q S. Per chunk:
//   1. tcgen05: K K^T and Q K^T (M=64 N=64), K S and Q S (M=64 N=64) into tensor memory;
//   2. CUDA cores: A = diag(beta) K K^T (strict lower) and R in fp32, P = lower(Q K^T) in bf16;
//   3. CUDA cores: X = T R by solving (I + A) X = R in fp32, row by row: once row t of X is
//      final it is subtracted from every later row (A[u][t] X[t] for u > t), so each row's value
//      is ready the moment the row before it is; thread = value column x every 4th row, the
//      rows in registers. X goes to bf16 as the B operand of the next products;
//   4. tcgen05: O = Q S + P X (onto the Q S accumulator), S += K^T X;
//   5. o = scale O (bf16, TMA store), the state's bf16 copy (and, for the backward, the state
//      entering the next chunk in fp32).
// K, Q and V tiles arrive by TMA into a two-stage ring, so the next chunk's loads overlap this
// chunk's work. Every phase runs on all 8 warps in turn; one elected lane of warp 0 issues the
// MMAs and the TMA copies. The backward's reverse walk and its per-chunk gradient kernel follow
// below in the same style.
#include <cudaTypedefs.h>

#include "gla_common.cuh"
#include "gla_plans.h"
#include "gla_tc_common.cuh"

namespace gla {
namespace tc {

using namespace sm100;

namespace {

constexpr int DT_NT = 256;   // 8 warps: two warpgroups
constexpr int DT_VT = 64;    // value columns per CTA
constexpr int DT_TS = 68;    // row stride (floats) of the fp32 A and R tiles (16-byte rows, spread banks)

template <int DK>
struct DtCfg {
    static constexpr uint32_t KB = TR * DK * 2;   // K tile (bf16, 128-byte swizzled 64-column blocks)
    static constexpr uint32_t QB = TR * DK * 2;   // Q tile
    static constexpr uint32_t VB = TR * DT_VT * 2;
    static constexpr uint32_t STAGE = KB + QB + VB;
    static constexpr int NS = 2;
    static constexpr uint32_t SB = DK * DT_VT * 2;        // bf16 state copy (MN-major B: row = key dim)
    static constexpr uint32_t MB = TR * TR * 2;           // one 64 x 64 bf16 operand (P, X, O staging)
    static constexpr uint32_t AF = TR * DT_TS * 4;        // diag(beta) K K^T, fp32 [t][s]
    static constexpr uint32_t RF = TR * DT_TS * 4;        // R, fp32 [t][value column]
    static constexpr uint32_t SMALL = 256 + 4 * TR;
    static constexpr uint32_t SMEM = NS * STAGE + SB + 3 * MB + AF + RF + SMALL + 1024;
    // TMEM columns: the state [0, 64) (M = Dk rows), then two M=64 accumulators, each pair in
    // lanes 0-15 / 16-31 of the same columns: K K^T | Q K^T at 64, K S | Q S (then O) at 128
    static constexpr uint32_t C_S = 0, C_KK = 64, C_KS = 128, NCOL = 256;
    static constexpr int MS = DK == 64 ? 64 : 128;        // M of the state product
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0 && SB % 1024 == 0, "alignment");
};

struct DtArgs {
    const float* beta;   // [BH*L]
    const float* h0;     // [BH, Dk, Dv] or null
    float* hT;           // [BH, Dk, Dv] or null
    __nv_bfloat16* saved;   // [BH, NC, Dk, Dv]: the state entering every chunk (bf16, the precision
                            // the backward's products read it in), or null
    int* status;         // device status word (a wait that gave up), or null
    int L, Dv;
    float scale;
};

__device__ __forceinline__ bool dt_wait(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __syncthreads_and(ok) != 0;
}

// 16 consecutive values to bf16 in global memory (32-byte aligned)
__device__ __forceinline__ void dt_store16_bf16(__nv_bfloat16* dst, const float* v) {
    uint32_t w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
        w[u] = *reinterpret_cast<uint32_t*>(&p);
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// 32 values to bf16 in global memory (64 contiguous bytes)
__device__ __forceinline__ void dt_put_row_bf16(__nv_bfloat16* dst, const float* v) {
    dt_store16_bf16(dst, v);
    dt_store16_bf16(dst + 16, v + 16);
}

// The CTA's [DK, 64] state slice, row `d` (this thread's TMEM lane), 32 columns from `c`: fp32 to
// global memory (saved / hT), 128 contiguous bytes per thread.
__device__ __forceinline__ void dt_put_row(float* dst, const uint32_t* r) {
#pragma unroll
    for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(dst + j) =
            make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                        __uint_as_float(r[j + 3]));
}

template <int DK, bool OUT>
__global__ void __launch_bounds__(DT_NT, 1)
    k_deltanet_tc_fwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, DtArgs A) {
    using C = DtCfg<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_align1024(smem_raw);
    uint8_t* sS = sm + C::NS * C::STAGE;
    uint8_t* sP = sS + C::SB;
    uint8_t* sX = sP + C::MB;
    uint8_t* sO = sX + C::MB;
    float* sA = reinterpret_cast<float*>(sO + C::MB);
    float* sRf = sA + TR * DT_TS;
    uint8_t* small = reinterpret_cast<uint8_t*>(sRf + TR * DT_TS);
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(small);   // [2]
    uint64_t* bar_mma = bar_full + 2;
    uint64_t* bar_drain = bar_full + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + 64);
    float* sB = reinterpret_cast<float*>(small + 256);   // beta of the chunk [64]

    const int bh = blockIdx.x, col0 = blockIdx.y * DT_VT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2, qd = warp & 3;
    const int L = A.L, Dv = A.Dv;
    const int nc = (L + TR - 1) / TR;
    const long rowbase = (long)bh * L;
    // state rows: this thread's TMEM lane holds key dim srow (M=64 state: lanes 0-15 only)
    const bool srow_ok = DK != 64 || lane < 16;
    const int srow = DK == 64 ? 16 * qd + (lane & 15) : 32 * qd + lane;
    // M=64 accumulators: lane l < 16 holds row 16 qd + l of the first, l >= 16 of the second
    const int mrow = 16 * qd + (lane & 15);
    const bool first = lane < 16;

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_drain, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, C::NCOL);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tq_lane = tbase + ((uint32_t)(32 * qd) << 16);

    auto issue_loads = [&](int c, int s) {
        uint8_t* st = sm + s * C::STAGE;
        const int t0 = c * TR;
        mbar_arrive_expect_tx(&bar_full[s], OUT ? C::STAGE : C::KB + C::VB);
        for (int cb = 0; cb < DK / 64; ++cb) {
            tma_load_3d(st + cb * BLK, &tk, cb * 64, t0, bh, &bar_full[s]);
            if (OUT) tma_load_3d(st + C::KB + cb * BLK, &tq, cb * 64, t0, bh, &bar_full[s]);
        }
        tma_load_3d(st + C::KB + C::QB, &tv, col0, t0, bh, &bar_full[s]);
    };
    if (tid == 0)
        for (int c = 0; c < C::NS && c < nc; ++c) issue_loads(c, c);

    // ---- the initial state: TMEM (fp32), its bf16 copy, and the state entering chunk 0
    {
        const float* src = A.h0 ? A.h0 + ((long)bh * DK + srow) * Dv + col0 : nullptr;
        const int c = 32 * wg;
        float f[32];
        if (src && srow_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = *reinterpret_cast<const float4*>(src + c + j);
                f[j] = x.x; f[j + 1] = x.y; f[j + 2] = x.z; f[j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = 0.f;
        }
        tmem_st32(tq_lane + C::C_S + c, reinterpret_cast<uint32_t*>(f));
        if (srow_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) store8_bf16(sS, sw128_off(srow, c + j, DK * 128), f + j);
            if (A.saved && nc > 0) dt_put_row_bf16(A.saved + (((long)bh * nc) * DK + srow) * Dv + col0 + c, f);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    int err = 0, n_mma = 0;
    for (int c = 0; c < nc; ++c) {
        const int s = c % C::NS;
        uint8_t* sk = sm + s * C::STAGE;
        uint8_t* sq = sk + C::KB;
        uint8_t* sv = sq + C::QB;
        const int t0 = c * TR;
        if (tid < TR) sB[tid] = t0 + tid < L ? A.beta[rowbase + t0 + tid] : 0.f;
        if (!dt_wait(&bar_full[s], (c / C::NS) & 1)) { err = 1; break; }

        // ---- 1. K K^T, Q K^T, K S, Q S
        if (warp == 0) {
            const bool leader = elect_one();
            tc_fence_after();
            const uint32_t ka = smem_u32(sk), qa = smem_u32(sq);
            const uint32_t idAA = idesc_bf16(64, 64, 0, 0), idAS = idesc_bf16(64, DT_VT, 0, 1);
            const uint64_t dS = sw128_desc(smem_u32(sS), DK * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader) {
                    mma_bf16(tbase + C::C_KK, sw128_desc(ka + koff, 16, 1024), sw128_desc(ka + koff, 16, 1024), idAA,
                             kk > 0);
                    mma_bf16(tbase + C::C_KS, sw128_desc(ka + koff, 16, 1024), dS + ((kk * 2048) >> 4), idAS, kk > 0);
                    if (OUT) {
                        mma_bf16(tbase + C::C_KK + (16u << 16), sw128_desc(qa + koff, 16, 1024),
                                 sw128_desc(ka + koff, 16, 1024), idAA, kk > 0);
                        mma_bf16(tbase + C::C_KS + (16u << 16), sw128_desc(qa + koff, 16, 1024), dS + ((kk * 2048) >> 4),
                                 idAS, kk > 0);
                    }
                }
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }
        tc_fence_after();

        // ---- 2a. A = diag(beta) K K^T (strict lower, fp32) and P = lower(Q K^T) (bf16): one TMEM
        //      read, K K^T rows in lanes 0-15, Q K^T rows in lanes 16-31; 32 columns per warpgroup
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_KK + 32 * wg, r);
            tmem_wait_ld();
            const int t = mrow;
            if (first) {
                const float bt = sB[t];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int sc = 32 * wg + j;
                    *reinterpret_cast<float4*>(sA + t * DT_TS + sc) =
                        make_float4(sc < t ? bt * __uint_as_float(r[j]) : 0.f, sc + 1 < t ? bt * __uint_as_float(r[j + 1]) : 0.f,
                                    sc + 2 < t ? bt * __uint_as_float(r[j + 2]) : 0.f,
                                    sc + 3 < t ? bt * __uint_as_float(r[j + 3]) : 0.f);
                }
            } else if (OUT) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int sc = 32 * wg + 8 * u + j;
                        f[j] = sc <= t ? __uint_as_float(r[8 * u + j]) : 0.f;
                    }
                    store8_bf16(sP, sw128_off(t, 32 * wg + 8 * u, BLK), f);
                }
            }
        }
        // ---- 2b. R = diag(beta) (V - K S), fp32 [t][value column]
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_KS + 32 * wg, r);
            tmem_wait_ld();
            if (first) {
                const int t = mrow;
                const float bt = sB[t];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int cc = 32 * wg + 8 * u;
                    const uint4 vw = *reinterpret_cast<const uint4*>(sv + sw128_off(t, cc, BLK));
                    const uint32_t* vp = reinterpret_cast<const uint32_t*>(&vw);
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vp[j]));
                        f[2 * j] = bt * (vf.x - __uint_as_float(r[8 * u + 2 * j]));
                        f[2 * j + 1] = bt * (vf.y - __uint_as_float(r[8 * u + 2 * j + 1]));
                    }
                    *reinterpret_cast<float4*>(sRf + t * DT_TS + cc) = make_float4(f[0], f[1], f[2], f[3]);
                    *reinterpret_cast<float4*>(sRf + t * DT_TS + cc + 4) = make_float4(f[4], f[5], f[6], f[7]);
                }
            }
        }
        __syncthreads();

        // ---- 3. X = (I + A)^{-1} R in fp32: thread = value column j x rows u = 4 m + sp (m = 0..15),
        //      their values in registers; row t, once final, is broadcast from its owner and
        //      subtracted from the thread's later rows. A is read four columns at a time.
        {
            const int j = warp * 8 + (lane >> 2), sp = lane & 3;
            float x[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) x[m] = sRf[(4 * m + sp) * DT_TS + j];
#pragma unroll
            for (int t4 = 0; t4 < TR; t4 += 4) {
                float4 a[16];   // A[u][t4 .. t4 + 3] of the thread's rows u >= t4
#pragma unroll
                for (int m = t4 / 4; m < 16; ++m) a[m] = *reinterpret_cast<const float4*>(sA + (4 * m + sp) * DT_TS + t4);
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const int t = t4 + tt;
                    const float xt = __shfl_sync(0xffffffffu, x[t >> 2], (lane & ~3) | (t & 3));
#pragma unroll
                    for (int m = t4 / 4; m < 16; ++m) {
                        const float at = tt == 0 ? a[m].x : tt == 1 ? a[m].y : tt == 2 ? a[m].z : a[m].w;
                        if (4 * m + sp > t) x[m] = fmaf(-at, xt, x[m]);
                    }
                }
            }
            // X to bf16, laid out like a V tile (the B operand of P X and K^T X)
#pragma unroll
            for (int m = 0; m < 16; ++m)
                *reinterpret_cast<__nv_bfloat16*>(sX + sw128_off(4 * m + sp, j, BLK)) = __float2bfloat16_rn(x[m]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- 4. O = Q S + P X, S += K^T X
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t idO = idesc_bf16(64, DT_VT, 0, 1), idS = idesc_bf16(C::MS, DT_VT, 1, 1);
            const uint64_t dP = sw128_desc(smem_u32(sP), 16, 1024), dX = sw128_desc(smem_u32(sX), BLK, 1024);
            const uint64_t dKm = sw128_desc(smem_u32(sk), BLK, 1024);
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks) {
                if (leader && OUT)
                    mma_bf16(tbase + C::C_KS + (16u << 16), dP + ((ks * 32) >> 4), dX + ((ks * 2048) >> 4), idO, 1);
                if (leader) mma_bf16(tbase + C::C_S, dKm + ((ks * 2048) >> 4), dX + ((ks * 2048) >> 4), idS, 1);
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }
        tc_fence_after();

        // ---- 5. o = scale O (bf16 tile -> TMA store); the state's bf16 copy and the state entering
        //      the next chunk
        if (OUT) {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_KS + 32 * wg, r);
            tmem_wait_ld();
            if (!first) {
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) f[j] = A.scale * __uint_as_float(r[j]);
#pragma unroll
                for (int u = 0; u < 4; ++u) store8_bf16(sO, sw128_off(mrow, 32 * wg + 8 * u, BLK), f + 8 * u);
            }
        }
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_S + 32 * wg, r);
            tmem_wait_ld();
            if (srow_ok) {
#pragma unroll
                for (int j = 0; j < 32; j += 8)
                    store8_bf16(sS, sw128_off(srow, 32 * wg + j, DK * 128), reinterpret_cast<const float*>(r + j));
                if (A.saved && c + 1 < nc)
                    dt_put_row_bf16(A.saved + (((long)bh * nc + c + 1) * DK + srow) * Dv + col0 + 32 * wg,
                                    reinterpret_cast<const float*>(r));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            if (OUT) {
                tma_store_3d(&to, sO, col0, t0, bh);
                bulk_commit();
            }
            // every product that read this stage is done: the chunk after next may take it
            if (c + C::NS < nc) issue_loads(c + C::NS, s);
            if (OUT) bulk_wait_read<0>();   // the o tile is read before the next chunk rewrites it
        }
    }

    if (err) {
        if (warp == 0) {
            // every product the issuing lane issued completes before TMEM and shared memory go away
            const bool leader = elect_one();
            if (leader) {
                if (A.status) atomicOr(A.status, kDevStatusTimeout);
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0, 1u << 20);
            }
            __syncwarp();
        }
    } else if (A.hT) {
        uint32_t r[32];
        tmem_ld32(tq_lane + C::C_S + 32 * wg, r);
        tmem_wait_ld();
        if (srow_ok) dt_put_row(A.hT + ((long)bh * DK + srow) * Dv + col0 + 32 * wg, r);
    }
    if (tid == 0) bulk_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, C::NCOL);
}

template <int DK, bool OUT>
cudaError_t dt_launch(int B, int H, int L, int Dv, const CUtensorMap& mq, const CUtensorMap& mk,
                      const CUtensorMap& mv, const CUtensorMap& mo, const DtArgs& a, cudaStream_t st) {
    auto kern = k_deltanet_tc_fwd<DK, OUT>;
    const uint32_t smem = DtCfg<DK>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(B * H, Dv / DT_VT);
    GLA_LAUNCH(OUT ? "deltanet_fwd" : "deltanet_state", st, (kern<<<grid, DT_NT, smem, st>>>(mq, mk, mv, mo, a)));
    return cudaGetLastError();
}

// ------------------------------------------------------------------ backward walk
// With U = V - K S, R = diag(beta) U, X = T R, P = lower(Q K^T) and dS' the gradient reaching the
// chunk's end state, a chunk's reverse step is
//   dX = scale P^T dO + K dS',   dR = T^T dX,   dV = diag(beta) dR,
//   dS = dS' + scale Q^T dO - K^T diag(beta) dR       (the gradient at the chunk's start).
// Only dS carries across chunks, and none of it needs S, X or U: those belong to the gradient
// kernel below, which runs all chunks in parallel. One CTA per (batch*head, 64-column value
// slice) walks the chunks in reverse with its dS slice in tensor memory. Per chunk:
//   1. q is scaled in place (so that Q K^T and Q^T dO carry the output scale); tcgen05: K K^T,
//      Q K^T, K dS';
//   2. A^T = strict_lower(diag(beta) K K^T)^T (fp32) and P = lower(Q K^T) (bf16); tcgen05:
//      dX = K dS' + P^T dO (onto the K dS' accumulator; P read as an MN-major A operand);
//   3. dR = (I + A)^{-T} dX: a right-looking substitution in fp32 from the last row (thread =
//      value column x every fourth row, the rows in registers; once row u is final it is
//      broadcast and A[u][t] dR[u] subtracted from every earlier row t);
//   4. dR (fp32) and dV = diag(beta) dR to global memory, -diag(beta) dR as a bf16 operand;
//   5. tcgen05: dS += Q^T dO + K^T (-diag(beta) dR); its bf16 copy for the next chunk, and the
//      gradient at the next chunk's end (bf16, for the gradient kernel).
template <int DK>
struct DwCfg {
    static constexpr uint32_t KB = TR * DK * 2, QB = TR * DK * 2, OB = TR * DT_VT * 2;
    static constexpr uint32_t STAGE = KB + QB + OB;
    static constexpr int NS = 2;
    static constexpr uint32_t GB = DK * DT_VT * 2;   // bf16 copy of dS'
    static constexpr uint32_t MB = TR * TR * 2;      // P; -diag(beta) dR
    static constexpr uint32_t F = TR * DT_TS * 4;    // fp32 tiles: A^T, W (dX, then dR)
    static constexpr uint32_t SMALL = 256 + 4 * TR;
    static constexpr uint32_t SMEM = NS * STAGE + GB + 2 * MB + 2 * F + SMALL + 1024;
    static constexpr uint32_t C_S = 0, C_KK = 64, C_KD = 128, NCOL = 256;
    static constexpr int MS = DK == 64 ? 64 : 128;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0 && GB % 1024 == 0, "alignment");
};

struct DwArgs {
    const float* beta;      // [BH*L]
    const float* dhT;       // [BH, Dk, Dv] or null
    float* drw;             // [BH*L, Dv] dR
    __nv_bfloat16* dsend;   // [BH, NC, Dk, Dv] the gradient at every chunk's end
    __nv_bfloat16* dv;      // [BH*L, Dv]
    float* dh0;             // [BH, Dk, Dv] or null
    int BH, L, Dv;
    float scale;
};

template <int DK>
__global__ void __launch_bounds__(DT_NT, 1)
    k_deltanet_tc_walk(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tdo, DwArgs A) {
    using C = DwCfg<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_align1024(smem_raw);
    uint8_t* sG = sm + C::NS * C::STAGE;
    uint8_t* sP = sG + C::GB;
    uint8_t* sBR = sP + C::MB;
    float* sAT = reinterpret_cast<float*>(sBR + C::MB);
    float* sW = sAT + TR * DT_TS;
    uint8_t* small = reinterpret_cast<uint8_t*>(sW + TR * DT_TS);
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(small);   // [2]
    uint64_t* bar_mma = bar_full + 2;
    uint64_t* bar_drain = bar_full + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + 64);
    float* sB = reinterpret_cast<float*>(small + 256);

    const int bh = blockIdx.x, col0 = blockIdx.y * DT_VT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2, qd = warp & 3;
    const int L = A.L, Dv = A.Dv;
    const int nc = (L + TR - 1) / TR;
    const long rowbase = (long)bh * L;
    const bool srow_ok = DK != 64 || lane < 16;
    const int srow = DK == 64 ? 16 * qd + (lane & 15) : 32 * qd + lane;
    const int mrow = 16 * qd + (lane & 15);
    const bool first = lane < 16;
    const int sj = warp * 8 + (lane >> 2), sp = lane & 3;   // substitution: value column, row phase
    const int rt = tid >> 2, rc = 16 * (tid & 3);           // row pass: token row, 16 value columns

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_drain, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, C::NCOL);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tq_lane = tbase + ((uint32_t)(32 * qd) << 16);

    auto chunk_at = [&](int i) { return nc - 1 - i; };
    auto issue_loads = [&](int i, int s) {
        uint8_t* st = sm + s * C::STAGE;
        const int t0 = chunk_at(i) * TR;
        mbar_arrive_expect_tx(&bar_full[s], C::STAGE);
        for (int cb = 0; cb < DK / 64; ++cb) {
            tma_load_3d(st + cb * BLK, &tk, cb * 64, t0, bh, &bar_full[s]);
            tma_load_3d(st + C::KB + cb * BLK, &tq, cb * 64, t0, bh, &bar_full[s]);
        }
        tma_load_3d(st + C::KB + C::QB, &tdo, col0, t0, bh, &bar_full[s]);
    };
    if (tid == 0)
        for (int i = 0; i < C::NS && i < nc; ++i) issue_loads(i, i);

    // ---- dS' at the sequence's end (dhT or zero): TMEM and its bf16 copy
    {
        const float* src = A.dhT ? A.dhT + ((long)bh * DK + srow) * Dv + col0 : nullptr;
        const int c = 32 * wg;
        float f[32];
        if (src && srow_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = *reinterpret_cast<const float4*>(src + c + j);
                f[j] = x.x; f[j + 1] = x.y; f[j + 2] = x.z; f[j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = 0.f;
        }
        tmem_st32(tq_lane + C::C_S + c, reinterpret_cast<uint32_t*>(f));
        if (srow_ok)
#pragma unroll
            for (int j = 0; j < 32; j += 8) store8_bf16(sG, sw128_off(srow, c + j, DK * 128), f + j);
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    int err = 0, n_mma = 0;
    for (int i = 0; i < nc; ++i) {
        const int s = i % C::NS, ci = chunk_at(i), t0 = ci * TR;
        uint8_t* sk = sm + s * C::STAGE;
        uint8_t* sq = sk + C::KB;
        uint8_t* sdo = sq + C::QB;
        const long cbase = (long)bh * nc + ci;
        if (tid < TR) sB[tid] = t0 + tid < L ? A.beta[rowbase + t0 + tid] : 0.f;
        // the gradient at this chunk's end, for the gradient kernel (its bf16 copy is in sG)
        if (srow_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 8)
                *reinterpret_cast<uint4*>(A.dsend + (cbase * DK + srow) * Dv + col0 + 32 * wg + j) =
                    *reinterpret_cast<const uint4*>(sG + sw128_off(srow, 32 * wg + j, DK * 128));
        }
        if (!dt_wait(&bar_full[s], (i / C::NS) & 1)) { err = 1; break; }
        // q scaled in place (bf16, layout-blind 16-byte chunks)
        for (int e = tid; e < (int)(C::QB / 16); e += DT_NT) {
            uint4 w = *reinterpret_cast<uint4*>(sq + 16 * e);
            uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pw[u]));
                __nv_bfloat162 h = __floats2bfloat162_rn(f.x * A.scale, f.y * A.scale);
                pw[u] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(sq + 16 * e) = w;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- 1. K K^T | Q K^T, K dS'
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t ka = smem_u32(sk), qa = smem_u32(sq);
            const uint32_t idAA = idesc_bf16(64, 64, 0, 0), idAS = idesc_bf16(64, DT_VT, 0, 1);
            const uint64_t dG = sw128_desc(smem_u32(sG), DK * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader) {
                    mma_bf16(tbase + C::C_KK, sw128_desc(ka + koff, 16, 1024), sw128_desc(ka + koff, 16, 1024), idAA,
                             kk > 0);
                    mma_bf16(tbase + C::C_KK + (16u << 16), sw128_desc(qa + koff, 16, 1024),
                             sw128_desc(ka + koff, 16, 1024), idAA, kk > 0);
                    mma_bf16(tbase + C::C_KD, sw128_desc(ka + koff, 16, 1024), dG + ((kk * 2048) >> 4), idAS, kk > 0);
                }
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }
        tc_fence_after();

        // ---- 2. A^T (fp32) and P (bf16); dX = K dS' + P^T dO
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_KK + 32 * wg, r);
            tmem_wait_ld();
            const int t = mrow;
            if (first) {
                const float bt = sB[t];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int sc = 32 * wg + j;
                    sAT[sc * DT_TS + t] = sc < t ? bt * __uint_as_float(r[j]) : 0.f;
                }
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int sc = 32 * wg + 8 * u + j;
                        f[j] = sc <= t ? __uint_as_float(r[8 * u + j]) : 0.f;
                    }
                    store8_bf16(sP, sw128_off(t, 32 * wg + 8 * u, BLK), f);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t idX = idesc_bf16(64, DT_VT, 1, 1);
            const uint64_t dPt = sw128_desc(smem_u32(sP), BLK, 1024), dO = sw128_desc(smem_u32(sdo), BLK, 1024);
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks)
                if (leader) mma_bf16(tbase + C::C_KD, dPt + ((ks * 2048) >> 4), dO + ((ks * 2048) >> 4), idX, 1);
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }
        tc_fence_after();
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_KD + 32 * wg, r);
            tmem_wait_ld();
            if (first)
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4*>(sW + mrow * DT_TS + 32 * wg + j) =
                        make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                    __uint_as_float(r[j + 3]));
        }
        __syncthreads();

        // ---- 3. dR = (I + A)^{-T} dX, rows from the last; A^T read four columns at a time
        {
            float x[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) x[m] = sW[(4 * m + sp) * DT_TS + sj];
#pragma unroll
            for (int u4 = TR - 4; u4 >= 0; u4 -= 4) {
                float4 a[16];
#pragma unroll
                for (int m = 0; m <= u4 / 4; ++m) a[m] = *reinterpret_cast<const float4*>(sAT + (4 * m + sp) * DT_TS + u4);
#pragma unroll
                for (int uu = 3; uu >= 0; --uu) {
                    const int u = u4 + uu;
                    const float xu = __shfl_sync(0xffffffffu, x[u >> 2], (lane & ~3) | (u & 3));
#pragma unroll
                    for (int m = 0; m <= u4 / 4; ++m) {
                        const float at = uu == 0 ? a[m].x : uu == 1 ? a[m].y : uu == 2 ? a[m].z : a[m].w;
                        if (4 * m + sp < u) x[m] = fmaf(-at, xu, x[m]);
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int m = 0; m < 16; ++m) sW[(4 * m + sp) * DT_TS + sj] = x[m];
        }
        __syncthreads();

        // ---- 4. dR and dV = diag(beta) dR to global memory, -diag(beta) dR (bf16)
        {
            const float bt = sB[rt];
            float dr[16];
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                const float4 x = *reinterpret_cast<const float4*>(sW + rt * DT_TS + rc + j);
                dr[j] = x.x; dr[j + 1] = x.y; dr[j + 2] = x.z; dr[j + 3] = x.w;
            }
            if (t0 + rt < L) {
                const long row = rowbase + t0 + rt;
                float* dst = A.drw + row * Dv + col0 + rc;
#pragma unroll
                for (int j = 0; j < 16; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(dr[j], dr[j + 1], dr[j + 2], dr[j + 3]);
                float bv[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) bv[j] = bt * dr[j];
                dt_store16_bf16(A.dv + row * Dv + col0 + rc, bv);
            }
            float nb[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) nb[j] = -bt * dr[j];
            store8_bf16(sBR, sw128_off(rt, rc, BLK), nb);
            store8_bf16(sBR, sw128_off(rt, rc + 8, BLK), nb + 8);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- 5. dS += Q^T dO + K^T (-diag(beta) dR)
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t idS = idesc_bf16(C::MS, DT_VT, 1, 1);
            const uint64_t dQm = sw128_desc(smem_u32(sq), BLK, 1024), dKm = sw128_desc(smem_u32(sk), BLK, 1024);
            const uint64_t dO = sw128_desc(smem_u32(sdo), BLK, 1024), dB = sw128_desc(smem_u32(sBR), BLK, 1024);
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks) {
                if (leader) {
                    mma_bf16(tbase + C::C_S, dQm + ((ks * 2048) >> 4), dO + ((ks * 2048) >> 4), idS, 1);
                    mma_bf16(tbase + C::C_S, dKm + ((ks * 2048) >> 4), dB + ((ks * 2048) >> 4), idS, 1);
                }
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }
        tc_fence_after();
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_S + 32 * wg, r);
            tmem_wait_ld();
            if (srow_ok)
#pragma unroll
                for (int j = 0; j < 32; j += 8)
                    store8_bf16(sG, sw128_off(srow, 32 * wg + j, DK * 128), reinterpret_cast<const float*>(r + j));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && i + C::NS < nc) issue_loads(i + C::NS, s);
    }

    if (err) {
        if (warp == 0) {
            const bool leader = elect_one();
            if (leader) {
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0, 1u << 20);
            }
            __syncwarp();
        }
    } else if (A.dh0) {
        uint32_t r[32];
        tmem_ld32(tq_lane + C::C_S + 32 * wg, r);
        tmem_wait_ld();
        if (srow_ok) dt_put_row(A.dh0 + ((long)bh * DK + srow) * Dv + col0 + 32 * wg, r);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, C::NCOL);
}

template <int DK>
cudaError_t dw_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mdo, const DwArgs& a,
                      cudaStream_t st) {
    auto kern = k_deltanet_tc_walk<DK>;
    const uint32_t smem = DwCfg<DK>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.BH, a.Dv / DT_VT);
    GLA_LAUNCH("deltanet_bwd_walk", st, (kern<<<grid, DT_NT, smem, st>>>(mq, mk, mdo, a)));
    return cudaGetLastError();
}

// ------------------------------------------------------------------ backward gradients
// Per chunk, all chunks in parallel, from the chunk's start state S (saved by the forward's state
// walk, bf16), the gradient at its end dS' and dR (both from the reverse walk), value columns in
// 64-wide slices summed in tensor memory:
//   A = strict_lower(diag(beta) K K^T),  U = V - K S,  X = (I + A)^{-1} diag(beta) U
//   dP = scale lower(dO X^T),  G = -strict_lower(dR X^T)
//   dQ = scale dO S^T + dP K
//   dK = X dS'^T - diag(beta) dR S^T + dP^T Q + diag(beta) (G K) + G^T diag(beta) K
//   dbeta_t = sum_j dR_tj U_tj + sum_i k_ti (G K)_ti
// One CTA per (chunk, batch*head). dO is scaled in place, so dO X^T and dO S^T carry the scale.
// X comes from the forward's substitution (fp32, rows in registers), once per value slice.
template <int DK>
struct DgCfg {
    static constexpr uint32_t KB = TR * DK * 2;      // K, Q (TMA), diag(beta) K
    static constexpr uint32_t MB = TR * TR * 2;      // 64 x 64 bf16: dO, V, X, dR, -diag(beta) dR, dP, G
    static constexpr uint32_t SB = DK * DT_VT * 2;   // S and dS' slices, bf16, rows of key dims
    static constexpr uint32_t F = TR * DT_TS * 4;    // fp32: A, U, R (then X)
    static constexpr uint32_t SMALL = 256 + 4 * TR + 8 * TR + 4 * TR;
    static constexpr uint32_t SMEM = 3 * KB + 7 * MB + 2 * SB + 3 * F + SMALL + 1024;
    // TMEM: dO X^T | dR X^T (lanes 0-15 | 16-31) at 0; dQ | dK at 64; G K (lanes 16-31) at
    // 64 + DK; K K^T at 64 + 2 DK; K S at 128 + 2 DK
    static constexpr uint32_t C_PG = 0, C_QK = 64, C_GK = 64 + DK, C_KK = 64 + 2 * DK, C_KS = 128 + 2 * DK;
    static constexpr uint32_t NCOL = 512;
    static_assert(C_KS + 64 <= NCOL, "tensor memory");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct DgArgs {
    const float* beta;            // [BH*L]
    const __nv_bfloat16* saved;   // [BH, NC, Dk, Dv] the state entering every chunk
    const float* drw;             // [BH*L, Dv]
    const __nv_bfloat16* dsend;   // [BH, NC, Dk, Dv] the gradient at every chunk's end
    __nv_bfloat16* dq;            // [BH*L, Dk]
    __nv_bfloat16* dk;
    float* dbeta;                 // [BH*L]
    int BH, L, Dv;
    float scale;
};

template <int DK>
__global__ void __launch_bounds__(DT_NT, 1)
    k_deltanet_tc_grads(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, DgArgs A) {
    using C = DgCfg<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_align1024(smem_raw);
    uint8_t* sK = sm;
    uint8_t* sQ = sK + C::KB;
    uint8_t* sBK = sQ + C::KB;      // diag(beta) K
    uint8_t* sDO = sBK + C::KB;
    uint8_t* sV = sDO + C::MB;
    uint8_t* sX = sV + C::MB;
    uint8_t* sDR = sX + C::MB;
    uint8_t* sNB = sDR + C::MB;     // -diag(beta) dR
    uint8_t* sDP = sNB + C::MB;
    uint8_t* sGm = sDP + C::MB;
    uint8_t* sSb = sGm + C::MB;
    uint8_t* sDS = sSb + C::SB;
    float* sAf = reinterpret_cast<float*>(sDS + C::SB);
    float* sU = sAf + TR * DT_TS;
    float* sRf = sU + TR * DT_TS;
    uint8_t* small = reinterpret_cast<uint8_t*>(sRf + TR * DT_TS);
    uint64_t* bar_kq = reinterpret_cast<uint64_t*>(small);
    uint64_t* bar_do = bar_kq + 1;
    uint64_t* bar_mma = bar_kq + 2;
    uint64_t* bar_drain = bar_kq + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + 64);
    float* sB = reinterpret_cast<float*>(small + 256);      // beta [64]
    float* sDB = sB + TR;                                   // [2][64] partial sums of k . (G K)
    float* sDU = sDB + 2 * TR;                              // [64] sum_j dR U over the slices

    const int ci = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2, qd = warp & 3;
    const int L = A.L, Dv = A.Dv, nsl = Dv / DT_VT;
    const int nc = (L + TR - 1) / TR, t0 = ci * TR;
    const long rowbase = (long)bh * L;
    const long cbase = (long)bh * nc + ci;
    const int mrow = 16 * qd + (lane & 15);
    const bool first = lane < 16;
    const int rt = tid >> 2, rc = 16 * (tid & 3);           // row pass: token row, 16 value columns
    const int sj = warp * 8 + (lane >> 2), sp = lane & 3;   // substitution: value column, row phase

    if (tid == 0) {
        mbar_init(bar_kq, 1);
        mbar_init(bar_do, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_drain, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, C::NCOL);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tq_lane = tbase + ((uint32_t)(32 * qd) << 16);
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_kq, 2 * C::KB);
        for (int cb = 0; cb < DK / 64; ++cb) {
            tma_load_3d(sK + cb * BLK, &tk, cb * 64, t0, bh, bar_kq);
            tma_load_3d(sQ + cb * BLK, &tq, cb * 64, t0, bh, bar_kq);
        }
    }
    if (tid < TR) {
        sB[tid] = t0 + tid < L ? A.beta[rowbase + t0 + tid] : 0.f;
        sDU[tid] = 0.f;
    }
    int err = 0, n_mma = 0, n_do = 0;
    // ---- K K^T, then A (fp32)
    if (!dt_wait(bar_kq, 0)) err = 1;
    if (!err) {
        if (warp == 0) {
            const bool leader = elect_one();
            tc_fence_after();
            const uint32_t ka = smem_u32(sK);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader)
                    mma_bf16(tbase + C::C_KK, sw128_desc(ka + koff, 16, 1024), sw128_desc(ka + koff, 16, 1024),
                             idesc_bf16(64, 64, 0, 0), kk > 0);
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) err = 1;
    }
    if (!err) {
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(tq_lane + C::C_KK + 32 * wg, r);
        tmem_wait_ld();
        if (first) {
            const int t = mrow;
            const float bt = sB[t];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const int sc = 32 * wg + j;
                *reinterpret_cast<float4*>(sAf + t * DT_TS + sc) =
                    make_float4(sc < t ? bt * __uint_as_float(r[j]) : 0.f, sc + 1 < t ? bt * __uint_as_float(r[j + 1]) : 0.f,
                                sc + 2 < t ? bt * __uint_as_float(r[j + 2]) : 0.f,
                                sc + 3 < t ? bt * __uint_as_float(r[j + 3]) : 0.f);
            }
        }
    }

    for (int sl = 0; sl < nsl && !err; ++sl) {
        const int col0 = sl * DT_VT;
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_do, 2 * C::MB);
            tma_load_3d(sDO, &tdo, col0, t0, bh, bar_do);
            tma_load_3d(sV, &tv, col0, t0, bh, bar_do);
        }
        // S and dS' slices (bf16, rows of key dims), copied as they are
        {
            constexpr int TPR = DT_NT / DK, CPT = DT_VT / TPR;   // threads per key row, columns per thread
            const int kr = tid / TPR, kc = (tid % TPR) * CPT;
            const long off = (cbase * DK + kr) * Dv + col0 + kc;
#pragma unroll
            for (int j = 0; j < CPT; j += 8) {
                *reinterpret_cast<uint4*>(sSb + sw128_off(kr, kc + j, BLK)) = __ldg(reinterpret_cast<const uint4*>(A.saved + off + j));
                *reinterpret_cast<uint4*>(sDS + sw128_off(kr, kc + j, BLK)) = __ldg(reinterpret_cast<const uint4*>(A.dsend + off + j));
            }
        }
        ++n_do;
        if (!dt_wait(bar_do, (n_do - 1) & 1)) { err = 1; break; }
        // dO scaled in place (the output scale of dO X^T and dO S^T)
        for (int e = tid; e < (int)(C::MB / 16); e += DT_NT) {
            uint4 w = *reinterpret_cast<uint4*>(sDO + 16 * e);
            uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pw[u]));
                __nv_bfloat162 h = __floats2bfloat162_rn(f.x * A.scale, f.y * A.scale);
                pw[u] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(sDO + 16 * e) = w;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // K S (the slice's S as an MN-major B operand)
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t ka = smem_u32(sK);
            const uint64_t dS = sw128_desc(smem_u32(sSb), DK * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader)
                    mma_bf16(tbase + C::C_KS, sw128_desc(ka + koff, 16, 1024), dS + ((kk * 2048) >> 4),
                             idesc_bf16(64, DT_VT, 0, 1), kk > 0);
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }
        tc_fence_after();
        // U = V - K S and R = diag(beta) U (fp32)
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_KS + 32 * wg, r);
            tmem_wait_ld();
            if (first) {
                const int t = mrow;
                const float bt = sB[t];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int cc = 32 * wg + 8 * u;
                    const uint4 vw = *reinterpret_cast<const uint4*>(sV + sw128_off(t, cc, BLK));
                    const uint32_t* vp = reinterpret_cast<const uint32_t*>(&vw);
                    float uu[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vp[j]));
                        uu[2 * j] = vf.x - __uint_as_float(r[8 * u + 2 * j]);
                        uu[2 * j + 1] = vf.y - __uint_as_float(r[8 * u + 2 * j + 1]);
                    }
                    *reinterpret_cast<float4*>(sU + t * DT_TS + cc) = make_float4(uu[0], uu[1], uu[2], uu[3]);
                    *reinterpret_cast<float4*>(sU + t * DT_TS + cc + 4) = make_float4(uu[4], uu[5], uu[6], uu[7]);
                    *reinterpret_cast<float4*>(sRf + t * DT_TS + cc) = make_float4(bt * uu[0], bt * uu[1], bt * uu[2], bt * uu[3]);
                    *reinterpret_cast<float4*>(sRf + t * DT_TS + cc + 4) =
                        make_float4(bt * uu[4], bt * uu[5], bt * uu[6], bt * uu[7]);
                }
            }
        }
        __syncthreads();
        // dR (fp32 from the walk): its bf16 operands, and sum_j dR U
        {
            const bool in = t0 + rt < L;
            const long off = (rowbase + t0 + rt) * Dv + col0 + rc;
            const float bt = sB[rt];
            float d[16], nb[16], acc = 0.f;
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                const float4 b = in ? __ldg(reinterpret_cast<const float4*>(A.drw + off + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 u4 = *reinterpret_cast<const float4*>(sU + rt * DT_TS + rc + j);
                d[j] = b.x; d[j + 1] = b.y; d[j + 2] = b.z; d[j + 3] = b.w;
                acc += b.x * u4.x + b.y * u4.y + b.z * u4.z + b.w * u4.w;
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if ((tid & 3) == 0) sDU[rt] += acc;
#pragma unroll
            for (int j = 0; j < 16; ++j) nb[j] = -bt * d[j];
            store8_bf16(sDR, sw128_off(rt, rc, BLK), d);
            store8_bf16(sDR, sw128_off(rt, rc + 8, BLK), d + 8);
            store8_bf16(sNB, sw128_off(rt, rc, BLK), nb);
            store8_bf16(sNB, sw128_off(rt, rc + 8, BLK), nb + 8);
        }
        // X = (I + A)^{-1} R, as in the forward; X to bf16
        {
            float x[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) x[m] = sRf[(4 * m + sp) * DT_TS + sj];
#pragma unroll
            for (int t4 = 0; t4 < TR; t4 += 4) {
                float4 a[16];
#pragma unroll
                for (int m = t4 / 4; m < 16; ++m) a[m] = *reinterpret_cast<const float4*>(sAf + (4 * m + sp) * DT_TS + t4);
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const int t = t4 + tt;
                    const float xt = __shfl_sync(0xffffffffu, x[t >> 2], (lane & ~3) | (t & 3));
#pragma unroll
                    for (int m = t4 / 4; m < 16; ++m) {
                        const float at = tt == 0 ? a[m].x : tt == 1 ? a[m].y : tt == 2 ? a[m].z : a[m].w;
                        if (4 * m + sp > t) x[m] = fmaf(-at, xt, x[m]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m)
                *reinterpret_cast<__nv_bfloat16*>(sX + sw128_off(4 * m + sp, sj, BLK)) = __float2bfloat16_rn(x[m]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t id64 = idesc_bf16(64, 64, 0, 0), idK = idesc_bf16(64, DK, 0, 0);
            const uint32_t a_do = smem_u32(sDO), a_x = smem_u32(sX), a_dr = smem_u32(sDR), a_nb = smem_u32(sNB);
            const uint32_t b_s = smem_u32(sSb), b_ds = smem_u32(sDS);
#pragma unroll
            for (int kk = 0; kk < DT_VT / 16; ++kk) {
                const uint32_t ko = kk * 32;
                const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
                if (leader) {
                    mma_bf16(tbase + C::C_PG, sw128_desc(a_do + ko, 16, 1024), sw128_desc(a_x + ko, 16, 1024), id64, acc);
                    mma_bf16(tbase + C::C_PG + (16u << 16), sw128_desc(a_dr + ko, 16, 1024), sw128_desc(a_x + ko, 16, 1024),
                             id64, acc);
                    mma_bf16(tbase + C::C_QK, sw128_desc(a_do + ko, 16, 1024), sw128_desc(b_s + ko, 16, 1024), idK, acc);
                    mma_bf16(tbase + C::C_QK + (16u << 16), sw128_desc(a_x + ko, 16, 1024), sw128_desc(b_ds + ko, 16, 1024),
                             idK, acc);
                    mma_bf16(tbase + C::C_QK + (16u << 16), sw128_desc(a_nb + ko, 16, 1024), sw128_desc(b_s + ko, 16, 1024),
                             idK, 1);
                }
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) { err = 1; break; }   // the slice's tiles may be rewritten
        tc_fence_after();
    }

    if (!err) {
        // dP = lower(dO X^T) (bf16; the scale came with dO) and G = -strict_lower(dR X^T); diag(beta) K
        {
            uint32_t r[32];
            tmem_ld32(tq_lane + C::C_PG + 32 * wg, r);
            tmem_wait_ld();
            const int t = mrow;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int sc = 32 * wg + 8 * u + j;
                    const float y = __uint_as_float(r[8 * u + j]);
                    f[j] = first ? (sc <= t ? y : 0.f) : (sc < t ? -y : 0.f);
                }
                store8_bf16(first ? sDP : sGm, sw128_off(t, 32 * wg + 8 * u, BLK), f);
            }
        }
        for (int e = tid; e < (int)(C::KB / 16); e += DT_NT) {
            // 16-byte chunk e of the K tile: row (e % 8 + 8 (e / 64 % 8)) ... the row of a chunk in
            // the 128-byte-swizzled layout is its byte offset / 128 within its 64-column block
            const int row = (int)(((uint32_t)e * 16 % BLK) / 128);
            uint4 w = *reinterpret_cast<const uint4*>(sK + 16 * e);
            uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
            const float b = sB[row];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pw[u]));
                __nv_bfloat162 h = __floats2bfloat162_rn(f.x * b, f.y * b);
                pw[u] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(sBK + 16 * e) = w;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t idKm = idesc_bf16(64, DK, 0, 1), idMM = idesc_bf16(64, DK, 1, 1);
            const uint64_t dPk = sw128_desc(smem_u32(sDP), 16, 1024), dPm = sw128_desc(smem_u32(sDP), BLK, 1024);
            const uint64_t dGk = sw128_desc(smem_u32(sGm), 16, 1024), dGm = sw128_desc(smem_u32(sGm), BLK, 1024);
            const uint64_t dKm = sw128_desc(smem_u32(sK), BLK, 1024), dQm = sw128_desc(smem_u32(sQ), BLK, 1024);
            const uint64_t dBm = sw128_desc(smem_u32(sBK), BLK, 1024);
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks) {
                const uint64_t ka = (ks * 32) >> 4, km = (ks * 2048) >> 4;
                if (leader) {
                    mma_bf16(tbase + C::C_QK, dPk + ka, dKm + km, idKm, 1);                      // dQ += dP K
                    mma_bf16(tbase + C::C_QK + (16u << 16), dPm + km, dQm + km, idMM, 1);        // dK += dP^T Q
                    mma_bf16(tbase + C::C_QK + (16u << 16), dGm + km, dBm + km, idMM, 1);        // dK += G^T diag(beta) K
                    mma_bf16(tbase + C::C_GK + (16u << 16), dGk + ka, dKm + km, idKm, ks > 0);   // G K
                }
            }
            if (leader) mma_commit(bar_mma);
            __syncwarp();
        }
        ++n_mma;
        if (!dt_wait(bar_mma, (n_mma - 1) & 1)) err = 1;
    }
    if (!err) {
        tc_fence_after();
        // dq (lanes 0-15) and dk = dK + diag(beta) G K (lanes 16-31); k_t . (G K)_t partial sums
        const int t = mrow;
        const bool in = t0 + t < L;
        float dbp = 0.f;
        for (int cc = 0; cc < DK / 2; cc += 32) {
            const int c = wg * (DK / 2) + cc;
            uint32_t r[32], g[32];
            tmem_ld32(tq_lane + C::C_QK + c, r);
            tmem_ld32(tq_lane + C::C_GK + c, g);
            tmem_wait_ld();
            if (first) {
                if (in) {
                    float f[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
                    dt_store16_bf16(A.dq + (rowbase + t0 + t) * DK + c, f);
                    dt_store16_bf16(A.dq + (rowbase + t0 + t) * DK + c + 16, f + 16);
                }
            } else {
                const float bt = sB[t];
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    const uint4 kw = *reinterpret_cast<const uint4*>(sK + sw128_off(t, c + j, BLK));
                    const uint32_t* kp = reinterpret_cast<const uint32_t*>(&kw);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kp[u]));
                        const float g0 = __uint_as_float(g[j + 2 * u]), g1 = __uint_as_float(g[j + 2 * u + 1]);
                        f[j + 2 * u] = __uint_as_float(r[j + 2 * u]) + bt * g0;
                        f[j + 2 * u + 1] = __uint_as_float(r[j + 2 * u + 1]) + bt * g1;
                        dbp += kf.x * g0 + kf.y * g1;
                    }
                }
                if (in) {
                    dt_store16_bf16(A.dk + (rowbase + t0 + t) * DK + c, f);
                    dt_store16_bf16(A.dk + (rowbase + t0 + t) * DK + c + 16, f + 16);
                }
            }
        }
        if (!first) sDB[wg * TR + t] = dbp;
        __syncthreads();
        if (tid < TR && t0 + tid < L) {
            float x = sDB[tid] + sDB[TR + tid];
            x += sDU[tid];
            A.dbeta[rowbase + t0 + tid] = x;
        }
    }
    if (err) {
        if (warp == 0) {
            const bool leader = elect_one();
            if (leader) {
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0, 1u << 20);
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, C::NCOL);
}

template <int DK>
cudaError_t dg_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                      const DgArgs& a, int nc, cudaStream_t st) {
    auto kern = k_deltanet_tc_grads<DK>;
    const uint32_t smem = DgCfg<DK>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    GLA_LAUNCH("deltanet_bwd_grads", st, (kern<<<dim3(nc, a.BH), DT_NT, smem, st>>>(mq, mk, mv, mdo, a)));
    return cudaGetLastError();
}

}  // namespace

cudaError_t deltanet_fwd(int B, int H, int L, int Dk, int Dv, float scale, const void* q, const void* k,
                         const void* v, const float* beta, const float* h0, void* o, float* hT, void* saved,
                         int* status, cudaStream_t st) {
    const int BH = B * H;
    if (BH == 0) return cudaSuccess;
    if (L == 0) {
        // no chunk (and no tensor map over an empty sequence): hT = h0 (or zero), nothing else
        if (hT) {
            const size_t n = (size_t)BH * Dk * Dv * sizeof(float);
            return h0 ? cudaMemcpyAsync(hT, h0, n, cudaMemcpyDeviceToDevice, st) : cudaMemsetAsync(hT, 0, n, st);
        }
        return cudaSuccess;
    }
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dk, L, BH, 64, true) ||
        !make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dv, L, BH, 64, true))
        return cudaErrorInvalidValue;
    if (o) {
        if (!make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dk, L, BH, 64, true) ||
            !make_map(&mo, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dv, L, BH, 64, true))
            return cudaErrorInvalidValue;
    } else {
        mq = mk;
        mo = mv;
    }
    DtArgs a{};
    a.beta = beta;
    a.h0 = h0;
    a.hT = hT;
    a.saved = static_cast<__nv_bfloat16*>(saved);
    a.status = status;
    a.L = L;
    a.Dv = Dv;
    a.scale = scale;
    if (Dk == 64)
        return o ? dt_launch<64, true>(B, H, L, Dv, mq, mk, mv, mo, a, st)
                 : dt_launch<64, false>(B, H, L, Dv, mq, mk, mv, mo, a, st);
    return o ? dt_launch<128, true>(B, H, L, Dv, mq, mk, mv, mo, a, st)
             : dt_launch<128, false>(B, H, L, Dv, mq, mk, mv, mo, a, st);
}


cudaError_t deltanet_walk(int B, int H, int L, int Dk, int Dv, float scale, const void* q, const void* k,
                          const float* beta, const void* dO, const float* dhT, float* drw, void* dsend, void* dv,
                          float* dh0, cudaStream_t st) {
    const int BH = B * H;
    if (BH == 0) return cudaSuccess;
    if (L == 0) {   // no chunk: dh0 = dhT (or zero)
        if (dh0) {
            const size_t n = (size_t)BH * Dk * Dv * sizeof(float);
            return dhT ? cudaMemcpyAsync(dh0, dhT, n, cudaMemcpyDeviceToDevice, st) : cudaMemsetAsync(dh0, 0, n, st);
        }
        return cudaSuccess;
    }
    CUtensorMap mq, mk, mdo;
    if (!make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dk, L, BH, 64, true) ||
        !make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dk, L, BH, 64, true) ||
        !make_map(&mdo, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dv, L, BH, 64, true))
        return cudaErrorInvalidValue;
    DwArgs a{};
    a.beta = beta;
    a.dhT = dhT;
    a.drw = drw;
    a.dsend = static_cast<__nv_bfloat16*>(dsend);
    a.dv = static_cast<__nv_bfloat16*>(dv);
    a.dh0 = dh0;
    a.BH = BH;
    a.L = L;
    a.Dv = Dv;
    a.scale = scale;
    return Dk == 64 ? dw_launch<64>(mq, mk, mdo, a, st) : dw_launch<128>(mq, mk, mdo, a, st);
}

cudaError_t deltanet_grads(int B, int H, int L, int Dk, int Dv, float scale, const void* q, const void* k,
                           const void* v, const float* beta, const void* dO, const void* saved, const float* drw,
                           const void* dsend, void* dq, void* dk, float* dbeta, cudaStream_t st) {
    const int BH = B * H, nc = (L + TR - 1) / TR;
    if (BH == 0 || nc == 0) return cudaSuccess;
    CUtensorMap mq, mk, mv, mdo;
    if (!make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dk, L, BH, 64, true) ||
        !make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dk, L, BH, 64, true) ||
        !make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dv, L, BH, 64, true) ||
        !make_map(&mdo, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Dv, L, BH, 64, true))
        return cudaErrorInvalidValue;
    DgArgs a{};
    a.beta = beta;
    a.saved = static_cast<const __nv_bfloat16*>(saved);
    a.drw = drw;
    a.dsend = static_cast<const __nv_bfloat16*>(dsend);
    a.dq = static_cast<__nv_bfloat16*>(dq);
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dbeta = dbeta;
    a.BH = BH;
    a.L = L;
    a.Dv = Dv;
    a.scale = scale;
    return Dk == 64 ? dg_launch<64>(mq, mk, mv, mdo, a, nc, st) : dg_launch<128>(mq, mk, mv, mdo, a, nc, st);
}

}  // namespace tc
}  // namespace gla
