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
// Here num is a pass of the gated linear attention kernels (per-head log-decay g, input gate
// e^{i~ - c}, values v), with c the largest i~ of the head: the same kind of constant shift as
// the stabiliser, it keeps every input gate <= 1 and turns the bound into e^{-c}. den is the same
// sum with a value of one: n_t = e^{g_t} n_{t-1} + e^{i~_t - c} k_t is a Dk-vector recurrence,
// which runs in fp32 on the CUDA cores (one thread per key dim, the sequence cut into 32-token
// segments joined by a scan over segment end states), den_t = (scale q_t) . n_t. Small kernels
// then form h, and in the backward the upstream gradients of the two sums,
//     dnum = dh / N,   dden = -(dh . h) / N * sign(den) where |den| > e^{-c} (else 0),
// and the sums of the two backward parts' dq, dk, dg and the chain rule through the input gate,
// d i~ = (di_num + di_den) e^{i~ - c} (h does not depend on c), formed by the normaliser's last
// kernel as it produces its part. The normaliser's backward is the recurrence's: with
// dn_t = scale dden_t q_t + e^{g_{t+1}} dn_{t+1},
//     dq_t = scale dden_t n_t,  dk_t = i_t dn_t,  di_t = k_t . dn_t,  dg_t = (n_t - i_t k_t) . dn_t
// (i_t the input gate, e^{g_t} n_{t-1} = n_t - i_t k_t).
#include <math.h>
#include <stdint.h>

#include "gla_common.cuh"
#include "sm100.cuh"

namespace gla {
namespace {

constexpr int ML_NT = 256;
constexpr int ML_SL = 32;   // tokens per segment of the normaliser recurrence

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

template <typename Tin, typename Tout>
__global__ void k_cast(const Tin* __restrict__ a, Tout* __restrict__ b, long n) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
        b[i] = from_f<Tout>(to_f(a[i]));
}

// ---- the normaliser recurrence n_t = e^{g_t} n_{t-1} + i_t k_t, fp32, one thread per key dim,
// grid (segment, batch*head) with blocks of Dk threads. A segment's rows of q and k (and of the
// value pass's dq and dk) are contiguous in memory: one bulk copy each brings them into shared
// memory (one memory round trip per block), and the chains over the segment's tokens, sequential
// per key dim, read them there. (Loads issued token by token from global memory left these
// kernels waiting on memory at about a third of the copy bandwidth.) The first warp stages the
// per-token scalars e^{g_t}, i_t and scale dden_t.

// sum over the block's threads of one value per thread, for token slot j: warp sums into part
template <int NW>
__device__ __forceinline__ void ml_warp_part(float x, float (*part)[NW], int j) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if ((threadIdx.x & 31) == 0) part[j][threadIdx.x >> 5] = x;
}

// The first warp stages e^{g_t} (se), and where given i_t (si) and scale dden_t (sd), of the
// segment's cnt <= 32 tokens from row r0; returns the segment's total log-decay (to every lane of
// warp 0). The caller synchronises before the others read them.
__device__ __forceinline__ float ml_stage_scalars(const float* __restrict__ g, const float* __restrict__ ig,
                                                  const float* __restrict__ dd, float scale, long r0, int cnt,
                                                  float* se, float* si, float* sd) {
    const int lane = threadIdx.x;
    const float gj = lane < cnt ? g[r0 + lane] : 0.f;
    if (lane < cnt) {
        se[lane] = __expf(gj);
        if (si) si[lane] = ig[r0 + lane];
        if (sd) sd[lane] = scale * dd[r0 + lane];
    }
    float G = gj;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) G += __shfl_xor_sync(0xffffffffu, G, off);
    return G;
}

// Shared-memory layout of a normaliser block: the mbarrier, the scalars and partial sums, then the
// row tiles (each ML_SL rows of Dk elements, 16-byte aligned).
struct MlSmem {
    static constexpr uint32_t BAR = 0;                   // uint64_t
    static constexpr uint32_t SE = 16;                   // float[ML_SL] each: se, si, sd
    static constexpr uint32_t SI = SE + 4 * ML_SL;
    static constexpr uint32_t SD = SI + 4 * ML_SL;
    static constexpr uint32_t PI = SD + 4 * ML_SL;       // float[ML_SL][8] each: pi, pg
    static constexpr uint32_t PG = PI + 4 * ML_SL * 8;
    static constexpr uint32_t TILES = PG + 4 * ML_SL * 8;
    static_assert(TILES % 16 == 0, "tile alignment");
};
__device__ __forceinline__ uint32_t ml_tile_bytes(int Dk, uint32_t esize) { return (uint32_t)ML_SL * Dk * esize; }

// Thread 0 initialises the block's mbarrier; after the block barrier it expects `bytes` and issues
// the copies (issue()). Everyone then waits (bounded, with the scalars staged in between by the
// caller); false when the copies did not complete, after setting the status word's timeout bit.
template <typename Issue>
__device__ __forceinline__ void ml_tiles_issue(uint64_t* bar, uint32_t bytes, Issue issue) {
    if (threadIdx.x == 0) {
        sm100::mbar_init(bar, 1);
        sm100::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        sm100::mbar_arrive_expect_tx(bar, bytes);
        issue();
    }
}
__device__ __forceinline__ bool ml_tiles_wait(uint64_t* bar, int* status) {
    const bool ok = sm100::mbar_wait(bar, 0);
    if (__syncthreads_and(ok)) return true;
    if (threadIdx.x == 0) atomicOr(status, kDevStatusTimeout);
    return false;
}
template <typename T>
__device__ __forceinline__ void ml_rows_load(T* dst, const T* src, long r0, int cnt, int Dk, uint64_t* bar) {
    sm100::bulk_load_1d(dst, src + r0 * Dk, (uint32_t)cnt * Dk * (uint32_t)sizeof(T), bar);
}

// the segment's end state from zero and its total log-decay
template <typename T>
__global__ void __launch_bounds__(256) k_mlstm_nloc(const T* __restrict__ k, const float* __restrict__ g,
                                                    const float* __restrict__ ig, int L, int Dk, int nseg,
                                                    float* __restrict__ nloc, float* __restrict__ gam, int* status) {
    extern __shared__ __align__(128) uint8_t ml_dsm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(ml_dsm + MlSmem::BAR);
    float* se = reinterpret_cast<float*>(ml_dsm + MlSmem::SE);
    float* si = reinterpret_cast<float*>(ml_dsm + MlSmem::SI);
    const T* sk = reinterpret_cast<const T*>(ml_dsm + MlSmem::TILES);
    const long bh = blockIdx.y;
    const int s = blockIdx.x, d = threadIdx.x;
    const int t0 = s * ML_SL, cnt = min(L - t0, ML_SL);
    const long r0 = bh * L + t0;
    ml_tiles_issue(bar, (uint32_t)cnt * Dk * sizeof(T),
                   [&] { ml_rows_load(const_cast<T*>(sk), k, r0, cnt, Dk, bar); });
    if (d < 32) {
        const float G = ml_stage_scalars(g, ig, nullptr, 0.f, r0, cnt, se, si, nullptr);
        if (d == 0) gam[bh * nseg + s] = G;
    }
    if (!ml_tiles_wait(bar, status)) return;
    float n = 0.f;
#pragma unroll 8
    for (int j = 0; j < cnt; ++j) n = se[j] * n + si[j] * to_f(sk[j * Dk + d]);
    nloc[(bh * nseg + s) * Dk + d] = n;
}

// The two scans over segments run in two levels, groups of ML_SG segments: a first kernel scans
// every group from zero (all groups in parallel) and leaves its total, a second carries the
// totals of the groups before (after) each group into it and adds them to its segments. (One
// block per head walking all segments in order ran only B*H blocks.)
constexpr int ML_SG = 16;

// the state entering every segment of a group from a zero state at the group's start, and the
// group's end state and total log-decay (grid (group, batch*head), blocks of Dk threads)
__global__ void k_mlstm_nscan_local(const float* __restrict__ nloc, const float* __restrict__ gam, int nseg, int Dk,
                                    float* __restrict__ nstart, float* __restrict__ gst, float* __restrict__ ggam) {
    const long bh = blockIdx.y;
    const int gi = blockIdx.x, ng = gridDim.x, d = threadIdx.x;
    const int s0 = gi * ML_SG, cnt = min(nseg - s0, ML_SG);
    float nl[ML_SG], ga[ML_SG];
#pragma unroll
    for (int u = 0; u < ML_SG; ++u)
        if (u < cnt) {
            nl[u] = nloc[(bh * nseg + s0 + u) * Dk + d];
            ga[u] = gam[bh * nseg + s0 + u];
        }
    float n = 0.f, G = 0.f;
#pragma unroll
    for (int u = 0; u < ML_SG; ++u)
        if (u < cnt) {
            nstart[(bh * nseg + s0 + u) * Dk + d] = n;
            n = __expf(ga[u]) * n + nl[u];
            G += ga[u];
        }
    gst[(bh * ng + gi) * Dk + d] = n;
    if (d == 0) ggam[bh * ng + gi] = G;
}

// the state entering group gi from the groups before it, carried into its segments
__global__ void k_mlstm_nscan_fix(const float* __restrict__ gam, const float* __restrict__ gst,
                                  const float* __restrict__ ggam, int nseg, int Dk, float* __restrict__ nstart) {
    const long bh = blockIdx.y;
    const int gi = blockIdx.x, ng = gridDim.x, d = threadIdx.x;
    if (gi == 0) return;   // the first group starts from the zero state
    float e = 0.f;   // groups 0 .. gi-1 in order, their totals loaded ML_SG at a time
    for (int b0 = 0; b0 < gi; b0 += ML_SG) {
        float gs[ML_SG], gg[ML_SG];
#pragma unroll
        for (int u = 0; u < ML_SG; ++u)
            if (b0 + u < gi) {
                gs[u] = gst[(bh * ng + b0 + u) * Dk + d];
                gg[u] = ggam[bh * ng + b0 + u];
            }
#pragma unroll
        for (int u = 0; u < ML_SG; ++u)
            if (b0 + u < gi) e = __expf(gg[u]) * e + gs[u];
    }
    const int s0 = gi * ML_SG, cnt = min(nseg - s0, ML_SG);
    float D = 1.f;   // decay from the group's start to the segment
#pragma unroll
    for (int u = 0; u < ML_SG; ++u)
        if (u < cnt) {
            nstart[(bh * nseg + s0 + u) * Dk + d] += D * e;
            D *= __expf(gam[bh * nseg + s0 + u]);
        }
}

// den_t = scale q_t . n_t over the segment (den [BH*L] fp32)
template <typename T>
__global__ void __launch_bounds__(256) k_mlstm_den(const T* __restrict__ q, const T* __restrict__ k,
                                                   const float* __restrict__ g, const float* __restrict__ ig,
                                                   const float* __restrict__ nstart, int L, int Dk, int nseg,
                                                   float scale, float* __restrict__ den, int* status) {
    extern __shared__ __align__(128) uint8_t ml_dsm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(ml_dsm + MlSmem::BAR);
    float* se = reinterpret_cast<float*>(ml_dsm + MlSmem::SE);
    float* si = reinterpret_cast<float*>(ml_dsm + MlSmem::SI);
    float(*part)[8] = reinterpret_cast<float(*)[8]>(ml_dsm + MlSmem::PI);
    const T* sq = reinterpret_cast<const T*>(ml_dsm + MlSmem::TILES);
    const T* sk = reinterpret_cast<const T*>(ml_dsm + MlSmem::TILES + ml_tile_bytes(Dk, sizeof(T)));
    const long bh = blockIdx.y;
    const int s = blockIdx.x, d = threadIdx.x, nw = Dk / 32;
    const int t0 = s * ML_SL, cnt = min(L - t0, ML_SL);
    const long r0 = bh * L + t0;
    ml_tiles_issue(bar, 2u * cnt * Dk * sizeof(T), [&] {
        ml_rows_load(const_cast<T*>(sq), q, r0, cnt, Dk, bar);
        ml_rows_load(const_cast<T*>(sk), k, r0, cnt, Dk, bar);
    });
    if (d < 32) ml_stage_scalars(g, ig, nullptr, 0.f, r0, cnt, se, si, nullptr);
    float n = nstart[(bh * nseg + s) * Dk + d];
    if (!ml_tiles_wait(bar, status)) return;
#pragma unroll 4
    for (int j = 0; j < cnt; ++j) {
        n = se[j] * n + si[j] * to_f(sk[j * Dk + d]);
        ml_warp_part<8>(to_f(sq[j * Dk + d]) * n, part, j);
    }
    __syncthreads();
    if (d < cnt) {
        float x = 0.f;
        for (int w = 0; w < nw; ++w) x += part[d][w];
        den[r0 + d] = scale * x;
    }
}

// backward, local: the gradient carried out of the segment's start from a zero carry at its end,
// c = e^{g_t} dn_t with dn_t = scale dden_t q_t + c (walking the segment backwards)
template <typename T>
__global__ void __launch_bounds__(256) k_mlstm_dnloc(const T* __restrict__ q, const float* __restrict__ g,
                                                     const float* __restrict__ dden, int L, int Dk, int nseg,
                                                     float scale, float* __restrict__ cloc, int* status) {
    extern __shared__ __align__(128) uint8_t ml_dsm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(ml_dsm + MlSmem::BAR);
    float* se = reinterpret_cast<float*>(ml_dsm + MlSmem::SE);
    float* sd = reinterpret_cast<float*>(ml_dsm + MlSmem::SD);
    const T* sq = reinterpret_cast<const T*>(ml_dsm + MlSmem::TILES);
    const long bh = blockIdx.y;
    const int s = blockIdx.x, d = threadIdx.x;
    const int t0 = s * ML_SL, cnt = min(L - t0, ML_SL);
    const long r0 = bh * L + t0;
    ml_tiles_issue(bar, (uint32_t)cnt * Dk * sizeof(T),
                   [&] { ml_rows_load(const_cast<T*>(sq), q, r0, cnt, Dk, bar); });
    if (d < 32) ml_stage_scalars(g, nullptr, dden, scale, r0, cnt, se, nullptr, sd);
    if (!ml_tiles_wait(bar, status)) return;
    float c = 0.f;
#pragma unroll 8
    for (int j = cnt - 1; j >= 0; --j) c = se[j] * (sd[j] * to_f(sq[j * Dk + d]) + c);
    cloc[(bh * nseg + s) * Dk + d] = c;
}

// the carry entering every segment of a group from a zero carry at the group's end, and the
// carry out of the group's start and its total log-decay (grid (group, batch*head))
__global__ void k_mlstm_cscan_local(const float* __restrict__ cloc, const float* __restrict__ gam, int nseg, int Dk,
                                    float* __restrict__ cin, float* __restrict__ gst, float* __restrict__ ggam) {
    const long bh = blockIdx.y;
    const int gi = blockIdx.x, ng = gridDim.x, d = threadIdx.x;
    const int s0 = gi * ML_SG, cnt = min(nseg - s0, ML_SG);
    float cl[ML_SG], ga[ML_SG];
#pragma unroll
    for (int u = 0; u < ML_SG; ++u)
        if (u < cnt) {
            cl[u] = cloc[(bh * nseg + s0 + u) * Dk + d];
            ga[u] = gam[bh * nseg + s0 + u];
        }
    float c = 0.f, G = 0.f;
#pragma unroll
    for (int u = ML_SG - 1; u >= 0; --u)
        if (u < cnt) {
            cin[(bh * nseg + s0 + u) * Dk + d] = c;
            c = __expf(ga[u]) * c + cl[u];
            G += ga[u];
        }
    gst[(bh * ng + gi) * Dk + d] = c;
    if (d == 0) ggam[bh * ng + gi] = G;
}

// the carry entering group gi's end from the groups after it, carried into its segments
__global__ void k_mlstm_cscan_fix(const float* __restrict__ gam, const float* __restrict__ gst,
                                  const float* __restrict__ ggam, int nseg, int Dk, float* __restrict__ cin) {
    const long bh = blockIdx.y;
    const int gi = blockIdx.x, ng = gridDim.x, d = threadIdx.x;
    if (gi == ng - 1) return;   // nothing comes after the last group
    float e = 0.f;   // groups ng-1 .. gi+1 in reverse order, their totals loaded ML_SG at a time
    for (int b1 = ng - 1; b1 > gi; b1 -= ML_SG) {
        float gs[ML_SG], gg[ML_SG];
#pragma unroll
        for (int u = 0; u < ML_SG; ++u)
            if (b1 - u > gi) {
                gs[u] = gst[(bh * ng + b1 - u) * Dk + d];
                gg[u] = ggam[bh * ng + b1 - u];
            }
#pragma unroll
        for (int u = 0; u < ML_SG; ++u)
            if (b1 - u > gi) e = __expf(gg[u]) * e + gs[u];
    }
    const int s0 = gi * ML_SG, cnt = min(nseg - s0, ML_SG);
    float D = 1.f;   // decay from the group's end back to the segment
#pragma unroll
    for (int u = ML_SG - 1; u >= 0; --u)
        if (u < cnt) {
            cin[(bh * nseg + s0 + u) * Dk + d] += D * e;
            D *= __expf(gam[bh * nseg + s0 + u]);
        }
}

// the normaliser's gradients over a segment: n_t forward from the segment's start state (kept in
// registers), then dn_t backwards from the carry entering the segment's end. They are added
// to the value pass's in the same step: dq = dq1 + scale dden n_t and dk = dk1 + i_t dn_t in the
// output dtype (dq1 / dk1 may be the outputs themselves: each thread reads its element of a row
// before it writes it), dg += (n_t - i_t k_t) . dn_t and d i~ = (di1 + k_t . dn_t) i_t. The
// segment's rows of q, k, dq1 and dk1 come into shared memory by bulk copies.
template <typename T, typename Ta>
__global__ void __launch_bounds__(256) k_mlstm_den_bwd(const T* __restrict__ q, const T* __restrict__ k,
                                                       const float* __restrict__ g, const float* __restrict__ ig,
                                                       const float* __restrict__ dden,
                                                       const float* __restrict__ nstart, const float* __restrict__ cin,
                                                       int L, int Dk, int nseg, float scale, const Ta* dq1,
                                                       const Ta* dk1, T* dq, T* dk, float* __restrict__ dg,
                                                       const float* __restrict__ di1, float* __restrict__ ditil,
                                                       int* status) {
    extern __shared__ __align__(128) uint8_t ml_dsm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(ml_dsm + MlSmem::BAR);
    float* se = reinterpret_cast<float*>(ml_dsm + MlSmem::SE);
    float* si = reinterpret_cast<float*>(ml_dsm + MlSmem::SI);
    float* sd = reinterpret_cast<float*>(ml_dsm + MlSmem::SD);
    float(*pi)[8] = reinterpret_cast<float(*)[8]>(ml_dsm + MlSmem::PI);
    float(*pg)[8] = reinterpret_cast<float(*)[8]>(ml_dsm + MlSmem::PG);
    const uint32_t tb = ml_tile_bytes(Dk, sizeof(T)), ta = ml_tile_bytes(Dk, sizeof(Ta));
    const T* sq = reinterpret_cast<const T*>(ml_dsm + MlSmem::TILES);
    const T* sk = reinterpret_cast<const T*>(ml_dsm + MlSmem::TILES + tb);
    const Ta* sa = reinterpret_cast<const Ta*>(ml_dsm + MlSmem::TILES + 2 * tb);
    const Ta* sb = reinterpret_cast<const Ta*>(ml_dsm + MlSmem::TILES + 2 * tb + ta);
    const long bh = blockIdx.y;
    const int s = blockIdx.x, d = threadIdx.x, nw = Dk / 32;
    const int t0 = s * ML_SL, cnt = min(L - t0, ML_SL);
    const long r0 = bh * L + t0;
    ml_tiles_issue(bar, 2u * cnt * Dk * (uint32_t)(sizeof(T) + sizeof(Ta)), [&] {
        ml_rows_load(const_cast<T*>(sq), q, r0, cnt, Dk, bar);
        ml_rows_load(const_cast<T*>(sk), k, r0, cnt, Dk, bar);
        ml_rows_load(const_cast<Ta*>(sa), dq1, r0, cnt, Dk, bar);
        ml_rows_load(const_cast<Ta*>(sb), dk1, r0, cnt, Dk, bar);
    });
    if (d < 32) ml_stage_scalars(g, ig, dden, scale, r0, cnt, se, si, sd);
    float n = nstart[(bh * nseg + s) * Dk + d];
    float c = cin[(bh * nseg + s) * Dk + d];
    if (!ml_tiles_wait(bar, status)) return;
    float nv[ML_SL];   // n_t of this key dim over the segment (fully unrolled: registers)
#pragma unroll
    for (int j = 0; j < ML_SL; ++j)
        if (j < cnt) {
            n = se[j] * n + si[j] * to_f(sk[j * Dk + d]);
            nv[j] = n;
        }
#pragma unroll
    for (int j = ML_SL - 1; j >= 0; --j)
        if (j < cnt) {
            const long o = (r0 + j) * Dk + d;
            const float sdj = sd[j], it = si[j], kt = to_f(sk[j * Dk + d]), nj = nv[j];
            const float dn = sdj * to_f(sq[j * Dk + d]) + c;
            dq[o] = from_f<T>(to_f(sa[j * Dk + d]) + sdj * nj);
            dk[o] = from_f<T>(to_f(sb[j * Dk + d]) + it * dn);
            ml_warp_part<8>(kt * dn, pi, j);
            ml_warp_part<8>((nj - it * kt) * dn, pg, j);
            c = se[j] * dn;
        }
    __syncthreads();
    if (d < cnt) {
        float xi = 0.f, xg = 0.f;
        for (int w = 0; w < nw; ++w) {
            xi += pi[d][w];
            xg += pg[d][w];
        }
        dg[r0 + d] += xg;
        ditil[r0 + d] = (di1[r0 + d] + xi) * si[d];
    }
}

// dynamic shared memory of the normaliser kernels: the fixed part and `tiles` row tiles of esize
// bytes per element (den_bwd: plus its fp32 n_t tile)
inline size_t ml_smem_bytes(int Dk, size_t tile_elem_bytes) {
    return MlSmem::TILES + (size_t)ML_SL * Dk * tile_elem_bytes;
}

// Eight consecutive elements (16 bytes of bf16, 32 of fp32) to / from fp32.
__device__ __forceinline__ void ld8(const float* p, float* f) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* f) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ void st8(float* p, const float* f) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16* p, const float* f) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 x = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        u[i] = *reinterpret_cast<const uint32_t*>(&x);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(u[0], u[1], u[2], u[3]);
}

// One warp per token row (eight elements a lane at a time): N = max(|den|, e^{-c}), h = num / N.
template <typename Ta, typename To>
__global__ void __launch_bounds__(ML_NT) k_mlstm_norm(const Ta* __restrict__ num, const float* __restrict__ den,
                                                      const float* __restrict__ cst, To* __restrict__ h, long rows,
                                                      int L, int Dv) {
    const long row = blockIdx.x * (long)(ML_NT / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float N = fmaxf(fabsf(den[row]), expf(-cst[row / L]));
    const float inv = 1.f / N;
    for (int e = 8 * lane; e < Dv; e += 256) {
        float f[8];
        ld8(num + row * Dv + e, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] *= inv;
        st8(h + row * Dv + e, f);
    }
}

// One warp per token row (eight elements a lane at a time): the upstream gradients of the two
// sums.
template <typename Ta, typename To>
__global__ void __launch_bounds__(ML_NT) k_mlstm_bwd_prep(const Ta* __restrict__ num, const float* __restrict__ den,
                                                          const float* __restrict__ cst, const To* __restrict__ dh,
                                                          Ta* __restrict__ dnum, float* __restrict__ dden, long rows,
                                                          int L, int Dv) {
    const long row = blockIdx.x * (long)(ML_NT / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float dn = den[row];
    const float bound = expf(-cst[row / L]);
    const float N = fmaxf(fabsf(dn), bound);
    const float inv = 1.f / N;
    float s = 0.f;   // dh . h
    for (int e = 8 * lane; e < Dv; e += 256) {
        float d[8], x[8];
        ld8(dh + row * Dv + e, d);
        ld8(num + row * Dv + e, x);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            s += d[i] * x[i] * inv;
            d[i] *= inv;
        }
        st8(dnum + row * Dv + e, d);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) dden[row] = fabsf(dn) > bound ? -s * inv * (dn > 0.f ? 1.f : -1.f) : 0.f;
}

bool ml_aligned16(const void* x) { return x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }

struct MlLayout {
    gla_problem pa;       // the value pass
    bool fa;              // the value pass runs with fp32 I/O
    bool cast_a;          // ... on bf16 I/O: converted copies of q, k, v, and its gradients are
                          // cast back
    int nseg;             // 32-token segments of the normaliser recurrence
    size_t wsa;           // the value pass's workspace bytes
    int ngrp;             // groups of ML_SG segments of the two-level scans over segments
    size_t o_qf, o_kf, o_vf, o_nloc, o_gst, o_ggam;
    size_t o_dnum, o_dden, o_dq1, o_dk1, o_dv1, o_di1, o_cloc, o_cin;
    size_t o_res;         // the forward's results (MlRes) when they live in the workspace
    size_t total;
    // The forward's results the backward reads, at offsets from their own base: the input gate,
    // the per-head shift, num, den, the normaliser's segment decays and start states, and (saved
    // buffer only) the value pass's saved states for gla_bwd_saved.
    size_t r_ig, r_c, r_num, r_den, r_gam, r_nst, r_gla, res_bytes, gla_saved, saved_total;
};

gla_status ml_layout(const gla_problem* p, bool bwd, MlLayout* w) {
    if (!p || p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_PER_HEAD) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->plan < GLA_PLAN_AUTO || p->plan > GLA_PLAN_TC) return GLA_ERR_INVALID_ARG;
    w->pa = *p;
    // h divides by |den| wherever |den| exceeds the bound, and den is a sum of terms of both
    // signs: an error proportional to the terms becomes a large relative error of h where |den|
    // sits just above the bound, and the gradients add the two sums' parts, which can nearly
    // cancel. So the normaliser always runs as its fp32 recurrence (a Dk-vector state, a small
    // share of the work). The value pass runs on the CUDA cores in fp32 (the automatic plan and
    // GLA_PLAN_SIMT; fp32 I/O always), or with GLA_PLAN_TC on the tensor cores in bf16: much
    // faster, with the bf16 pass's error carried into h and, through the cancellation, into dq
    // and dk.
    const bool bf = p->io == GLA_BF16;
    w->fa = !bf || p->plan != GLA_PLAN_TC;
    w->cast_a = bf && w->fa;
    w->pa.plan = w->fa ? GLA_PLAN_SIMT : GLA_PLAN_TC;
    if (w->fa) w->pa.io = GLA_F32;
    const size_t f = gla_workspace_bytes(&w->pa, 0);
    const size_t b = bwd ? gla_workspace_bytes(&w->pa, 1) : 0;
    w->wsa = (f == 0 || (bwd && b == 0)) ? 0 : (f > b ? f : b);
    if (w->wsa == 0) return GLA_ERR_UNSUPPORTED;   // the verdict gla_fwd / gla_bwd give
    const size_t BHL = (size_t)p->B * p->H * p->L, BH = (size_t)p->B * p->H;
    const size_t ea = w->fa ? 4 : 2;   // bytes of the value pass's elements
    w->nseg = (p->L + ML_SL - 1) / ML_SL;
    const size_t NS = BH * (size_t)w->nseg;
    size_t off = align_up(w->wsa, 256);
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    {
        size_t r = 0;
        auto rtake = [&](size_t bytes) {
            const size_t o = r;
            r = align_up(r + bytes, 256);
            return o;
        };
        w->r_ig = rtake(4 * BHL);
        w->r_c = rtake(4 * BH);
        w->r_num = rtake(ea * BHL * p->Dv);
        w->r_den = rtake(4 * BHL);
        w->r_gam = rtake(4 * NS);
        w->r_nst = rtake(4 * NS * p->Dk);
        w->res_bytes = r;
        w->gla_saved = gla_saved_states_bytes(&w->pa);
        w->r_gla = w->gla_saved ? rtake(w->gla_saved) : 0;
        w->saved_total = r;
    }
    w->o_res = take(w->res_bytes);
    if (w->cast_a) {
        w->o_qf = take(4 * BHL * p->Dk);
        w->o_kf = take(4 * BHL * p->Dk);
        w->o_vf = take(4 * BHL * p->Dv);
    }
    w->o_nloc = take(4 * NS * p->Dk);
    w->ngrp = (w->nseg + ML_SG - 1) / ML_SG;
    w->o_gst = take(4 * BH * (size_t)w->ngrp * p->Dk);
    w->o_ggam = take(4 * BH * (size_t)w->ngrp);
    if (bwd) {
        w->o_dnum = take(ea * BHL * p->Dv);
        w->o_dden = take(4 * BHL);
        if (w->cast_a) {
            w->o_dq1 = take(4 * BHL * p->Dk);
            w->o_dk1 = take(4 * BHL * p->Dk);
            w->o_dv1 = take(4 * BHL * p->Dv);
        }
        w->o_cloc = take(4 * NS * p->Dk);
        w->o_cin = take(4 * NS * p->Dk);
        w->o_di1 = take(4 * BHL);
    }
    w->total = off;
    return GLA_OK;
}

unsigned ml_grid(long n, int nt) {
    const long b = (n + nt - 1) / nt;
    return (unsigned)(b < 1 ? 1 : b > 148L * 16 ? 148L * 16 : b);
}

// The inputs the value pass reads (the caller's, or converted fp32 copies in the workspace).
struct MlInputs {
    const void *qa, *ka, *va;
};

// Where the forward's results live: in the workspace, or (a training pair) in the caller's
// saved buffer, which then also takes the value pass's saved states.
struct MlRes {
    float* ig;
    float* c;
    void* num;
    float* den;
    float* gam;
    float* nst;
    float* gla;   // value pass's saved states, or null
};

MlRes ml_res(const MlLayout& w, char* ws, char* saved) {
    char* b = saved ? saved : ws + w.o_res;
    MlRes r;
    r.ig = reinterpret_cast<float*>(b + w.r_ig);
    r.c = reinterpret_cast<float*>(b + w.r_c);
    r.num = b + w.r_num;
    r.den = reinterpret_cast<float*>(b + w.r_den);
    r.gam = reinterpret_cast<float*>(b + w.r_gam);
    r.nst = reinterpret_cast<float*>(b + w.r_nst);
    r.gla = (saved && w.gla_saved) ? reinterpret_cast<float*>(b + w.r_gla) : nullptr;
    return r;
}

// fp32 copies of bf16 inputs where the value pass runs in fp32 (else the caller's inputs).
template <typename To>
gla_status ml_inputs(const gla_problem* p, const MlLayout& w, const void* q, const void* k, const void* v, char* ws,
                     MlInputs* in, cudaStream_t st) {
    *in = MlInputs{q, k, v};
    if (!w.cast_a) return GLA_OK;
    const long BHL = (long)p->B * p->H * p->L;
    const long nq = BHL * p->Dk, nv = BHL * p->Dv;
    float* qf = reinterpret_cast<float*>(ws + w.o_qf);
    float* kf = reinterpret_cast<float*>(ws + w.o_kf);
    float* vf = reinterpret_cast<float*>(ws + w.o_vf);
    GLA_LAUNCH("mlstm_cast", st, (k_cast<To, float><<<ml_grid(nq, 256), 256, 0, st>>>(static_cast<const To*>(q), qf, nq)));
    GLA_LAUNCH("mlstm_cast", st, (k_cast<To, float><<<ml_grid(nq, 256), 256, 0, st>>>(static_cast<const To*>(k), kf, nq)));
    GLA_LAUNCH("mlstm_cast", st, (k_cast<To, float><<<ml_grid(nv, 256), 256, 0, st>>>(static_cast<const To*>(v), vf, nv)));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e, "mLSTM input conversion launch");
    *in = MlInputs{qf, kf, vf};
    return GLA_OK;
}

// Shared by the forward and the backward (unless the backward reads a training pair's saved
// results): the input gate, num (the value pass) and den (the normaliser recurrence) into `r`.
template <typename Ta, typename To>
gla_status ml_forward_passes(const gla_problem* p, const MlLayout& w, const MlInputs& in, const void* q,
                             const void* k, const float* g, const float* itil, char* ws, const MlRes& r,
                             cudaStream_t st) {
    const long BH = (long)p->B * p->H;
    GLA_LAUNCH("mlstm_prep", st, k_mlstm_prep<<<(unsigned)BH, ML_NT, 0, st>>>(itil, p->L, r.ig, r.c));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e, "mLSTM gate launch");
    gla_status s = gla_fwd_save(&w.pa, in.qa, in.ka, in.va, g, r.ig, nullptr, r.num, nullptr, r.gla, ws, w.wsa, st);
    if (s != GLA_OK) return s;
    // the normaliser recurrence, reading q and k in the I/O dtype
    const To* tq = static_cast<const To*>(q);
    const To* tk = static_cast<const To*>(k);
    float* nloc = reinterpret_cast<float*>(ws + w.o_nloc);
    const dim3 grid(w.nseg, (unsigned)BH);
    int* status = reinterpret_cast<int*>(ws);
    const size_t s1 = ml_smem_bytes(p->Dk, sizeof(To)), s2 = ml_smem_bytes(p->Dk, 2 * sizeof(To));
    static std::atomic<bool> attr_nloc[kMaxDevices], attr_den[kMaxDevices];
    {
        cudaError_t ea = smem_attr_once(k_mlstm_nloc<To>, ml_smem_bytes(256, sizeof(To)), attr_nloc);
        if (ea == cudaSuccess) ea = smem_attr_once(k_mlstm_den<To>, ml_smem_bytes(256, 2 * sizeof(To)), attr_den);
        if (ea != cudaSuccess) return record_cuda(ea, "mLSTM normaliser shared-memory attribute");
    }
    GLA_LAUNCH("mlstm_nloc", st,
               k_mlstm_nloc<To><<<grid, p->Dk, s1, st>>>(tk, g, r.ig, p->L, p->Dk, w.nseg, nloc, r.gam, status));
    float* gst = reinterpret_cast<float*>(ws + w.o_gst);
    float* ggam = reinterpret_cast<float*>(ws + w.o_ggam);
    const dim3 ggrid(w.ngrp, (unsigned)BH);
    GLA_LAUNCH("mlstm_nscan", st,
               k_mlstm_nscan_local<<<ggrid, p->Dk, 0, st>>>(nloc, r.gam, w.nseg, p->Dk, r.nst, gst, ggam));
    GLA_LAUNCH("mlstm_nscan", st, k_mlstm_nscan_fix<<<ggrid, p->Dk, 0, st>>>(r.gam, gst, ggam, w.nseg, p->Dk, r.nst));
    GLA_LAUNCH("mlstm_den", st,
               k_mlstm_den<To><<<grid, p->Dk, s2, st>>>(tq, tk, g, r.ig, r.nst, p->L, p->Dk, w.nseg, p->scale, r.den,
                                                        status));
    return record_cuda(cudaGetLastError(), "mLSTM normaliser launch");
}

// saved: a training pair's buffer (gla_mlstm_saved_bytes) that receives the forward's results, or
// null to keep them in the workspace.
template <typename Ta, typename To>
gla_status ml_fwd(const gla_problem* p, const MlLayout& w, const void* q, const void* k, const void* v,
                  const float* g, const float* itil, void* h, char* ws, char* saved, cudaStream_t st) {
    MlInputs in;
    gla_status s = ml_inputs<To>(p, w, q, k, v, ws, &in, st);
    if (s != GLA_OK) return s;
    const MlRes r = ml_res(w, ws, saved);
    s = ml_forward_passes<Ta, To>(p, w, in, q, k, g, itil, ws, r, st);
    if (s != GLA_OK) return s;
    const long rows = (long)p->B * p->H * p->L;
    GLA_LAUNCH("mlstm_norm", st,
               (k_mlstm_norm<Ta, To><<<(unsigned)((rows + ML_NT / 32 - 1) / (ML_NT / 32)), ML_NT, 0, st>>>(
                   static_cast<const Ta*>(r.num), r.den, r.c, static_cast<To*>(h), rows, p->L, p->Dv)));
    return record_cuda(cudaGetLastError(), "mLSTM normalise launch");
}

// saved: the buffer the forward of a training pair filled (its results are read from there and
// the forward passes are not run again), or null to run them.
template <typename Ta, typename To>
gla_status ml_bwd(const gla_problem* p, const MlLayout& w, const void* q, const void* k, const void* v,
                  const float* g, const float* itil, const void* dh, void* dq, void* dk, void* dv, float* dg,
                  float* ditil, char* ws, char* saved, cudaStream_t st) {
    MlInputs in;
    gla_status s = ml_inputs<To>(p, w, q, k, v, ws, &in, st);
    if (s != GLA_OK) return s;
    const MlRes r = ml_res(w, ws, saved);
    if (!saved) {
        s = ml_forward_passes<Ta, To>(p, w, in, q, k, g, itil, ws, r, st);
        if (s != GLA_OK) return s;
    }
    const long rows = (long)p->B * p->H * p->L;
    Ta* dnum = reinterpret_cast<Ta*>(ws + w.o_dnum);
    float* dden = reinterpret_cast<float*>(ws + w.o_dden);
    GLA_LAUNCH("mlstm_bwd_prep", st,
               (k_mlstm_bwd_prep<Ta, To><<<(unsigned)((rows + ML_NT / 32 - 1) / (ML_NT / 32)), ML_NT, 0, st>>>(
                   static_cast<const Ta*>(r.num), r.den, r.c, static_cast<const To*>(dh), dnum, dden, rows, p->L,
                   p->Dv)));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return record_cuda(e, "mLSTM backward prep launch");
    const float* ig = r.ig;
    float* di1 = reinterpret_cast<float*>(ws + w.o_di1);
    // the value pass writes its gradients straight into the outputs unless they are cast back
    void* dq1 = w.cast_a ? ws + w.o_dq1 : dq;
    void* dk1 = w.cast_a ? ws + w.o_dk1 : dk;
    void* dv1 = w.cast_a ? ws + w.o_dv1 : dv;
    s = gla_bwd_saved(&w.pa, in.qa, in.ka, in.va, g, ig, nullptr, dnum, nullptr, r.gla, dq1, dk1, dv1, dg, di1,
                      nullptr, ws, w.wsa, st);
    if (s != GLA_OK) return s;
    // the normaliser recurrence's backward, reading q and k in the I/O dtype
    {
        const long BH = (long)p->B * p->H;
        const To* tq = static_cast<const To*>(q);
        const To* tk = static_cast<const To*>(k);
        float* cloc = reinterpret_cast<float*>(ws + w.o_cloc);
        float* cin = reinterpret_cast<float*>(ws + w.o_cin);
        const dim3 grid(w.nseg, (unsigned)BH);
        int* status = reinterpret_cast<int*>(ws);
        const size_t s1 = ml_smem_bytes(p->Dk, sizeof(To));
        const size_t sb = ml_smem_bytes(p->Dk, 2 * sizeof(To) + 2 * sizeof(Ta));
        static std::atomic<bool> attr_dnloc[kMaxDevices], attr_dbwd[kMaxDevices];
        {
            cudaError_t ea = smem_attr_once(k_mlstm_dnloc<To>, ml_smem_bytes(256, sizeof(To)), attr_dnloc);
            if (ea == cudaSuccess)
                ea = smem_attr_once(k_mlstm_den_bwd<To, Ta>, ml_smem_bytes(256, 2 * sizeof(To) + 2 * sizeof(Ta)),
                                    attr_dbwd);
            if (ea != cudaSuccess) return record_cuda(ea, "mLSTM normaliser shared-memory attribute");
        }
        GLA_LAUNCH("mlstm_dnloc", st,
                   k_mlstm_dnloc<To><<<grid, p->Dk, s1, st>>>(tq, g, dden, p->L, p->Dk, w.nseg, p->scale, cloc, status));
        float* gst = reinterpret_cast<float*>(ws + w.o_gst);
        float* ggam = reinterpret_cast<float*>(ws + w.o_ggam);
        const dim3 ggrid(w.ngrp, (unsigned)BH);
        GLA_LAUNCH("mlstm_cscan", st,
                   k_mlstm_cscan_local<<<ggrid, p->Dk, 0, st>>>(cloc, r.gam, w.nseg, p->Dk, cin, gst, ggam));
        GLA_LAUNCH("mlstm_cscan", st,
                   k_mlstm_cscan_fix<<<ggrid, p->Dk, 0, st>>>(r.gam, gst, ggam, w.nseg, p->Dk, cin));
        GLA_LAUNCH("mlstm_den_bwd", st,
                   (k_mlstm_den_bwd<To, Ta><<<grid, p->Dk, sb, st>>>(
                       tq, tk, g, ig, dden, r.nst, cin, p->L, p->Dk, w.nseg,
                       p->scale, static_cast<const Ta*>(dq1), static_cast<const Ta*>(dk1), static_cast<To*>(dq),
                       static_cast<To*>(dk), dg, di1, ditil, status)));
        if ((e = cudaGetLastError()) != cudaSuccess) return record_cuda(e, "mLSTM normaliser backward launch");
    }
    if (w.cast_a) {   // dv of the fp32 value pass, cast back
        const long nv = rows * p->Dv;
        GLA_LAUNCH("mlstm_cast", st,
                   (k_cast<float, To><<<ml_grid(nv, 256), 256, 0, st>>>(static_cast<const float*>(dv1),
                                                                        static_cast<To*>(dv), nv)));
    }
    return record_cuda(cudaGetLastError(), "mLSTM backward cast launch");
}

}  // namespace
}  // namespace gla

namespace gla {
namespace {

gla_status ml_fwd_entry(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                        const float* itil, void* h, void* saved, void* ws, size_t ws_bytes, void* stream) {
    MlLayout w;
    const gla_status s = ml_layout(p, false, &w);
    if (s != GLA_OK) return s;
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!q || !k || !v || !g || !itil || !h)) return GLA_ERR_INVALID_ARG;
    if (!ws) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, itil, h, saved, ws};
    for (const void* x : ptrs)
        if (!ml_aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return GLA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
    if (e != cudaSuccess) return record_cuda(e, "status word reset");
    if (empty) return GLA_OK;
    char* wsb = static_cast<char*>(ws);
    char* sv = static_cast<char*>(saved);
    using bf16 = __nv_bfloat16;
    if (p->io == GLA_F32) return ml_fwd<float, float>(p, w, q, k, v, g, itil, h, wsb, sv, st);
    return w.fa ? ml_fwd<float, bf16>(p, w, q, k, v, g, itil, h, wsb, sv, st)
                : ml_fwd<bf16, bf16>(p, w, q, k, v, g, itil, h, wsb, sv, st);
}

gla_status ml_bwd_entry(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                        const float* itil, const void* dh, const void* saved, void* dq, void* dk, void* dv, float* dg,
                        float* ditil, void* ws, size_t ws_bytes, void* stream) {
    MlLayout w;
    const gla_status s = ml_layout(p, true, &w);
    if (s != GLA_OK) return s;
    const bool empty = (size_t)p->B * p->H * p->L == 0;
    if (!empty && (!q || !k || !v || !g || !itil || !dh || !dq || !dk || !dv || !dg || !ditil))
        return GLA_ERR_INVALID_ARG;
    if (!ws) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, itil, dh, saved, dq, dk, dv, dg, ditil, ws};
    for (const void* x : ptrs)
        if (!ml_aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return GLA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
    if (e != cudaSuccess) return record_cuda(e, "status word reset");
    if (empty) return GLA_OK;
    char* wsb = static_cast<char*>(ws);
    char* sv = const_cast<char*>(static_cast<const char*>(saved));   // read only
    using bf16 = __nv_bfloat16;
    if (p->io == GLA_F32)
        return ml_bwd<float, float>(p, w, q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, wsb, sv, st);
    return w.fa ? ml_bwd<float, bf16>(p, w, q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, wsb, sv, st)
                : ml_bwd<bf16, bf16>(p, w, q, k, v, g, itil, dh, dq, dk, dv, dg, ditil, wsb, sv, st);
}

}  // namespace
}  // namespace gla

extern "C" {

size_t gla_mlstm_workspace_bytes(const gla_problem* p, int for_backward) {
    gla::MlLayout w;
    if (gla::ml_layout(p, for_backward != 0, &w) != GLA_OK) return 0;
    return w.total;
}

size_t gla_mlstm_saved_bytes(const gla_problem* p) {
    gla::MlLayout w;
    if (gla::ml_layout(p, true, &w) != GLA_OK) return 0;
    if ((size_t)p->B * p->H * p->L == 0) return 0;
    return w.saved_total;
}

gla_status gla_mlstm_fwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                         const float* itil, void* h, void* ws, size_t ws_bytes, void* stream) {
    return gla::ml_fwd_entry(p, q, k, v, g, itil, h, nullptr, ws, ws_bytes, stream);
}

gla_status gla_mlstm_fwd_save(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                              const float* itil, void* h, void* saved, void* ws, size_t ws_bytes, void* stream) {
    return gla::ml_fwd_entry(p, q, k, v, g, itil, h, saved, ws, ws_bytes, stream);
}

gla_status gla_mlstm_bwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                         const float* itil, const void* dh, void* dq, void* dk, void* dv, float* dg, float* ditil,
                         void* ws, size_t ws_bytes, void* stream) {
    return gla::ml_bwd_entry(p, q, k, v, g, itil, dh, nullptr, dq, dk, dv, dg, ditil, ws, ws_bytes, stream);
}

gla_status gla_mlstm_bwd_saved(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                               const float* itil, const void* dh, const void* saved, void* dq, void* dk, void* dv,
                               float* dg, float* ditil, void* ws, size_t ws_bytes, void* stream) {
    return gla::ml_bwd_entry(p, q, k, v, g, itil, dh, saved, dq, dk, dv, dg, ditil, ws, ws_bytes, stream);
}

}  // extern "C"
