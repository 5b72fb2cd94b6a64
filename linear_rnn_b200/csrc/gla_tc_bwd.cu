// Tensor-core (tcgen05 / TMEM / TMA) backward of chunkwise gated linear attention, bf16 I/O.
//
// Per 64-token tile, with b the in-tile cumulative log-gate, Gamma its total, k' = i k,
// q~ = q e^b, k~ = k' e^-b, S the state before the tile and G = dL/dS after it (the
// chunkwise backward restated from the forward of the talk summary "Hardware-Efficient
// Training of Linear Attention Models", section 11:58, with the GLA abstract's gates):
//   dq   = scale e^b * ( dO S^T + mask(dO V^T) k~ )
//   G~   = diag(e^Gamma) G
//   dk'  = e^-b * ( mask(dO V^T)^T (scale q~) + V G~^T ),   dk = i dk'
//   dv   = mask(scale q~ k~^T)^T dO + k~ G~
//   G_prev = G~ + (scale q~)^T dO
//   dg   = reverse cumulative sum over the whole sequence of q*dq - k*dk (+ sum_e dhT*hT),
//          (k*dk = k'*dk' because dk = i dk')
// Kernels:
//   tc_bwd_dq    forward tile walk per (b*h, key-dim block, segment); S in TMEM (fp32, the
//                state MMA accumulates onto it, a TMEM pass applies e^Gamma) and bf16 in
//                shared memory as the B operand of dO S^T.
//   tc_bwd_dkdv  reverse tile walk per (b*h, segment); G in TMEM, bf16 G~ in shared memory.
//                Dk = 256 (G does not fit one SM's TMEM next to the accumulators): a cluster
//                of two CTAs per (b*h, segment), CTA kb holding G's key rows [128 kb, 128 kb
//                + 128). Everything but dv (and the per-row sums behind di and a per-head dg)
//                is complete in each CTA, because key dims only meet in those contractions;
//                each CTA owns half of dv's value dims, receives the other CTA's partial sum
//                of them into its shared memory (distributed shared memory, fp32) and adds it.
// dg in fp32 without a separate pass: the dq kernel writes the in-segment exclusive prefix
// of q*dq (into the dg buffer) and its segment total; the dk/dv kernel forms the in-segment
// reverse sum of k*dk and finishes dg_t = (total - prefix_t) - revsum_t + carry, where the
// carry (everything after the segment, incl. the final-state term) is
// sum_e G_end[d][e] S_end[d][e]: adding a constant to the log-gate at the segment's first
// token scales the state entering it, so that sum is exactly the gradient of the
// shifted cumulative decay.
// Segment boundary states come from the forward state pass + scan; segment boundary
// state gradients from the reverse state pass (gla_tc_fwd.cu, mode 2) + reverse scan.
#include <mutex>

#include "gla_plans.h"
#include "gla_tc_common.cuh"

namespace gla {
namespace tc {

using namespace sm100;

constexpr int NT_B = 256;  // 8 warps: two warpgroups; thread 0 also issues TMA and MMA

struct BwdArgs {
    const __nv_bfloat16 *q, *k, *v, *dO;   // inputs (L2 prefetches of whole tile rows)
    const float* g;       // per-key log-gate [BH*L*Dk] (L2 prefetch) or null
    const float* gh;      // per-head log-gate [BH*L]
    const float* ig;      // input gate [BH*L] or null
    const float* sinit;   // initial state per (bh, segment) [BH, nseg, Dk, Dv] or null (then h0 / 0)
    const float* h0;
    const float* gend;    // state gradient at the end of each segment [BH, nseg, Dk, Dv] or null (then dhT / 0)
    const float* dhT;
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* di;            // [BH*L] or null
    float* dh0;           // [BH, Dk, Dv] or null
    float* hT_ws;         // final state (for the dg term) or null
    float* dg;            // dg output; the dq kernel first stores there the in-segment
                          // exclusive prefix of q*dq, the dk/dv kernel finishes it
    float* tq;            // [BH, nseg, Dk] in-segment totals of q*dq (per-head gates: the
                          // total of key block kb at key index 128 kb)
    float* pre;           // per-head gates: [key blocks][BH*L] in-segment exclusive prefixes of
                          // q*dq, one row per key block (the dg buffer when there is one block)
    int* status;
    int tiles_per_seg;
    int nseg;
};

__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __syncthreads_and(ok) != 0;
}
__device__ __forceinline__ float4 f4_add(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 f4_zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
// four consecutive key dims d..d+3 (d a multiple of 4) of row r of a swizzled fp32 tile (gsw)
__device__ __forceinline__ float4 gsw_ld4(const float* sg, int r, int d) {
    return *reinterpret_cast<const float4*>(sg + gsw(r, d));
}

// The same for a barrier that the other CTA of the cluster arrives on.
__device__ __forceinline__ bool block_wait_cluster(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait_cluster(bar, parity);
    return __syncthreads_and(ok) != 0;
}

// Tile rows [t, t + 64) (clipped at L) of the inputs of CTA (bh, key block kb of nkb) into L2,
// one contiguous bulk prefetch per tensor (a tile's rows are contiguous in the BHLD layout);
// the first key block fetches q, k, g, the last v and dO.
__device__ __forceinline__ void prefetch_tile_rows(const BwdArgs& A, const Dims& P, long rowbase, int t, int kb,
                                                   int nkb, bool with_q) {
    if (t >= P.L) return;
    const long r0 = rowbase + t;
    const uint32_t rows = (uint32_t)min(TR, P.L - t);
    if (kb == 0) {
        if (with_q) prefetch_l2_bulk(A.q + r0 * P.Dk, rows * P.Dk * 2);
        prefetch_l2_bulk(A.k + r0 * P.Dk, rows * P.Dk * 2);
        if (A.g) prefetch_l2_bulk(A.g + r0 * P.Dk, rows * P.Dk * 4);
    }
    if (kb == nkb - 1) {
        prefetch_l2_bulk(A.v + r0 * P.Dv, rows * P.Dv * 2);
        prefetch_l2_bulk(A.dO + r0 * P.Dv, rows * P.Dv * 2);
    }
}

__device__ __forceinline__ void store16_bf16_global(__nv_bfloat16* dst, const float* v) {
    uint32_t w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
        w[u] = *reinterpret_cast<uint32_t*>(&p);
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

constexpr uint32_t pow2cols(uint32_t n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512; }

// In-place transform of one 64-token tile by all NT_B threads:
//   step A (per-key gates): b = column cumsum of the log-gate in row segments (thread = key
//     dim x segment) joined through the segment totals, written over g; gam[d] = e^Gamma;
//   step B: every 16-byte chunk (8 key dims of one row): k~ = i * k * e^-b (k tile),
//     DO_Q: q~ = scale * q * e^b (q tile), and the g slot keeps e^b (G_SLOT_EB) or e^-b.
// Per-head gates use the row factors rowE / rowEi (warp 0 scans the 64 gates) instead.
// Both backward kernels use this one routine so they form bit-identical q~ and k~. The g tile
// is in the swizzled fp32 layout (gsw).
//
// Per-key gates (GATE 1) run it in one pass instead: thread = key-dim pair x run of RSF rows;
// the column cumsum of its rows stays in registers, the run totals are exchanged once, and each
// row's k (and q) pair is scaled right away, with the products formed in the same order as
// above ((k i) e^-b, (q scale) e^b) so that both kernels, and the dq kernel's q*dq, see the same
// bf16 values.
template <int D, bool DO_Q, bool G_SLOT_EB>
__device__ __forceinline__ void bwd_transform_key(uint8_t* sq, uint8_t* sk, float* sg, float* tot, float* gam,
                                                  const float* igs, float scale, int tid, int* status) {
    constexpr int NP = D / 2, SEGF = NT_B / NP, RSF = TR / SEGF;
    static_assert(NT_B % NP == 0 && TR % SEGF == 0 && SEGF * NP * 2 <= 2048, "fused transform mapping");
    const int p = tid % NP, sgi = tid / NP, d0 = 2 * p;
    float2* tot2 = reinterpret_cast<float2*>(tot);   // [SEGF][NP] run totals
    float2 cs[RSF];
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < RSF; ++u) {
        const float2 x = *reinterpret_cast<const float2*>(sg + gsw(sgi * RSF + u, d0));
        acc.x += x.x;
        acc.y += x.y;
        cs[u] = acc;
    }
    tot2[sgi * NP + p] = acc;
    __syncthreads();
    float2 off = make_float2(0.f, 0.f), G = make_float2(0.f, 0.f);
#pragma unroll
    for (int s2 = 0; s2 < SEGF; ++s2) {
        const float2 t = tot2[s2 * NP + p];
        if (s2 < sgi) {
            off.x += t.x;
            off.y += t.y;
        }
        G.x += t.x;
        G.y += t.y;
    }
    if (sgi == 0) {
        gam[d0] = __expf(G.x);
        gam[d0 + 1] = __expf(G.y);
        if (G.x < kMinTileLogDecay || G.y < kMinTileLogDecay) atomicOr(status, kDevStatusRange);
    }
#pragma unroll
    for (int u = 0; u < RSF; ++u) {
        const int r = sgi * RSF + u;
        const float ex = __expf(cs[u].x + off.x), ey = __expf(cs[u].y + off.y);
        const float dx = rcp_approx(ex), dy = rcp_approx(ey);
        *reinterpret_cast<float2*>(sg + gsw(r, d0)) = G_SLOT_EB ? make_float2(ex, ey) : make_float2(dx, dy);
        // byte offset of (r, d0) in a 128-byte-swizzled bf16 tile
        const uint32_t ob = (uint32_t)(d0 >> 6) * BLK + (uint32_t)r * 128 +
                            ((((uint32_t)((d0 & 63) >> 3)) ^ (uint32_t)(r & 7)) << 4) + (uint32_t)(d0 & 7) * 2;
        const float iv = igs[r];
        __nv_bfloat162* pk = reinterpret_cast<__nv_bfloat162*>(sk + ob);
        const float2 kf = __bfloat1622float2(*pk);
        *pk = __floats2bfloat162_rn(kf.x * iv * dx, kf.y * iv * dy);
        if (DO_Q) {
            __nv_bfloat162* pq = reinterpret_cast<__nv_bfloat162*>(sq + ob);
            const float2 qf = __bfloat1622float2(*pq);
            *pq = __floats2bfloat162_rn(qf.x * scale * ex, qf.y * scale * ey);
        }
    }
}

template <int D, int GATE, bool DO_Q, bool G_SLOT_EB>
__device__ __forceinline__ void bwd_transform(uint8_t* sq, uint8_t* sk, float* sg, float* tot, float* gam,
                                              float* rowE, float* rowEi, const float* ghs, const float* igs,
                                              float scale, int tid, int* status) {
    if constexpr (GATE == 1 && D <= 128) {
        bwd_transform_key<D, DO_Q, G_SLOT_EB>(sq, sk, sg, tot, gam, igs, scale, tid, status);
        return;
    }
    constexpr int SEG = NT_B / D, RS = TR / SEG;   // step A
    constexpr int NO = D / 8, NPOS = TR * NO;       // step B
    constexpr int NB = 2;
    static_assert(NT_B % D == 0 && NPOS % (NB * NT_B) == 0, "transform mapping");
    const int warp = tid >> 5, lane = tid & 31;
    if (GATE == 1) {
        const int dA = tid % D, sA = tid / D;
        float x[RS];
#pragma unroll
        for (int u = 0; u < RS; ++u) x[u] = sg[gsw(sA * RS + u, dA)];
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < RS; ++u) {
            acc += x[u];
            x[u] = acc;
        }
        float off = 0.f, G = acc;
        if constexpr (SEG > 1) {
            tot[tid] = acc;
            __syncthreads();
            G = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < SEG; ++s2) {
                const float t = tot[s2 * D + dA];
                if (s2 < sA) off += t;
                G += t;
            }
        }
#pragma unroll
        for (int u = 0; u < RS; ++u) sg[gsw(sA * RS + u, dA)] = x[u] + off;
        if (sA == 0) {
            gam[dA] = __expf(G);
            if (G < kMinTileLogDecay) atomicOr(status, kDevStatusRange);
        }
    } else if (GATE == 2 && warp == 0) {
        const float g0 = ghs[2 * lane], g1 = ghs[2 * lane + 1];
        float v = g0 + g1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += n;
        }
        const float b1 = v, b0 = v - g1;
        rowE[2 * lane] = __expf(b0);
        rowE[2 * lane + 1] = __expf(b1);
        rowEi[2 * lane] = __expf(-b0);
        rowEi[2 * lane + 1] = __expf(-b1);
        const float G = __shfl_sync(0xffffffffu, b1, 31);
        if (lane == 0) {
            gam[0] = __expf(G);
            if (G < kMinTileLogDecay) atomicOr(status, kDevStatusRange);
        }
    }
    __syncthreads();
#pragma unroll
    for (int it0 = 0; it0 < NPOS / NT_B; it0 += NB) {
        float bv[NB][8];
        uint4 wq[NB], wk[NB];
        uint32_t offs[NB];
        int rows[NB], d0s[NB];
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            const int c = tid + (it0 + k) * NT_B;
            const int r = c / NO, d0 = 8 * (c % NO);
            rows[k] = r;
            d0s[k] = d0;
            if (GATE == 1) {
                const float4 b0 = *reinterpret_cast<const float4*>(sg + gsw(r, d0));
                const float4 b1 = *reinterpret_cast<const float4*>(sg + gsw(r, d0 + 4));
                bv[k][0] = b0.x; bv[k][1] = b0.y; bv[k][2] = b0.z; bv[k][3] = b0.w;
                bv[k][4] = b1.x; bv[k][5] = b1.y; bv[k][6] = b1.z; bv[k][7] = b1.w;
            }
            offs[k] = (uint32_t)(d0 >> 6) * BLK + (uint32_t)r * 128 +
                      ((((uint32_t)((d0 & 63) >> 3)) ^ (uint32_t)(r & 7)) << 4);
            if (DO_Q) wq[k] = *reinterpret_cast<const uint4*>(sq + offs[k]);
            wk[k] = *reinterpret_cast<const uint4*>(sk + offs[k]);
        }
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            const int r = rows[k], d0 = d0s[k];
            float eq[8], ek[8];
            if (GATE == 1) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    eq[u] = __expf(bv[k][u]);
                    ek[u] = rcp_approx(eq[u]);
                }
                const float* keep = G_SLOT_EB ? eq : ek;
                *reinterpret_cast<float4*>(sg + gsw(r, d0)) = make_float4(keep[0], keep[1], keep[2], keep[3]);
                *reinterpret_cast<float4*>(sg + gsw(r, d0 + 4)) = make_float4(keep[4], keep[5], keep[6], keep[7]);
            } else {
                const float e1 = GATE == 2 ? rowE[r] : 1.f, e2 = GATE == 2 ? rowEi[r] : 1.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    eq[u] = e1;
                    ek[u] = e2;
                }
            }
            const float iv = igs[r];
            uint32_t* pk = reinterpret_cast<uint32_t*>(&wk[k]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pk[u]));
                __nv_bfloat162 h = __floats2bfloat162_rn(f.x * iv * ek[2 * u], f.y * iv * ek[2 * u + 1]);
                pk[u] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(sk + offs[k]) = wk[k];
            if (DO_Q) {
                uint32_t* pq = reinterpret_cast<uint32_t*>(&wq[k]);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pq[u]));
                    __nv_bfloat162 h = __floats2bfloat162_rn(f.x * scale * eq[2 * u], f.y * scale * eq[2 * u + 1]);
                    pq[u] = *reinterpret_cast<uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(sq + offs[k]) = wq[k];
            }
        }
    }
}

// ============================================================================ dq
template <int DKB, int DV, int GATE>
struct QCfg {
    static constexpr uint32_t QB = GATE != 0 ? TR * DKB * 2 : 0;  // raw q (for q*dq)
    static constexpr uint32_t KB = TR * DKB * 2;
    static constexpr uint32_t GB = GATE != 0 ? TR * DKB * 4 : 0;  // g (per key), then q*dq scratch
    static constexpr uint32_t VB = TR * DV * 2;
    static constexpr uint32_t OB = TR * DV * 2;
    static constexpr uint32_t STAGE = QB + KB + GB + VB + OB;
    static constexpr uint32_t TXA = QB + KB + (GATE == 1 ? GB : 0);  // bytes of the q, k, g loads
    static constexpr uint32_t TXV = VB + OB;                         // bytes of the v, dO loads
    static constexpr uint32_t SB = DKB * DV * 2;
    static constexpr uint32_t AB = TR * TR * 2;
    static constexpr uint32_t SMALL = 256 + 8192 + 8 * DKB + 1024 + 512;
    static constexpr int NS = (2 * STAGE + SB + AB + SMALL + 1024 <= 227 * 1024) ? 2 : 1;
    static constexpr uint32_t SMEM = NS * STAGE + SB + AB + SMALL + 1024;
    // TMEM: S [0, DV). From COL_R the M=64 accumulators of D = dO S^T + mask(dA) k~ (rows in
    // lanes 16-31) and dA (lanes 0-15); with SPLIT, D's two column halves sit in lanes 0-15 and
    // 16-31 of the same columns, so that every lane of the epilogue holds a row, and dA follows.
    static constexpr bool SPLIT = DKB == 128;
    static constexpr uint32_t COL_R = DV;
    static constexpr uint32_t COL_A = SPLIT ? COL_R + DKB / 2 : COL_R;
    static constexpr uint32_t NCOL = pow2cols(DV + (SPLIT ? DKB / 2 + 64 : (DKB > 64 ? DKB : 64)));
    static constexpr int HC = DV / 2;    // state columns per warpgroup
    static constexpr int QC = SPLIT ? DKB / 4 : DKB / 2;   // D columns (TMEM) per warpgroup
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0, "stage alignment");
};

template <int DKB, int DV, int GATE>
__global__ void __launch_bounds__(NT_B, 1)
    k_tc_bwd_dq(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tg, const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tout, BwdArgs A,
                Dims P) {
    using C = QCfg<DKB, DV, GATE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_align1024(smem_raw);
    uint8_t* sS = sm + C::NS * C::STAGE;
    uint8_t* sA = sS + C::SB;
    uint8_t* small = sA + C::AB;
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(small);  // [2]
    uint64_t* bar_mma1 = bar_full + 2;
    uint64_t* bar_mma2 = bar_full + 3;
    uint64_t* bar_drain = bar_full + 4;   // error path: completion of every product issued
    uint64_t* bar_fullv = bar_full + 5;   // [2] v and dO landed (bar_full: q, k, g)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + 64);
    float* tot = reinterpret_cast<float*>(small + 256);
    float* gam = tot + 2048;            // [DKB]
    float* rowE = gam + DKB;            // [64]
    float* rowEi = rowE + TR;
    float* igs = rowEi + TR;
    float* ghs = igs + TR;
    float* carry = ghs + TR;            // [DKB] running in-segment sum of q*dq per key dim
    float* rows = carry + DKB;          // [64] per-row sums (per-head gate)

    const int bh = blockIdx.x, kb = blockIdx.y, z = blockIdx.z;
    const int d0 = kb * DKB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2, qd = warp & 3;
    const int ntiles_all = cdiv(P.L, TR);
    const int tile0 = z * A.tiles_per_seg;
    const int ntiles = min(ntiles_all, tile0 + A.tiles_per_seg) - tile0;
    const long rowbase = (long)bh * P.L;
    const bool srow_ok = (DKB != 64) || (lane < 16);
    const int srow = DKB == 64 ? 16 * qd + (lane & 15) : 32 * qd + lane;

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        mbar_init(bar_drain, 1);
        mbar_init(&bar_fullv[0], 1);
        mbar_init(&bar_fullv[1], 1);
        mbar_fence_init();
    }
    if (tid < DKB) carry[tid] = 0.f;
    if (warp == 0) tmem_alloc(tmem_slot, C::NCOL);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(32 * qd) << 16);

    // ---- initial state into TMEM (fp32) and shared memory (bf16)
    {
        const float* src = nullptr;
        if (z == 0) src = A.h0 ? A.h0 + ((long)bh * P.Dk + d0) * P.Dv : nullptr;
        else src = A.sinit + (((long)bh * A.nseg + z) * P.Dk + d0) * P.Dv;
        // staged through the ring stages (free until the first tile's loads), in column halves
        // where the whole block does not fit
        constexpr int CW = (DKB * DV * 4 <= C::NS * C::STAGE) ? DV : DV / 2;
        static_assert(DKB * CW * 4 <= C::NS * C::STAGE, "state staging");
        float* stg = reinterpret_cast<float*>(sm);
        for (int c0 = 0; c0 < DV; c0 += CW) {
            if (src) {
                stage_rows<DKB, CW, NT_B>(stg, src + c0, nullptr, P.Dv, nullptr, tid);
                __syncthreads();
            }
            for (int c = wg * C::HC; c < (wg + 1) * C::HC; c += 16) {
                if (c < c0 || c >= c0 + CW) continue;
                float f[16];
                if (src && srow_ok) staged_row16<CW>(stg, srow, c - c0, f);
                else
#pragma unroll
                    for (int j = 0; j < 16; ++j) f[j] = 0.f;
                tmem_st16(tlane + c, reinterpret_cast<uint32_t*>(f));
                if (srow_ok) {
                    store8_bf16(sS, sw128_off(srow, c, DKB * 128), f);
                    store8_bf16(sS, sw128_off(srow, c + 8, DKB * 128), f + 8);
                }
            }
            if (src) __syncthreads();   // the next column block overwrites the staging
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // q, k, g of a tile are read until its epilogue ends; v and dO only by the first product
    // group, so the next tile's v and dO are loaded as soon as that group completes
    auto issue_qkg = [&](int i, int s) {
        uint8_t* st = sm + s * C::STAGE;
        const int t0 = (tile0 + i) * TR;
        mbar_arrive_expect_tx(&bar_full[s], C::TXA);
        for (int cb = 0; cb < DKB / 64; ++cb) {
            if (GATE != 0) tma_load_3d(st + cb * BLK, &tq, d0 + cb * 64, t0, bh, &bar_full[s]);
            tma_load_3d(st + C::QB + cb * BLK, &tk, d0 + cb * 64, t0, bh, &bar_full[s]);
        }
        if (GATE == 1)
            for (int gb = 0; gb < DKB / 32; ++gb)
                tma_load_3d(st + C::QB + C::KB + gb * BLK, &tg, d0 + 32 * gb, t0, bh, &bar_full[s]);
    };
    // tile i into L2, ahead of its loads (issued by another warp than the loads and products)
    auto issue_prefetch = [&](int i) {
        prefetch_tile_rows(A, P, rowbase, (tile0 + i) * TR, kb, P.Dk / DKB, GATE != 0);
    };
    auto issue_vo = [&](int i, int s) {
        uint8_t* st = sm + s * C::STAGE;
        const int t0 = (tile0 + i) * TR;
        mbar_arrive_expect_tx(&bar_fullv[s], C::TXV);
        for (int vb = 0; vb < DV / 64; ++vb) {
            tma_load_3d(st + C::QB + C::KB + C::GB + vb * BLK, &tv, vb * 64, t0, bh, &bar_fullv[s]);
            tma_load_3d(st + C::QB + C::KB + C::GB + C::VB + vb * BLK, &tdo, vb * 64, t0, bh, &bar_fullv[s]);
        }
    };
    if (tid == 0)
        for (int i = 0; i < C::NS && i < ntiles; ++i) {
            issue_qkg(i, i);
            issue_vo(i, i);
        }
    if (tid == 32)
        for (int i = C::NS; i < 2 * C::NS && i < ntiles; ++i) issue_prefetch(i);
    // input and per-head gates of the next tile, loaded a tile ahead into registers
    float nig = 1.f, ngh = 0.f;
    auto fetch_gates = [&](int i) {
        const int t = (tile0 + i) * TR + tid;
        if (A.ig) nig = t < P.L ? A.ig[rowbase + t] : 1.f;
        if (GATE == 2) ngh = t < P.L ? A.gh[rowbase + t] : 0.f;
    };
    if (tid < TR) fetch_gates(0);

    int err = 0, n_mma = 0;
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::NS;
        uint8_t* st = sm + s * C::STAGE;
        uint8_t* sqr = st;
        uint8_t* sk = st + C::QB;
        float* sg = reinterpret_cast<float*>(st + C::QB + C::KB);
        uint8_t* sv = st + C::QB + C::KB + C::GB;
        uint8_t* so = sv + C::VB;
        const int t0 = (tile0 + i) * TR;
        if (tid < TR) {
            igs[tid] = nig;
            if (GATE == 2) ghs[tid] = ngh;
            if (i + 1 < ntiles) fetch_gates(i + 1);
        }
        if (!block_wait(&bar_full[s], (i / C::NS) & 1)) { err = 1; break; }

        // ---- transform: k~ = i k e^-b in place; e^b kept (in place of g) for the dq epilogue
        bwd_transform<DKB, GATE, false, true>(sqr, sk, sg, tot, gam, rowE, rowEi, ghs, igs, P.scale, tid, A.status);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (!block_wait(&bar_fullv[s], (i / C::NS) & 1)) { err = 1; break; }

        // ---- MMA group 1: dA = dO V^T, D = dO S^T, S += k~^T V
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t ka = smem_u32(sk), va = smem_u32(sv), oa = smem_u32(so), sa = smem_u32(sS);
            const uint32_t idA = idesc_bf16(64, 64, 0, 0), idQ = idesc_bf16(64, C::SPLIT ? DKB / 2 : DKB, 0, 0);
            const uint32_t idS = idesc_bf16(DKB, DV, 1, 1);
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader) mma_bf16(tbase + C::COL_A, sw128_desc(oa + koff, 16, 1024), sw128_desc(va + koff, 16, 1024), idA,
                         kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                const uint32_t soff = (kk >> 2) * (DKB * 128) + (kk & 3) * 32;
                if (C::SPLIT) {
                    // key dims [0, 64) into lanes 0-15, [64, 128) (state rows 64 on) into lanes 16-31
                    if (leader) mma_bf16(tbase + C::COL_R, sw128_desc(oa + koff, 16, 1024), sw128_desc(sa + soff, 16, 1024),
                             idQ, kk > 0);
                    if (leader) mma_bf16(tbase + (16u << 16) + C::COL_R, sw128_desc(oa + koff, 16, 1024),
                             sw128_desc(sa + soff + (DKB / 2) * 128, 16, 1024), idQ, kk > 0);
                } else {
                    if (leader) mma_bf16(tbase + (16u << 16) + C::COL_R, sw128_desc(oa + koff, 16, 1024),
                             sw128_desc(sa + soff, 16, 1024), idQ, kk > 0);
                }
            }
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks)
                if (leader) mma_bf16(tbase, sw128_desc(ka + ks * 2048, BLK, 1024), sw128_desc(va + ks * 2048, BLK, 1024), idS, 1);
            if (leader) mma_commit(bar_mma1);
            __syncwarp();
        } else if (tid == 32 && i + 2 * C::NS < ntiles) {
            issue_prefetch(i + 2 * C::NS);   // while warp 0 issues the products
        }
        ++n_mma;
        if (!block_wait(bar_mma1, i & 1)) { err = 1; break; }
        tc_fence_after();
        if (tid == 0 && i + C::NS < ntiles) issue_vo(i + C::NS, s);

        // ---- masked dA -> shared; state pass S = e^Gamma (S + dS') in TMEM, bf16 copy
        {
            uint32_t r[32];
            tmem_ld32(tlane + C::COL_A + 32 * wg, r);
            tmem_wait_ld();
            if (lane < 16) {
                const int t = 16 * qd + lane;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int sidx = 32 * wg + 8 * u + j;
                        f[j] = (sidx <= t) ? __uint_as_float(r[8 * u + j]) : 0.f;
                    }
                    store8_bf16(sA, sw128_off(t, 32 * wg + 8 * u, BLK), f);
                }
            }
        }
        {
            const float eg = GATE == 0 ? 1.f : gam[GATE == 1 ? srow : 0];
            const uint64_t eg2 = f2(eg, eg);
            for (int c = wg * C::HC; c < (wg + 1) * C::HC; c += 32) {
                uint32_t r[32];
                float f[32];
                tmem_ld32(tlane + c, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const uint64_t x = f2_mul(f2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), eg2);
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(f[j]), "=f"(f[j + 1]) : "l"(x));
                    r[j] = __float_as_uint(f[j]);
                    r[j + 1] = __float_as_uint(f[j + 1]);
                }
                tmem_st32(tlane + c, r);
                if (srow_ok)
#pragma unroll
                    for (int j = 0; j < 32; j += 8) store8_bf16(sS, sw128_off(srow, c + j, DKB * 128), f + j);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- MMA group 2: D += mask(dA) k~
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t aa = smem_u32(sA), ka = smem_u32(sk);
            const uint32_t idQ = idesc_bf16(64, C::SPLIT ? DKB / 2 : DKB, 0, 1);
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks) {
                if (C::SPLIT) {   // key-dim blocks 0 and 1 of k~ into the two lane halves
                    if (leader) mma_bf16(tbase + C::COL_R, sw128_desc(aa + ks * 32, 16, 1024),
                             sw128_desc(ka + ks * 2048, BLK, 1024), idQ, 1);
                    if (leader) mma_bf16(tbase + (16u << 16) + C::COL_R, sw128_desc(aa + ks * 32, 16, 1024),
                             sw128_desc(ka + BLK + ks * 2048, BLK, 1024), idQ, 1);
                } else {
                    if (leader) mma_bf16(tbase + (16u << 16) + C::COL_R, sw128_desc(aa + ks * 32, 16, 1024),
                             sw128_desc(ka + ks * 2048, BLK, 1024), idQ, 1);
                }
            }
            if (leader) mma_commit(bar_mma2);
            __syncwarp();
        }
        if (!block_wait(bar_mma2, i & 1)) { err = 1; break; }
        tc_fence_after();

        // ---- dq = scale e^b D -> bf16 tile staged in the k slot (k~ is no longer read) -> TMA
        //      store; q*dq into the g slot for dg. Row t of D sits in lane (t % 16) of quadrant
        //      t / 16, lanes 16-31 (SPLIT: lanes 0-15 hold key dims [0, DKB/2), 16-31 the rest);
        //      the g slot holds e^b in the swizzled fp32 layout (gsw).
        {
            const int t = 16 * qd + (lane & 15);
            const bool row_ok = t0 + t < P.L;
            uint8_t* sdq = sk;
            float rsum = 0.f;   // per-head gates: this lane's part of the row's sum of q*dq
            for (int ct = wg * C::QC; ct < (wg + 1) * C::QC; ct += 16) {
                uint32_t r[16];
                tmem_ld16(tlane + C::COL_R + ct, r);
                tmem_wait_ld();
                const int c = C::SPLIT ? (lane >> 4) * (DKB / 2) + ct : ct;   // key dim of r[0]
                if (C::SPLIT || lane >= 16) {
                    float eb[16];
                    if (GATE == 1) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 e4 = *reinterpret_cast<const float4*>(sg + gsw(t, c + 4 * q4));
                            eb[4 * q4] = e4.x; eb[4 * q4 + 1] = e4.y; eb[4 * q4 + 2] = e4.z; eb[4 * q4 + 3] = e4.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) eb[j] = GATE == 2 ? rowE[t] : 1.f;
                    }
                    float f[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) f[j] = P.scale * eb[j] * __uint_as_float(r[j]);
                    store8_bf16(sdq, sw128_off(t, c, BLK), f);
                    store8_bf16(sdq, sw128_off(t, c + 8, BLK), f + 8);
                    if (GATE != 0) {
                        // q*dq, formed as bf16(scale q e^b) * D with the rounding the dk/dv kernel
                        // applies to q~, so the pairwise cancellation inside dg's reverse sum survives
                        uint4 qw[2];
                        qw[0] = *reinterpret_cast<const uint4*>(sqr + sw128_off(t, c, BLK));
                        qw[1] = *reinterpret_cast<const uint4*>(sqr + sw128_off(t, c + 8, BLK));
                        const uint32_t* qp = reinterpret_cast<const uint32_t*>(qw);
                        float x[16];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qp[u]));
                            const float qs0 = __bfloat162float(__float2bfloat16_rn(qf.x * P.scale * eb[2 * u]));
                            const float qs1 = __bfloat162float(__float2bfloat16_rn(qf.y * P.scale * eb[2 * u + 1]));
                            x[2 * u] = row_ok ? qs0 * __uint_as_float(r[2 * u]) : 0.f;
                            x[2 * u + 1] = row_ok ? qs1 * __uint_as_float(r[2 * u + 1]) : 0.f;
                            rsum += x[2 * u] + x[2 * u + 1];
                        }
                        if (GATE == 1)
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                *reinterpret_cast<float4*>(sg + gsw(t, c + 4 * q4)) =
                                    make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
                    }
                }
            }
            if (GATE == 2) {   // the row's sum over this warpgroup's key dims (tot is free here)
                if (C::SPLIT) rsum += __shfl_xor_sync(0xffffffffu, rsum, 16);
                if (C::SPLIT ? lane < 16 : lane >= 16) tot[wg * TR + t] = rsum;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            for (int cb = 0; cb < DKB / 64; ++cb) tma_store_3d(&tout, sk + cb * BLK, d0 + 64 * cb, t0, bh);
            bulk_commit();
        }
        // ---- in-segment exclusive prefix of q*dq (fp32) into the dg buffer
        if (GATE == 1) {
            // thread = (key dims dc..dc+3, group of RPR rows): local sums, exchange, then the
            // prefix walk with 16-byte stores
            constexpr int NC4 = DKB / 4, NGR = NT_B / NC4, RPR = TR / NGR;
            const int c4 = tid % NC4, gr = tid / NC4, dc = 4 * c4;
            float4* tot4 = reinterpret_cast<float4*>(tot);
            float4* carry4 = reinterpret_cast<float4*>(carry);
            float4 x[RPR];   // the thread's rows of q*dq, read once
            float4 loc = f4_zero();
#pragma unroll
            for (int rr = 0; rr < RPR; ++rr) {
                x[rr] = gsw_ld4(sg, gr * RPR + rr, dc);
                loc = f4_add(loc, x[rr]);
            }
            tot4[gr * NC4 + c4] = loc;
            __syncthreads();
            float4 px = carry4[c4], T = f4_zero();
#pragma unroll
            for (int g2 = 0; g2 < NGR; ++g2) {
                const float4 v = tot4[g2 * NC4 + c4];
                if (g2 < gr) px = f4_add(px, v);
                T = f4_add(T, v);
            }
            float4* dgp = reinterpret_cast<float4*>(A.dg + (rowbase + t0 + gr * RPR) * P.Dk + d0 + dc);
#pragma unroll
            for (int rr = 0; rr < RPR; ++rr) {
                if (t0 + gr * RPR + rr < P.L) dgp[(long)rr * (P.Dk / 4)] = px;
                px = f4_add(px, x[rr]);
            }
            __syncthreads();
            if (gr == 0) carry4[c4] = f4_add(carry4[c4], T);
        } else if (GATE == 2) {
            __syncthreads();
            if (tid < TR) rows[tid] = tot[tid] + tot[TR + tid];
            __syncthreads();
            if (warp == 0) {  // exclusive scan over 64 rows, two per lane
                const float a0 = rows[2 * lane], a1 = rows[2 * lane + 1];
                float v = a0 + a1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float n = __shfl_up_sync(0xffffffffu, v, off);
                    if (lane >= off) v += n;
                }
                const float base = carry[0];
                const float e0 = base + v - a0 - a1, e1 = base + v - a1;
                float* pre = A.pre + (long)kb * P.B * P.H * P.L + rowbase + t0;
                if (t0 + 2 * lane < P.L) pre[2 * lane] = e0;
                if (t0 + 2 * lane + 1 < P.L) pre[2 * lane + 1] = e1;
                const float total = __shfl_sync(0xffffffffu, v, 31);
                __syncwarp();
                if (lane == 0) carry[0] = base + total;
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) bulk_wait_read<0>();   // the dq store has read the k slot before it is reloaded
        if (tid == 0 && i + C::NS < ntiles) issue_qkg(i + C::NS, s);
    }

    if (!err) {
        __syncthreads();
        if (GATE == 1 && tid < DKB) A.tq[((long)bh * A.nseg + z) * P.Dk + d0 + tid] = carry[tid];
        if (GATE == 2 && tid == 0) A.tq[((long)bh * A.nseg + z) * P.Dk + d0] = carry[0];
    }
    if (err) {
        if (warp == 0) {
            // every product the issuing lane issued completes before TMEM and shared memory go away
            const bool leader = elect_one();
            if (leader) {
                atomicOr(A.status, kDevStatusTimeout);
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0, 1u << 20);
            }
            __syncwarp();
        }
    } else if (A.hT_ws && z == A.nseg - 1) {
        // final state (for the dg term of an upstream final-state gradient)
        for (int c = wg * C::HC; c < (wg + 1) * C::HC; c += 16) {
            uint32_t r[16];
            tmem_ld16(tlane + c, r);
            tmem_wait_ld();
            if (srow_ok) {
                float* dst = A.hT_ws + ((long)bh * P.Dk + d0 + srow) * P.Dv + c;
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                                      __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            }
        }
    }
    if (tid == 0) bulk_wait<0>();   // the last output stores have completed
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, C::NCOL);
}

// ============================================================================ dk, dv
template <int DK, int DV, int GATE>
struct KVCfg {
    static constexpr uint32_t QB = TR * DK * 2;
    static constexpr uint32_t KB = TR * DK * 2;
    static constexpr uint32_t GB = TR * DK * 4;  // g (per key: loaded; e^-b after the transform), k*dk scratch
    static constexpr uint32_t VB = TR * DV * 2;
    static constexpr uint32_t OB = TR * DV * 2;
    static constexpr uint32_t STAGE = QB + KB + GB + VB + OB;
    static constexpr uint32_t TXB = STAGE - (GATE == 1 ? 0 : GB);
    static constexpr uint32_t GTB = DK * DV * 2;
    static constexpr uint32_t AB = TR * TR * 2;
    static constexpr uint32_t SMALL = 256 + 8192 + 4 * DK + 1024 + 512 + 16 * DK + 256 + 64;
    static constexpr int NS = (2 * STAGE + GTB + 2 * AB + SMALL + 1024 <= 227 * 1024) ? 2 : 1;
    static constexpr uint32_t SMEM = NS * STAGE + GTB + 2 * AB + SMALL + 1024;
    // TMEM: G [0, DV); from COL_R the dv accumulator (lanes 16-31, DV columns) and, in lanes
    // 0-15, the dk' accumulator (DK columns) followed by A and dA (64 columns each)
    static constexpr uint32_t COL_R = DV;
    static constexpr uint32_t COL_A = COL_R + DK;
    static constexpr uint32_t COL_DA = COL_A + 64;
    static constexpr uint32_t WR = DV > DK + 128 ? DV : DK + 128;
    // SPLIT layout (whole 64-column blocks on both halves): from COL_K the dk' accumulator with
    // key dims [0, DK/2) in lanes 0-15 and [DK/2, DK) in lanes 16-31, from COL_V dv likewise over
    // the value dims, from COL_AD dA (lanes 0-15) and A (lanes 16-31), so that every epilogue
    // lane holds a row.
    static constexpr bool SPLIT = DK == 128 && DV >= 128;
    static constexpr uint32_t COL_K = DV;
    static constexpr uint32_t COL_V = COL_K + DK / 2;
    static constexpr uint32_t COL_AD = COL_V + DV / 2;
    static constexpr uint32_t NCOL = SPLIT ? pow2cols(COL_AD + 64) : pow2cols(DV + WR);
    static constexpr int HC = DV / 2;
    static constexpr int KC = DK / 2;
    // key split: the G~ slot receives the other CTA's fp32 dv partial (half the value dims)
    // and, from XROWS on, its 64 per-row sums of k' dk'
    static constexpr uint32_t XROWS = (DV / 2) * TR * 4;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert((SPLIT ? COL_AD + 64 : DV + WR) <= 512, "tensor memory");
    static_assert(STAGE % 1024 == 0, "stage alignment");
};

// KS = key blocks of DK key dims (1, or 2 as a two-CTA cluster along x with DV >= 128).
template <int DK, int DV, int GATE, int KS>
__global__ void __launch_bounds__(NT_B, 1)
    k_tc_bwd_dkdv(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tg, const __grid_constant__ CUtensorMap tv,
                  const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tout,
                  const __grid_constant__ CUtensorMap tout2, BwdArgs A, Dims P) {
    using C = KVCfg<DK, DV, GATE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_align1024(smem_raw);
    uint8_t* sG = sm + C::NS * C::STAGE;
    uint8_t* sAm = sG + C::GTB;
    uint8_t* sdA = sAm + C::AB;
    uint8_t* small = sdA + C::AB;
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(small);
    uint64_t* bar_mma1 = bar_full + 2;
    uint64_t* bar_mma2 = bar_full + 3;
    uint64_t* bar_drain = bar_full + 4;   // error path: completion of every product issued
    uint64_t* bar_free = bar_full + 5;    // KS = 2: the other CTA's G~ slot may take its dv partial
    uint64_t* bar_recv = bar_full + 6;    // KS = 2: the other CTA's dv partial is in this G~ slot
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + 64);
    float* czs_peer = reinterpret_cast<float*>(small + 128);   // KS = 2: key block 1's part of czs
    float* tot = reinterpret_cast<float*>(small + 256);
    float* gam = tot + 2048;      // [DK]
    float* rowE = gam + DK;       // [64]
    float* rowEi = rowE + TR;
    float* igs = rowEi + TR;
    float* ghs = igs + TR;
    float* sdi = ghs + TR;        // [2][64]
    float* cz = sdi + 2 * TR;     // [DK] in-segment q*dq total + carry from later segments
    float* rk = cz + DK;          // [DK] running reverse sum of k*dk
    float* red = rk + DK;         // [2][DK]
    float* rows = red + 2 * DK;   // [64]
    float* czs = rows + TR;       // [1] per-head: sum over key dims of cz

    static_assert(KS == 1 || (KS == 2 && C::SPLIT), "key split needs the split TMEM layout");
    constexpr uint32_t kXRows = C::XROWS;
    static_assert(KS == 1 || kXRows + 4 * TR <= C::GTB, "key-split exchange area");
    const int bh = KS == 1 ? blockIdx.x : blockIdx.x >> 1, z = blockIdx.y;
    const int kb = KS == 1 ? 0 : blockIdx.x & 1;   // = the CTA's rank in its cluster
    const int d0 = kb * DK;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2, qd = warp & 3;
    const int ntiles_all = cdiv(P.L, TR);
    const int tile0 = z * A.tiles_per_seg;
    const int ntiles = min(ntiles_all, tile0 + A.tiles_per_seg) - tile0;
    const long rowbase = (long)bh * P.L;
    const bool srow_ok = (DK != 64) || (lane < 16);
    const int srow = DK == 64 ? 16 * qd + (lane & 15) : 32 * qd + lane;
    auto tile_at = [&](int j) { return tile0 + ntiles - 1 - j; };

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        mbar_init(bar_drain, 1);
        if (KS == 2) {
            mbar_init(bar_free, 1);
            mbar_init(bar_recv, NT_B / 2);   // one arrival per sending thread of the other CTA
        }
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, C::NCOL);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (KS == 2) cluster_sync();   // both CTAs' barriers are initialised before either touches the other
    const uint32_t tbase = *tmem_slot;
    // launched to overlap the reverse scan (or the dq kernel) before it: everything read from
    // earlier kernels of the call is read after this
    grid_dep_wait();
    const uint32_t tlane = tbase + ((uint32_t)(32 * qd) << 16);

    // ---- state gradient at the end of the segment into TMEM
    {
        const float* src = nullptr;
        if (z == A.nseg - 1) src = A.dhT ? A.dhT + ((long)bh * P.Dk + d0) * P.Dv : nullptr;
        else src = A.gend + (((long)bh * A.nseg + z) * P.Dk + d0) * P.Dv;
        // dg at the segment's end: sum_e G_end[d][e] * S_end[d][e] (shift invariance of the
        // cumulative log-decay), with S_end the forward state after the segment
        const float* send = nullptr;
        if (GATE != 0 && src) {
            if (z < A.nseg - 1) send = A.sinit + (((long)bh * A.nseg + z + 1) * P.Dk + d0) * P.Dv;
            else send = A.hT_ws ? A.hT_ws + ((long)bh * P.Dk + d0) * P.Dv : nullptr;
        }
        // staged through the ring stages, which are free until the first tile's loads
        static_assert(DK * DV * 4 <= C::NS * C::STAGE, "state staging");
        float* stg = reinterpret_cast<float*>(sm);
        if (src) stage_rows<DK, DV, NT_B>(stg, src, send, P.Dv, red, tid);
        if (!send && tid < DK) red[tid] = 0.f;
        if (tid < DK) rk[tid] = 0.f;
        __syncthreads();
        for (int c = wg * C::HC; c < (wg + 1) * C::HC; c += 16) {
            float f[16];
            if (src && srow_ok) staged_row16<DV>(stg, srow, c, f);
            else
#pragma unroll
                for (int j = 0; j < 16; ++j) f[j] = 0.f;
            tmem_st16(tlane + c, reinterpret_cast<uint32_t*>(f));
        }
        tmem_wait_st();
        if (tid < DK) {
            const float tqv = GATE == 1 ? A.tq[((long)bh * A.nseg + z) * P.Dk + d0 + tid] : 0.f;
            cz[tid] = red[tid] + tqv;
        }
        __syncthreads();
        if (GATE == 2 && tid == 0) {
            float sacc = A.tq[((long)bh * A.nseg + z) * P.Dk + d0];
            for (int dd = 0; dd < DK; ++dd) sacc += cz[dd];
            czs[0] = sacc;
            if (KS == 2 && kb == 1) st_cluster_f32(mapa_shared(czs_peer, 0), sacc);
        }
        if (KS == 2) {
            cluster_sync();   // key block 1's part of czs has reached key block 0
            if (GATE == 2 && kb == 0 && tid == 0) czs[0] += czs_peer[0];
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    auto issue_loads = [&](int i, int s) {
        uint8_t* st = sm + s * C::STAGE;
        const int t0 = tile_at(i) * TR;
        mbar_arrive_expect_tx(&bar_full[s], C::TXB);
        for (int cb = 0; cb < DK / 64; ++cb) {
            tma_load_3d(st + cb * BLK, &tq, d0 + cb * 64, t0, bh, &bar_full[s]);
            tma_load_3d(st + C::QB + cb * BLK, &tk, d0 + cb * 64, t0, bh, &bar_full[s]);
        }
        if (GATE == 1)
            for (int gb = 0; gb < DK / 32; ++gb)
                tma_load_3d(st + C::QB + C::KB + gb * BLK, &tg, d0 + 32 * gb, t0, bh, &bar_full[s]);
        for (int vb = 0; vb < DV / 64; ++vb) {
            tma_load_3d(st + C::QB + C::KB + C::GB + vb * BLK, &tv, vb * 64, t0, bh, &bar_full[s]);
            tma_load_3d(st + C::QB + C::KB + C::GB + C::VB + vb * BLK, &tdo, vb * 64, t0, bh, &bar_full[s]);
        }
    };
    // the i-th tile of the walk into L2, ahead of its loads
    auto issue_prefetch = [&](int i) { prefetch_tile_rows(A, P, rowbase, tile_at(i) * TR, kb, KS, true); };
    if (tid == 0) {
        for (int i = 0; i < C::NS && i < ntiles; ++i) issue_loads(i, i);
        for (int i = C::NS; i < 2 * C::NS && i < ntiles; ++i) issue_prefetch(i);
    }
    // input and per-head gates of the next tile, loaded a tile ahead into registers
    float nig = 1.f, ngh = 0.f;
    auto fetch_gates = [&](int i) {
        const int t = tile_at(i) * TR + tid;
        if (A.ig) nig = t < P.L ? A.ig[rowbase + t] : 1.f;
        if (GATE == 2) ngh = t < P.L ? A.gh[rowbase + t] : 0.f;
    };
    if (tid < TR) fetch_gates(0);

    int err = 0, n_mma = 0;
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::NS;
        uint8_t* st = sm + s * C::STAGE;
        uint8_t* sq = st;
        uint8_t* sk = st + C::QB;
        float* sg = reinterpret_cast<float*>(st + C::QB + C::KB);
        uint8_t* sv = st + C::QB + C::KB + C::GB;
        uint8_t* so = sv + C::VB;
        const int t0 = tile_at(i) * TR;
        if (tid < TR) {
            igs[tid] = nig;
            if (GATE == 2) ghs[tid] = ngh;
            if (i + 1 < ntiles) fetch_gates(i + 1);
        }
        // per-key gates: the dq kernel's exclusive prefixes of q*dq for this tile, fetched now so
        // that the loads have the whole tile to land; thread = (key dims dc..dc+3, RPR rows)
        constexpr int NC4 = DK / 4, NGR = NT_B / NC4, RPR = TR / NGR;
        const int c4 = tid % NC4, gr = tid / NC4, dc = 4 * c4;
        float4* dgp = reinterpret_cast<float4*>(A.dg + (rowbase + t0 + gr * RPR) * P.Dk + d0 + dc);
        float4 pre[GATE == 1 ? RPR : 1];
        if (GATE == 1)
#pragma unroll
            for (int rr = 0; rr < RPR; ++rr) pre[rr] = (t0 + gr * RPR + rr < P.L) ? dgp[(long)rr * (P.Dk / 4)] : f4_zero();
        if (!block_wait(&bar_full[s], (i / C::NS) & 1)) { err = 1; break; }

        // ---- transform: q~ = scale q e^b, k~ = i k e^-b (in place); e^-b kept in place of g
        bwd_transform<DK, GATE, true, false>(sq, sk, sg, tot, gam, rowE, rowEi, ghs, igs, P.scale, tid, A.status);
        fence_proxy_async_smem();
        __syncthreads();
        // ---- MMA group 1 (needs only this tile): A = (scale q~) k~^T, dA = dO V^T, both M=64 in
        //      TMEM lanes 0-15 next to the dk' accumulator
        if (warp == 0) {
            const bool leader = elect_one();
            tc_fence_after();
            const uint32_t qa = smem_u32(sq), ka = smem_u32(sk), va = smem_u32(sv), oa = smem_u32(so);
            const uint32_t id64 = idesc_bf16(64, 64, 0, 0);
            const uint32_t tA = C::SPLIT ? tbase + (16u << 16) + C::COL_AD : tbase + C::COL_A;
            const uint32_t tdA = C::SPLIT ? tbase + C::COL_AD : tbase + C::COL_DA;
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader) mma_bf16(tA, sw128_desc(qa + koff, 16, 1024), sw128_desc(ka + koff, 16, 1024), id64, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (leader) mma_bf16(tdA, sw128_desc(oa + koff, 16, 1024), sw128_desc(va + koff, 16, 1024), id64, kk > 0);
            }
            if (leader) mma_commit(bar_mma1);
            __syncwarp();
        }
        ++n_mma;
        // ---- G~ = e^Gamma G in TMEM; bf16 copy (runs while group 1 is in flight)
        {
            const float eg = GATE == 0 ? 1.f : gam[GATE == 1 ? srow : 0];
            const uint64_t eg2 = f2(eg, eg);
            for (int c = wg * C::HC; c < (wg + 1) * C::HC; c += 32) {
                uint32_t r[32];
                float f[32];
                tmem_ld32(tlane + c, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const uint64_t x = f2_mul(f2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), eg2);
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(f[j]), "=f"(f[j + 1]) : "l"(x));
                    r[j] = __float_as_uint(f[j]);
                    r[j + 1] = __float_as_uint(f[j + 1]);
                }
                tmem_st32(tlane + c, r);
                if (srow_ok)
#pragma unroll
                    for (int j = 0; j < 32; j += 8) store8_bf16(sG, sw128_off(srow, c + j, DK * 128), f + j);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- MMA group 2a (needs G~, not P): dk' = V G~^T, dv = k~ G~, G += (scale q~)^T dO
        const uint32_t tdk = C::SPLIT ? tbase + C::COL_K : tbase + C::COL_R;
        const uint32_t tdv = C::SPLIT ? tbase + C::COL_V : tbase + (16u << 16) + C::COL_R;
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t qa = smem_u32(sq), ka = smem_u32(sk), va = smem_u32(sv), oa = smem_u32(so);
            const uint32_t ga = smem_u32(sG);
            const uint32_t idK2 = idesc_bf16(64, C::SPLIT ? DK / 2 : DK, 0, 0);
            const uint32_t idV2 = idesc_bf16(64, C::SPLIT ? DV / 2 : DV, 0, 1);
            const uint32_t idG = idesc_bf16(DK, DV, 1, 1);
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk) {  // V G~^T
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                const uint32_t goff = (kk >> 2) * (DK * 128) + (kk & 3) * 32;
                if (C::SPLIT) {   // key dims (rows of G~) [0, DK/2) and [DK/2, DK) into the two lane halves
                    if (leader) mma_bf16(tdk, sw128_desc(va + koff, 16, 1024), sw128_desc(ga + goff, 16, 1024), idK2, kk > 0);
                    if (leader) mma_bf16(tdk + (16u << 16), sw128_desc(va + koff, 16, 1024),
                             sw128_desc(ga + goff + (DK / 2) * 128, 16, 1024), idK2, kk > 0);
                } else {
                    if (leader) mma_bf16(tdk, sw128_desc(va + koff, 16, 1024), sw128_desc(ga + goff, 16, 1024), idK2, kk > 0);
                }
            }
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {  // k~ G~
                const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
                if (C::SPLIT) {   // value-dim blocks [0, DV/2) and [DV/2, DV) into the two lane halves
                    if (leader) mma_bf16(tdv, sw128_desc(ka + koff, 16, 1024), sw128_desc(ga + kk * 2048, DK * 128, 1024),
                             idV2, kk > 0);
                    if (leader) mma_bf16(tdv + (16u << 16), sw128_desc(ka + koff, 16, 1024),
                             sw128_desc(ga + (DV / 128) * (DK * 128) + kk * 2048, DK * 128, 1024), idV2, kk > 0);
                } else {
                    if (leader) mma_bf16(tdv, sw128_desc(ka + koff, 16, 1024), sw128_desc(ga + kk * 2048, DK * 128, 1024), idV2,
                             kk > 0);
                }
            }
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks)  // G += (scale q~)^T dO
                if (leader) mma_bf16(tbase, sw128_desc(qa + ks * 2048, BLK, 1024), sw128_desc(oa + ks * 2048, BLK, 1024), idG, 1);
            __syncwarp();
        }
        if (!block_wait(bar_mma1, i & 1)) { err = 1; break; }
        tc_fence_after();
        // ---- P pass: masked A and masked dA -> bf16 in shared memory (rows in lanes 0-15;
        //      SPLIT: one read, dA rows in lanes 0-15 and A rows in lanes 16-31)
        if (C::SPLIT) {
            uint32_t r[32];
            tmem_ld32(tlane + C::COL_AD + 32 * wg, r);
            tmem_wait_ld();
            const int t = 16 * qd + (lane & 15);
            uint8_t* dst = lane < 16 ? sdA : sAm;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int sidx = 32 * wg + 8 * u + j;
                    f[j] = (sidx <= t) ? __uint_as_float(r[8 * u + j]) : 0.f;
                }
                store8_bf16(dst, sw128_off(t, 32 * wg + 8 * u, BLK), f);
            }
        } else {
            uint32_t ra[32], rd[32];
            tmem_ld32(tlane + C::COL_A + 32 * wg, ra);
            tmem_ld32(tlane + C::COL_DA + 32 * wg, rd);
            tmem_wait_ld();
            if (lane < 16) {
                const int t = 16 * qd + lane;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float fa[8], fd[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int sidx = 32 * wg + 8 * u + j;
                        fa[j] = (sidx <= t) ? __uint_as_float(ra[8 * u + j]) : 0.f;
                        fd[j] = (sidx <= t) ? __uint_as_float(rd[8 * u + j]) : 0.f;
                    }
                    store8_bf16(sAm, sw128_off(t, 32 * wg + 8 * u, BLK), fa);
                    store8_bf16(sdA, sw128_off(t, 32 * wg + 8 * u, BLK), fd);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- MMA group 2b: dk' += mask(dA)^T (scale q~), dv += mask(A)^T dO
        if (warp == 0) {
            const bool leader = elect_one();
            const uint32_t qa = smem_u32(sq), oa = smem_u32(so);
            const uint32_t ama = smem_u32(sAm), dama = smem_u32(sdA);
            const uint32_t idK1 = idesc_bf16(64, C::SPLIT ? DK / 2 : DK, 1, 1);
            const uint32_t idV1 = idesc_bf16(64, C::SPLIT ? DV / 2 : DV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks) {
                if (leader) mma_bf16(tdk, sw128_desc(dama + ks * 2048, BLK, 1024), sw128_desc(qa + ks * 2048, BLK, 1024), idK1, 1);
                if (C::SPLIT && leader)   // key-dim block 1 of q~ into lanes 16-31
                    mma_bf16(tdk + (16u << 16), sw128_desc(dama + ks * 2048, BLK, 1024),
                             sw128_desc(qa + BLK + ks * 2048, BLK, 1024), idK1, 1);
            }
#pragma unroll
            for (int ks = 0; ks < TR / 16; ++ks) {
                if (leader) mma_bf16(tdv, sw128_desc(ama + ks * 2048, BLK, 1024), sw128_desc(oa + ks * 2048, BLK, 1024), idV1, 1);
                if (C::SPLIT && leader)   // value-dim blocks [DV/2, DV) of dO into lanes 16-31
                    mma_bf16(tdv + (16u << 16), sw128_desc(ama + ks * 2048, BLK, 1024),
                             sw128_desc(oa + (DV / 128) * BLK + ks * 2048, BLK, 1024), idV1, 1);
            }
            if (leader) mma_commit(bar_mma2);
            __syncwarp();
        }
        // per-head gates: the dq kernel's exclusive prefixes of this tile's rows, in flight during
        // the epilogue (per-key gates fetched theirs at the top of the tile)
        float pre2[2];
        if (GATE == 2 && kb == 0 && warp == 0) {   // rows 2 lane, 2 lane + 1: both key blocks' prefixes
            const long bhl = (long)P.B * P.H * P.L;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int ta = t0 + 2 * lane + u;
                pre2[u] = ta < P.L ? A.pre[rowbase + ta] + (KS == 2 ? A.pre[bhl + rowbase + ta] : 0.f) : 0.f;
            }
        }
        if (!block_wait(bar_mma2, i & 1)) { err = 1; break; }
        tc_fence_after();
        // every product that reads G~ is done: the other CTA may write its dv partial there
        if (KS == 2 && tid == 0) mbar_arrive_remote(mapa_shared(bar_free, kb ^ 1));

        // ---- dk = i e^-b X (bf16, staged in the q slot), k*dk = k~ X (into the g slot for dg),
        //      di = sum_d k~ X / i, and dv (bf16, staged in the v slot); q~ and V are no longer
        //      read. Row s of X / dv sits in TMEM lane (s % 16) / 16 + (s % 16) of quadrant s / 16
        //      (SPLIT: both accumulators in both lane halves, by column half).
        {
            const int srw = 16 * qd + (lane & 15);
            const bool row_ok = t0 + srw < P.L;
            float dsum = 0.f;
            constexpr int KCW = C::SPLIT ? DK / 4 : C::KC, VCW = C::SPLIT ? DV / 4 : C::HC;   // TMEM columns per warpgroup
            // key split: dv over this key block is a partial sum. This CTA owns value dims
            // [kb DV/2, (kb + 1) DV/2), the TMEM lane half kb; the lanes of the other half send
            // theirs to the other CTA first (so that the transfer overlaps the dk epilogue), as
            // fp32, 16-byte chunk j of row s at byte (64 j + s) * 16 of its G~ slot, followed
            // (key block 1 only) by the rows' sums of k' dk'.
            const bool own = (lane >> 4) == kb;
            const uint32_t peer_g = KS == 2 ? mapa_shared(sG, kb ^ 1) : 0u;
            if (KS == 2) {
                if (!block_wait_cluster(bar_free, i & 1)) { err = 1; break; }
                for (int ct = wg * VCW; ct < (wg + 1) * VCW; ct += 16) {
                    uint32_t r[16];
                    tmem_ld16(tlane + C::COL_V + ct, r);
                    tmem_wait_ld();
                    if (!own)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            st_cluster_v4(peer_g + (uint32_t)((((ct >> 2) + u) * TR + srw) * 16),
                                          __uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                                          __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3]));
                }
            }
            for (int ct = wg * KCW; ct < (wg + 1) * KCW; ct += 16) {
                uint32_t r[16];
                tmem_ld16(tlane + (C::SPLIT ? C::COL_K : C::COL_R) + ct, r);
                tmem_wait_ld();
                const int c = C::SPLIT ? (lane >> 4) * (DK / 2) + ct : ct;   // key dim of r[0]
                if (C::SPLIT || lane < 16) {
                    const float iv = igs[srw];
                    float em[16];
                    if (GATE == 1) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 e4 = *reinterpret_cast<const float4*>(sg + gsw(srw, c + 4 * q4));
                            em[4 * q4] = e4.x; em[4 * q4 + 1] = e4.y; em[4 * q4 + 2] = e4.z; em[4 * q4 + 3] = e4.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) em[j] = GATE == 2 ? rowEi[srw] : 1.f;
                    }
                    uint4 kw[2];
                    kw[0] = *reinterpret_cast<const uint4*>(sk + sw128_off(srw, c, BLK));
                    kw[1] = *reinterpret_cast<const uint4*>(sk + sw128_off(srw, c + 8, BLK));
                    const uint32_t* kp = reinterpret_cast<const uint32_t*>(kw);
                    float f[16], kx[16];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kp[u]));
                        const float x0 = __uint_as_float(r[2 * u]), x1 = __uint_as_float(r[2 * u + 1]);
                        f[2 * u] = iv * em[2 * u] * x0;
                        f[2 * u + 1] = iv * em[2 * u + 1] * x1;
                        kx[2 * u] = row_ok ? kf.x * x0 : 0.f;         // k' dk' = k~ X
                        kx[2 * u + 1] = row_ok ? kf.y * x1 : 0.f;
                        dsum += kx[2 * u] + kx[2 * u + 1];
                    }
                    store8_bf16(sq, sw128_off(srw, c, BLK), f);
                    store8_bf16(sq, sw128_off(srw, c + 8, BLK), f + 8);
                    if (GATE == 1)
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<float4*>(sg + gsw(srw, c + 4 * q4)) =
                                make_float4(kx[4 * q4], kx[4 * q4 + 1], kx[4 * q4 + 2], kx[4 * q4 + 3]);
                }
            }
            if (C::SPLIT) dsum += __shfl_xor_sync(0xffffffffu, dsum, 16);
            if (lane < 16) sdi[wg * TR + srw] = dsum;
            if (KS == 1) {
                for (int ct = wg * VCW; ct < (wg + 1) * VCW; ct += 16) {
                    uint32_t r[16];
                    tmem_ld16(tlane + (C::SPLIT ? C::COL_V : C::COL_R) + ct, r);
                    tmem_wait_ld();
                    const int c = C::SPLIT ? (lane >> 4) * (DV / 2) + ct : ct;   // value dim of r[0]
                    if (C::SPLIT || lane >= 16) {
                        store8_bf16(sv, sw128_off(srw, c, BLK), reinterpret_cast<const float*>(r));
                        store8_bf16(sv, sw128_off(srw, c + 8, BLK), reinterpret_cast<const float*>(r + 8));
                    }
                }
            } else {
                __syncthreads();   // sdi is complete
                if (!own) {
                    if (kb == 1 && wg == 0) st_cluster_f32(peer_g + kXRows + 4 * srw, sdi[srw] + sdi[TR + srw]);
                    mbar_arrive_remote(mapa_shared(bar_recv, kb ^ 1));
                }
                if (!block_wait_cluster(bar_recv, i & 1)) { err = 1; break; }
                // the owning lanes add the other CTA's part to theirs
                const float* rx = reinterpret_cast<const float*>(sG);
                for (int ct = wg * VCW; ct < (wg + 1) * VCW; ct += 16) {
                    uint32_t r[16];
                    tmem_ld16(tlane + C::COL_V + ct, r);
                    tmem_wait_ld();
                    if (own) {
                        float f[16];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float4 x = *reinterpret_cast<const float4*>(rx + (((ct >> 2) + u) * TR + srw) * 4);
                            f[4 * u] = __uint_as_float(r[4 * u]) + x.x;
                            f[4 * u + 1] = __uint_as_float(r[4 * u + 1]) + x.y;
                            f[4 * u + 2] = __uint_as_float(r[4 * u + 2]) + x.z;
                            f[4 * u + 3] = __uint_as_float(r[4 * u + 3]) + x.w;
                        }
                        store8_bf16(sv, sw128_off(srw, ct, BLK), f);
                        store8_bf16(sv, sw128_off(srw, ct + 8, BLK), f + 8);
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            for (int cb = 0; cb < DK / 64; ++cb) tma_store_3d(&tout, sq + cb * BLK, d0 + 64 * cb, t0, bh);
            for (int vb = 0; vb < DV / 64 / KS; ++vb)
                tma_store_3d(&tout2, sv + vb * BLK, kb * (DV / KS) + 64 * vb, t0, bh);
            bulk_commit();
        }
        const float* prow = reinterpret_cast<const float*>(sG + kXRows);   // KS = 2, key block 0
        if (A.di && kb == 0 && tid < TR && t0 + tid < P.L)
            A.di[rowbase + t0 + tid] = (sdi[tid] + sdi[TR + tid] + (KS == 2 ? prow[tid] : 0.f)) / igs[tid];
        // ---- dg = (in-segment q*dq total - exclusive prefix) - reverse sum of k*dk + carry
        if (GATE == 1) {
            // thread = (key dims dc..dc+3, group of RPR rows; the prefixes were fetched above):
            // local sums, exchange, then the reverse walk with 16-byte stores
            float4* tot4 = reinterpret_cast<float4*>(tot);
            float4* rk4 = reinterpret_cast<float4*>(rk);
            float4 x[RPR];   // the thread's rows of k*dk, read once
            float4 loc = f4_zero();
#pragma unroll
            for (int rr = 0; rr < RPR; ++rr) {
                x[rr] = gsw_ld4(sg, gr * RPR + rr, dc);
                loc = f4_add(loc, x[rr]);
            }
            tot4[gr * NC4 + c4] = loc;
            __syncthreads();
            float4 sx = rk4[c4], T = f4_zero();
#pragma unroll
            for (int g2 = 0; g2 < NGR; ++g2) {
                const float4 v = tot4[g2 * NC4 + c4];
                if (g2 > gr) sx = f4_add(sx, v);
                T = f4_add(T, v);
            }
            const float4 cx = reinterpret_cast<const float4*>(cz)[c4];
#pragma unroll
            for (int rr = RPR - 1; rr >= 0; --rr) {
                sx = f4_add(sx, x[rr]);
                if (t0 + gr * RPR + rr < P.L)
                    dgp[(long)rr * (P.Dk / 4)] = make_float4(cx.x - pre[rr].x - sx.x, cx.y - pre[rr].y - sx.y,
                                                             cx.z - pre[rr].z - sx.z, cx.w - pre[rr].w - sx.w);
            }
            __syncthreads();
            if (gr == 0) rk4[c4] = f4_add(rk4[c4], T);
        } else if (GATE == 2 && kb == 0) {
            // key block 0 forms the per-head dg of both blocks; a row's sum of k' dk' over the
            // key dims is the epilogue's per-row sum (sdi, and prow from key block 1)
            if (tid < TR) rows[tid] = sdi[tid] + sdi[TR + tid] + (KS == 2 ? prow[tid] : 0.f);
            __syncthreads();
            if (warp == 0) {  // reverse inclusive scan over 64 rows, two per lane
                const float a0 = rows[2 * lane], a1 = rows[2 * lane + 1];
                float v = a0 + a1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float n = __shfl_down_sync(0xffffffffu, v, off);
                    if (lane + off < 32) v += n;
                }
                const float base = rk[0], cc = czs[0];
                const float s0 = base + v, s1 = base + v - a0;
                const int ta = t0 + 2 * lane;
                // pre: the dq kernel's exclusive prefixes of q*dq (both key blocks), fetched above
                if (ta < P.L) A.dg[rowbase + ta] = cc - pre2[0] - s0;
                if (ta + 1 < P.L) A.dg[rowbase + ta + 1] = cc - pre2[1] - s1;
                const float total = __shfl_sync(0xffffffffu, v, 0);
                __syncwarp();
                if (lane == 0) rk[0] = base + total;
            }
        }
        __syncthreads();
        if (tid == 0) bulk_wait_read<0>();   // the dk / dv stores have read the q and v slots
        // the next tile's loads, then the tile after it into L2 (issued from the same thread
        // after the loads: an earlier prefetch, or one from another warp, measured slower)
        if (tid == 0 && i + C::NS < ntiles) {
            issue_loads(i + C::NS, s);
            if (i + 2 * C::NS < ntiles) issue_prefetch(i + 2 * C::NS);
        }
    }

    if (err) {
        if (warp == 0) {
            // every product the issuing lane issued completes before TMEM and shared memory go away
            const bool leader = elect_one();
            if (leader) {
                atomicOr(A.status, kDevStatusTimeout);
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0, 1u << 20);
            }
            __syncwarp();
        }
    } else if (A.dh0 && z == 0) {
        for (int c = wg * C::HC; c < (wg + 1) * C::HC; c += 16) {
            uint32_t r[16];
            tmem_ld16(tlane + c, r);
            tmem_wait_ld();
            if (srow_ok) {
                float* dst = A.dh0 + ((long)bh * P.Dk + d0 + srow) * P.Dv + c;
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                                      __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            }
        }
    }
    if (tid == 0) bulk_wait<0>();   // the last output stores have completed
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, C::NCOL);
    // neither CTA of a pair leaves while the other may still write into its shared memory
    if (KS == 2) cluster_sync();
}

// ============================================================================ host side
// A second stream per device, created on first use, on which the state-gradient pass and its
// reverse scan run beside the dq kernel (they do not depend on it): their CTAs fill the SMs the
// dq kernel's last partial wave leaves idle. nullptr if it cannot be created.
static cudaStream_t aux_stream() {
    static std::once_flag once[kMaxDevices];
    static cudaStream_t streams[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(once[dev], [dev] {
        if (cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) streams[dev] = nullptr;
    });
    return streams[dev];
}

struct BwdPlan {
    int nseg, tiles_per_seg, dkb;
};

static BwdPlan plan_bwd(const Dims& P) {
    BwdPlan pl{};
    pl.dkb = P.Dk > 128 ? 128 : P.Dk;
    const int ntiles = cdiv(P.L, TR);
    const long base = (long)P.B * P.H;
    const int sms = num_sms();
    int nseg = 1;
    if (base * 4 < (long)sms * 3 && ntiles > 1) nseg = (int)((long)sms / base);
    if (nseg < 1) nseg = 1;
    // dg's reverse sum restarts from an exact fp32 carry at every segment boundary; keeping
    // segments to about ten tiles bounds how far bf16 operand rounding can accumulate
    const int acc_seg = cdiv(ntiles, 10);
    if (nseg < acc_seg) nseg = acc_seg;
    const int tiles_per_chunk = P.C / TR;
    const int nchunks = cdiv(P.L, P.C);
    if (nseg > nchunks) nseg = nchunks;
    if (nchunks == 0) {   // L = 0: one empty segment
        pl.nseg = 1;
        pl.tiles_per_seg = 0;
        return pl;
    }
    const int chunks_per_seg = cdiv(nchunks, nseg);
    pl.tiles_per_seg = chunks_per_seg * tiles_per_chunk;
    pl.nseg = cdiv(ntiles, pl.tiles_per_seg);
    if (pl.nseg < 1) pl.nseg = 1;
    return pl;
}

// Dk = 256 splits the key dims over a CTA pair whose dv exchange needs the split TMEM layout
// (Dv >= 128).
bool bwd_supports(const Dims& P) {
    if (P.C % TR != 0) return false;
    if (P.Dk == 64 || P.Dk == 128) return P.Dv == 64 || P.Dv == 128 || P.Dv == 256;
    return P.Dk == 256 && (P.Dv == 128 || P.Dv == 256);
}

struct BwdWs {
    float *seg_state, *seg_gamma, *sinit, *gend, *hT, *tq, *pre;
    size_t total;
};

static BwdWs bwd_layout(const Dims& P, char* base) {
    const BwdPlan pl = plan_bwd(P);
    const size_t BH = (size_t)P.B * P.H, st = 4 * BH * (size_t)P.Dk * P.Dv;
    BwdWs w{};
    size_t off = kStatusBytes;
    w.hT = reinterpret_cast<float*>(base + off);
    off = align_up(off + st, 256);
    w.tq = reinterpret_cast<float*>(base + off);
    off = align_up(off + 4 * BH * (size_t)pl.nseg * P.Dk, 256);
    if (P.gate == GLA_GATE_PER_HEAD && P.Dk > 128) {   // per-key-block prefixes of q*dq
        w.pre = reinterpret_cast<float*>(base + off);
        off = align_up(off + 4 * BH * (size_t)(P.Dk / 128) * P.L, 256);
    }
    if (pl.nseg > 1) {
        w.seg_state = reinterpret_cast<float*>(base + off);
        off = align_up(off + st * pl.nseg, 256);
        w.seg_gamma = reinterpret_cast<float*>(base + off);
        off = align_up(off + 4 * BH * pl.nseg * P.Dk, 256);
        w.sinit = reinterpret_cast<float*>(base + off);
        off = align_up(off + st * pl.nseg, 256);
        w.gend = reinterpret_cast<float*>(base + off);
        off = align_up(off + st * pl.nseg, 256);
    }
    w.total = off;
    return w;
}

size_t bwd_workspace_bytes(const Dims& P) { return bwd_layout(P, nullptr).total; }

void bwd_plan_info(const Dims& P, int* nseg, int* tiles_per_seg) {
    const BwdPlan pl = plan_bwd(P);
    *nseg = pl.nseg;
    *tiles_per_seg = pl.tiles_per_seg;
}

template <int DKB, int DV, int GATE>
static cudaError_t launch_dq(const Dims& P, const BwdPlan& pl, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mg, const CUtensorMap& mv, const CUtensorMap& mo,
                             const CUtensorMap& mdq, const BwdArgs& a, cudaStream_t st) {
    using C = QCfg<DKB, DV, GATE>;
    auto kern = k_tc_bwd_dq<DKB, DV, GATE>;
    static std::atomic<bool> attr[kMaxDevices];
    {
        const cudaError_t e = smem_attr_once(kern, C::SMEM, attr);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(P.B * P.H, P.Dk / DKB, pl.nseg);
    GLA_LAUNCH("tc_bwd_dq", st, kern<<<grid, NT_B, C::SMEM, st>>>(mq, mk, mg, mv, mo, mdq, a, P));
    return cudaGetLastError();
}

template <int DK, int DV, int GATE, int KS>
static cudaError_t launch_dkdv(const Dims& P, const BwdPlan& pl, const CUtensorMap& mq, const CUtensorMap& mk,
                               const CUtensorMap& mg, const CUtensorMap& mv, const CUtensorMap& mo,
                               const CUtensorMap& mdk, const CUtensorMap& mdv, const BwdArgs& a, cudaStream_t st,
                               bool pdl) {
    using C = KVCfg<DK, DV, GATE>;
    auto kern = k_tc_bwd_dkdv<DK, DV, GATE, KS>;
    static std::atomic<bool> attr[kMaxDevices];
    {
        const cudaError_t e = smem_attr_once(kern, C::SMEM, attr);
        if (e != cudaSuccess) return e;
    }
    // the two key blocks of a (b*h, segment) run as one cluster of two CTAs; with pdl the kernel
    // may start before the kernel ahead of it in the stream (reverse scan or dq) ends, and waits
    // for it in grid_dep_wait
    cudaError_t e = cudaSuccess;
    GLA_LAUNCH("tc_bwd_dkdv", st,
               e = launch_ex(kern, dim3(KS * P.B * P.H, pl.nseg), dim3(NT_B), C::SMEM, st, pdl, KS, mq, mk, mg, mv, mo,
                             mdk, mdv, a, P));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int DK, int DV, int GATE>
static cudaError_t run_bwd(const Dims& P, const void* q, const void* k, const void* v, const float* g,
                           const float* ig, const float* h0, const void* dO, const float* dhT, void* dq, void* dk,
                           void* dv, float* dg, float* di, float* dh0, const float* saved, void* ws,
                           cudaStream_t st) {
    const BwdPlan pl = plan_bwd(P);
    const BwdWs w = bwd_layout(P, static_cast<char*>(ws));
    const int BH = P.B * P.H;
    constexpr int DKB = DK > 128 ? 128 : DK;
    constexpr int KS = DK / DKB;
    CUtensorMap mq, mk, mv, mo, mg, mdq, mdk, mdv;
    if (!make_map(&mdq, dq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mdk, dk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mdv, dv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dv, P.L, BH, 64, true) ||
        !make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dv, P.L, BH, 64, true) ||
        !make_map(&mo, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dv, P.L, BH, 64, true))
        return cudaErrorInvalidValue;
    if (GATE == 1) {
        // 32-column fp32 boxes with the 128-byte swizzle (see gsw)
        if (!make_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P.Dk, P.L, BH, 32, true))
            return cudaErrorInvalidValue;
    } else {
        mg = mk;
    }
    int* status = static_cast<int*>(ws);
    cudaError_t e;
    // segment initial states: from the forward that saved them, else a state pass + scan
    const float* sinit = saved ? saved : w.sinit;
    if (pl.nseg > 1 && !saved) {
        e = state_pass(P, 1, k, v, g, ig, pl.nseg, pl.tiles_per_seg, w.seg_state, w.seg_gamma, status, st);
        if (e != cudaSuccess) return e;
        e = seg_scan(P, pl.nseg, w.seg_state, w.seg_gamma, h0, w.sinit, st);
        if (e != cudaSuccess) return e;
    }
    BwdArgs a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.dO = static_cast<const __nv_bfloat16*>(dO);
    a.g = GATE == 1 ? g : nullptr;
    a.gh = GATE == 2 ? g : nullptr;
    a.ig = ig;
    a.sinit = sinit;
    a.h0 = h0;
    a.gend = w.gend;
    a.dhT = dhT;
    a.dq = static_cast<__nv_bfloat16*>(dq);
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dv = static_cast<__nv_bfloat16*>(dv);
    a.di = di;
    a.dh0 = dh0;
    a.hT_ws = (dhT && GATE != 0) ? w.hT : nullptr;
    a.dg = dg;
    a.tq = w.tq;
    a.pre = (GATE == 2 && KS == 2) ? w.pre : dg;
    a.status = status;
    a.tiles_per_seg = pl.tiles_per_seg;
    a.nseg = pl.nseg;
    // the state-gradient pass and reverse scan (segment-end state gradients for the dk/dv kernel)
    // depend on the inputs only: forked onto a second stream after everything the call has
    // enqueued so far (the forward state pass and scan above use the same segment buffers), and
    // joined before the dk/dv kernel
    cudaStream_t st2 = (pl.nseg > 1 && !prof_enabled()) ? aux_stream() : nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    if (st2 && (cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess)) {
        if (ev_fork) cudaEventDestroy(ev_fork);
        ev_fork = nullptr;
        st2 = nullptr;
    }
    auto release = [&] {
        if (ev_fork) cudaEventDestroy(ev_fork);
        if (ev_join) cudaEventDestroy(ev_join);
    };
    cudaStream_t sg = st;
    if (st2) {
        if ((e = cudaEventRecord(ev_fork, st)) != cudaSuccess || (e = cudaStreamWaitEvent(st2, ev_fork, 0)) != cudaSuccess) {
            release();
            return e;
        }
        sg = st2;
    }
    e = launch_dq<DKB, DV, GATE>(P, pl, mq, mk, mg, mv, mo, mdq, a, st);
    if (e == cudaSuccess && pl.nseg > 1) {
        e = state_pass(P, 2, q, dO, g, ig, pl.nseg, pl.tiles_per_seg, w.seg_state, w.seg_gamma, status, sg);
        if (e == cudaSuccess) e = seg_rscan(P, pl.nseg, w.seg_state, w.seg_gamma, dhT, w.gend, sg);
    }
    if (st2) {
        // the join is enqueued even after a launch error, so that st never races ahead of st2
        const cudaError_t e1 = cudaEventRecord(ev_join, st2);
        const cudaError_t e2 = e1 == cudaSuccess ? cudaStreamWaitEvent(st, ev_join, 0) : e1;
        if (e == cudaSuccess) e = e2;
    }
    release();
    if (e != cudaSuccess) return e;
    // after the join the kernel ahead of it in st is an event wait: launched without overlap
    e = launch_dkdv<DKB, DV, GATE, KS>(P, pl, mq, mk, mg, mv, mo, mdk, mdv, a, st, st2 == nullptr);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int DK, int DV>
static cudaError_t bwd_gate(const Dims& P, const void* q, const void* k, const void* v, const float* g,
                            const float* ig, const float* h0, const void* dO, const float* dhT, void* dq, void* dk,
                            void* dv, float* dg, float* di, float* dh0, const float* saved, void* ws,
                            cudaStream_t st) {
    switch (P.gate) {
        case GLA_GATE_NONE: return run_bwd<DK, DV, 0>(P, q, k, v, g, ig, h0, dO, dhT, dq, dk, dv, dg, di, dh0, saved, ws, st);
        case GLA_GATE_PER_KEY:
            return run_bwd<DK, DV, 1>(P, q, k, v, g, ig, h0, dO, dhT, dq, dk, dv, dg, di, dh0, saved, ws, st);
        default: return run_bwd<DK, DV, 2>(P, q, k, v, g, ig, h0, dO, dhT, dq, dk, dv, dg, di, dh0, saved, ws, st);
    }
}

cudaError_t bwd(const Dims& P, const void* q, const void* k, const void* v, const float* g, const float* ig,
                const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dg, float* di,
                float* dh0, const float* saved, void* ws, cudaStream_t st) {
#define GLA_BWD_CASE(DK_, DV_)                                                                      \
    if (P.Dk == DK_ && P.Dv == DV_)                                                                 \
        return bwd_gate<DK_, DV_>(P, q, k, v, g, ig, h0, dO, dhT, dq, dk, dv, dg, di, dh0, saved, ws, st);
    GLA_BWD_CASE(64, 64)
    GLA_BWD_CASE(64, 128)
    GLA_BWD_CASE(64, 256)
    GLA_BWD_CASE(128, 64)
    GLA_BWD_CASE(128, 128)
    GLA_BWD_CASE(128, 256)
    GLA_BWD_CASE(256, 128)
    GLA_BWD_CASE(256, 256)
#undef GLA_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace tc
}  // namespace gla
