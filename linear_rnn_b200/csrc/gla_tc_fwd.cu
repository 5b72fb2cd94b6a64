// Tensor-core (tcgen05 / TMEM / TMA) forward of chunkwise gated linear attention, bf16 I/O.
//
// One CTA owns a (batch*head, Dv tile, sequence segment) and walks its segment in tiles
// of 64 tokens, keeping the Dk x DVT state on chip: fp32 in tensor memory, where the
// state product accumulates onto it, and a bf16 copy in shared memory as the B operand
// of the inter-chunk product. Per tile (the chunk ("trunk") step of the talk summary
// "Hardware-Efficient Training of Linear Attention Models", section 11:58, with the gates
// of the GLA abstract):
//   b      = in-tile inclusive cumsum of the log-gate (fp32), Gamma = b at the last row
//   q~     = q * e^b,   k~ = i * k * e^-b            (bf16, in place in the TMA tile)
//   A      = q~ k~^T                (tcgen05, M=64 N=64 K=Dk, TMEM lanes 0-15 of each quadrant)
//   O      = q~ S_prev              (tcgen05, M=64 N=DVT K=Dk, TMEM lanes 16-31)
//   S     += k~^T V                 (tcgen05, M=128 (or 64) N=DVT K=64, onto the TMEM state)
//   S      = diag(e^Gamma) S        (TMEM load, scale, store; bf16 copy for the next tile)
//   P      = causal mask of A (bf16 in shared memory);  O += P V   (tcgen05)
//   o      = scale * O
// q~ k~^T equals sum_d q_td k_sd e^(b_td - b_sd): the single in-tile reference point keeps
// every exponent inside the tile's span. The state update uses k~ (not k e^(Gamma-b))
// and applies e^Gamma to the rows afterwards, so one bf16 key tile serves both products.
//
// Plans: a single pass per (bh, Dv tile) when that fills the GPU; otherwise the
// sequence is cut into segments (a multiple of the chunk size) processed in parallel:
// a state-only pass gives each segment's local end state and total log-decay, a small
// scan turns them into each segment's initial state, and the output pass starts every
// segment from its initial state -- the two-level chunking of the Tiled Flash Linear
// Attention abstract (large chunks, tiled inside, few materialised states).
#include <cudaTypedefs.h>

#include "gla_common.cuh"
#include "gla_plans.h"
#include "gla_tc_common.cuh"

namespace gla {
namespace tc {

using namespace sm100;


// Thread roles: warps [0, 4*NEWG) run the epilogues (state, P, output), warps
// [4*NEWG, 4*(NEWG+NTWG)) transform tiles in place, warp W_MMA issues the tcgen05 MMAs
// and warp W_TMA the TMA loads. They hand tiles to each other through mbarriers: the
// transform runs up to two tiles ahead, the MMAs of tile i+1 overlap the epilogues of
// tile i (two TMEM buffers for A and O). Epilogue warp w reads TMEM lane quadrant w % 4;
// each epilogue warpgroup owns DVT/NEWG state columns.
constexpr int NEWG = 2;
constexpr int NTWG = 2;
constexpr int NEP = NEWG * 128;
constexpr int NTRF = NTWG * 128;
constexpr int W_MMA = (NEP + NTRF) / 32;
constexpr int W_TMA = W_MMA + 1;
constexpr int NTHR_WS = NEP + NTRF + 64;
constexpr int BAR_S = 1;    // named barrier of the state-epilogue threads
constexpr int BAR_TR = 2;   // named barrier of the transform threads
constexpr int BAR_PO = 3;   // named barrier of the P/output-epilogue threads (output pass)
constexpr float kLog2e = 1.4426950408889634f;
// Tiles at the start of each segment that the state-only pass loads with the evict_last L2
// policy (k, g, v: 64 KB a tile at Dk = Dv = 128, so ~9 tiles over ~140 CTAs keep about
// 80 MB of the 126 MB L2)
constexpr int kL2KeepTiles = 9;

// 2^x on the special-function unit (inputs here are log-gate sums times log2(e))
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


constexpr uint32_t pow2_cols(uint32_t n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512; }

template <int DK, int DVT, int GATE, int MODE>
struct Cfg {
    // MODE 0: output pass (q, k, g, v). MODE 1: state-only pass (k, g, v), walked from the
    // segment's end with every k scaled by its whole decay to that end, e^(D + Gamma - b) <= 1
    // (D: decay of the tiles after this one), so that the state only accumulates.
    // MODE 2: state-gradient pass (q in the k slot, g, dO in the v slot), walked from the
    // segment's start with every q scaled by its whole decay from that start, e^(D + b) <= 1.
    static constexpr uint32_t QB = MODE == 0 ? TR * DK * 2 : 0;
    static constexpr uint32_t KB = TR * DK * 2;
    static constexpr uint32_t GB = GATE == 1 ? TR * DK * 4 : 0;
    static constexpr uint32_t VB = TR * DVT * 2;
    static constexpr uint32_t STAGE = QB + KB + GB + VB;
    static constexpr uint32_t PB = MODE == 0 ? TR * TR * 2 : 0;       // P
    static constexpr uint32_t SB = MODE == 0 ? DK * DVT * 2 : 0;      // bf16 state
    static constexpr uint32_t OB = MODE == 0 ? TR * DVT * 2 : 0;      // output tile staged for the TMA store
    // (+ a ring of NS + 1 row-factor vectors of the output pass)
    static constexpr uint32_t SMALL = 256 + 8 * NTRF + 16 * DK + 1024 + 256 * 5;
    // Output pass with per-head or no gates: q enters the products untransformed, the O
    // accumulator holds q S_prev + P V, and the output pass scales row t by scale e^(b_t)
    // (P = mask(q k~^T) already carries e^(-b_s)). Per-key gates transform q (scale q e^b).
    static constexpr bool XQ = MODE == 0 && GATE == 1;
    static constexpr uint32_t FIXED = PB + SB + OB + SMALL + 1024;
    // as many ring stages (up to 4) as shared memory holds: the loads of a tile are in
    // flight while the tiles before it are transformed and multiplied
    static constexpr int NS = (4 * STAGE + FIXED <= 227 * 1024) ? 4 : (3 * STAGE + FIXED <= 227 * 1024) ? 3
                              : (2 * STAGE + FIXED <= 227 * 1024) ? 2 : 1;
    static constexpr uint32_t SMEM = NS * STAGE + FIXED;
    static constexpr int NF = NS + 1;   // row-factor ring: a tile's factors live until its output pass
    static constexpr int NH = DK == 256 ? 2 : 1;            // M=128 halves of the state
    static constexpr int MS = DK == 64 ? 64 : 128;           // M of the state MMA
    // TMEM columns: the fp32 state [0, COLS_S), then NAB buffers of COLA columns holding
    // A (lanes 0-15 of each quadrant) and O (lanes 16-31) of a tile
    static constexpr int NAB = 3;
    static constexpr uint32_t COLS_S = NH * DVT;
    static constexpr uint32_t COLA = MODE == 0 ? (DVT > 64 ? DVT : 64) : 0;
    static constexpr uint32_t NCOL = pow2_cols(COLS_S + NAB * COLA);
    // Epilogue split. Output pass: warpgroup 0 runs the state pass over all DVT columns
    // (the recurrence's critical path), warpgroup 1 the P and output passes. State-only
    // passes: both warpgroups run the state pass, DVT/2 columns each.
    static constexpr int SCOLS = MODE == 0 ? DVT : DVT / 2;  // state columns per state-pass thread
    static constexpr int NSW = MODE == 0 ? 128 : 256;        // state-pass threads
    static constexpr int CH = 32;                            // TMEM columns per tcgen05.ld / st
    static_assert(STAGE % 1024 == 0, "stage alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(SCOLS % CH == 0 && DVT % CH == 0 && TR % CH == 0, "column chunks");
    static_assert(COLS_S + NAB * COLA <= 512, "tensor memory");
    static_assert(DK <= NTRF, "one transform thread per key dim in the cumsum");
};

struct FwdArgs {
    const float* gh;      // per-head log-gate [BH*L] (GATE == 2)
    const float* ig;      // input gate [BH*L] or null
    const float* h0;      // [BH, Dk, Dv] or null
    const float* sinit;   // [BH, sinit_nseg, Dk, Dv] initial states of the state pass's segments
                          // (output pass: segment z starts from entry z * sinit_step)
    int sinit_nseg;
    int sinit_step;
    __nv_bfloat16* o;     // [BH, L, Dv]
    float* hT;            // [BH, Dk, Dv] or null
    float* seg_state;     // state-only pass: [BH, nseg, Dk, Dv] local end states
    float* seg_gamma;     // state-only pass: [BH, nseg, Dk] total log-decay of the segment
    int* status;
    int tiles_per_seg;
    int nseg;
    int seg_offset;       // segment index = blockIdx.z + seg_offset
    float* saved;         // output pass: [BH, save_nseg, Dk, Dv] states entering the backward's
                          // segments (entry z after save_tps * z tiles), or null
    int save_tps;
    int save_nseg;
};

template <int DK, int DVT, int GATE, int MODE>
__global__ void __launch_bounds__(NTHR_WS, 1)
    k_tc_fwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
             const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tg,
             const __grid_constant__ CUtensorMap to, FwdArgs A, Dims P) {
    using C = Cfg<DK, DVT, GATE, MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_align1024(smem_raw);
    uint8_t* sPb = sm + C::NS * C::STAGE;
    uint8_t* sS = sPb + C::PB;
    uint8_t* sO = sS + C::SB;
    uint8_t* small = sO + C::OB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(small);
    uint64_t* bar_full = bars + 0;     // [NS] TMA landed
    uint64_t* bar_empty = bars + 4;    // [NS] stage's MMAs done
    uint64_t* bar_trans = bars + 8;    // [NS] stage transformed
    uint64_t* bar_mma1 = bars + 12;    // [2] O_inter and the state product of the tile done
    uint64_t* bar_mma2 = bars + 14;    // [NAB] P V done
    uint64_t* bar_pready = bars + 17;  // [2] P written
    uint64_t* bar_tfree = bars + 19;   // [NAB] A/O buffer read out
    uint64_t* bar_gfree = bars + 22;   // [2] e^Gamma buffer read by the state epilogue
    uint64_t* bar_sready = bars + 24;  // state of the last tile decayed (and its bf16 copy written)
    uint64_t* bar_aready = bars + 25;  // [NAB] A of the tile done
    constexpr int NBARS = 28;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + 224);
    volatile int* abortp = reinterpret_cast<volatile int*>(small + 228);
    int* n_issued = reinterpret_cast<int*>(small + 232);
    int* n_consumed = reinterpret_cast<int*>(small + 236);
    int* n_mma1 = reinterpret_cast<int*>(small + 240);
    int* n_mma2 = reinterpret_cast<int*>(small + 244);
    float* tot = reinterpret_cast<float*>(small + 256);      // [2 NTRF] cumsum segment totals
    float* gamb = tot + 2 * NTRF;                            // [2][DK] e^Gamma per buffer
    float* gamlb = gamb + 2 * DK;                            // [2][DK] Gamma per buffer
    float* rowE = gamlb + 2 * DK;                            // [64] e^b   (per-head gate)
    float* rowEi = rowE + TR;                                // [64] e^-b
    float* igs = rowEi + TR;                                 // [64] input gate
    float* ghs = igs + TR;                                   // [64] per-head gate
    float* orf = ghs + TR;                                   // [NF][64] output row factors (!XQ)

    const int bh = blockIdx.x, vt = blockIdx.y, z = blockIdx.z + A.seg_offset;
    const int e0 = vt * DVT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, qd = warp & 3;   // meaningful for the epilogue warps
    const int ntiles_all = cdiv(P.L, TR);
    const int tile0 = z * A.tiles_per_seg;
    const int ntiles = min(ntiles_all, tile0 + A.tiles_per_seg) - tile0;
    const long rowbase = (long)bh * P.L;
    // the j-th tile this CTA processes (the forward state-only pass walks its segment backwards)
    auto tile_at = [&](int j) { return MODE == 1 ? tile0 + ntiles - 1 - j : tile0 + j; };
    const bool is_ep = tid < NEP;
    // epilogue threads: key-dim row of the state this lane holds (M=64 state: lanes 0-15)
    const bool srow_ok = (DK != 64) || (lane < 16);
    auto srow = [&](int h) { return (DK == 64 ? 16 * qd + (lane & 15) : 32 * qd + lane) + 128 * h; };

    grid_dep_launch();   // a kernel launched after this one to overlap it may start now
    if (tid == 0) {
        for (int j = 0; j < NBARS; ++j) mbar_init(&bars[j], 1);
        *abortp = 0;
        *n_issued = 0;
        *n_consumed = 0;
        *n_mma1 = 0;
        *n_mma2 = 0;
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, C::NCOL);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    grid_dep_wait();   // output pass after a segment scan: the initial states are written

    // ---- initial state -> TMEM (fp32) and its bf16 copy -> shared memory
    const bool s_worker = is_ep && (MODE != 0 || wg == 0);
    const int scol0 = MODE == 0 ? 0 : wg * C::SCOLS;   // first state column of this state-pass thread
    float glog[C::NH];
    // the output pass starts from h0 or the segment's initial state: all threads stage this
    // CTA's [DK, DVT] block through the ring stages (free until the first loads), coalesced
    static_assert(MODE != 0 || DK * DVT * 4 <= C::NS * C::STAGE, "state staging");
    const float* src = nullptr;
    if (MODE == 0) {
        if (z == 0) src = A.h0 ? A.h0 + (long)bh * DK * P.Dv + e0 : nullptr;
        else src = A.sinit + ((long)bh * A.sinit_nseg + (long)z * A.sinit_step) * DK * P.Dv + e0;
    }
    const float* stg = reinterpret_cast<const float*>(sm);
    if (src) {
        stage_rows<DK, DVT, NTHR_WS>(reinterpret_cast<float*>(sm), src, nullptr, P.Dv, nullptr, tid);
        __syncthreads();
    }
    if (s_worker) {
#pragma unroll
        for (int h = 0; h < C::NH; ++h) {
            const int d = srow(h);
            glog[h] = 0.f;
#pragma unroll
            for (int c = 0; c < C::SCOLS; c += C::CH) {
                const int col = scol0 + c;
                float f[C::CH];
#pragma unroll
                for (int j = 0; j < C::CH; j += 16) {
                    if (src && srow_ok) staged_row16<DVT>(stg, d, col + j, f + j);
                    else
#pragma unroll
                        for (int u = 0; u < 16; ++u) f[j + u] = 0.f;
                }
                tmem_stn<C::CH>(tbase + ((uint32_t)(32 * qd) << 16) + h * DVT + col, reinterpret_cast<uint32_t*>(f));
                if (MODE == 0 && srow_ok)
#pragma unroll
                    for (int j = 0; j < C::CH; j += 8) store8_bf16(sS, sw128_off(d, col + j, DK * 128), &f[j]);
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == W_TMA) {
        // ================================================================ TMA producer
        if (lane == 0) {
            if (MODE == 0) tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            if (GATE == 1) tma_prefetch_desc(&tg);
            for (int j = 0; j < ntiles; ++j) {
                const int s = j % C::NS;
                if (j >= C::NS && !mbar_wait_abort(&bar_empty[s], ((j / C::NS) - 1) & 1, abortp)) break;
                uint8_t* st = sm + s * C::STAGE;
                const int t0 = tile_at(j) * TR;
                mbar_arrive_expect_tx(&bar_full[s], C::STAGE);
                if (MODE == 0)
                    for (int cb = 0; cb < DK / 64; ++cb)
                        tma_load_3d(st + cb * BLK, &tq, cb * 64, t0, bh, &bar_full[s]);
                if (MODE == 1) {
                    // the state-only pass walks its segment backwards, so the last tiles it
                    // loads are the first ones the output pass loads next: those stay in L2
                    const uint64_t pol = j >= ntiles - kL2KeepTiles ? l2_policy_evict_last() : l2_policy_evict_first();
                    for (int cb = 0; cb < DK / 64; ++cb)
                        tma_load_3d_hint(st + C::QB + cb * BLK, &tk, cb * 64, t0, bh, &bar_full[s], pol);
                    if (GATE == 1) tma_load_3d_hint(st + C::QB + C::KB, &tg, 0, t0, bh, &bar_full[s], pol);
                    for (int vb = 0; vb < DVT / 64; ++vb)
                        tma_load_3d_hint(st + C::QB + C::KB + C::GB + vb * BLK, &tv, e0 + vb * 64, t0, bh, &bar_full[s],
                                         pol);
                } else {
                    for (int cb = 0; cb < DK / 64; ++cb)
                        tma_load_3d(st + C::QB + cb * BLK, &tk, cb * 64, t0, bh, &bar_full[s]);
                    if (GATE == 1) tma_load_3d(st + C::QB + C::KB, &tg, 0, t0, bh, &bar_full[s]);
                    for (int vb = 0; vb < DVT / 64; ++vb)
                        tma_load_3d(st + C::QB + C::KB + C::GB + vb * BLK, &tv, e0 + vb * 64, t0, bh, &bar_full[s]);
                }
                *n_issued = j + 1;
                // with a shallow ring (output pass, two stages) the tile that takes this stage
                // next is brought into L2 now, so that its load (issued once the stage is
                // released) does not wait on DRAM; deeper rings and the streaming state-only
                // passes keep enough loads in flight without it
                if (MODE == 0 && C::NS <= 2 && j + C::NS < ntiles) {
                    const int tp = tile_at(j + C::NS) * TR;
                    if (MODE == 0)
                        for (int cb = 0; cb < DK / 64; ++cb) tma_prefetch_l2_3d(&tq, cb * 64, tp, bh);
                    for (int cb = 0; cb < DK / 64; ++cb) tma_prefetch_l2_3d(&tk, cb * 64, tp, bh);
                    if (GATE == 1) tma_prefetch_l2_3d(&tg, 0, tp, bh);
                    for (int vb = 0; vb < DVT / 64; ++vb) tma_prefetch_l2_3d(&tv, e0 + vb * 64, tp, bh);
                }
            }
        }
    } else if (warp == W_MMA) {
        // ================================================================ MMA issuer
        // Per tile i: P V of tile i-1 (once its P is written; this releases its ring stage),
        // A(i) = q~ k~^T (commit: the P epilogue may start), then, once the state of tile
        // i-1 is decayed, O(i) = q~ S_prev and S += k~^T V (commit: the state epilogue may
        // start).
        {
            const bool leader = elect_one();
            // every lane waits; the vote keeps the warp's decision uniform
            auto warp_wait = [&](uint64_t* bar, uint32_t parity, volatile int* ab) -> bool {
                return __all_sync(0xffffffffu, mbar_wait_abort(bar, parity, ab));
            };
            const uint32_t idA = idesc_bf16(64, 64, 0, 0);
            const uint32_t idO = idesc_bf16(64, DVT, 0, 1);
            const uint32_t idS = idesc_bf16(C::MS, DVT, 1, 1);
            const uint64_t dS0 = sw128_desc(smem_u32(sS), DK * 128, 1024);
            const uint64_t dP = sw128_desc(smem_u32(sPb), 16, 1024);
            auto issue_pv = [&](int j) -> bool {
                const int sj = j % C::NS, aj = j % C::NAB;
                if (!warp_wait(&bar_pready[j & 1], (j >> 1) & 1, abortp)) return false;
                tc_fence_after();
                const uint64_t dVj = sw128_desc(smem_u32(sm + sj * C::STAGE + C::QB + C::KB + C::GB), BLK, 1024);
                const uint32_t tOj = tbase + C::COLS_S + aj * C::COLA + (16u << 16);
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < TR / 16; ++ks)
                        mma_bf16(tOj, dP + ((ks * 32) >> 4), dVj + ((ks * 2048) >> 4), idO, 1);
                    mma_commit(&bar_mma2[aj]);
                    *n_mma2 = j + 1;
                    if (j + C::NS < ntiles) mma_commit(&bar_empty[sj]);
                }
                __syncwarp();
                return true;
            };
            bool alive = true;
            for (int i = 0; i < ntiles && alive; ++i) {
                const int s = i % C::NS, b = i & 1, ab = i % C::NAB;
                // P V of the previous tile first: it releases that tile's ring stage
                if (MODE == 0 && i >= 1 && !issue_pv(i - 1)) break;
                if (!warp_wait(&bar_trans[s], (i / C::NS) & 1, abortp)) break;
                if (MODE == 0 && i >= C::NAB &&
                    !warp_wait(&bar_tfree[ab], ((i / C::NAB) - 1) & 1, abortp))
                    break;
                tc_fence_after();
                uint8_t* st = sm + s * C::STAGE;
                // descriptors of the stage's tiles; K steps advance the 16-byte start field
                const uint64_t dQ = sw128_desc(smem_u32(st), 16, 1024);
                const uint64_t dKk = sw128_desc(smem_u32(st + C::QB), 16, 1024);       // k~, K-major
                const uint64_t dKm = sw128_desc(smem_u32(st + C::QB), BLK, 1024);      // k~, MN-major
                const uint64_t dV = sw128_desc(smem_u32(st + C::QB + C::KB + C::GB), BLK, 1024);
                const uint32_t tAO = tbase + C::COLS_S + ab * C::COLA;
                if (MODE == 0 && leader) {
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint64_t ko = ((kk >> 2) * BLK + (kk & 3) * 32) >> 4;
                        mma_bf16(tAO, dQ + ko, dKk + ko, idA, kk > 0);
                    }
                    mma_commit(&bar_aready[ab]);
                }
                __syncwarp();
                // the state of the previous tile must be decayed (and copied) first
                if (MODE == 0 && i >= 1) {
                    if (!warp_wait(bar_sready, (i - 1) & 1, abortp)) break;
                    tc_fence_after();
                }
                if (leader) {
                    if (MODE == 0) {
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk) {
                            const uint64_t ko = ((kk >> 2) * BLK + (kk & 3) * 32) >> 4;
                            mma_bf16(tAO + (16u << 16), dQ + ko, dS0 + ((kk * 2048) >> 4), idO, kk > 0);
                        }
                    }
#pragma unroll
                    for (int h = 0; h < C::NH; ++h)
#pragma unroll
                        for (int ks = 0; ks < TR / 16; ++ks)
                            mma_bf16(tbase + h * DVT, dKm + ((h * 2 * BLK + ks * 2048) >> 4),
                                     dV + ((ks * 2048) >> 4), idS, 1);
                    mma_commit(&bar_mma1[b]);
                    *n_mma1 = i + 1;
                    if (MODE != 0 && i + C::NS < ntiles) mma_commit(&bar_empty[s]);
                }
                __syncwarp();
                if (MODE == 0 && i == ntiles - 1) alive = issue_pv(i);
            }
        }
    } else if (!is_ep) {
        // ================================================================ transform warpgroups
        // Step A: b = inclusive column cumsum of the log-gate, in row segments (thread = key
        // dim x segment) joined through the segment totals, written over g in place in
        // base-2 units (b * log2 e; MODE 1 writes (b - Gamma - D), MODE 2 (b + D) * log2 e). Step B: every 16-byte
        // chunk (8 key dims of one row) of the k tile, and of the q tile in the output pass,
        // is scaled in place by its exponentials and rounded to bf16 (q also by the output
        // scale, so that A, P and O carry it).
        const int ttid = tid - NEP;
        constexpr int NO = DK / 8;
        constexpr int SEG = NTRF / DK, RS = TR / SEG;        // step A: segments, rows per segment
        constexpr int NPOS = TR * NO;                        // step B: (row, chunk) positions
        constexpr int NB = 2;                                // positions per batch of loads
        static_assert(NPOS % (NB * NTRF) == 0 && TR % SEG == 0, "transform mapping");
        const int dA = ttid % DK, sA = ttid / DK;
        float dlat1 = 0.f;   // MODE 1/2: log-decay of the tiles walked so far (key dim dA, or per head)
        constexpr bool kFused = GATE == 1 && DK <= 128;
        if constexpr (kFused) {
            // Per-key gates, one pass per tile: thread = key-dim pair x run of RSF rows. The
            // column cumsum of its rows stays in registers (b never goes through shared
            // memory), the run totals are exchanged once, and each row's q, k pairs are scaled
            // right away (MODE 1: k only; MODE 2, q in the k slot: scale q e^(D + b)).
            constexpr int NP = DK / 2, SEGF = NTRF / NP, RSF = TR / SEGF;
            static_assert(NTRF % NP == 0 && TR % SEGF == 0 && 2 * NTRF >= SEGF * DK, "fused transform mapping");
            const int p = ttid % NP, sgi = ttid / NP, d0 = 2 * p;
            float2* tot2 = reinterpret_cast<float2*>(tot);   // [SEGF][NP] run totals
            const uint64_t sc2 = f2(P.scale, P.scale);
            float2 dlat = make_float2(0.f, 0.f);   // MODE 1/2: log-decay of the tiles walked so far
            for (int j = 0; j < ntiles; ++j) {
                const int s = j % C::NS, b = j & 1;
                uint8_t* st = sm + s * C::STAGE;
                uint8_t* sq = st;
                uint8_t* sk = st + C::QB;
                const float* sgt = reinterpret_cast<const float*>(st + C::QB + C::KB);
                const int t0 = tile_at(j) * TR;
                if (ttid < TR) {
                    const int t = t0 + ttid;
                    igs[ttid] = (A.ig && t < P.L) ? A.ig[rowbase + t] : 1.f;
                }
                bool ok = mbar_wait_abort(&bar_full[s], (j / C::NS) & 1, abortp);
                if (ok && j >= 2) ok = mbar_wait_abort(&bar_gfree[b], ((j >> 1) - 1) & 1, abortp);
                float2 cs[RSF];
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int u = 0; u < RSF; ++u) {
                    const float2 x = *reinterpret_cast<const float2*>(sgt + (sgi * RSF + u) * DK + d0);
                    acc.x += x.x;
                    acc.y += x.y;
                    cs[u] = acc;
                }
                tot2[sgi * NP + p] = acc;
                if (!named_bar_and(BAR_TR, NTRF, ok)) break;
                if (ttid == 0) *n_consumed = j + 1;
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
                // exponent of row u = cs[u] + c: b (output pass), D + b (MODE 2, D the decay of
                // the tiles before this one), and in MODE 1 b - Gamma - D (D the decay of the tiles
                // after it), whose negation scales k
                const float cx = MODE == 0 ? off.x : MODE == 2 ? off.x + dlat.x : off.x - G.x - dlat.x;
                const float cy = MODE == 0 ? off.y : MODE == 2 ? off.y + dlat.y : off.y - G.y - dlat.y;
                if (MODE != 0) {
                    dlat.x += G.x;
                    dlat.y += G.y;
                }
                if (sgi == 0) {
                    float* gam = gamb + b * DK;
                    float* gaml = gamlb + b * DK;
                    gam[d0] = __expf(G.x);
                    gam[d0 + 1] = __expf(G.y);
                    gaml[d0] = G.x;
                    gaml[d0 + 1] = G.y;
                    // (the state-only passes scale by whole decays <= 1: any gate strength)
                    if (MODE == 0 && (G.x < kMinTileLogDecay || G.y < kMinTileLogDecay)) atomicOr(A.status, kDevStatusRange);
                }
#pragma unroll
                for (int u = 0; u < RSF; ++u) {
                    const int r = sgi * RSF + u;
                    // byte offset of (r, d0) in a 128-byte-swizzled bf16 tile
                    const uint32_t ob = (uint32_t)(d0 >> 6) * BLK + (uint32_t)r * 128 +
                                        ((((uint32_t)((d0 & 63) >> 3)) ^ (uint32_t)(r & 7)) << 4) + (uint32_t)(d0 & 7) * 2;
                    const float bx = (cs[u].x + cx) * kLog2e, by = (cs[u].y + cy) * kLog2e;
                    uint32_t* pk = reinterpret_cast<uint32_t*>(sk + ob);
                    if (MODE == 2) {
                        *pk = f2_to_bf2(f2_mul(bf2_to_f2(*pk), f2_mul(sc2, f2(ex2_approx(bx), ex2_approx(by)))));
                    } else {
                        const float m = igs[r];
                        float ex = 1.f, ey = 1.f, dx, dy;
                        if (MODE == 0) {
                            // e^-b = 1 / e^b (one exponential and one reciprocal per element)
                            ex = ex2_approx(bx);
                            ey = ex2_approx(by);
                            dx = rcp_approx(ex);
                            dy = rcp_approx(ey);
                        } else {
                            dx = ex2_approx(-bx);
                            dy = ex2_approx(-by);
                        }
                        *pk = f2_to_bf2(f2_mul(bf2_to_f2(*pk), f2_mul(f2(m, m), f2(dx, dy))));
                        if (MODE == 0) {
                            uint32_t* pq = reinterpret_cast<uint32_t*>(sq + ob);
                            *pq = f2_to_bf2(f2_mul(bf2_to_f2(*pq), f2_mul(sc2, f2(ex, ey))));
                        }
                    }
                }
                fence_proxy_async_smem();
                named_bar_sync(BAR_TR, NTRF);
                if (ttid == 0) mbar_arrive(&bar_trans[s]);
            }
        } else
        for (int j = 0; j < ntiles; ++j) {
            const int s = j % C::NS, b = j & 1;
            uint8_t* st = sm + s * C::STAGE;
            uint8_t* sq = st;
            uint8_t* sk = st + C::QB;
            float* sg = reinterpret_cast<float*>(st + C::QB + C::KB);
            float* gam = gamb + b * DK;
            float* gaml = gamlb + b * DK;
            const int t0 = tile_at(j) * TR;
            if (ttid < TR) {
                const int t = t0 + ttid;
                igs[ttid] = (A.ig && t < P.L) ? A.ig[rowbase + t] : 1.f;
                if (GATE == 2) ghs[ttid] = (t < P.L) ? A.gh[rowbase + t] : 0.f;
            }
            bool ok = mbar_wait_abort(&bar_full[s], (j / C::NS) & 1, abortp);
            if (ok && j >= 2) ok = mbar_wait_abort(&bar_gfree[b], ((j >> 1) - 1) & 1, abortp);
            if (!named_bar_and(BAR_TR, NTRF, ok)) break;
            if (ttid == 0) *n_consumed = j + 1;
            // ---- step A
            if (GATE == 1) {
                float* col = sg + sA * RS * DK + dA;
                float x[RS];
#pragma unroll
                for (int u = 0; u < RS; ++u) x[u] = col[u * DK];
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < RS; ++u) {
                    acc += x[u];
                    x[u] = acc;
                }
                float off = 0.f, G = acc;
                if constexpr (SEG > 1) {
                    tot[ttid] = acc;
                    named_bar_sync(BAR_TR, NTRF);
                    G = 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < SEG; ++s2) {
                        const float t = tot[s2 * DK + dA];
                        if (s2 < sA) off += t;
                        G += t;
                    }
                }
                const float sub = MODE == 0 ? -off : MODE == 2 ? -off - dlat1 : G - off + dlat1;
                if (MODE != 0) dlat1 += G;
#pragma unroll
                for (int u = 0; u < RS; ++u) col[u * DK] = (x[u] - sub) * kLog2e;
                if (sA == 0) {
                    gam[dA] = __expf(G);
                    gaml[dA] = G;
                    if (MODE == 0 && G < kMinTileLogDecay) atomicOr(A.status, kDevStatusRange);
                }
            } else if (GATE == 2) {
                if (ttid < 32) {  // warp scan over 64 rows, two rows per lane
                    const float g0 = ghs[2 * lane], g1 = ghs[2 * lane + 1];
                    float v = g0 + g1;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float n = __shfl_up_sync(0xffffffffu, v, off);
                        if (lane >= off) v += n;
                    }
                    const float b1 = v, b0 = v - g1;
                    const float G = __shfl_sync(0xffffffffu, b1, 31);
                    // MODE 2 scales q by its decay from the segment's start, e^(D + b)
                    const float bq0 = MODE == 2 ? b0 + dlat1 : b0, bq1 = MODE == 2 ? b1 + dlat1 : b1;
                    rowE[2 * lane] = __expf(bq0);
                    if (MODE == 0) {   // the output pass's row factors of this tile
                        orf[(j % C::NF) * TR + 2 * lane] = P.scale * rowE[2 * lane];
                        orf[(j % C::NF) * TR + 2 * lane + 1] = P.scale * __expf(bq1);
                    }
                    rowE[2 * lane + 1] = __expf(bq1);
                    // MODE 1: e^(D + Gamma - b), the decay from the token to the segment's end
                    rowEi[2 * lane] = __expf(MODE == 1 ? dlat1 + G - b0 : -b0);
                    rowEi[2 * lane + 1] = __expf(MODE == 1 ? dlat1 + G - b1 : -b1);
                    if (MODE != 0) dlat1 += G;
                    if (lane == 0) {
                        gam[0] = __expf(G);
                        gaml[0] = G;
                        if (MODE == 0 && G < kMinTileLogDecay) atomicOr(A.status, kDevStatusRange);
                    }
                }
            }
            named_bar_sync(BAR_TR, NTRF);
            // ---- step B: MODE 0/1 k -> i k e^-b, MODE 0 q -> q e^b, MODE 2 (q in the k slot) -> scale q e^(D+b)
#pragma unroll
            for (int it0 = 0; it0 < NPOS / NTRF; it0 += NB) {
                float bv[NB][8];
                uint4 wq[NB], wk[NB];
                uint32_t offs[NB];
                int rows[NB];
#pragma unroll
                for (int k = 0; k < NB; ++k) {
                    const int c = ttid + (it0 + k) * NTRF;
                    const int r = c / NO, d0 = 8 * (c % NO);
                    rows[k] = r;
                    if (GATE == 1) {
                        const float4 b0 = *reinterpret_cast<const float4*>(sg + r * DK + d0);
                        const float4 b1 = *reinterpret_cast<const float4*>(sg + r * DK + d0 + 4);
                        bv[k][0] = b0.x; bv[k][1] = b0.y; bv[k][2] = b0.z; bv[k][3] = b0.w;
                        bv[k][4] = b1.x; bv[k][5] = b1.y; bv[k][6] = b1.z; bv[k][7] = b1.w;
                    }
                    offs[k] = (uint32_t)(d0 >> 6) * BLK + (uint32_t)r * 128 +
                              ((((uint32_t)((d0 & 63) >> 3)) ^ (uint32_t)(r & 7)) << 4);
                    if (C::XQ) wq[k] = *reinterpret_cast<const uint4*>(sq + offs[k]);
                    wk[k] = *reinterpret_cast<const uint4*>(sk + offs[k]);
                }
#pragma unroll
                for (int k = 0; k < NB; ++k) {
                    const int r = rows[k];
                    const float mk = MODE == 2 ? P.scale : igs[r];
                    float eu[8], ed[8];   // e^(+b) for q (MODE 0 and 2), e^(-b) for k (MODE 0 and 1)
                    if (GATE == 1) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            // output pass: e^-b = 1 / e^b (one exponential per element)
                            eu[u] = MODE != 1 ? ex2_approx(bv[k][u]) : 1.f;
                            ed[u] = MODE == 0 ? rcp_approx(eu[u]) : MODE == 1 ? ex2_approx(-bv[k][u]) : 1.f;
                        }
                    } else {
                        const float fu = GATE == 2 ? rowE[r] : 1.f, fd = GATE == 2 ? rowEi[r] : 1.f;
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            eu[u] = fu;
                            ed[u] = fd;
                        }
                    }
                    // factors first (m * e), then one packed multiply per element pair
                    uint32_t* pk = reinterpret_cast<uint32_t*>(&wk[k]);
                    const uint64_t mk2 = f2(mk, mk);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint64_t e2 = MODE == 2 ? f2(eu[2 * u], eu[2 * u + 1]) : f2(ed[2 * u], ed[2 * u + 1]);
                        pk[u] = f2_to_bf2(f2_mul(bf2_to_f2(pk[u]), f2_mul(mk2, e2)));
                    }
                    *reinterpret_cast<uint4*>(sk + offs[k]) = wk[k];
                    if (C::XQ) {
                        uint32_t* pq = reinterpret_cast<uint32_t*>(&wq[k]);
                        const uint64_t sc2 = f2(P.scale, P.scale);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            pq[u] = f2_to_bf2(f2_mul(bf2_to_f2(pq[u]), f2_mul(sc2, f2(eu[2 * u], eu[2 * u + 1]))));
                        *reinterpret_cast<uint4*>(sq + offs[k]) = wq[k];
                    }
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(BAR_TR, NTRF);
            if (ttid == 0) mbar_arrive(&bar_trans[s]);
        }
    } else if (s_worker) {
        // ================================================================ state epilogue
        // S = e^Gamma (S_prev + dS'), where the MMA has added dS' onto S_prev in TMEM; the
        // decayed state goes back to TMEM and, as bf16, to shared memory (next tile's q~ S)
        const uint32_t lq = (uint32_t)(32 * qd) << 16;   // this warp's TMEM lane quadrant
        for (int i = 0; i < ntiles; ++i) {
            const int b = i & 1;
            {
                const bool ok = mbar_wait_abort(&bar_mma1[b], (i >> 1) & 1, abortp);
                if (!named_bar_and(BAR_S, C::NSW, ok)) break;
            }
            tc_fence_after();
            const float* gam = gamb + b * DK;
            const float* gaml = gamlb + b * DK;
            // the state after this tile enters backward segment save_z when a boundary follows it
            int save_z = 0;
            if (MODE == 0 && A.saved) {
                const int nxt = tile_at(i) + 1;
                if (nxt % A.save_tps == 0 && nxt / A.save_tps < A.save_nseg) save_z = nxt / A.save_tps;
            }
#pragma unroll
            for (int h = 0; h < C::NH; ++h) {
                const int d = srow(h);
                const int gi = GATE == 1 ? d : 0;
                const float egv = GATE == 0 ? 1.f : gam[gi];
                if (GATE != 0) glog[h] += gaml[gi];
                // the state-only passes scaled k (q) by whole decays to the segment's end (from its
                // start): nothing to decay
#pragma unroll
                for (int c = 0; c < (MODE != 0 ? 0 : C::SCOLS); c += C::CH) {
                    const int col = scol0 + c;
                    float f[C::CH];
                    uint32_t* r = reinterpret_cast<uint32_t*>(f);
                    tmem_ldn<C::CH>(tbase + lq + h * DVT + col, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < C::CH; j += 2) {
                        const uint64_t x = f2_mul(f2(f[j], f[j + 1]), f2(egv, egv));
                        asm("mov.b64 {%0, %1}, %2;" : "=f"(f[j]), "=f"(f[j + 1]) : "l"(x));
                    }
                    tmem_stn<C::CH>(tbase + lq + h * DVT + col, r);
                    if (MODE == 0 && srow_ok)
#pragma unroll
                        for (int j = 0; j < C::CH; j += 8) store8_bf16(sS, sw128_off(d, col + j, DK * 128), &f[j]);
                    if (MODE == 0 && save_z > 0 && srow_ok) {
                        float* dst = A.saved + (((long)bh * A.save_nseg + save_z) * DK + d) * P.Dv + e0 + col;
#pragma unroll
                        for (int j = 0; j < C::CH; j += 4)
                            *reinterpret_cast<float4*>(dst + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
                    }
                }
            }
            tmem_wait_st();
            if (MODE == 0) fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(BAR_S, C::NSW);
            if (tid == 0) {
                mbar_arrive(bar_sready);
                mbar_arrive(&bar_gfree[b]);
            }
        }
    } else if (MODE == 0 && is_ep) {
        // ================================================================ P and output epilogue
        const uint32_t lq = (uint32_t)(32 * qd) << 16;
        const int ptid = tid - 128;
        for (int i = 0; i < ntiles; ++i) {
            const int b = i & 1;
            const int ab = i % C::NAB;
            const uint32_t tAO = tbase + C::COLS_S + ab * C::COLA;
            {
                const bool ok = mbar_wait_abort(&bar_aready[ab], (i / C::NAB) & 1, abortp);
                if (!named_bar_and(BAR_PO, 128, ok)) break;
            }
            tc_fence_after();
            const int t0 = tile_at(i) * TR;
            // ---- P = causal mask of A -> shared (single buffer: P V of the previous tile is
            //      complete, its output pass waited for it)
            {
                uint8_t* sP = sPb;
#pragma unroll
                for (int c0 = 0; c0 < TR; c0 += C::CH) {
                    uint32_t r[C::CH];
                    tmem_ldn<C::CH>(tAO + lq + c0, r);
                    tmem_wait_ld();
                    if (lane < 16) {
                        const int t = 16 * qd + lane;
#pragma unroll
                        for (int u = 0; u < C::CH / 8; ++u) {
                            float f[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int sidx = c0 + 8 * u + j;
                                f[j] = (sidx <= t) ? __uint_as_float(r[8 * u + j]) : 0.f;
                            }
                            store8_bf16(sP, sw128_off(t, c0 + 8 * u, BLK), f);
                        }
                    }
                }
                fence_proxy_async_smem();
                named_bar_sync(BAR_PO, 128);
                if (ptid == 0) mbar_arrive(&bar_pready[b]);
            }
            // ---- output tile: TMEM -> bf16 tile in shared memory -> TMA store
            {
                bool ok = mbar_wait_abort(&bar_mma2[ab], (i / C::NAB) & 1, abortp);
                if (ptid == 0) bulk_wait_read<0>();   // the previous tile's store has read the staging tile
                if (!named_bar_and(BAR_PO, 128, ok)) break;
                tc_fence_after();
                const int t = 16 * qd + (lane & 15);
                // per-head or no gates: row t of O is q S_prev + P V, scaled here by scale e^(b_t)
                const float rf = C::XQ ? 1.f : GATE == 2 ? orf[(i % C::NF) * TR + t] : P.scale;
#pragma unroll
                for (int c = 0; c < DVT; c += C::CH) {
                    uint32_t r[C::CH];
                    tmem_ldn<C::CH>(tAO + lq + c, r);
                    tmem_wait_ld();
                    if (lane >= 16)
#pragma unroll
                        for (int u = 0; u < C::CH / 8; ++u) {
                            float f[8];
#pragma unroll
                            for (int jj = 0; jj < 8; ++jj) f[jj] = C::XQ ? __uint_as_float(r[8 * u + jj]) : rf * __uint_as_float(r[8 * u + jj]);
                            store8_bf16(sO, sw128_off(t, c + 8 * u, BLK), f);
                        }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            named_bar_sync(BAR_PO, 128);
            if (ptid == 0) {
                for (int vb = 0; vb < DVT / 64; ++vb) tma_store_3d(&to, sO + vb * BLK, e0 + 64 * vb, t0, bh);
                bulk_commit();
            }
            if (ptid == 0) mbar_arrive(&bar_tfree[ab]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abortp) {
        if (tid == 0) {
            atomicOr(A.status, kDevStatusTimeout);
            // let every issued copy and product land before shared memory and TMEM go away
            for (int j = *n_consumed; j < *n_issued; ++j)
                mbar_wait(&bar_full[j % C::NS], (j / C::NS) & 1, 1u << 20);
            if (*n_mma1) mbar_wait(&bar_mma1[(*n_mma1 - 1) & 1], ((*n_mma1 - 1) >> 1) & 1, 1u << 20);
            if (*n_mma2) mbar_wait(&bar_mma2[(*n_mma2 - 1) % C::NAB], ((*n_mma2 - 1) / C::NAB) & 1, 1u << 20);
        }
    } else {
        // final state of the segment: TMEM -> rows in shared memory (the ring stages are idle
        // now) -> coalesced rows in global memory
        float* dst = nullptr;   // row 0, column e0 of this CTA's block
        if (MODE == 0) {
            if (z == A.nseg - 1 && A.hT) dst = A.hT + (long)bh * DK * P.Dv + e0;
        } else {
            dst = A.seg_state + ((long)bh * A.nseg + z) * DK * P.Dv + e0;
        }
        static_assert(DK * DVT * 4 <= C::NS * C::STAGE, "state staging");
        float* stg = reinterpret_cast<float*>(sm);
        if (s_worker) {
            const uint32_t lq = (uint32_t)(32 * qd) << 16;
#pragma unroll
            for (int h = 0; h < C::NH; ++h) {
                const int d = srow(h);
                if (MODE != 0 && vt == 0 && scol0 == 0 && srow_ok)
                    A.seg_gamma[((long)bh * A.nseg + z) * DK + d] = glog[h];
                if (!dst) continue;
#pragma unroll
                for (int c = 0; c < C::SCOLS; c += C::CH) {
                    const int col = scol0 + c;
                    float f[C::CH];
                    tmem_ldn<C::CH>(tbase + lq + h * DVT + col, reinterpret_cast<uint32_t*>(f));
                    tmem_wait_ld();
                    if (srow_ok)
#pragma unroll
                        for (int j = 0; j < C::CH; j += 16) staged_put16<DVT>(stg, d, col + j, f + j);
                }
            }
        }
        if (dst) {   // uniform over the block
            __syncthreads();
            unstage_rows<DK, DVT, NTHR_WS>(stg, dst, P.Dv, tid);
        }
    }
    if (MODE == 0 && tid == 128) bulk_wait<0>();   // the last output stores have completed
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, C::NCOL);
}

// Segment scan: sinit[z] = e^{Gamma_{z-1}} sinit[z-1] + dS_{z-1}, sinit[0] = h0 (or 0).
// One thread per four consecutive state elements of one (bh, d) row; the loads of SEGU
// segments are issued before their dependent chain, so that the walk is bandwidth-bound.
constexpr int SEGU = 8;
__global__ void __launch_bounds__(256) k_seg_scan(const float* __restrict__ seg_state,
                                                  const float* __restrict__ seg_gamma, const float* __restrict__ h0,
                                                  float* __restrict__ sinit, int BH, int Dk, int Dv, int nseg) {
    grid_dep_launch();
    grid_dep_wait();   // the state pass has written seg_state, seg_gamma
    const int per4 = Dk * Dv / 4;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)BH * per4) return;
    const int bh = (int)(idx / per4), de4 = (int)(idx - (long)bh * per4), d = 4 * de4 / Dv;
    const float4* src = reinterpret_cast<const float4*>(seg_state) + (size_t)bh * nseg * per4 + de4;
    const float* gam = seg_gamma + (size_t)bh * nseg * Dk + d;
    float4* dst = reinterpret_cast<float4*>(sinit) + (size_t)bh * nseg * per4 + de4;
    float4 S = h0 ? __ldg(reinterpret_cast<const float4*>(h0) + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int z0 = 0; z0 < nseg - 1; z0 += SEGU) {
        float4 x[SEGU];
        float e[SEGU];
#pragma unroll
        for (int u = 0; u < SEGU; ++u)
            if (z0 + u < nseg - 1) {
                x[u] = __ldg(src + (size_t)(z0 + u) * per4);
                e[u] = __expf(__ldg(gam + (size_t)(z0 + u) * Dk));
            }
#pragma unroll
        for (int u = 0; u < SEGU; ++u)
            if (z0 + u < nseg - 1) {
                S = make_float4(fmaf(e[u], S.x, x[u].x), fmaf(e[u], S.y, x[u].y), fmaf(e[u], S.z, x[u].z),
                                fmaf(e[u], S.w, x[u].w));
                dst[(size_t)(z0 + u + 1) * per4] = S;
            }
    }
}

// Reverse segment scan for the backward: gend[z] = gradient w.r.t. the state at the end of
// segment z; gend[nseg-1] = dhT (or 0), gend[z] = e^{Gamma_{z+1}} gend[z+1] + dG_{z+1},
// where dG_z (seg_state[z]) is segment z's own state-gradient accumulated from zero at
// its end and Gamma_z (seg_gamma[z]) its total log-decay. Same layout as k_seg_scan.
__global__ void __launch_bounds__(256) k_seg_rscan(const float* __restrict__ seg_state,
                                                   const float* __restrict__ seg_gamma, const float* __restrict__ dhT,
                                                   float* __restrict__ gend, int BH, int Dk, int Dv, int nseg) {
    grid_dep_launch();
    grid_dep_wait();   // the state-gradient pass has written seg_state, seg_gamma
    const int per4 = Dk * Dv / 4;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)BH * per4) return;
    const int bh = (int)(idx / per4), de4 = (int)(idx - (long)bh * per4), d = 4 * de4 / Dv;
    const float4* src = reinterpret_cast<const float4*>(seg_state) + (size_t)bh * nseg * per4 + de4;
    const float* gam = seg_gamma + (size_t)bh * nseg * Dk + d;
    float4* dst = reinterpret_cast<float4*>(gend) + (size_t)bh * nseg * per4 + de4;
    float4 G = dhT ? __ldg(reinterpret_cast<const float4*>(dhT) + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
    dst[(size_t)(nseg - 1) * per4] = G;
    for (int z0 = nseg - 1; z0 >= 1; z0 -= SEGU) {
        float4 x[SEGU];
        float e[SEGU];
#pragma unroll
        for (int u = 0; u < SEGU; ++u)
            if (z0 - u >= 1) {
                x[u] = __ldg(src + (size_t)(z0 - u) * per4);
                e[u] = __expf(__ldg(gam + (size_t)(z0 - u) * Dk));
            }
#pragma unroll
        for (int u = 0; u < SEGU; ++u)
            if (z0 - u >= 1) {
                G = make_float4(fmaf(e[u], G.x, x[u].x), fmaf(e[u], G.y, x[u].y), fmaf(e[u], G.z, x[u].z),
                                fmaf(e[u], G.w, x[u].w));
                dst[(size_t)(z0 - u - 1) * per4] = G;
            }
    }
}

// ------------------------------------------------------------------ host side
// pdl: the kernel follows the segment scan of the same call and may start before it ends
template <int DK, int DVT, int GATE, int MODE>
static cudaError_t launch_one(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const CUtensorMap& mg, const CUtensorMap& mo, const FwdArgs& a, const Dims& P, int nseg,
                              cudaStream_t st, bool pdl = false) {
    using C = Cfg<DK, DVT, GATE, MODE>;
    auto kern = k_tc_fwd<DK, DVT, GATE, MODE>;
    static std::atomic<bool> attr[kMaxDevices];
    {
        const cudaError_t e = smem_attr_once(kern, C::SMEM, attr);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(P.B * P.H, P.Dv / DVT, nseg);
    cudaError_t e = cudaSuccess;
    GLA_LAUNCH(MODE == 0 ? "tc_fwd" : MODE == 1 ? "tc_state" : "tc_gstate", st,
               e = launch_ex(kern, grid, dim3(NTHR_WS), C::SMEM, st, pdl, 1, mq, mk, mv, mg, mo, a, P));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

int pick_dvt(const Dims& P) { return (P.Dk == 256 || P.Dv % 128 != 0) ? 64 : 128; }

int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

FwdPlan plan_fwd(const Dims& P) {
    FwdPlan pl{};
    pl.dvt = pick_dvt(P);
    const int ntiles = cdiv(P.L, TR);
    const long base = (long)P.B * P.H * (P.Dv / pl.dvt);
    const int sms = num_sms();
    int nseg = 1;
    if (base * 4 < (long)sms * 3 && ntiles > 1) nseg = (int)((long)sms / base);
    if (nseg < 1) nseg = 1;
    // Segments are whole 64-token tiles, as equal as the tile count allows: the tensor-core
    // plan carries the state through every tile, so the chunk size does not constrain them
    // (segments of whole 256-token chunks cut 1024 tiles into 17 of 60 tiles and one of 4).
    if (nseg > ntiles) nseg = ntiles;
    if (ntiles == 0) {   // L = 0: one empty segment
        pl.nseg = 1;
        pl.tiles_per_seg = 0;
        return pl;
    }
    pl.tiles_per_seg = cdiv(ntiles, nseg);
    pl.nseg = cdiv(ntiles, pl.tiles_per_seg);
    if (pl.nseg < 1) pl.nseg = 1;
    return pl;
}

// Dv tile of the state-only passes: the widest whose ring keeps several stages, so that the k
// (q) and gate tiles a CTA loads serve as many state columns as possible. Dv = 256 in one tile
// for Dk <= 128 (256 TMEM columns; the final state, up to 128 KB, is staged through the ring);
// Dk = 256 takes 128 columns, or 64 with per-key gates (a 128-column stage already holds 112 KB
// and the ring a single stage).
static int pick_state_dvt(const Dims& P) {
    if (P.Dv % 128 != 0) return 64;
    if (P.Dk == 256) return P.gate == GLA_GATE_PER_KEY ? 64 : 128;
    return P.Dv == 256 ? 256 : 128;
}

// The forward's state pass covers segments 0..nseg-2 of the output pass. It runs in R
// sub-segments per output segment (R divides the segment's tiles), as many as keep its CTAs
// within one wave; the scan then yields the initial state of every sub-segment and the
// output pass reads every R-th.
static int state_subsegments(const Dims& P, const FwdPlan& pl) {
    if (pl.nseg <= 1) return 1;
    const long per = (long)P.B * P.H * (P.Dv / pick_state_dvt(P)) * (pl.nseg - 1);
    const long sms = num_sms();
    int R = 1;
    for (int r = 2; r <= pl.tiles_per_seg; ++r)
        if (pl.tiles_per_seg % r == 0 && per * r <= sms) R = r;
    return R;
}

size_t fwd_workspace_bytes(const Dims& P) {
    const FwdPlan pl = plan_fwd(P);
    if (pl.nseg <= 1) return kStatusBytes;
    const size_t BH = (size_t)P.B * P.H;
    const size_t nsub = (size_t)(pl.nseg - 1) * state_subsegments(P, pl) + 1;
    size_t off = kStatusBytes;
    off = align_up(off + 4 * BH * nsub * P.Dk * P.Dv, 256);   // local end states
    off = align_up(off + 4 * BH * nsub * P.Dk, 256);          // log-decay totals
    off = align_up(off + 4 * BH * nsub * P.Dk * P.Dv, 256);   // initial states
    return off;
}

bool supports(const Dims& P) {
    return P.C % TR == 0 && (P.Dk == 64 || P.Dk == 128 || P.Dk == 256) && P.Dv % 64 == 0;
}

cudaError_t seg_scan(const Dims& P, int nseg, const float* seg_state, const float* seg_gamma, const float* h0,
                     float* sinit, cudaStream_t st);

// State-only pass over every segment but one: MODE 1 (forward states: a = k, b = v) runs
// segments 0..nseg-2, MODE 2 (state gradients: a = q, b = dO) segments 1..nseg-1.
template <int DK, int DVT, int GATE>
static cudaError_t state_run(const Dims& P, int mode, const void* a_src, const void* b_src, const float* g,
                             const float* ig, int nseg, int tps, float* seg_state, float* seg_gamma, int* status,
                             cudaStream_t st) {
    CUtensorMap mk, mv, mg;
    const int BH = P.B * P.H;
    if (!make_map(&mk, a_src, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mv, b_src, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dv, P.L, BH, 64, true))
        return cudaErrorInvalidValue;
    if (GATE == 1) {
        if (!make_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P.Dk, P.L, BH, P.Dk, false))
            return cudaErrorInvalidValue;
    } else {
        mg = mk;
    }
    FwdArgs a{};
    a.gh = GATE == 2 ? g : nullptr;
    a.ig = ig;
    a.seg_state = seg_state;
    a.seg_gamma = seg_gamma;
    a.status = status;
    a.tiles_per_seg = tps;
    a.nseg = nseg;
    a.seg_offset = mode == 2 ? 1 : 0;
    // modes 3 and 4: the forward state / the state gradient of every segment (a sequence shard
    // as one segment)
    if (mode == 1 || mode == 3)
        return launch_one<DK, DVT, GATE, 1>(mk, mk, mv, mg, mk, a, P, mode == 3 ? nseg : nseg - 1, st);
    return launch_one<DK, DVT, GATE, 2>(mk, mk, mv, mg, mk, a, P, mode == 4 ? nseg : nseg - 1, st);
}

template <int DK, int DVT, int GATE>
static cudaError_t run(const Dims& P, const void* q, const void* k, const void* v, const float* g,
                       const float* ig, const float* h0, void* o, float* hT, float* saved, void* ws,
                       cudaStream_t st) {
    const FwdPlan pl = plan_fwd(P);
    CUtensorMap mq, mk, mv, mg, mo;
    const int BH = P.B * P.H;
    if (!make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dk, P.L, BH, 64, true) ||
        !make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dv, P.L, BH, 64, true) ||
        !make_map(&mo, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P.Dv, P.L, BH, 64, true))
        return cudaErrorInvalidValue;
    if (GATE == 1) {
        if (!make_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P.Dk, P.L, BH, P.Dk, false))
            return cudaErrorInvalidValue;
    } else {
        mg = mk;  // unused
    }
    FwdArgs a{};
    a.gh = GATE == 2 ? g : nullptr;
    a.ig = ig;
    a.h0 = h0;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.hT = hT;
    a.status = static_cast<int*>(ws);
    a.tiles_per_seg = pl.tiles_per_seg;
    a.nseg = pl.nseg;
    a.seg_offset = 0;
    a.sinit_nseg = pl.nseg;
    a.sinit_step = 1;
    if (saved) {
        a.saved = saved;
        bwd_plan_info(P, &a.save_nseg, &a.save_tps);
    }
    if (pl.nseg > 1) {
        const int R = state_subsegments(P, pl);
        const int nsub = (pl.nseg - 1) * R + 1;
        char* w = static_cast<char*>(ws);
        size_t off = kStatusBytes;
        float* seg_state = reinterpret_cast<float*>(w + off);
        off = align_up(off + 4 * (size_t)BH * nsub * P.Dk * P.Dv, 256);
        float* seg_gamma = reinterpret_cast<float*>(w + off);
        off = align_up(off + 4 * (size_t)BH * nsub * P.Dk, 256);
        float* sinit = reinterpret_cast<float*>(w + off);
        a.sinit = sinit;
        a.sinit_nseg = nsub;
        a.sinit_step = R;
        cudaError_t e = state_pass(P, 1, k, v, g, ig, nsub, pl.tiles_per_seg / R, seg_state, seg_gamma, a.status, st);
        if (e != cudaSuccess) return e;
        e = seg_scan(P, nsub, seg_state, seg_gamma, h0, sinit, st);
        if (e != cudaSuccess) return e;
    }
    return launch_one<DK, DVT, GATE, 0>(mq, mk, mv, mg, mo, a, P, pl.nseg, st, pl.nseg > 1);
}

cudaError_t seg_scan(const Dims& P, int nseg, const float* seg_state, const float* seg_gamma, const float* h0,
                     float* sinit, cudaStream_t st) {
    const long n = (long)P.B * P.H * P.Dk * P.Dv / 4;
    // follows the state pass of the same call, and may start before it ends
    cudaError_t e = cudaSuccess;
    GLA_LAUNCH("tc_seg_scan", st,
               e = launch_ex(k_seg_scan, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true, 1, seg_state,
                             seg_gamma, h0, sinit, P.B * P.H, P.Dk, P.Dv, nseg));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t seg_rscan(const Dims& P, int nseg, const float* seg_state, const float* seg_gamma, const float* dhT,
                      float* gend, cudaStream_t st) {
    const long n = (long)P.B * P.H * P.Dk * P.Dv / 4;
    // follows the state-gradient pass of the same call, and may start before it ends
    cudaError_t e = cudaSuccess;
    GLA_LAUNCH("tc_seg_rscan", st,
               e = launch_ex(k_seg_rscan, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true, 1, seg_state,
                             seg_gamma, dhT, gend, P.B * P.H, P.Dk, P.Dv, nseg));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int DK, int DVT>
static cudaError_t run_gate(const Dims& P, const void* q, const void* k, const void* v, const float* g,
                            const float* ig, const float* h0, void* o, float* hT, float* saved, void* ws,
                            cudaStream_t st) {
    switch (P.gate) {
        case GLA_GATE_NONE: return run<DK, DVT, 0>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
        case GLA_GATE_PER_KEY: return run<DK, DVT, 1>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
        default: return run<DK, DVT, 2>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
    }
}

template <int DK, int DVT>
static cudaError_t state_gate(const Dims& P, int mode, const void* a_src, const void* b_src, const float* g,
                              const float* ig, int nseg, int tps, float* ss, float* sg, int* status, cudaStream_t st) {
    switch (P.gate) {
        case GLA_GATE_NONE: return state_run<DK, DVT, 0>(P, mode, a_src, b_src, g, ig, nseg, tps, ss, sg, status, st);
        case GLA_GATE_PER_KEY:
            // (pick_state_dvt keeps per-key gates with Dk = 256 on 64-column tiles)
            if constexpr (DK == 256 && DVT == 128) return cudaErrorInvalidValue;
            else return state_run<DK, DVT, 1>(P, mode, a_src, b_src, g, ig, nseg, tps, ss, sg, status, st);
        default: return state_run<DK, DVT, 2>(P, mode, a_src, b_src, g, ig, nseg, tps, ss, sg, status, st);
    }
}

cudaError_t state_pass(const Dims& P, int mode, const void* a_src, const void* b_src, const float* g,
                       const float* ig, int nseg, int tiles_per_seg, float* seg_state, float* seg_gamma, int* status,
                       cudaStream_t st) {
    const int dvt = pick_state_dvt(P);
    if (P.Dk == 64) {
        if (dvt == 256) return state_gate<64, 256>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
        if (dvt == 128) return state_gate<64, 128>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
        return state_gate<64, 64>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
    }
    if (P.Dk == 128) {
        if (dvt == 256) return state_gate<128, 256>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
        if (dvt == 128) return state_gate<128, 128>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
        return state_gate<128, 64>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
    }
    if (dvt == 128) return state_gate<256, 128>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
    return state_gate<256, 64>(P, mode, a_src, b_src, g, ig, nseg, tiles_per_seg, seg_state, seg_gamma, status, st);
}

cudaError_t fwd(const Dims& P, const void* q, const void* k, const void* v, const float* g, const float* ig,
                const float* h0, void* o, float* hT, float* saved, void* ws, cudaStream_t st) {
    const int dvt = pick_dvt(P);
    if (P.Dk == 64) {
        if (dvt == 128) return run_gate<64, 128>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
        return run_gate<64, 64>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
    }
    if (P.Dk == 128) {
        if (dvt == 128) return run_gate<128, 128>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
        return run_gate<128, 64>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
    }
    return run_gate<256, 64>(P, q, k, v, g, ig, h0, o, hT, saved, ws, st);
}

}  // namespace tc
}  // namespace gla
