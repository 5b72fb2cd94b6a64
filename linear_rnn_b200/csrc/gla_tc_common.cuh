// Helpers shared by the tensor-core forward and backward kernels.
#pragma once
#include <cudaTypedefs.h>

#include <utility>

#include "gla_common.cuh"
#include "sm100.cuh"

namespace gla {
namespace tc {

// Launch with optional programmatic stream serialization (the kernel may start before the
// previous kernel in the stream ends, and waits in grid_dep_wait for what it reads from it) and
// an optional cluster of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                             int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    unsigned n = 0;
    if (pdl) {
        at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 1) {
        at[n].id = cudaLaunchAttributeClusterDimension;
        at[n].val.clusterDim.x = cluster_x;
        at[n].val.clusterDim.y = 1;
        at[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = at;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr int TR = 64;          // tokens per tile
constexpr uint32_t BLK = 8192;  // one 64-column bf16 block of a 64-row tile (64 x 128 B)

// Float index of element (r, d) of a 64-row fp32 tile loaded by TMA in 32-column boxes with
// the 128-byte swizzle: boxes of 64 rows x 128 B, 16-byte chunks XOR-ed with the row. Eight
// consecutive rows reading the same column range then hit eight different bank groups, and a
// row read column-wise stays conflict-free.
__device__ __forceinline__ int gsw(int r, int d) {
    return ((d >> 5) << 11) + (r << 5) + ((((d >> 2) & 7) ^ (r & 7)) << 2) + (d & 3);
}

// 1/x on the special-function unit (PTX rcp.approx.ftz: at most 1 ulp of error over the whole
// input range per the PTX ISA, subnormal results flushed to zero). Its results e^-b go into bf16
// operands (relative rounding 2^-9) or fp32 epilogue factors.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pairs of fp32 in one 64-bit register, multiplied lane-wise by the sm_100 packed
// fp32 instruction (IEEE round-to-nearest per lane, like two separate multiplies).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// bf16 pair (element 0 in the low half) -> fp32 pair
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
    return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// fp32 pair -> bf16 pair, round to nearest even
__device__ __forceinline__ uint32_t f2_to_bf2(uint64_t x) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Coalesced staging of a row-major fp32 block (NR rows x CW columns, row stride ld floats) in
// shared memory, for consumers that each want one whole row (a state row goes to one TMEM lane).
// Loading rows thread by thread straight from global memory touches 32 rows per warp access and
// thrashes L1; here a warp reads whole rows with 16-byte loads, several rows in flight, and
// 16-byte chunk j of row r lands at chunk j ^ (r & 7) of that row, so that eight consecutive rows
// read at one column hit eight different bank groups (staged_row16).  With b given (same shape
// and stride as a), dot[r] = sum_c a[r][c] b[r][c] for every row.  All NT threads take part.
template <int NR, int CW, int NT>
__device__ __forceinline__ void stage_rows(float* stg, const float* __restrict__ a, const float* __restrict__ b,
                                           long ld, float* dot, int tid) {
    constexpr int CPR = CW / 4;                // 16-byte chunks per row
    constexpr int LPR = CPR < 32 ? CPR : 32;   // lanes sharing a row
    constexpr int RPI = 32 / LPR;              // rows per warp access
    constexpr int CPL = CPR / LPR;             // chunks per lane and row
    constexpr int W = NT / 32;
    constexpr int U = 4;                       // row groups in flight per warp
    static_assert(CPR >= 8 && CPR % LPR == 0 && NR % RPI == 0 && NT % 32 == 0, "staged block shape");
    const int warp = tid >> 5, lane = tid & 31;
    const int rsub = lane / LPR, csub = lane % LPR;
    for (int r0 = warp * RPI; r0 < NR; r0 += U * W * RPI) {
        float4 xa[U][CPL], xb[U][CPL];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = r0 + u * W * RPI + rsub;
            if (r < NR) {
                const float4* pa = reinterpret_cast<const float4*>(a + r * ld) + csub;
                const float4* pb = b ? reinterpret_cast<const float4*>(b + r * ld) + csub : nullptr;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    xa[u][j] = __ldg(pa + j * LPR);
                    if (b) xb[u][j] = __ldg(pb + j * LPR);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = r0 + u * W * RPI + rsub;  // r < NR is uniform over the lanes of a row
            if (r < NR) {
                float part = 0.f;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    const int ch = (csub + j * LPR) ^ (r & 7);
                    *reinterpret_cast<float4*>(stg + r * CW + 4 * ch) = xa[u][j];
                    if (b)
                        part += xa[u][j].x * xb[u][j].x + xa[u][j].y * xb[u][j].y + xa[u][j].z * xb[u][j].z +
                                xa[u][j].w * xb[u][j].w;
                }
                if (b) {
#pragma unroll
                    for (int off = LPR / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                    if (csub == 0) dot[r] = part;
                }
            }
        }
    }
}

// The reverse of stage_rows: rows written into shared memory one per thread (staged_put16)
// go out to global memory with coalesced 16-byte stores, whole rows per warp.
template <int NR, int CW, int NT>
__device__ __forceinline__ void unstage_rows(const float* stg, float* __restrict__ dst, long ld, int tid) {
    constexpr int CPR = CW / 4;
    constexpr int LPR = CPR < 32 ? CPR : 32;
    constexpr int RPI = 32 / LPR;
    constexpr int CPL = CPR / LPR;
    constexpr int W = NT / 32;
    static_assert(CPR >= 8 && CPR % LPR == 0 && NR % RPI == 0 && NT % 32 == 0, "staged block shape");
    const int warp = tid >> 5, lane = tid & 31;
    const int rsub = lane / LPR, csub = lane % LPR;
    for (int r = warp * RPI + rsub; r < NR; r += W * RPI) {
        float4* pd = reinterpret_cast<float4*>(dst + r * ld) + csub;
#pragma unroll
        for (int j = 0; j < CPL; ++j)
            pd[j * LPR] = *reinterpret_cast<const float4*>(stg + r * CW + 4 * ((csub + j * LPR) ^ (r & 7)));
    }
}

// Columns [c, c + 16) of row r into a block laid out as stage_rows does (c a multiple of 16).
template <int CW>
__device__ __forceinline__ void staged_put16(float* stg, int r, int c, const float* f) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(stg + r * CW + 4 * (((c >> 2) + u) ^ (r & 7))) =
            make_float4(f[4 * u], f[4 * u + 1], f[4 * u + 2], f[4 * u + 3]);
}

// Columns [c, c + 16) of row r of a block staged by stage_rows (c a multiple of 16).
template <int CW>
__device__ __forceinline__ void staged_row16(const float* stg, int r, int c, float* f) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const float4 x = *reinterpret_cast<const float4*>(stg + r * CW + 4 * (((c >> 2) + u) ^ (r & 7)));
        f[4 * u] = x.x;
        f[4 * u + 1] = x.y;
        f[4 * u + 2] = x.z;
        f[4 * u + 3] = x.w;
    }
}

__device__ __forceinline__ void store8_bf16(uint8_t* base, uint32_t off, const float* v) {
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
        w[u] = *reinterpret_cast<uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(base + off) = make_uint4(w[0], w[1], w[2], w[3]);
}


inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3D map over [BH][L][D] (D innermost) with a box of {box0, 64, 1}.
inline bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int D, int L, int BH,
                     int box0, bool swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * esize, (cuuint64_t)D * esize * L};
    cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)TR, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


}  // namespace tc
}  // namespace gla
