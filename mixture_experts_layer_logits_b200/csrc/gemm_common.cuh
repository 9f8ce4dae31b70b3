// gemm_common.cuh -- pieces shared by the two tcgen05 grouped-GEMM kernels
// (grouped_ffn.cu: one launch per GEMM; fused_ffn.cu: both GEMMs and the
// combine in one persistent launch for weight-streaming shapes): tile sizes,
// the shared-memory ring layout, barrier helpers, the SwiGLU epilogue math and
// the TMA tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"
#include "ptx.cuh"

namespace moe {
namespace gemm {

constexpr int kBM = 128;        // weight rows per tile (MMA M)
constexpr int kBK = 64;         // K elements per stage (one 128-byte swizzle row)
constexpr int kUmmaK = 16;      // K per tcgen05.mma (bf16)
constexpr int kThreads = 512;   // 16 warps, roles below
constexpr int kGatherWarps = 6;  // warps 2..7
constexpr int kEpiWarp0 = 8;     // warps 8..15: two epilogue groups of four
constexpr int kStageRows = 8;    // token rows per epilogue staging buffer
constexpr int kStageRowBytes = 512;  // one token row: 256 bf16 outputs
constexpr int kATileBytes = kBM * kBK * 2;

// Shared-memory ring of one CTA.  MODE 0: the B operand (token rows) is written by
// the gather warps; MODE 1: it is loaded by TMA with the weights.  RESERVE bytes
// after the aux area are left for the kernel's own tables.
template <int MODE, int NT, int RESERVE = 0>
struct Cfg {
    static constexpr int kNA = 2;                                  // A tiles per stage
    static constexpr int kBTileBytes = NT * kBK * 2;
    static constexpr int kStageBytes = kNA * kATileBytes + kBTileBytes;
    // shared memory: 1 KB alignment slack | ring | epilogue staging | Aux | token offsets
    static constexpr int kMaxSmem = 232448;  // 227 KB per CTA
    static constexpr int kAuxBytes = 1024 + kGatherWarps * NT * 4;
    static constexpr int kStagingBytes = 2 * 2 * kStageRows * kStageRowBytes;  // 2 groups x 2 bufs
    static constexpr int kStagesRaw =
        (kMaxSmem - 1024 - kAuxBytes - kStagingBytes - RESERVE) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kAccCols = 2 * NT;                        // per accumulator buffer
    static constexpr int kNBufRaw = 512 / kAccCols;                // accumulators in flight
    static constexpr int kNBuf = kNBufRaw > 8 ? 8 : kNBufRaw;
    static constexpr int kUsedCols = kAccCols * kNBuf;
    static constexpr int kTmemCols = kUsedCols <= 32 ? 32 : kUsedCols <= 64 ? 64
                                   : kUsedCols <= 128 ? 128 : kUsedCols <= 256 ? 256 : 512;
    static constexpr uint32_t kTxBytes = kNA * kATileBytes + (MODE == 1 ? kBTileBytes : 0);
    // shared memory: 1 KB alignment slack + ring + barriers/aux
    // Gather groups.  A waiter on a ring slot's mbarrier must never be more than one
    // phase ahead of it (a parity wait cannot tell phase n from n - 2); group g
    // handles stages g, g + G, ..., so G <= kStages guarantees it.  The W warps of
    // a group split the rows of its stages.
    static constexpr int kG = kGatherWarps < kStages ? kGatherWarps : kStages;
    static constexpr int kW = kGatherWarps / kG;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kStagingBytes + kAuxBytes;
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "MMA N tile");
    static_assert(kStages >= 2, "pipeline depth");
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
};

constexpr int kBarSlots = 20;  // ring barriers in Aux

struct Aux {
    uint64_t full[kBarSlots];
    uint64_t empty[kBarSlots];
    uint64_t tfull[8];
    uint64_t tempty[8];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// TMEM columns an epilogue group reads per tcgen05.ld: 16, or 8 when a group's
// half of the token columns is narrower (NT = 16), so no load reaches past the
// group's columns -- and past the allocation in the last accumulator buffer.
template <int NT>
constexpr int kEpiCols = NT / 2 >= 16 ? 16 : 8;

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N])
{
    static_assert(N == 8 || N == 16, "tcgen05.ld width");
    if constexpr (N == 16)
        tmem_ld16(taddr, r);
    else
        tmem_ld8(taddr, r);
}

// Split-K slices wanted for `units` (tile, feature block) pairs: enough
// (tile, feature block, slice) units for `waves` waves of CTAs, each slice at
// least min_kt K tiles long.
__device__ __forceinline__ int split_count(int units, int s_max, int num_kt, int min_kt,
                                           int waves = 16)
{
    if (units <= 0) return 1;
    int s = (waves * (int)gridDim.x + units - 1) / units;
    s = min(s, s_max);
    s = min(s, max(1, num_kt / min_kt));
    return max(s, 1);
}

// silu(g) * u = g * u / (1 + e^-g).  The result is rounded to bf16 (8-bit
// significand), so the fast exponential and the approximate reciprocal (one
// MUFU instruction each, a few ulp of fp32) are far inside that rounding; when
// e^-g overflows, the reciprocal of inf is 0.
__device__ __forceinline__ float silu_mul(float g, float u)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + __expf(-g)));
    return g * r * u;
}

__device__ __forceinline__ void named_bar_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// bar.red.or over `n` threads: true in every thread if any thread passed true.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}


// Tile list entries are read through L2 (they may be read before this grid's
// dependency wait; see the kernel).
__device__ __forceinline__ Tile load_tile(const Tile* p)
{
    const int4 lo = __ldcg(reinterpret_cast<const int4*>(p));
    const int4 hi = __ldcg(reinterpret_cast<const int4*>(p) + 1);
    Tile t;
    t.expert = lo.x;
    t.row_start = lo.y;
    t.rows = lo.z;
    t.first = lo.w;
    t.count = hi.x;
    t.pad[0] = hi.y;
    t.pad[1] = hi.z;
    t.pad[2] = hi.w;
    return t;
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2D bf16 row-major [rows, cols] tensor map with a [box_rows, 64] box, 128-byte swizzle.
inline cudaError_t make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows)
{
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2D byte tensor (E4M3 weight codes) [rows, cols] with a [box_rows, box_cols] box:
// box_cols 64 unswizzled, or 128 with the 128-byte swizzle (16-byte chunk c of box
// row r lands at chunk c ^ (r % 8) of its 128-byte shared-memory row).
inline cudaError_t make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows, uint32_t box_cols = kBK)
{
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (box_cols != 64 && box_cols != 128) return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box_cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace gemm
}  // namespace moe
