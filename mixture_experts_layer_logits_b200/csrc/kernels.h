// kernels.h -- host-side launch interface between the C ABI (moe_api.cu) and the
// kernels (route_permute.cu, grouped_ffn.cu, combine.cu).  Internal only.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Value a kernel stores in the workspace's error word when it gives up on a
// bounded wait.  A fresh workspace holds arbitrary bytes, so only this exact
// value counts as an error.
constexpr int32_t kDeviceErrorMagic = 0x4D4F4554;

// Value a kernel of the debug build (compiled with MOE_DEBUG) stores in the error
// word when an index read from its inputs -- an expert id, an expert offset, a
// permuted row -- is out of range; the access it would have made is skipped or
// redirected to index 0.
constexpr int32_t kDeviceBoundsMagic = 0x4D4F4542;

#ifdef MOE_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Debug build: true when lo <= v < hi; otherwise records kDeviceBoundsMagic in
// *err (when err is not null) and returns false.  Release build: always true,
// and the check compiles away.
__device__ __forceinline__ bool debug_in_range(long long v, long long lo, long long hi,
                                               int32_t* err)
{
    if constexpr (!kDebugChecks) return true;
    const bool ok = v >= lo && v < hi;
    if (!ok && err) atomicExch(err, kDeviceBoundsMagic);
    return ok;
}

// One tile of the grouped GEMMs: `rows` (1..NT) consecutive permuted rows of one
// expert, starting at permuted position `row_start`.  `first` is the index of the
// expert's first tile and `count` its number of tiles.
struct Tile {
    int expert;
    int row_start;
    int rows;
    int first;
    int count;
    int pad[3];
};

// The grid barrier of the multi-CTA permutation (32 bytes of device memory;
// needs no initialisation).  CTA 0 of a call zeroes `count`, then publishes the
// call's generation in `gen` (release); every CTA waits for that before its
// first arrival.  A CTA that gives up on a wait stores the call's generation in
// `abort`, so the others stop too.
struct GridBar {
    uint32_t count;
    uint32_t pad;
    unsigned long long gen;
    unsigned long long abort;
    unsigned long long pad2;
};

// Everything the route/permute kernels write besides the user-visible outputs.
struct PermuteAux {
    Tile* tiles;           // [max_tiles]
    int32_t* num_tiles;    // device scalar
    int nt;                // token rows per tile (the GEMM's N tile)
    int32_t* err;          // the error word (bounded-wait timeouts, debug-build index checks)
    int max_tiles;         // entries of `tiles`
    int32_t* chunk_counts; // [max_chunks + 1, E] scratch of the multi-CTA path
    int max_chunks;        // its chunk rows (the multi-CTA path's grid bound)
    GridBar* bar;          // the multi-CTA path's grid barrier
    unsigned long long gen;  // a value unique to this call (next_generation())
};

// A value unique to each call that synchronises CTAs through workspace words
// (the one-launch FFN, the multi-CTA permutation): a per-process random start
// plus a counter, so that neither an earlier call's value nor stale workspace
// bytes match it.
unsigned long long next_generation();

// Streaming multiprocessors of the current device (cached per device).
int device_sms();

// Records the cudaError_t that moe_last_cuda_error() reports on this host thread.
void set_last_cuda_error(int err);

// The shape rules of moe_route / moe_permute (1 <= E <= 1024, 1 <= k <= min(E, 16),
// T >= 1, T*k <= 2^30); H and I are not looked at.
bool routing_shape_ok(const moe_shape_t& s);

// Launch helper: programmatic dependent launch unless MOE_DISABLE_PDL=1.
bool pdl_enabled();

// Launches kern<<<grid, block, smem, st>>>(args...) with programmatic dependent
// launch allowed (unless MOE_DISABLE_PDL=1): the kernel may start while its
// predecessor on `st` is finishing, and waits for it with griddepcontrol.wait
// before reading that predecessor's results.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* weights,
                         cudaStream_t st);

// Single-CTA path (T*k <= kSmallRows): optional routing, then histogram, scan,
// stable scatter, tile list.  logits == nullptr: ids are an input.
constexpr int kSmallRows = 4096;
cudaError_t launch_small_route_permute(const float* logits, int T, int E, int k, int32_t* ids,
                                       float* weights, int32_t* offsets, int32_t* rows,
                                       const PermuteAux& aux, cudaStream_t st);

// Multi-CTA path, one launch of at most min(SMs, aux.max_chunks) CTAs that must
// all be resident at once: every CTA counts and ranks its chunk of rows, then
// (after a grid barrier) the per-expert prefixes over the chunks are formed, and
// (after a second) every CTA places its chunk stably; the CTAs also write the
// offsets and the tile list.  Waits are bounded (2 s, then kDeviceErrorMagic in
// aux.err).
cudaError_t launch_large_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                                 int32_t* rows, const PermuteAux& aux, cudaStream_t st);

// Tile list from expert_offsets alone (moe_grouped_ffn called on its own).
cudaError_t launch_build_tiles(const int32_t* offsets, int E, int R, const PermuteAux& aux,
                               cudaStream_t st);

struct FfnPlan {
    int nt;            // token rows per tile (16..256, multiple of 16)
    int max_tiles;     // upper bound of the tile count
    int s13_max;       // split-K bounds (the device picks the actual split)
    int s2_max;
    int grid;          // persistent CTAs
};
FfnPlan plan_ffn(int T, int E, int k, int H, int I, int num_sms);

struct FfnBuffers {
    const void* x;
    const void* w13;
    const void* w2;
    const int32_t* permuted_rows;
    const Tile* tiles;
    const int32_t* num_tiles;
    void* act;         // bf16 [R, I]
    void* y;           // bf16 [R, H]; written directly only when the w2 split is 1
    float* partials;   // fp32 split-K partials (w13's, then reused by w2)
    int32_t* splits;   // [2]: split counts the w13 and w2 kernels used
    int32_t* err;
};
// w13 (+ SwiGLU finalize when split) and w2 (+ y reduction when split and
// reduce_y): y is complete when the launches finish, unless reduce_y is false,
// in which case a split w2 leaves its partials for launch_combine_partials.
// between_gemms: if not null, recorded on `st` after the w13 stage.
cudaError_t launch_grouped_ffn(const FfnBuffers& b, int T, int E, int k, int H, int I,
                               const FfnPlan& plan, cudaStream_t st,
                               cudaEvent_t between_gemms = nullptr, bool reduce_y = true);

// Routing, the permutation, w13 + SwiGLU, w2 and the combine in one persistent
// launch (fused_ffn.cu), for weight-streaming shapes: at most 64 tokens, so every
// expert's rows fit one tile.  Every CTA routes the tokens itself; CTA 0 writes
// the routing outputs and zeroes the arrival counters of this call, then sets
// *ready = gen (a value unique to the call) for the others.
struct FusedBuffers {
    const void* x;
    const float* logits;
    const void* w13;   // bf16 weights, or E4M3 codes when s13 is set
    const void* w2;
    const float* s13;  // E4M3 weights: [E, 2I] and [E, H] fp32 row scales; else nullptr
    const float* s2;
    int32_t* topk_ids;        // routing outputs [R], [R], [E + 1], [R]
    float* topk_weights;
    int32_t* expert_offsets;
    int32_t* permuted_rows;
    void* act;         // bf16 [I / 64, R, 64] (K-blocked)
    float* part2;      // fp32 [s2_max, R, H]
    void* y;           // bf16 [R, H]
    void* out;         // bf16 [T, H]
    int32_t* counters; // [fused_ffn_counters()]
    unsigned long long* ready;
    void* xmax;        // [T] 16-byte words (largest |x| per token, E4M3 weights)
    unsigned long long gen;
    int32_t* splits;   // [2]
    int32_t* err;
};
bool fused_ffn_eligible(int T, int E, int k, int H, int I, const FfnPlan& plan);
int fused_ffn_counters(int T, int k, int H, const FfnPlan& plan);
cudaError_t launch_fused_ffn(const FusedBuffers& b, int T, int E, int k, int H, int I,
                             const FfnPlan& plan, cudaStream_t st);
// moe_forward uses the fused launch where eligible unless MOE_DISABLE_FUSED=1.
bool fused_enabled();

// Failure-detection self-test (selftest.cu): a kernel whose bounded waits give
// up after limit_us and record the timeout in the error word at ws[0].
cudaError_t launch_wait_timeout_selftest(void* ws, unsigned limit_us, cudaStream_t st);

// out[t] = sum_j w[t,j] * y[t*k+j] (k <= 16).
cudaError_t launch_combine(const void* y, const float* weights, int T, int k, int H, void* out,
                           cudaStream_t st);

// The combine reading w2's split-K partials (k <= 16, splits <= 8): y[r] =
// bf16(sum_s partial_s[r]) in slice order (y itself when *splits <= 1), then
// the combine.  Used when w2 may be split.
cudaError_t launch_combine_partials(const float* partials, const int32_t* splits, const void* y,
                                   const float* weights, int T, int k, int H, void* out,
                                   cudaStream_t st);

// act[p, f] = bf16(silu(sum_s gate_s) * sum_s up_s) when *splits > 1 (else no-op).
cudaError_t launch_swiglu_finalize(const float* partials, const int32_t* splits, int R, int I,
                                   void* act, cudaStream_t st);

// y[r, h] = bf16(sum_s partial_s[r, h]) when *splits > 1 (else no-op).
cudaError_t launch_reduce_y(const float* partials, const int32_t* splits, int R, int H, void* y,
                            cudaStream_t st);

}  // namespace moe
