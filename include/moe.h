/*
 * moe.h -- C ABI of the B200 (sm_100a) Mixture-of-Experts layer forward.
 *
 * The layer (token t, expert e, top_k = k, hidden H, intermediate I):
 *   route    : topk_ids[t, 0..k) = the k experts with the largest raw fp32 router
 *              logit, ties to the lower expert index (-0.0 == +0.0), listed in
 *              that order; topk_weights[t, j] = exp(l_j - l_0) / sum_i exp(l_i - l_0)
 *              over the selected logits ("softmax_sum" routing: FlashInfer PR #3751
 *              page "Optimizing TRTLLM-Gen MoE routing", section "performance
 *              numbers"; a softmax over all E followed by division by the sum of
 *              the selected k is the same thing).
 *   permute  : expanded row r = t*k + j.  expert_offsets[e+1] = expert_offsets[e] +
 *              #{r : topk_ids[r] == e}; permuted_rows[expert_offsets[e] + q] = the
 *              q-th smallest r routed to e (a stable sort by expert).
 *   ffn      : for permuted position p of expert e, token t = permuted_rows[p] / k
 *              (the `members[m] // input_route_divisor` map of the FlashInfer
 *              PR #7368 page "overlap grouped activation staging", section
 *              "1. Ampere", with the divisor equal to top_k):
 *                h = w13[e] . x[t] (2I values), gate = h[0:I], up = h[I:2I],
 *                act = silu(gate) * up  (silu(z) = z / (1 + exp(-z))),
 *                y[permuted_rows[p]] = w2[e] . act  (H values).
 *              The gate/up split of w13's rows is this library's reading: the
 *              page elides its `split_gate` logic (section "2. Hopper").
 *   combine  : out[t] = sum_{j=0..k-1} topk_weights[t, j] * y[t*k + j], in fp32,
 *              j ascending, rounded once to bf16 (a fixed-order merge; cf. the
 *              "FP32 partials" section of the FlashInfer PR #5586 page).
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer to caller-owned memory, row-major
 *     and contiguous.  The library never allocates, frees, synchronises (except
 *     moe_device_status) or keeps a pointer past the completion of the call's
 *     work on `stream`.
 *   - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream).  Kernels are chained with programmatic
 *     dependent launch; set MOE_DISABLE_PDL=1 in the environment to turn it off.
 *   - All arguments are validated on the host before anything is launched; on an
 *     error no work is queued and no output is touched:
 *       NULL pointer                                      -> MOE_ERR_INVALID_ARG
 *       T < 1, E < 1 or E > 1024, k < 1 or k > min(E, 16) -> MOE_ERR_UNSUPPORTED_SHAPE
 *       (ffn/combine/forward) H or I < 128 or not a multiple of 128
 *                                                         -> MOE_ERR_UNSUPPORTED_SHAPE
 *       T*k > 2^30 or a size overflow                      -> MOE_ERR_UNSUPPORTED_SHAPE
 *       a base pointer not 16-byte aligned                 -> MOE_ERR_MISALIGNED
 *       ws_bytes < moe_workspace_size(shape)               -> MOE_ERR_WORKSPACE_TOO_SMALL
 *     A failed launch returns MOE_ERR_CUDA; moe_last_cuda_error() then gives the
 *     cudaError_t (per host thread).
 *   - Inputs and outputs must not alias.  NaN logits are outside the contract.
 *   - Element types: "bf16" is IEEE bfloat16 passed as its 16-bit pattern.
 *   - The workspace is device memory of at least moe_workspace_size(shape) bytes,
 *     256-byte aligned, owned by the caller; calls that share one workspace must
 *     be ordered on one stream.  Its contents need no initialisation.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED_SHAPE = 2,
    MOE_ERR_MISALIGNED = 3,
    MOE_ERR_WORKSPACE_TOO_SMALL = 4,
    MOE_ERR_CUDA = 5,
    MOE_ERR_DEVICE_TIMEOUT = 6,
    MOE_ERR_DEVICE_BOUNDS = 7   /* debug build only: see moe_device_status */
} moe_status_t;

/* T tokens, E experts, top_k, H hidden, I intermediate (H, I unused by route/permute). */
typedef struct {
    int32_t T, E, top_k, H, I;
} moe_shape_t;

typedef uint16_t moe_bf16_t;  /* bf16 bit pattern */
typedef void* moe_stream_t;   /* cudaStream_t */

/* Bytes of device workspace that moe_forward / moe_permute / moe_grouped_ffn need
 * for `shape` (one size covers all three); 0 if the shape is unsupported.  Pure
 * host function: touches no device. */
size_t moe_workspace_size(moe_shape_t shape);

/* route.  logits fp32 [T, E] -> topk_ids int32 [T, k], topk_weights fp32 [T, k]
 * (both ordered by selection rank).  Needs no workspace, so it takes none: each
 * token's selection and softmax stay in registers and shared memory. */
moe_status_t moe_route(const float* logits, moe_shape_t shape, int32_t* topk_ids,
                       float* topk_weights, moe_stream_t stream);

/* permute.  topk_ids int32 [T*k] (values in [0, E)) -> expert_offsets int32 [E+1],
 * permuted_rows int32 [T*k].  Ids outside [0, E) are outside the contract.
 * Up to 4096 rows one CTA does the whole permutation.  Beyond that it is one
 * launch of at most one CTA per SM whose CTAs meet at two grid barriers (the
 * chunk counts must all be in before the prefixes over the chunks are formed,
 * and those before any row is placed); the workspace holds the count table and
 * the barrier.  Co-residency: as for the one-launch layer (moe_forward), the
 * launch assumes all of its CTAs run at once; every wait is bounded (2 s, then
 * moe_device_status reports MOE_ERR_DEVICE_TIMEOUT and the outputs are
 * unspecified), so it never hangs. */
moe_status_t moe_permute(const int32_t* topk_ids, moe_shape_t shape, int32_t* expert_offsets,
                         int32_t* permuted_rows, void* workspace, size_t ws_bytes,
                         moe_stream_t stream);

/* ffn.  x bf16 [T, H]; w13 bf16 [E, 2I, H]; w2 bf16 [E, H, I]; expert_offsets and
 * permuted_rows as produced by moe_permute -> y bf16 [T*k, H] in expanded-id
 * order (row r = t*k + j).  Activation rows are gathered straight from x (no
 * permuted copy of x is made); gate/up accumulate in fp32 in tensor memory, act
 * is rounded to bf16, the down projection accumulates in fp32 and y is rounded
 * to bf16. */
moe_status_t moe_grouped_ffn(const moe_bf16_t* x, const moe_bf16_t* w13, const moe_bf16_t* w2,
                             const int32_t* expert_offsets, const int32_t* permuted_rows,
                             moe_shape_t shape, moe_bf16_t* y, void* workspace, size_t ws_bytes,
                             moe_stream_t stream);

/* combine.  y bf16 [T*k, H] (expanded-id order), topk_weights fp32 [T, k]
 * -> out bf16 [T, H].  Needs no workspace; shape.E and shape.I are not used. */
moe_status_t moe_combine(const moe_bf16_t* y, const float* topk_weights, moe_shape_t shape,
                         moe_bf16_t* out, moe_stream_t stream);

/* The whole layer: route -> permute -> ffn -> combine, one stream, no host sync.
 * x bf16 [T, H], logits fp32 [T, E], w13 bf16 [E, 2I, H], w2 bf16 [E, H, I]
 * -> out bf16 [T, H].  topk_ids, topk_weights, expert_offsets and permuted_rows
 * are optional outputs: pass NULL to keep them inside the workspace.
 * For weight-streaming shapes (T <= 64, see moe_forward_fused) the whole layer
 * runs as ONE persistent launch: every CTA routes and permutes the tokens itself
 * (the same ids and, bit for bit, the same weights as moe_route), and the CTAs
 * hand act rows and finished y rows to each other through arrival counters in
 * the workspace.  It sums w13
 * over the whole K range in one fp32 chain, so its result equals the
 * multi-launch path's (MOE_DISABLE_FUSED=1 in the environment selects that
 * path) bit for bit where that path leaves w13 unsplit (H < 512), and up to
 * bf16 rounding of the differently ordered sum otherwise.  Either way every
 * wait is bounded (2 s; then moe_device_status reports MOE_ERR_DEVICE_TIMEOUT).
 * Co-residency: that one launch has at most one CTA per SM, and its CTAs wait for each
 * other's rows, so it assumes all of its CTAs run at once.  Kernels on other
 * streams that hold SMs while it starts delay some of its CTAs; the call stays
 * correct as long as they get an SM within the 2 s bound, and otherwise its
 * output is unspecified and moe_device_status reports MOE_ERR_DEVICE_TIMEOUT
 * (it never hangs).  Give it the device to itself for guaranteed progress. */
moe_status_t moe_forward(const moe_bf16_t* x, const float* logits, const moe_bf16_t* w13,
                         const moe_bf16_t* w2, moe_shape_t shape, moe_bf16_t* out,
                         int32_t* topk_ids, float* topk_weights, int32_t* expert_offsets,
                         int32_t* permuted_rows, void* workspace, size_t ws_bytes,
                         moe_stream_t stream);

/* moe_forward for measurement: identical work, and additionally records
 * events[i] (cudaEvent_t, created by the caller) on `stream` at the stage
 * boundaries: [0] before routing, [1] after route+permute, [2] after the
 * w13/SwiGLU kernel, [3] after the w2 kernel, [4] after the combine.  n_events
 * must be 5.  When the layer is one launch (moe_forward_fused), [1] is
 * recorded right after [0] and [2], [3] and [4] after the launch.  A recorded event is a
 * stream operation, so the launch overlap between the stages it separates is
 * lost while measuring. */
moe_status_t moe_forward_timed(const moe_bf16_t* x, const float* logits, const moe_bf16_t* w13,
                               const moe_bf16_t* w2, moe_shape_t shape, moe_bf16_t* out,
                               int32_t* topk_ids, float* topk_weights, int32_t* expert_offsets,
                               int32_t* permuted_rows, void* workspace, size_t ws_bytes,
                               moe_stream_t stream, void* const* events, int n_events);

/* moe_permute without a workspace argument, for callers that cannot allocate
 * device memory: code that must not grow its device footprint after start-up,
 * code whose device memory is all owned by another allocator, or callers that
 * are handed only the input and output buffers.  The FlashInfer pages have no
 * counterpart of this entry point; it computes exactly what moe_permute
 * computes (same kernels, same bit-exact result).
 *
 * Scratch: a file-scope device array of MOE_PERMUTE_NOALLOC_SCRATCH_BYTES
 * (about 1 MiB) inside the library; every GPU on which the library is used holds
 * it until the process exits.  The caller still passes topk_ids, expert_offsets
 * and permuted_rows (device pointers, 16-byte aligned).
 * Limits: T*k <= MOE_PERMUTE_NOALLOC_MAX_ROWS and the moe_permute shape rules,
 * else MOE_ERR_UNSUPPORTED_SHAPE before anything is launched.
 * The first call on each device looks up the array's device address for that
 * device (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.
 * Every call shares the one array, which holds the per-chunk expert counts and
 * also the per-expert tile list and its count: every call rewrites all of them,
 * so after a later call only the caller's own output buffers still hold this
 * call's results.  Calls whose GPU work can overlap (on other streams or host
 * threads, same device) race and may return wrong results; order them on one
 * stream. */
#define MOE_PERMUTE_NOALLOC_MAX_ROWS (1 << 20)
#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (1052672 + 32768 + 256)
moe_status_t moe_permute_noalloc(const int32_t* topk_ids, moe_shape_t shape,
                                 int32_t* expert_offsets, int32_t* permuted_rows,
                                 moe_stream_t stream);

/* The layer with FP8 expert weights (the E4M3 format of "FP8 Formats for Deep
 * Learning": sign, 4 exponent bits with bias 7, 3 significand bits, no
 * infinities).  w13 uint8 [E, 2I, H] and w2 uint8 [E, H, I] hold E4M3 codes,
 * w13_scale fp32 [E, 2I] and w2_scale fp32 [E, H] one scale per weight row:
 * weight (e, r, c) = e4m3(code) * scale(e, r).  Everything else -- arguments,
 * outputs, workspace (moe_workspace_size), routing, roundings, error reporting
 * -- is moe_forward's.  The weights stream at one byte each and the tensor
 * cores multiply the codes as they are (E4M3 MMAs).  The other operand, each
 * token row (x for w13, the bf16 act for w2), is made E4M3 without loss: it is
 * scaled by a power of two chosen from its largest magnitude and written as two
 * E4M3 terms that sum to it exactly (entries smaller than 2^-9 of the row's
 * largest to within 2^-17 of it).  E4M3 products are exact in fp32, so the
 * accumulators hold the bf16 products; the power of two is undone and each
 * weight row's scale multiplies its fp32 accumulator row.  Runs only as the
 * one-launch layer (moe_forward_w8_supported; 1 kernel):
 * MOE_ERR_UNSUPPORTED_SHAPE otherwise, whatever MOE_DISABLE_FUSED says.  Codes
 * 0x7F / 0xFF (NaN) propagate as NaN; a token whose x row holds an inf or a NaN
 * gets NaN outputs.  All pointers 16-byte aligned. */
moe_status_t moe_forward_w8(const moe_bf16_t* x, const float* logits, const uint8_t* w13,
                            const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                            moe_shape_t shape, moe_bf16_t* out, int32_t* topk_ids,
                            float* topk_weights, int32_t* expert_offsets, int32_t* permuted_rows,
                            void* workspace, size_t ws_bytes, moe_stream_t stream);

/* moe_forward_w8 recording the 5 stage events of moe_forward_timed ([0] and [1]
 * before its one launch, [2] .. [4] after it). */
moe_status_t moe_forward_w8_timed(const moe_bf16_t* x, const float* logits, const uint8_t* w13,
                                  const float* w13_scale, const uint8_t* w2,
                                  const float* w2_scale, moe_shape_t shape, moe_bf16_t* out,
                                  int32_t* topk_ids, float* topk_weights,
                                  int32_t* expert_offsets, int32_t* permuted_rows,
                                  void* workspace, size_t ws_bytes, moe_stream_t stream,
                                  void* const* events, int n_events);

/* 1 if moe_forward_w8 accepts `shape` (the one-launch layer's shapes), else 0. */
int moe_forward_w8_supported(moe_shape_t shape);

/* Number of kernels one moe_forward call launches for `shape` (0 if unsupported). */
int moe_forward_kernel_count(moe_shape_t shape);

/* Failure detection without a GPU fault.  Launches one small kernel whose two
 * bounded waits cannot be satisfied -- an mbarrier that nothing arrives on and
 * a workspace flag that nothing sets (workspace bytes [4, 8), zeroed first) --
 * built from the same wait primitives as the layer's kernels.  Each gives up
 * after limit_us microseconds and records the timeout in the workspace's error
 * word exactly as a layer kernel does, so the next moe_device_status(workspace)
 * returns MOE_ERR_DEVICE_TIMEOUT (and clears it); the CUDA context stays usable.
 * workspace: device memory of at least 8 bytes, 16-byte aligned.
 * limit_us: 1 .. 2,000,000, else MOE_ERR_INVALID_ARG. */
moe_status_t moe_selftest_wait_timeout(void* workspace, size_t ws_bytes, unsigned limit_us,
                                       moe_stream_t stream);

/* 1 if moe_forward runs the whole layer of `shape` as one persistent launch
 * (T <= 64, unless MOE_DISABLE_FUSED=1), else 0. */
int moe_forward_fused(moe_shape_t shape);

/* Waits for `stream`, then reads and clears the device error word kept in the
 * workspace.  MOE_ERR_DEVICE_TIMEOUT means a kernel gave up on a bounded
 * intra-kernel wait (its outputs for that call are then unspecified).
 * MOE_ERR_DEVICE_BOUNDS comes only from the debug build of the library
 * (libmoe_debug.so, compiled with MOE_DEBUG): one of its kernels read an index
 * out of range from its inputs -- an expert id outside [0, E) given to
 * moe_permute, expert offsets outside [0, T*k] or a permuted row outside
 * [0, T*k) given to moe_grouped_ffn -- and skipped (or redirected to index 0)
 * the access it would have made; that call's outputs are unspecified.  The
 * release build does not check these out-of-contract inputs. */
moe_status_t moe_device_status(void* workspace, size_t ws_bytes, moe_stream_t stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status_t status);

/* The cudaError_t behind the last MOE_ERR_CUDA returned on this host thread. */
int moe_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
