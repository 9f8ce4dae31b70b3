// grouped_ffn.cu -- the gathered grouped expert FFN on tcgen05 tensor cores.
//
// Two launches of one persistent, warp-specialised kernel template:
//   w13 (MODE 0): act[p, f] = silu(gate) * up with gate/up = w13[e] rows f and
//                 I + f dotted with x[permuted_rows[p] / k]; act is bf16 [R, I]
//                 in permuted order.
//   w2  (MODE 1): y[permuted_rows[p], h] = w2[e] row h dotted with act[p];
//                 y is bf16 [R, H] in expanded-id order.
//
// Orientation ("swap AB", as on the FlashInfer PR #7368 page, section
// "2. Hopper": weights are the TMA-fed operand, the few routed activation rows
// the other one): the MMA's M = 128 rows are weight rows (output features), its
// N = the routed token rows of one expert (16..256, rounded up to 16 per tile, so
// a ragged tail costs at most 15 padded columns).  Accumulators live in tensor
// memory (fp32); MODE 0 keeps a gate and an up accumulator of equal shape so the
// epilogue thread that owns feature f holds both halves of its SwiGLU pair.
//
// Warp roles:
//   warp 0      TMA producer: weight tiles [128 x 64] (and, MODE 1, the act tile
//               [NT x 64]) with the 128-byte swizzle into a STAGES-deep ring.
//   warp 1      TMEM allocator and the single MMA-issuing thread.
//   MODE 0: warps 2-5 activation gather.  Every gather thread copies part of
//               every stage: 16-byte cp.async copies of the x rows selected by
//               permuted_rows[p] / k straight into the swizzled B tile (no
//               permuted copy of x exists).  Each thread's copies arrive on the
//               stage's mbarrier when they land (cp.async.mbarrier.arrive), so no
//               gather thread waits for its own copies; the MMA thread issues the
//               async-proxy fence after that barrier and before its MMAs read the
//               tile -- the proxy fence plus barrier that the FlashInfer PR #7368
//               page ("2. Hopper") requires before an async proxy reads
//               generic-proxy writes.  The weight TMA of a stage is issued
//               independently of its gather, so the two overlap (the BF16 ordering
//               of the same section).
//   epilogue    MODE 0: warps 6-13, two groups of four; MODE 1: warps 2-17, four
//               groups of four (two when NT < 64).  Warp w reads TMEM lanes
//               32*(w%4) ..; group g owns a contiguous range of token columns.  It
//               drains its columns into registers as packed bf16 (MODE 0: SwiGLU
//               applied), hands them back to the MMA thread at once, and only then
//               stages and stores the rows, so the stores overlap the next unit's
//               main loop.  MODE 1 hands back its two 128-row output blocks one at
//               a time, and the MMA thread starts the next unit on the first block
//               while the second is still being drained.  Split-K units write fp32
//               partials instead.
//
// Split-K: when there are too few (tile, feature block) units to fill the GPU
// (decode), each unit's K range is cut into S slices (S chosen on the device
// from the tile count and written to the workspace).  Every slice stores its
// fp32 partial with plain stores and moves on -- no fence, atomic or wait on the
// critical path.  The slices are added in slice order later, by the SwiGLU
// finalize kernel (w13) and by the combine (w2), so results are bit-reproducible.
//
// Every mbarrier wait is bounded (mbar_wait); on a timeout the kernel records
// an error word, stops issuing work, drains what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "gemm_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

using namespace gemm;

struct FfnArgs {
    const __nv_bfloat16* x;
    const int32_t* permuted_rows;
    const Tile* tiles;
    const int32_t* num_tiles;
    __nv_bfloat16* out;       // MODE 0: act [R, I]; MODE 1: y [R, H]
    float* partials;          // MODE 0: [S, R, 2I] by permuted row; MODE 1: [S, R, H] by expanded id
    int32_t* split_out;       // CTA 0 records the split count S here
    int32_t* err;
    int k, H, I, R;
    int num_kt;               // K / 64
    int fb_count;             // MODE 0: gate/up block pairs (I / 128); MODE 1: 256-row blocks
    int s_max;                // split-K upper bound
    int max_tiles;
    int min_kt_per_split;
    int weights_evict_first;  // weights are streamed once (few tokens per expert)
};

// Thread roles of the grouped GEMM:
//   warp 0              TMA producer
//   warp 1              TMEM allocator and MMA issuer
//   MODE 0 (14 warps):  warps 2-5 activation gather; warps 6-13 epilogue (2 groups of 4)
//   MODE 1 (18 warps):  warps 2-17 epilogue (4 groups of 4; 2 groups, warps 2-9, when
//                       NT < 64)
constexpr int kGGatherWarps = 4;
constexpr int kGGatherThreads = kGGatherWarps * 32;

template <int MODE, int NT>
struct GCfg {
    // MODE 0: 2 + 4 gather + 8 epilogue warps; MODE 1: 2 + 16 epilogue warps
    static constexpr int kThreads = MODE == 0 ? 448 : 576;
    static constexpr int kNA = 2;                                  // A tiles per stage
    static constexpr int kBTileBytes = NT * kBK * 2;
    static constexpr int kStageBytes = kNA * kATileBytes + kBTileBytes;
    static constexpr int kMaxSmem = 232448;                        // 227 KB per CTA
    // epilogue groups: 4 warps each (one per TMEM lane quarter), each group owning
    // kGroupCols consecutive token columns of the accumulator
    static constexpr int kGroups = (MODE == 1 && NT >= 64) ? 4 : 2;
    static constexpr int kEpiWarp0 = MODE == 0 ? 2 + kGGatherWarps : 2;
    static constexpr int kEpiWarps = 4 * kGroups;
    static constexpr int kGroupCols = NT / kGroups;
    static constexpr int kRows = 8;                                // token rows per staging chunk
    static constexpr int kRowBytes = 256;                          // one staged row segment
    static constexpr int kStagingBytes = kGroups * 2 * kRows * kRowBytes;
    // rows of the B tile one gather thread copies per stage (8 16-byte chunks a row)
    static constexpr int kGIters = (NT * 8 + kGGatherThreads - 1) / kGGatherThreads;
    static constexpr int kAuxBytes = 1024;
    static constexpr int kStagesRaw = (kMaxSmem - 1024 - kAuxBytes - kStagingBytes) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kAccCols = 2 * NT;                        // per accumulator buffer
    static constexpr int kNBufRaw = 512 / kAccCols;
    static constexpr int kNBuf = kNBufRaw > 8 ? 8 : kNBufRaw;
    static constexpr int kUsedCols = kAccCols * kNBuf;
    static constexpr int kTmemCols = kUsedCols <= 32 ? 32 : kUsedCols <= 64 ? 64
                                   : kUsedCols <= 128 ? 128 : kUsedCols <= 256 ? 256 : 512;
    static constexpr uint32_t kTxBytes = kNA * kATileBytes + (MODE == 1 ? kBTileBytes : 0);
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kStagingBytes + kAuxBytes;
    // token columns per tcgen05.ld in the split-K epilogue (within the group's columns)
    static constexpr int kLdCols = kGroupCols >= 16 ? 16 : 8;
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "MMA N tile");
    static_assert(kGroupCols % 8 == 0 && kGroupCols % kRows == 0, "epilogue column split");
    static_assert(kStages >= 2, "pipeline depth");
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kSmemBytes <= kMaxSmem, "shared memory");
    static_assert(kEpiWarp0 + kEpiWarps <= kThreads / 32, "warp roles");
};

// Barriers of one CTA.  tempty[b] frees accumulator buffer b (MODE 1: its first
// 128-row block's columns only) and tempty2[b] (MODE 1) its second block's, so
// the next unit's MMAs into the first block can start while the epilogue still
// drains the second.
struct GAux {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t tfull[8];
    uint64_t tempty[8];
    uint64_t tempty2[8];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void flag_error(const FfnArgs& a, GAux* aux)
{
    atomicExch(a.err, kDeviceErrorMagic);
    aux->abort = 1;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <int MODE, int NT>
__global__ void __launch_bounds__(GCfg<MODE, NT>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_act, const FfnArgs a)
{
    using C = GCfg<MODE, NT>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* ring = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* staging = ring + C::kStages * C::kStageBytes;
    GAux* aux = reinterpret_cast<GAux*>(staging + C::kStagingBytes);
    static_assert(sizeof(GAux) <= C::kAuxBytes, "aux area");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // MODE 0: the producer's expect_tx plus one arrival per gather warp
            mbar_init(&aux->full[s], MODE == 0 ? 1 + kGGatherWarps : 1);
            mbar_init(&aux->empty[s], 1);
        }
        for (int b = 0; b < C::kNBuf; ++b) {
            mbar_init(&aux->tfull[b], 1);
            mbar_init(&aux->tempty[b], C::kEpiWarps);
            mbar_init(&aux->tempty2[b], C::kEpiWarps);
        }
        mbar_init(&aux->drain, 1);
        aux->abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_w);
        if (MODE == 1) tma_prefetch_desc(&tm_act);
    }
    if (warp == 1) {
        tmem_alloc(&aux->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;

    // Programmatic dependent launch.  w13 reads the tile list that the kernel
    // right before it wrote, so all of it waits here.  w2 only needs its
    // predecessor (the SwiGLU finalize, or w13) for the act rows it loads and for
    // the partials region its epilogue overwrites: its producer waits right before
    // the first act load and its epilogue before its first store, so the weight
    // loads of its first stages overlap the end of the w13 stage.  The tile list
    // it reads before waiting was written two or more launches earlier: w2 is
    // only launched once every w13 CTA has passed its own wait, i.e. after the
    // permutation and everything before it completed.  It is read with L2 loads.
    if (MODE == 0) pdl_wait();
    pdl_launch_dependents();

    const int ntiles = __ldcg(a.num_tiles);
    const int s_want = split_count(ntiles * a.fb_count, a.s_max, a.num_kt, a.min_kt_per_split);
    const int kt_per_split = (a.num_kt + s_want - 1) / s_want;
    const int S = (a.num_kt + kt_per_split - 1) / kt_per_split;  // every slice non-empty
    const int units = ntiles * a.fb_count * S;
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.split_out = S;
    volatile int* abort_flag = &aux->abort;

    // unit u -> (slice, tile, feature block), expert-grouped: the units of expert e
    // occupy [fb_count * first_e, fb_count * (first_e + count_e)), feature block
    // major and tile minor, so the tiles that share a weight block are adjacent
    // (they run at the same time on neighbouring CTAs and share it in L2), and the
    // feature blocks of a tile run close together (its x rows stay in L2).  Since
    // fb_count * first_e <= rest < fb_count * first_{e+1}, tile rest / fb_count
    // belongs to expert e and carries first_e and count_e.  Slice fastest.
    auto decode = [&](int u, int& split, int& tile, int& fb) {
        split = u % S;
        const int rest = u / S;
        const Tile probe = load_tile(a.tiles + rest / a.fb_count);
        const int local = rest - a.fb_count * probe.first;
        fb = local / probe.count;
        tile = probe.first + local % probe.count;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // decode streams each weight block once; larger batches share a block
            // between the tiles of one expert, so leave those at normal priority
            const uint64_t pol = a.weights_evict_first ? l2_policy_evict_first()
                                                       : l2_policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0;
            int fills = 0;  // ring stage fills so far (fill q went to stage q % stages)
            bool ok = true;
            bool dep_ready = MODE == 0;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int split, tile, fb;
                decode(u, split, tile, fb);
                const Tile t = load_tile(a.tiles + tile);
                const int kt0 = split * kt_per_split, kt1 = min(a.num_kt, kt0 + kt_per_split);
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!mbar_wait(&aux->empty[stage], phase ^ 1u, abort_flag)) {
                        flag_error(a, aux);
                        ok = false;
                        break;
                    }
                    uint8_t* st = ring + stage * C::kStageBytes;
                    mbar_arrive_expect_tx(&aux->full[stage], C::kTxBytes);
                    if (MODE == 0) {
                        const int row = t.expert * 2 * a.I + fb * kBM;
                        tma_load_2d(st, &tm_w, &aux->full[stage], kt * kBK, row, pol);
                        tma_load_2d(st + kATileBytes, &tm_w, &aux->full[stage], kt * kBK, row + a.I,
                                    pol);
                    } else {
                        // two consecutive 128-row blocks of w2[e]; when H is an odd number
                        // of 128-row blocks the second block of the last pair belongs to
                        // the next expert (or lies past the tensor and is zero-filled)
                        // and its accumulator is never stored
                        const int row = t.expert * a.H + fb * 2 * kBM;
                        tma_load_2d(st, &tm_w, &aux->full[stage], kt * kBK, row, pol);
                        tma_load_2d(st + kATileBytes, &tm_w, &aux->full[stage], kt * kBK,
                                    row + kBM, pol);
                        if (!dep_ready) {  // act comes from the previous kernel
                            pdl_wait();
                            dep_ready = true;
                        }
                        tma_load_2d_nohint(st + 2 * kATileBytes, &tm_act, &aux->full[stage],
                                           kt * kBK, t.row_start);
                    }
                    ++fills;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!dep_ready) pdl_wait();  // (no unit here) the grid still depends on it
            if (!ok || *abort_flag) {
                // let every TMA load already issued land before the CTA can exit
                for (int s = 0; s < C::kStages; ++s) {
                    // fills of stage s
                    const int n_s = fills > s ? (fills - s + C::kStages - 1) / C::kStages : 0;
                    if (n_s > 0) {
                        volatile int never = 0;
                        mbar_wait(&aux->full[s], (uint32_t)((n_s - 1) & 1), &never,
                                  500000000ull);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per K tile: two MMAs (gate and up blocks, or two 128-row w2 blocks) into
        // accumulators d0 and d0 + NT.  MODE 1 starts a unit with the first
        // block's MMAs of up to kStages K tiles, which need only tempty[b], and
        // waits for tempty2[b] (the epilogue still draining the previous unit's
        // second block) before the second block's.
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int lu = 0;
            bool ok = true;
            auto wait_full = [&](int st_, uint32_t ph_) {
                if (!mbar_wait(&aux->full[st_], ph_, abort_flag)) {
                    flag_error(a, aux);
                    return false;
                }
                // MODE 0: the B tile was written by cp.async (generic proxy); the
                // tensor core reads it through the async proxy
                if (MODE == 0) fence_proxy_async_smem();
                tc_fence_after();
                return true;
            };
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++lu) {
                int split, tile, fb;
                decode(u, split, tile, fb);
                const Tile t = load_tile(a.tiles + tile);
                const int kt0 = split * kt_per_split, kt1 = min(a.num_kt, kt0 + kt_per_split);
                const int b = lu % C::kNBuf;
                const uint32_t aphase = (uint32_t)((lu / C::kNBuf) & 1);
                if (!mbar_wait(&aux->tempty[b], aphase ^ 1u, abort_flag)) {
                    flag_error(a, aux);
                    break;
                }
                tc_fence_after();
                const int n = (t.rows + 15) & ~15;
                const uint32_t idesc = umma_idesc_bf16(kBM, n);
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::kAccCols);
                auto issue = [&](uint32_t d, int st_, int blk, bool first_kt) {
                    const uint32_t sa = smem_u32(ring + st_ * C::kStageBytes);
                    const uint32_t bt = sa + C::kNA * kATileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
                        umma_bf16(d, umma_desc_sw128(sa + blk * kATileBytes + kk * 32),
                                  umma_desc_sw128(bt + kk * 32), idesc,
                                  (!first_kt || kk > 0) ? 1u : 0u);
                };
                int kt = kt0;
                if (MODE == 1) {
                    // first block over the first n_pre K tiles, then the second block
                    const int n_pre = min(C::kStages, kt1 - kt0);
                    for (int i = 0; i < n_pre && ok; ++i) {
                        const int st_ = (stage + i) % C::kStages;
                        const uint32_t ph_ = phase ^ (uint32_t)((stage + i) / C::kStages);
                        ok = wait_full(st_, ph_);
                        if (ok) issue(d0, st_, 0, i == 0);
                    }
                    if (ok && !mbar_wait(&aux->tempty2[b], aphase ^ 1u, abort_flag)) {
                        flag_error(a, aux);
                        ok = false;
                    }
                    if (!ok) break;
                    tc_fence_after();
                    for (int i = 0; i < n_pre; ++i) {
                        issue(d0 + NT, stage, 1, i == 0);
                        umma_commit(&aux->empty[stage]);  // frees the smem stage when read
                        if (++stage == C::kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    kt += n_pre;
                }
                for (; kt < kt1; ++kt) {
                    if (!wait_full(stage, phase)) {
                        ok = false;
                        break;
                    }
                    issue(d0, stage, 0, kt == kt0);
                    issue(d0 + NT, stage, 1, kt == kt0);
                    umma_commit(&aux->empty[stage]);  // frees the smem stage when read
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit(&aux->tfull[b]);
            }
            // all MMAs issued by this thread are complete before TMEM is freed
            umma_commit(&aux->drain);
            volatile int never = 0;
            if (!mbar_wait(&aux->drain, 0, &never, 500000000ull)) atomicExch(a.err, kDeviceErrorMagic);
        }
    } else if (MODE == 0 && warp < 2 + kGGatherWarps) {
        // ------------------------------------------------------------ gather (MODE 0)
        // Every gather warp fills part of every stage: gather thread g copies the
        // 16-byte chunks g, g + 128, ... of the tile's B rows (row = chunk / 8), so a
        // warp instruction covers 4 whole 128-byte row segments.  Each thread's
        // copies arrive on the stage's full barrier when they land
        // (cp.async.mbarrier.arrive), then the warp arrives once: no thread waits
        // for its own copies, and the barrier completes only when every copy and
        // the weight TMA have landed.  The MMA thread fences the async proxy
        // before reading the tile.
        const int g = threadIdx.x - 64;  // 0 .. kGGatherThreads - 1
        const uint64_t x_policy = l2_policy_evict_last();  // x rows are re-read per block
        int off[C::kGIters];  // element offset of this thread's x row per iteration (-1: none)
        int q = 0;            // global stage sequence number (same as the producer's)
        int cur_tile = -1;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int split, tile, fb;
            decode(u, split, tile, fb);
            const int kt0 = split * kt_per_split, kt1 = min(a.num_kt, kt0 + kt_per_split);
            if (tile != cur_tile) {
                const Tile t = load_tile(a.tiles + tile);
#pragma unroll
                for (int i = 0; i < C::kGIters; ++i) {
                    const int j = (g + i * kGGatherThreads) >> 3;
                    int r = j < t.rows ? a.permuted_rows[t.row_start + j] : -1;
                    if (r >= 0 && !debug_in_range(r, 0, a.R, a.err)) r = 0;  // debug build
                    off[i] = r >= 0 ? (r / a.k) * a.H + (g & 7) * 8 : -1;
                }
                cur_tile = tile;
            }
            for (int kt = kt0; kt < kt1; ++kt, ++q) {
                const int stage = q % C::kStages;
                const uint32_t phase = (uint32_t)((q / C::kStages) & 1);
                // warp-uniform decision, so no lane is left behind at __syncwarp
                if (!__all_sync(0xffffffffu, mbar_wait(&aux->empty[stage], phase ^ 1u,
                                                       abort_flag))) {
                    if (lane == 0) flag_error(a, aux);
                    ok = false;
                    break;
                }
                const uint32_t bt = smem_u32(ring + stage * C::kStageBytes + C::kNA * kATileBytes);
                const __nv_bfloat16* src0 = a.x + kt * kBK;
#pragma unroll
                for (int i = 0; i < C::kGIters; ++i) {
                    const int c8 = g + i * kGGatherThreads;
                    const int j = c8 >> 3, c = c8 & 7;
                    if (off[i] >= 0)
                        cp_async_16_hint(bt + j * 128 + ((c ^ (j & 7)) << 4), src0 + off[i],
                                         x_policy);
                }
                cp_async_mbar_arrive(&aux->full[stage]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&aux->full[stage]);
            }
        }
        cp_async_commit();
        cp_async_wait<0>();  // no copy is still in flight when the CTA exits
    } else if (warp >= C::kEpiWarp0 && warp < C::kEpiWarp0 + C::kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        if (MODE == 1) pdl_wait();  // the outputs and partials the predecessor reads
        const int grp = (warp - C::kEpiWarp0) >> 2;  // token-column group
        const int q = warp & 3;                      // TMEM lane quarter
        const int f_local = q * 32 + lane;           // feature inside the 128-row block
        const int gt = (warp - C::kEpiWarp0 - grp * 4) * 32 + lane;  // 0..127 in the group
        const int pcols = (MODE == 0) ? 2 * a.I : a.H;
        const int ocols = (MODE == 0) ? a.I : a.H;
        uint8_t* gstage = staging + grp * 2 * (C::kRows * C::kRowBytes);
        int chunk = 0;  // staging chunks written by this group (buffer parity)
        int lu = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++lu) {
            int split, tile, fb;
            decode(u, split, tile, fb);
            const Tile t = load_tile(a.tiles + tile);
            const int b = lu % C::kNBuf;
            const uint32_t aphase = (uint32_t)((lu / C::kNBuf) & 1);
            const bool got = mbar_wait(&aux->tfull[b], aphase, abort_flag);
            if (!got) flag_error(a, aux);
            if (named_bar_or(1 + grp, 128, !got || *abort_flag)) break;  // same in all 4 warps
            tc_fence_after();
            // MODE 0: feature f of the gate block (accumulator 0) and of the up block
            // (accumulator 1); MODE 1: output features f and f + 128
            const int f = (MODE == 0 ? fb * kBM : fb * 2 * kBM) + f_local;
            const bool f1_ok = MODE == 0 || f + kBM < a.H;
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::kAccCols);
            const int jbeg = grp * C::kGroupCols;
            const int jend = min(t.rows, jbeg + C::kGroupCols);
            if (S == 1) {
                // For each output block (MODE 0: act; MODE 1: the two 128-row w2
                // blocks in turn):
                // 1. drain this group's accumulator columns into registers as packed
                //    bf16 (MODE 0: act = silu(gate) * up), then hand the columns back
                //    to the MMA thread at once, so the next unit's main loop overlaps
                //    the stores below;
                // 2. stage kRows token rows at a time in shared memory (one 256-byte
                //    row segment each) and copy them out with 16-byte loads and
                //    stores, each row segment written whole.  Two buffers per group:
                //    one barrier per chunk separates a buffer's readers from its next
                //    writers.
                constexpr int kPk = C::kGroupCols / 2;
                constexpr int kBlocks = MODE == 0 ? 1 : 2;
#pragma unroll
                for (int h = 0; h < kBlocks; ++h) {
                    uint32_t pk[kPk];
#pragma unroll
                    for (int c = 0; c < C::kGroupCols; c += 8) {
                        if (jbeg + c < jend) {  // warp-uniform
                            uint32_t gv[8];
                            tmem_ld8(tacc + h * NT + jbeg + c, gv);
                            if (MODE == 0) {
                                uint32_t vv[8];
                                tmem_ld8(tacc + NT + jbeg + c, vv);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < 8; i += 2)
                                    pk[(c + i) / 2] = pack_bf16x2(
                                        silu_mul(__uint_as_float(gv[i]), __uint_as_float(vv[i])),
                                        silu_mul(__uint_as_float(gv[i + 1]),
                                                 __uint_as_float(vv[i + 1])));
                            } else {
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < 8; i += 2)
                                    pk[(c + i) / 2] = pack_bf16x2(__uint_as_float(gv[i]),
                                                                  __uint_as_float(gv[i + 1]));
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(h == 0 ? &aux->tempty[b] : &aux->tempty2[b]);
                    // MODE 1: the second block of the last pair may lie past H
                    if (h == 1 && !f1_ok) continue;
                    // one 16-byte vector per group thread: kRows rows of 16 vectors
                    const int jj = gt >> 4, cc = gt & 15;
                    const int col0 = MODE == 0 ? fb * kBM : fb * 2 * kBM + h * kBM;
#pragma unroll
                    for (int c = 0; c < C::kGroupCols; c += C::kRows) {
                        if (jbeg + c < jend) {  // group-uniform
                            uint8_t* buf = gstage + (chunk & 1) * (C::kRows * C::kRowBytes);
#pragma unroll
                            for (int r = 0; r < C::kRows; ++r) {
                                const uint32_t w = pk[(c + r) / 2];
                                reinterpret_cast<uint16_t*>(buf + r * C::kRowBytes)[f_local] =
                                    (uint16_t)(((c + r) & 1) ? (w >> 16) : (w & 0xFFFFu));
                            }
                            named_bar_sync(1 + grp, 128);  // staged; the other buffer is free again
                            if (jj < jend - (jbeg + c)) {
                                const int p = t.row_start + jbeg + c + jj;
                                const uint4 val = *reinterpret_cast<const uint4*>(
                                    buf + jj * C::kRowBytes + cc * 16);
                                const int row = MODE == 0 ? p : a.permuted_rows[p];
                                if (debug_in_range(row, 0, a.R, a.err))
                                    *reinterpret_cast<uint4*>(a.out + (size_t)row * ocols + col0 +
                                                              cc * 8) = val;
                            }
                            ++chunk;
                        }
                    }
                }
                continue;
            }
            constexpr int kCols = C::kLdCols;
            for (int j0 = jbeg; j0 < jend; j0 += kCols) {
                uint32_t gv[kCols], vv[kCols];
                tmem_ld_cols(tacc + j0, gv);
                tmem_ld_cols(tacc + NT + j0, vv);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < kCols; ++jj) {
                    const int j = j0 + jj;
                    if (j >= jend) break;
                    const int p = t.row_start + j;
                    const float gvf = __uint_as_float(gv[jj]);
                    if (MODE == 0) {
                        float* prow = a.partials + ((size_t)split * a.R + p) * pcols;
                        prow[f] = gvf;
                        prow[a.I + f] = __uint_as_float(vv[jj]);
                    } else {
                        const int r = a.permuted_rows[p];
                        if (!debug_in_range(r, 0, a.R, a.err)) continue;
                        float* prow = a.partials + ((size_t)split * a.R + r) * pcols;
                        prow[f] = gvf;
                        if (f1_ok) prow[f + kBM] = __uint_as_float(vv[jj]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&aux->tempty[b]);
                mbar_arrive(&aux->tempty2[b]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side


template <int MODE, int NT>
cudaError_t launch_mode(const CUtensorMap& tw, const CUtensorMap& ta, const FfnArgs& a, int grid,
                        cudaStream_t st)
{
    using C = GCfg<MODE, NT>;
    auto kern = grouped_gemm_kernel<MODE, NT>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (err != cudaSuccess) return err;
    return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, st, tw, ta, a);
}

template <int MODE>
cudaError_t launch_nt(int nt, const CUtensorMap& tw, const CUtensorMap& ta, const FfnArgs& a,
                      int grid, cudaStream_t st)
{
    switch (nt) {
    case 16: return launch_mode<MODE, 16>(tw, ta, a, grid, st);
    case 32: return launch_mode<MODE, 32>(tw, ta, a, grid, st);
    case 64: return launch_mode<MODE, 64>(tw, ta, a, grid, st);
    case 128: return launch_mode<MODE, 128>(tw, ta, a, grid, st);
    case 256: return launch_mode<MODE, 256>(tw, ta, a, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

FfnPlan plan_ffn(int T, int E, int k, int H, int I, int num_sms)
{
    FfnPlan p;
    const long R = (long)T * k;
    // one tile per expert whenever an expert can hold every token (each token
    // picks an expert at most once), so decode streams each weight block once
    int nt = 16;
    while (nt < 256 && nt < T) nt *= 2;
    p.nt = nt;
    p.max_tiles = (int)((R + nt - 1) / nt + (E < R ? E : R));
    // split-K only pays when even the smallest possible tile count leaves the GPU
    // idle, and only for weight-streaming shapes: with >= 128 routed rows per
    // expert on average the GEMMs are tensor-bound and a split only adds traffic
    const long min_units13 = ((R + nt - 1) / nt) * (I / kBM);
    const long min_units2 = ((R + nt - 1) / nt) * (H / kBM);
    const long target = 16L * num_sms;
    const bool skinny = R < 128L * (E < R ? E : R);
    p.s13_max = (skinny && min_units13 < target) ? 8 : 1;
    p.s2_max = (skinny && min_units2 < target) ? 8 : 1;
    p.grid = num_sms;
    return p;
}

cudaError_t launch_grouped_ffn(const FfnBuffers& b, int T, int E, int k, int H, int I,
                               const FfnPlan& plan, cudaStream_t st, cudaEvent_t between_gemms,
                               bool reduce_y)
{
    const int R = T * k;
    CUtensorMap tw13, tw2, tact;
    cudaError_t err = make_tmap(&tw13, b.w13, (uint64_t)E * 2 * I, (uint64_t)H, kBM);
    if (err == cudaSuccess) err = make_tmap(&tw2, b.w2, (uint64_t)E * H, (uint64_t)I, kBM);
    if (err == cudaSuccess) err = make_tmap(&tact, b.act, (uint64_t)R, (uint64_t)I, (uint32_t)plan.nt);
    if (err != cudaSuccess) return err;

    FfnArgs a = {};
    a.x = static_cast<const __nv_bfloat16*>(b.x);
    a.permuted_rows = b.permuted_rows;
    a.tiles = b.tiles;
    a.num_tiles = b.num_tiles;
    a.partials = b.partials;
    a.err = b.err;
    a.k = k;
    a.H = H;
    a.I = I;
    a.R = R;
    a.max_tiles = plan.max_tiles;
    a.min_kt_per_split = 4;
    a.weights_evict_first = plan.nt <= 64 ? 1 : 0;

    // w13 + SwiGLU: K = H
    a.out = static_cast<__nv_bfloat16*>(b.act);
    a.split_out = b.splits;
    a.num_kt = H / kBK;
    a.fb_count = I / kBM;
    a.s_max = plan.s13_max;
    err = launch_nt<0>(plan.nt, tw13, tw13, a, plan.grid, st);
    if (err != cudaSuccess) return err;
    if (plan.s13_max > 1) {
        err = launch_swiglu_finalize(b.partials, b.splits, R, I, b.act, st);
        if (err != cudaSuccess) return err;
    }
    if (between_gemms) {
        err = cudaEventRecord(between_gemms, st);
        if (err != cudaSuccess) return err;
    }

    // w2: K = I
    a.out = static_cast<__nv_bfloat16*>(b.y);
    a.split_out = b.splits + 1;
    a.num_kt = I / kBK;
    a.fb_count = (H / kBM + 1) / 2;
    a.s_max = plan.s2_max;
    err = launch_nt<1>(plan.nt, tw2, tact, a, plan.grid, st);
    if (err != cudaSuccess || plan.s2_max <= 1 || !reduce_y) return err;
    return launch_reduce_y(b.partials, b.splits + 1, R, H, b.y, st);
}

}  // namespace moe
