// route_permute.cu -- top-k routing of fp32 router logits and the stable
// per-expert permutation of the expanded rows.
//
// Routing ("softmax_sum", FlashInfer PR #3751 page "Optimizing TRTLLM-Gen MoE
// routing", sections "1. dynamic thread-block size" and "performance numbers"):
// one warp owns one token; each lane keeps E/32 logits in registers; a warp
// bitonic sort of the lane maxima gives a threshold that leaves only a handful of
// candidates, which are sorted by (logit desc, expert asc) keys; the k weights
// are a softmax over the selected logits, summed in selection order.  The pages size the routing CTA by token count to keep
// register pressure down; here the register footprint is fixed by the
// per-lane value count V (a template), and the grid scales with T.
//
// Permutation: count -> exclusive scan -> stable scatter.  Ranks inside a warp
// come from __match_any_sync peer masks, ranks across warps from a per-warp
// count table and a column scan, ranks across CTAs from a per-chunk count table
// that every scatter CTA reads whole, so the result (ascending expanded id inside every expert)
// never depends on atomic ordering.  No kernel waits on another CTA.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "kernels.h"
#include "ptx.cuh"
#include "route_common.cuh"

namespace moe {

namespace {


// Sorts one float per lane across the warp, largest in lane 0.
__device__ __forceinline__ float warp_sort_desc(float v, int lane)
{
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const float o = __shfl_xor_sync(kFull, v, stride);
            const bool take_max = ((lane & stride) == 0) == ((lane & size) == 0);
            v = take_max ? fmaxf(v, o) : fminf(v, o);
        }
    }
    return v;
}

// Expert held in value slot `s` of lane `lane`.  With VEC (E % 4 == 0, V % 4 == 0)
// lane l loads float4 groups: slot 4m + c holds expert 128m + 4l + c; otherwise
// slot s holds expert 32s + l.  Either way a lane's slots are in ascending expert
// order.
template <int V, bool VEC>
__device__ __forceinline__ int slot_expert(int s, int lane)
{
    return VEC ? (s >> 2) * 128 + lane * 4 + (s & 3) : s * 32 + lane;
}

// Routes one token with the calling warp.  row: E logits.  Writes ids/weights
// (k each) to global memory and, if ids_s != nullptr, the ids to shared memory.
// `cand` is this warp's shared scratch of 32 (value, index) pairs.
//
// Selection.  Let tau be the k-th largest of the 32 per-lane maxima: the k lanes
// with the largest maxima hold k distinct experts with logit >= tau, so every
// expert of the top k has logit >= tau.  The experts with logit >= tau are
// gathered (one per lane) and sorted by (logit desc, expert asc); the first k
// are the answer.  If more than 32 experts reach tau (ties, -inf rows), the
// exact fallback takes the k winners one by one with a warp arg-max.
template <int V, bool VEC>
__device__ __forceinline__ void warp_load_row(const float* __restrict__ row, int E, int lane,
                                              float (&v)[V])
{
    if (VEC) {
#pragma unroll
        for (int m = 0; m < V / 4; ++m) {
            const int e = m * 128 + lane * 4;
            float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (e < E) q = __ldg(reinterpret_cast<const float4*>(row + e));
            v[4 * m] = q.x;
            v[4 * m + 1] = q.y;
            v[4 * m + 2] = q.z;
            v[4 * m + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int m = 0; m < V; ++m) {
            const int e = m * 32 + lane;
            v[m] = (e < E) ? __ldg(row + e) : -INFINITY;
        }
    }
}

// Exact selection when more than 32 experts reach the threshold (ties, -inf
// rows): the k winners one by one with a warp arg-max.
template <int V, bool VEC>
__device__ __forceinline__ void select_exhaustive(const float (&v)[V], int E, int k, int lane,
                                                  float& my_l, int& my_id)
{
    uint32_t taken = 0;
    // best not-yet-taken value of this lane; slots ascend with the expert, so a
    // strict '>' keeps the lower expert on equal values
    auto lane_best = [&](float& bv, int& bi) {
        bv = -INFINITY;
        bi = kNoIndex;
#pragma unroll
        for (int m = 0; m < V; ++m) {
            const int e = slot_expert<V, VEC>(m, lane);
            const bool ok = e < E && !((taken >> m) & 1u);
            if (ok && (bi == kNoIndex || v[m] > bv)) {
                bv = v[m];
                bi = e;
            }
        }
    };
    float bv;
    int bi;
    lane_best(bv, bi);
    for (int j = 0; j < k; ++j) {
        float wv = bv;
        int wi = bi;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(kFull, wv, off);
            const int oi = __shfl_xor_sync(kFull, wi, off);
            if (key_before(ov, oi, wv, wi)) {
                wv = ov;
                wi = oi;
            }
        }
        if (lane == j) {
            my_l = wv;
            my_id = wi;
        }
        const int owner = VEC ? (wi & 127) >> 2 : (wi & 31);
        if (owner == lane) {  // the owner drops the winner and finds its next best
            const int slot = VEC ? (wi >> 7) * 4 + (wi & 3) : (wi >> 5);
            taken |= 1u << slot;
            lane_best(bv, bi);
        }
    }
}

template <int V, bool VEC>
__device__ __forceinline__ void warp_select_token(const float (&v)[V], int E, int k, int lane,
                                                  int32_t* __restrict__ ids,
                                                  float* __restrict__ weights, int* ids_s,
                                                  float2* cand)
{
    // slots past E hold -inf; they are kept out of the candidates explicitly
    float mv = -INFINITY;
#pragma unroll
    for (int m = 0; m < V; ++m) mv = fmaxf(mv, v[m]);
    const float tau = __shfl_sync(kFull, warp_sort_desc(mv, lane), k - 1);

    // when E = 32 V every slot holds an expert and the range test can go
    const bool full = E == 32 * V;
    int c = 0;
    if (full) {
#pragma unroll
        for (int m = 0; m < V; ++m) c += v[m] >= tau ? 1 : 0;
    } else {
#pragma unroll
        for (int m = 0; m < V; ++m) c += (slot_expert<V, VEC>(m, lane) < E && v[m] >= tau) ? 1 : 0;
    }
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += n;
    }
    const int total = __shfl_sync(kFull, incl, 31);

    float my_l = 0.f;
    int my_id = 0;
    if (total <= 32) {
        int pos = incl - c;
        if (full) {
#pragma unroll
            for (int m = 0; m < V; ++m)
                if (v[m] >= tau)
                    cand[pos++] = make_float2(v[m], __int_as_float(slot_expert<V, VEC>(m, lane)));
        } else {
#pragma unroll
            for (int m = 0; m < V; ++m) {
                const int e = slot_expert<V, VEC>(m, lane);
                if (e < E && v[m] >= tau) cand[pos++] = make_float2(v[m], __int_as_float(e));
            }
        }
        __syncwarp();
        sort_candidates(total, lane, cand, my_l, my_id);
    } else {
        select_exhaustive<V, VEC>(v, E, k, lane, my_l, my_id);
    }
    write_selection(my_l, my_id, k, lane, ids, weights, ids_s);
}

// warp_select_token for a row that is also staged in shared memory (rowf[e] =
// logit of expert e; float4 slot layout, E % 4 == 0).  The threshold comes from
// warp max reductions, each lane marks its slots that reach it in a bit mask,
// and only the marked slots are read back (from shared memory) as candidates.
template <int V, bool FULL>
__device__ __forceinline__ void warp_select_staged(const float (&v)[V], const float* rowf, int E,
                                                   int k, int lane, int32_t* __restrict__ ids,
                                                   float* __restrict__ weights, float2* cand)
{
    float mv = -INFINITY;
#pragma unroll
    for (int m = 0; m < V; ++m) mv = fmaxf(mv, v[m]);
    const float tau = warp_kth_largest(mv, k);
    uint32_t mask = 0;
#pragma unroll
    for (int m = 0; m < V; ++m)
        if ((FULL || slot_expert<V, true>(m, lane) < E) && v[m] >= tau) mask |= 1u << m;
    const int c = __popc(mask);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += n;
    }
    const int total = __shfl_sync(kFull, incl, 31);
    float my_l = 0.f;
    int my_id = 0;
    if (total <= 32) {
        int pos = incl - c;
        while (mask) {
            const int m = __ffs(mask) - 1;
            mask &= mask - 1;
            const int e = slot_expert<V, true>(m, lane);
            cand[pos++] = make_float2(rowf[e], __int_as_float(e));
        }
        __syncwarp();
        sort_candidates(total, lane, cand, my_l, my_id);
    } else {
        select_exhaustive<V, true>(v, E, k, lane, my_l, my_id);
    }
    write_selection(my_l, my_id, k, lane, ids, weights, nullptr);
}

template <int V, bool VEC>
__device__ __forceinline__ void warp_route_token(const float* __restrict__ row, int E, int k,
                                                 int lane, int32_t* __restrict__ ids,
                                                 float* __restrict__ weights, int* ids_s,
                                                 float2* cand)
{
    float v[V];
    warp_load_row<V, VEC>(row, E, lane, v);
    warp_select_token<V, VEC>(v, E, k, lane, ids, weights, ids_s, cand);
}

// Thread e (< E) owns expert e with `count` rows at permuted offset `off` and
// writes its tiles: as few as ceil(count / nt) allows, of near-equal size rounded
// to the MMA's 16-column granule (so no tile is a short tail that streams a whole
// weight block for a few rows), the last one taking the remainder.
__device__ __forceinline__ void write_tiles_and_reset(bool owns, int e, int count, int off,
                                                      const PermuteAux& aux, int* sums)
{
    int n = 0, q = aux.nt;
    if (owns && count > 0) {
        const int n0 = (count + aux.nt - 1) / aux.nt;
        const int even = (count + n0 - 1) / n0;
        q = min(aux.nt, (even + 15) & ~15);
        n = (count + q - 1) / q;
    }
    int total;
    const int start = block_exclusive_scan(n, sums, total);
    // debug build: never past the tile array (only out-of-contract offsets can
    // ask for more tiles than it holds)
    if (n > 0 && !debug_in_range(start + n - 1, 0, aux.max_tiles, aux.err))
        n = max(0, aux.max_tiles - start);
    if (kDebugChecks) total = min(total, aux.max_tiles);
    for (int i = 0; i < n; ++i) {
        Tile t;
        t.expert = e;
        t.row_start = off + i * q;
        t.rows = min(q, count - i * q);
        t.first = start;
        t.count = n;
        t.pad[0] = t.pad[1] = t.pad[2] = 0;
        aux.tiles[start + i] = t;
    }
    if (threadIdx.x == 0) *aux.num_tiles = total;
}

// Per-warp histogram of rows [r0, r1) of ids_s into table[warp*E + e].
__device__ __forceinline__ void warp_count(const int* ids_s, int r0, int r1, int* table_row)
{
    const int lane = threadIdx.x & 31;
    for (int base = r0; base < r1; base += 32) {
        const int r = base + lane;
        const bool valid = r < r1;
        const int e = valid ? ids_s[r] : -1;
        const unsigned vm = __ballot_sync(kFull, valid);
        if (valid) {
            const unsigned peers = __match_any_sync(vm, e);
            if (lane == __ffs(peers) - 1) table_row[e] += __popc(peers);
        }
        __syncwarp();
    }
}

// Stable scatter of rows [r0, r1): table_row[e] holds the absolute position of
// the next row of expert e owned by this warp.
__device__ __forceinline__ void warp_scatter(const int* ids_s, int r0, int r1, int id_base,
                                             int* table_row, int32_t* __restrict__ rows_out)
{
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = r0; base < r1; base += 32) {
        const int r = base + lane;
        const bool valid = r < r1;
        const int e = valid ? ids_s[r] : -1;
        const unsigned vm = __ballot_sync(kFull, valid);
        unsigned peers = 0;
        int pos = 0;
        if (valid) {
            peers = __match_any_sync(vm, e);
            pos = table_row[e] + __popc(peers & lt);
        }
        __syncwarp();
        if (valid) {
            rows_out[pos] = id_base + r;
            if (lane == __ffs(peers) - 1) table_row[e] += __popc(peers);
        }
        __syncwarp();
    }
}

// ----------------------------------------------------------------- kernels

template <int V, bool VEC>
__global__ void __launch_bounds__(256, 4) route_kernel(const float* __restrict__ logits, int T,
                                                       int E, int k, int32_t* __restrict__ ids,
                                                       float* __restrict__ weights)
{
    __shared__ float2 cand[8][32];
    pdl_wait();
    pdl_launch_dependents();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    warp_route_token<V, VEC>(logits + (size_t)t * E, E, k, threadIdx.x & 31, ids + (size_t)t * k,
                             weights + (size_t)t * k, nullptr, cand[threadIdx.x >> 5]);
}

// Routing with many experts per token (E = 32 V logits, V >= 16, E % 4 == 0):
// persistent warps, warp w of the grid routing tokens w, w + W, ... (W = all warps).
// A token row is E * 4 bytes; each lane copies its own 16-byte pieces of it (the
// float4 slot layout of warp_load_row: piece m of lane l = experts 128 m + 4 l ..)
// with cp.async into the warp's ring of kRouteDepth rows in shared memory,
// kRouteDepth - 1 tokens ahead of the one being selected (one ahead: a second
// row per warp measured slower than the third CTA per SM it costs), and reads
// back only
// what it copied itself -- its own cp.async.wait_group makes those visible, so no
// barrier is involved.  The logits of later tokens stream from HBM while the
// current one is selected.
constexpr int kRouteWarps = 8;
constexpr int kRouteDepth = 2;

template <int V, bool FULL>
__global__ void __launch_bounds__(kRouteWarps * 32, 3)
    route_stream_kernel(const float* __restrict__ logits, int T, int E, int k,
                        int32_t* __restrict__ ids, float* __restrict__ weights)
{
    static_assert(V % 4 == 0, "float4 slots");
    constexpr int kPieces = V / 4;  // 16-byte pieces per lane and row
    extern __shared__ float4 ring[];  // [kRouteWarps][kRouteDepth][kPieces][32]
    __shared__ float2 cand[kRouteWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float4* my = ring + (size_t)warp * kRouteDepth * kPieces * 32;
    pdl_wait();
    pdl_launch_dependents();
    const uint64_t pol = l2_policy_evict_first();  // each logit is read once
    const int W = gridDim.x * kRouteWarps;
    const int w0 = blockIdx.x * kRouteWarps + warp;
    auto issue = [&](int t, int slot) {
        if (t < T) {
            const float* row = logits + (size_t)t * E;
#pragma unroll
            for (int m = 0; m < kPieces; ++m) {
                const int e = m * 128 + lane * 4;
                if (e < E)
                    cp_async_16_hint(smem_u32(my + (slot * kPieces + m) * 32 + lane), row + e, pol);
            }
        }
        cp_async_commit();  // one group per token, empty or not
    };
#pragma unroll
    for (int d = 0; d < kRouteDepth - 1; ++d) issue(w0 + d * W, d);
    int slot = 0;
    for (int t = w0; t < T; t += W) {
        // the slot refilled now held the previous token, whose values were
        // consumed by its selection
        issue(t + (kRouteDepth - 1) * W, (slot + kRouteDepth - 1) % kRouteDepth);
        cp_async_wait<kRouteDepth - 1>();  // this token's pieces have landed
        float v[V];
#pragma unroll
        for (int m = 0; m < kPieces; ++m) {
            float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (m * 128 + lane * 4 < E) q = my[(slot * kPieces + m) * 32 + lane];
            v[4 * m] = q.x;
            v[4 * m + 1] = q.y;
            v[4 * m + 2] = q.z;
            v[4 * m + 3] = q.w;
        }
        warp_select_staged<V, FULL>(v, reinterpret_cast<const float*>(my + slot * kPieces * 32), E, k,
                              lane, ids + (size_t)t * k, weights + (size_t)t * k, cand[warp]);
        slot = (slot + 1) % kRouteDepth;
    }
    cp_async_wait<0>();
}

// One CTA: (route) + count + scan + stable scatter + tile list, for T*k <= kSmallRows.
template <int V, bool VEC>
__global__ void __launch_bounds__(1024, 1)
    small_route_permute_kernel(const float* __restrict__ logits, int T, int E, int k,
                               int32_t* __restrict__ ids, float* __restrict__ weights,
                               int32_t* __restrict__ offsets, int32_t* __restrict__ rows_out,
                               PermuteAux aux)
{
    extern __shared__ int smem[];
    __shared__ int sums[32];
    __shared__ float2 cand[32][32];
    const int R = T * k;
    int* ids_s = smem;
    int* table = smem + ((R + 3) & ~3);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    pdl_wait();
    pdl_launch_dependents();

    if (logits) {
        // a warp's next token is loaded while its current one is selected
        float v[V];
        if (warp < T) warp_load_row<V, VEC>(logits + (size_t)warp * E, E, lane, v);
        for (int t = warp; t < T; t += 32) {
            float nv[V];
            if (t + 32 < T) warp_load_row<V, VEC>(logits + (size_t)(t + 32) * E, E, lane, nv);
            warp_select_token<V, VEC>(v, E, k, lane, ids + (size_t)t * k, weights + (size_t)t * k,
                                      ids_s + t * k, cand[warp]);
#pragma unroll
            for (int m = 0; m < V; ++m) v[m] = nv[m];
        }
    } else {
        for (int r = threadIdx.x; r < R; r += blockDim.x) {
            const int e = ids[r];
            ids_s[r] = debug_in_range(e, 0, E, aux.err) ? e : 0;
        }
    }
    // counting warps: as many as there are 32-row groups, up to 32
    const int W = min(32, (R + 31) / 32);
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) table[i] = 0;
    __syncthreads();

    const int per_warp = (R + W - 1) / W;
    const int r0 = min(R, warp * per_warp), r1 = warp < W ? min(R, r0 + per_warp) : r0;
    if (warp < W) warp_count(ids_s, r0, r1, table + warp * E);
    __syncthreads();

    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    int cnt = 0;
    if (owns)
        for (int w = 0; w < W; ++w) {
            const int c = table[w * E + e];
            table[w * E + e] = cnt;
            cnt += c;
        }
    int total;
    const int off = block_exclusive_scan(owns ? cnt : 0, sums, total);
    if (owns) {
        offsets[e] = off;
        for (int w = 0; w < W; ++w) table[w * E + e] += off;
    }
    if (threadIdx.x == 0) offsets[E] = total;
    write_tiles_and_reset(owns, e, cnt, off, aux, sums);
    __syncthreads();

    if (warp < W) warp_scatter(ids_s, r0, r1, 0, table + warp * E, rows_out);
}

__global__ void __launch_bounds__(1024) chunk_count_kernel(const int32_t* __restrict__ ids, int R,
                                                           int E, int32_t* __restrict__ counts,
                                                           int32_t* err)
{
    extern __shared__ int hist[];
    pdl_wait();
    pdl_launch_dependents();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int r0 = blockIdx.x * kChunkRows, r1 = min(R, r0 + kChunkRows);
    for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
        const int e = ids[r];
        atomicAdd(&hist[debug_in_range(e, 0, E, err) ? e : 0], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// After chunk_count_kernel, for experts 32 b .. 32 b + 31 (CTA b, lane = expert):
// warp w walks the chunks [w L, (w + 1) L) (L = ceil(n_chunks / 32)) of its
// expert, the 32 warps' sums are scanned in shared memory, and counts[c][e] is
// overwritten with P[c][e] = the rows of e in the chunks before c.  Row n_chunks
// of the table receives the expert's total.  Every chunk read is coalesced over
// the 32 experts of a warp.
__global__ void __launch_bounds__(1024, 1)
    chunk_prefix_kernel(int32_t* __restrict__ counts, int n_chunks, int E)
{
    __shared__ int part[32][33];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    const int L = (n_chunks + 31) / 32;
    const int c0 = min(n_chunks, warp * L), c1 = min(n_chunks, c0 + L);
    int sum = 0;
    if (e < E)
        for (int c = c0; c < c1; ++c) sum += __ldcg(counts + (size_t)c * E + e);
    part[warp][lane] = sum;
    __syncthreads();
    int pre = 0;
    for (int w = 0; w < warp; ++w) pre += part[w][lane];
    if (e < E) {
        int run = pre;
        for (int c = c0; c < c1; ++c) {
            const int v = __ldcg(counts + (size_t)c * E + e);
            counts[(size_t)c * E + e] = run;
            run += v;
        }
        if (warp == 31) counts[(size_t)n_chunks * E + e] = run;  // the expert's total
    }
}

constexpr int kRankWarps = 8;

// One CTA per chunk of kChunkRows expanded rows, after chunk_prefix_kernel.  The
// expert totals (row n_chunks of the table) give expert_offsets by an exclusive
// scan over experts (CTA 0 also writes them and the tile list); base[e] =
// expert_offsets[e] + P[chunk][e] is where the chunk's first row of expert e
// goes.  The chunk's rows are ranked stably with per-warp count tables (a warp's
// rows in order, warps in order) and scattered.
__global__ void __launch_bounds__(1024, 1)
    chunk_scatter_kernel(const int32_t* __restrict__ ids, int R, int E, int n_chunks,
                         const int32_t* __restrict__ prefix, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ rows_out, PermuteAux aux)
{
    extern __shared__ int smem[];
    __shared__ int sums[32];
    int* ids_s = smem;                 // kChunkRows
    int* table = smem + kChunkRows;    // [kRankWarps][E]
    const int warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_launch_dependents();
    const int c0 = blockIdx.x * kChunkRows, n = min(kChunkRows, R - c0);
    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    // the three loads are independent: issue them before anything waits
    const int total_e = owns ? __ldcg(prefix + (size_t)n_chunks * E + e) : 0;
    const int pre_e = owns ? __ldcg(prefix + (size_t)blockIdx.x * E + e) : 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int id = ids[c0 + i];
        ids_s[i] = debug_in_range(id, 0, E, aux.err) ? id : 0;
    }
    for (int i = threadIdx.x; i < kRankWarps * E; i += blockDim.x) table[i] = 0;
    int total;
    const int off = block_exclusive_scan(total_e, sums, total);  // ends with a barrier
    if (blockIdx.x == 0) {
        if (owns) offsets[e] = off;
        if (threadIdx.x == 0) offsets[E] = total;
        write_tiles_and_reset(owns, e, total_e, off, aux, sums);
    }

    // kRankWarps warps rank the chunk's rows, kChunkRows / kRankWarps each, in
    // order: fewer count rows to clear and to scan than one per warp of the CTA
    constexpr int per_warp = kChunkRows / kRankWarps;
    const int r0 = min(n, warp * per_warp), r1 = min(n, r0 + per_warp);
    if (warp < kRankWarps) warp_count(ids_s, r0, r1, table + warp * E);
    __syncthreads();
    if (owns) {
        // the ranking warps' counts of expert e, read before any is overwritten
        int v[kRankWarps];
#pragma unroll
        for (int w = 0; w < kRankWarps; ++w) v[w] = table[w * E + e];
        int run = off + pre_e;
#pragma unroll
        for (int w = 0; w < kRankWarps; ++w) {
            table[w * E + e] = run;
            run += v[w];
        }
    }
    __syncthreads();
    if (warp < kRankWarps) warp_scatter(ids_s, r0, r1, c0, table + warp * E, rows_out);
}

__global__ void __launch_bounds__(1024) build_tiles_kernel(const int32_t* __restrict__ offsets,
                                                           int E, int R, PermuteAux aux)
{
    __shared__ int sums[32];
    pdl_wait();
    pdl_launch_dependents();
    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    int off = owns ? offsets[e] : 0;
    int cnt = owns ? offsets[e + 1] - off : 0;
    // debug build: an expert's rows must lie inside [0, R); otherwise it gets no tile
    if (owns && !(debug_in_range(off, 0, R + 1, aux.err) && debug_in_range(cnt, 0, R - off + 1, aux.err)))
        off = cnt = 0;
    write_tiles_and_reset(owns, e, cnt, off, aux, sums);
}

template <typename Kern, typename... Args>
cudaError_t launch(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args)
{
    return launch_pdl(kern, grid, block, smem, st, args...);
}

int values_per_lane(int E)
{
    const int v = (E + 31) / 32;
    return v <= 1 ? 1 : v <= 2 ? 2 : v <= 4 ? 4 : v <= 8 ? 8 : v <= 16 ? 16 : 32;
}

}  // namespace

template <int V>
static cudaError_t launch_route_v(bool vec, const float* logits, int T, int E, int k, int32_t* ids,
                                  float* weights, cudaStream_t st)
{
    if constexpr (V >= 16) {
        if (vec) {
            const size_t smem = sizeof(float) * (size_t)kRouteWarps * kRouteDepth * 32 * V;
            int dev = 0, sms = 148;
            if (cudaGetDevice(&dev) == cudaSuccess)
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            // three CTAs per SM (64 KB of rings each at V = 32), no more than the tokens need
            const int want = (T + kRouteWarps - 1) / kRouteWarps;
            const int grid = want < 3 * sms ? want : 3 * sms;
            auto go = [&](auto kern) {
                cudaError_t err = cudaFuncSetAttribute(
                    kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (err != cudaSuccess) return err;
                return launch(kern, dim3(grid), dim3(kRouteWarps * 32), smem, st, logits, T, E, k,
                              ids, weights);
            };
            return E == 32 * V ? go(route_stream_kernel<V, true>)
                               : go(route_stream_kernel<V, false>);
        }
    }
    const dim3 grid((T + 7) / 8), block(256);
    if (vec && V >= 4)
        return launch(route_kernel<V, (V >= 4)>, grid, block, 0, st, logits, T, E, k, ids, weights);
    return launch(route_kernel<V, false>, grid, block, 0, st, logits, T, E, k, ids, weights);
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* weights,
                         cudaStream_t st)
{
    const bool vec = (E % 4) == 0;
    switch (values_per_lane(E)) {
    case 1: return launch_route_v<1>(vec, logits, T, E, k, ids, weights, st);
    case 2: return launch_route_v<2>(vec, logits, T, E, k, ids, weights, st);
    case 4: return launch_route_v<4>(vec, logits, T, E, k, ids, weights, st);
    case 8: return launch_route_v<8>(vec, logits, T, E, k, ids, weights, st);
    case 16: return launch_route_v<16>(vec, logits, T, E, k, ids, weights, st);
    default: return launch_route_v<32>(vec, logits, T, E, k, ids, weights, st);
    }
}

template <int V, bool VEC>
static cudaError_t launch_small_v(const float* logits, int T, int E, int k, int32_t* ids,
                                  float* weights, int32_t* offsets, int32_t* rows,
                                  const PermuteAux& aux, cudaStream_t st)
{
    const int R = T * k;
    const size_t smem = sizeof(int) * (size_t)(((R + 3) & ~3) + 32 * E);  // >= E ints
    cudaError_t err = cudaFuncSetAttribute(small_route_permute_kernel<V, VEC>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch(small_route_permute_kernel<V, VEC>, dim3(1), dim3(1024), smem, st, logits, T, E,
                  k, ids, weights, offsets, rows, aux);
}

cudaError_t launch_small_route_permute(const float* logits, int T, int E, int k, int32_t* ids,
                                       float* weights, int32_t* offsets, int32_t* rows,
                                       const PermuteAux& aux, cudaStream_t st)
{
    const bool vec = (E % 4) == 0;
#define MOE_SMALL(V)                                                                              \
    (vec && (V) >= 4 ? launch_small_v<V, ((V) >= 4)>(logits, T, E, k, ids, weights, offsets, rows, \
                                                     aux, st)                                     \
                     : launch_small_v<V, false>(logits, T, E, k, ids, weights, offsets, rows, aux, \
                                                st))
    switch (logits ? values_per_lane(E) : 1) {
    case 1: return MOE_SMALL(1);
    case 2: return MOE_SMALL(2);
    case 4: return MOE_SMALL(4);
    case 8: return MOE_SMALL(8);
    case 16: return MOE_SMALL(16);
    default: return MOE_SMALL(32);
    }
#undef MOE_SMALL
}

size_t large_permute_smem(int E) { return sizeof(int) * (size_t)(kChunkRows + kRankWarps * E); }

cudaError_t launch_large_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                                 int32_t* rows, const PermuteAux& aux, cudaStream_t st)
{
    const int R = T * k;
    const int n_chunks = (R + kChunkRows - 1) / kChunkRows;
    cudaError_t err = launch(chunk_count_kernel, dim3(n_chunks), dim3(1024), sizeof(int) * E, st,
                             ids, R, E, aux.chunk_counts, aux.err);
    if (err != cudaSuccess) return err;
    err = launch(chunk_prefix_kernel, dim3((E + 31) / 32), dim3(1024), 0, st, aux.chunk_counts,
                 n_chunks, E);
    if (err != cudaSuccess) return err;
    const size_t smem = large_permute_smem(E);
    err = cudaFuncSetAttribute(chunk_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (err != cudaSuccess) return err;
    return launch(chunk_scatter_kernel, dim3(n_chunks), dim3(1024), smem, st, ids, R, E, n_chunks,
                  (const int32_t*)aux.chunk_counts, offsets, rows, aux);
}

cudaError_t launch_build_tiles(const int32_t* offsets, int E, int R, const PermuteAux& aux,
                               cudaStream_t st)
{
    return launch(build_tiles_kernel, dim3(1), dim3(1024), 0, st, offsets, E, R, aux);
}

}  // namespace moe
