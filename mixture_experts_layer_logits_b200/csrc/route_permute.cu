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
// come from peer masks (one ballot per bit of the expert id), ranks across warps from a per-warp
// count table and a column scan, ranks across CTAs from a per-chunk count table
// whose columns are scanned over the chunks, so the result (ascending expanded id
// inside every expert) never depends on atomic ordering.  Up to kSmallRows rows
// one CTA does it all; beyond, one launch of at most one CTA per SM does it in
// three phases separated by two grid barriers (bounded waits).
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

// The tiles of an expert with `count` rows: as few as ceil(count / nt) allows, of
// near-equal size q rounded to the MMA's 16-column granule (so no tile is a short
// tail that streams a whole weight block for a few rows), the last one taking the
// remainder.  Returns the tile count (0 for an empty expert).
__device__ __forceinline__ int expert_tile_count(int count, int nt, int& q)
{
    q = nt;
    if (count <= 0) return 0;
    const int n0 = (count + nt - 1) / nt;
    const int even = (count + n0 - 1) / n0;
    q = min(nt, (even + 15) & ~15);
    return (count + q - 1) / q;
}

// Writes expert e's n tiles (size q, the expert's rows from permuted offset
// `off`) at tile index `start`.
__device__ __forceinline__ void write_expert_tiles(int e, int count, int off, int n, int q,
                                                   int start, const PermuteAux& aux)
{
    // debug build: never past the tile array (only out-of-contract offsets can
    // ask for more tiles than it holds)
    if (n > 0 && !debug_in_range(start + n - 1, 0, aux.max_tiles, aux.err))
        n = max(0, aux.max_tiles - start);
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
}

// Thread e (< E) owns expert e with `count` rows at permuted offset `off` and
// writes its tiles; thread 0 writes the tile count.
__device__ __forceinline__ void write_tiles_and_reset(bool owns, int e, int count, int off,
                                                      const PermuteAux& aux, int* sums)
{
    int q;
    const int n = owns ? expert_tile_count(count, aux.nt, q) : 0;
    int total;
    const int start = block_exclusive_scan(n, sums, total);
    if (kDebugChecks) total = min(total, aux.max_tiles);
    if (n > 0) write_expert_tiles(e, count, off, n, q, start, aux);
    if (threadIdx.x == 0) *aux.num_tiles = total;
}

// Expert ids of a range of rows: staged in shared memory, or read from global
// memory (the debug build redirects an out-of-range id to expert 0 on each read).
struct StagedIds {
    const int* s;
    __device__ __forceinline__ int operator()(int r) const { return s[r]; }
};
struct GlobalIds {
    const int32_t* g;
    int E;
    int32_t* err;
    __device__ __forceinline__ int operator()(int r) const
    {
        const int id = g[r];
        return debug_in_range(id, 0, E, err) ? id : 0;
    }
};

// Bits of an expert id below E (0 for E = 1).
__device__ __forceinline__ int expert_bits(int E) { return E <= 1 ? 0 : 32 - __clz(E - 1); }

// Mask of the valid lanes whose key equals this lane's key e (in [0, 2^nbits),
// nbits <= 10).  Up to 16 experts: __match_any_sync, whose cost grows with the
// number of distinct keys in the warp.  Beyond: one ballot per key bit (two keys
// are equal exactly when they agree on every bit), a constant cost, lower than
// __match_any_sync's once a warp holds many distinct experts.
__device__ __forceinline__ unsigned warp_peers(int e, bool valid, int nbits)
{
    if (nbits <= 4) {
        const unsigned vm = __ballot_sync(kFull, valid);
        return valid ? __match_any_sync(vm, e) : 0u;
    }
    unsigned peers = __ballot_sync(kFull, valid);
    for (int b = 0; b < nbits; ++b) {
        const bool bit = (e >> b) & 1;
        const unsigned m = __ballot_sync(kFull, bit);
        peers &= bit ? m : ~m;
    }
    return peers;
}

// Per-warp histogram of rows [r0, r1) into table_row[e] (ids below 2^nbits).
template <typename Ids>
__device__ __forceinline__ void warp_count(const Ids& id_at, int r0, int r1, int* table_row,
                                           int nbits)
{
    const int lane = threadIdx.x & 31;
    for (int base = r0; base < r1; base += 32) {
        const int r = base + lane;
        const bool valid = r < r1;
        const int e = valid ? id_at(r) : 0;
        const unsigned peers = warp_peers(e, valid, nbits);
        if (valid && lane == __ffs(peers) - 1) table_row[e] += __popc(peers);
        __syncwarp();
    }
}

// Stable scatter of rows [r0, r1): the next row of expert e owned by this warp
// goes to position (base ? base[e] : 0) + table_row[e].
template <typename Ids>
__device__ __forceinline__ void warp_scatter(const Ids& id_at, int r0, int r1, int id_base,
                                             const int* base, int* table_row,
                                             int32_t* __restrict__ rows_out, int nbits)
{
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    for (int b = r0; b < r1; b += 32) {
        const int r = b + lane;
        const bool valid = r < r1;
        const int e = valid ? id_at(r) : 0;
        const unsigned peers = warp_peers(e, valid, nbits);
        int pos = 0;
        if (valid) pos = (base ? base[e] : 0) + table_row[e] + __popc(peers & lt);
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
                if (FULL || e < E)
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
            if (FULL || m * 128 + lane * 4 < E) q = my[(slot * kPieces + m) * 32 + lane];
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
    if (warp < W) warp_count(StagedIds{ids_s}, r0, r1, table + warp * E, expert_bits(E));
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

    if (warp < W)
        warp_scatter(StagedIds{ids_s}, r0, r1, 0, nullptr, table + warp * E, rows_out,
                     expert_bits(E));
}

// ------------------------------------------- one-launch multi-CTA permutation

constexpr int kPermWarps = 32;         // warps per CTA
constexpr int kPermRankWarps = 8;      // of which rank the chunk, one contiguous piece each
constexpr int kPermStageRows = 8192;   // chunks up to this many rows are staged in shared memory
constexpr int kPermMaxChunks = 256;    // grid bound (the prefix phase's chunks per lane <= 8)
constexpr int kPermLaneChunks = kPermMaxChunks / 32;

// Thread 0 of a CTA: bounded wait (2 s) until `ok()` holds.  Gives up early when
// another CTA recorded an abort of this call; on its own timeout records the
// abort and kDeviceErrorMagic in *err.
template <typename Pred>
__device__ bool grid_wait(GridBar* bar, unsigned long long gen, int32_t* err, Pred ok)
{
    if (ok()) return true;
    const uint64_t t0 = globaltimer_ns();
    volatile unsigned long long* abort = &bar->abort;
    for (;;) {
        __nanosleep(32);
        if (ok()) return true;
        if (*abort == gen) return false;
        if (globaltimer_ns() - t0 > 2000000000ull) {
            *abort = gen;
            atomicExch(err, kDeviceErrorMagic);
            return false;
        }
    }
}

// The stable permutation of R > kSmallRows rows in one launch of G CTAs (all
// resident at once; at most one per SM), CTA c owning the S rows from c*S (S a
// multiple of 32).
//   1. The CTA counts its chunk's experts into counts[c][*] and arrives at the
//      grid barrier; while the others arrive, each of kPermRankWarps warps counts
//      its contiguous piece of the chunk, and per expert the pieces' counts
//      become exclusive prefixes over the pieces.
//   2. After the barrier, warp w of CTA c takes experts e = w G + c, ...: its
//      lanes split the G chunks into contiguous runs, and the warp turns column
//      e of the table into exclusive prefixes over the chunks (in place) with the
//      expert's total in row G.  Second barrier.
//   3. Every CTA scans the totals (and the experts' tile counts) into expert
//      offsets (and first tiles); CTA c writes the offsets and tiles of experts
//      c, c + G, ...  Then each of the kPermRankWarps warps places its piece in
//      order: row r of expert e goes to offset[e] + rows of e in earlier chunks +
//      rows of e in earlier pieces + rows of e before r in the piece (peer masks).
// A chunk too large to stage in shared memory (STAGED false) is read from global
// memory both times.
template <bool STAGED>
__global__ void __launch_bounds__(kPermWarps * 32, 1)
    grid_permute_kernel(const int32_t* __restrict__ ids, int R, int E, int S,
                        int32_t* __restrict__ offsets, int32_t* __restrict__ rows_out,
                        PermuteAux aux)
{
    extern __shared__ int smem[];
    __shared__ int2 sums2[32];
    __shared__ int go;
    int* table = smem;                      // [kPermRankWarps][E]
    int* hist = smem + kPermRankWarps * E;  // [E]: the chunk's counts, later its bases
    int* ids_s = smem + ((kPermRankWarps * E + E + 3) & ~3);  // [S] when STAGED (16-byte aligned)
    const int G = gridDim.x, c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    GridBar* bar = aux.bar;
    int32_t* counts = aux.chunk_counts;
    const unsigned long long gen = aux.gen;
    pdl_wait();
    pdl_launch_dependents();
    if (c == 0 && threadIdx.x == 0) {  // this call's barrier count starts at 0
        bar->count = 0;
        __threadfence();
        st_release_gpu_u64(&bar->gen, gen);
    }
    const int c0 = c * S, n = min(S, R - c0);
    for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
    for (int i = threadIdx.x; i < kPermRankWarps * E / 4; i += blockDim.x)
        reinterpret_cast<int4*>(table)[i] = make_int4(0, 0, 0, 0);
    if (STAGED) {
        // 16-byte loads, all in flight before any store (c0 is a multiple of 32,
        // so ids + c0 keeps the 16-byte alignment of ids)
        constexpr int kVec = kPermStageRows / 4 / (kPermWarps * 32);
        const int4* src = reinterpret_cast<const int4*>(ids + c0);
        int4 v[kVec];
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const int i = (threadIdx.x + j * kPermWarps * 32) * 4;
            v[j] = i + 3 < n ? src[i / 4] : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const int i = (threadIdx.x + j * kPermWarps * 32) * 4;
            if (i + 3 < n) reinterpret_cast<int4*>(ids_s)[i / 4] = v[j];
        }
        const int tail = n & ~3;  // the last n % 4 rows
        if (threadIdx.x < n - tail) ids_s[tail + threadIdx.x] = ids[c0 + tail + threadIdx.x];
    }
    __syncthreads();

    // 1. the chunk's counts
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        int id = STAGED ? ids_s[i] : ids[c0 + i];
        if (!debug_in_range(id, 0, E, aux.err)) id = 0;
        if (STAGED) ids_s[i] = id;
        atomicAdd(&hist[id], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) counts[(size_t)c * E + i] = hist[i];
    __syncthreads();
    if (threadIdx.x == 0) {
        go = grid_wait(bar, gen, aux.err,
                       [&] { return ld_acquire_gpu_u64(&bar->gen) == gen; });
        if (go) red_release_gpu_add(reinterpret_cast<int*>(&bar->count), 1);
    }
    // the pieces' counts while the other CTAs arrive
    const int nbits = expert_bits(E);
    const int per = (n + kPermRankWarps - 1) / kPermRankWarps;
    const int r0 = min(n, warp * per), r1 = warp < kPermRankWarps ? min(n, r0 + per) : r0;
    if (STAGED)
        warp_count(StagedIds{ids_s}, r0, r1, table + warp * E, nbits);
    else
        warp_count(GlobalIds{ids + c0, E, aux.err}, r0, r1, table + warp * E, nbits);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int v[kPermRankWarps];
#pragma unroll
        for (int w = 0; w < kPermRankWarps; ++w) v[w] = table[w * E + e];
        int run = 0;
#pragma unroll
        for (int w = 0; w < kPermRankWarps; ++w) {
            table[w * E + e] = run;
            run += v[w];
        }
    }
    if (threadIdx.x == 0 && go)
        go = grid_wait(bar, gen, aux.err, [&] {
            return (uint32_t)ld_acquire_gpu(reinterpret_cast<const int*>(&bar->count)) >= (uint32_t)G;
        });
    __syncthreads();
    if (!go) return;

    // 2. per expert: exclusive prefixes over the chunks, and the total
    {
        const int L = (G + 31) / 32;
        const int cb = min(G, lane * L), ce = min(G, cb + L);
        for (int e = warp * G + c; e < E; e += kPermWarps * G) {
            int v[kPermLaneChunks];
#pragma unroll
            for (int i = 0; i < kPermLaneChunks; ++i)  // all loads in flight at once
                v[i] = __ldcg(counts + (size_t)min(cb + i, G - 1) * E + e);
            int sum = 0;
#pragma unroll
            for (int i = 0; i < kPermLaneChunks; ++i) {
                if (cb + i >= ce) v[i] = 0;
                sum += v[i];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += t;
            }
            int run = incl - sum;
#pragma unroll
            for (int i = 0; i < kPermLaneChunks; ++i)
                if (cb + i < ce) {
                    counts[(size_t)(cb + i) * E + e] = run;
                    run += v[i];
                }
            if (lane == 31) counts[(size_t)G * E + e] = incl;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        red_release_gpu_add(reinterpret_cast<int*>(&bar->count), 1);
        go = grid_wait(bar, gen, aux.err, [&] {
            return (uint32_t)ld_acquire_gpu(reinterpret_cast<const int*>(&bar->count)) >=
                   2u * (uint32_t)G;
        });
    }
    __syncthreads();
    if (!go) return;

    // 3. offsets and tiles, the chunk's bases, the placement
    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    const int total_e = owns ? __ldcg(counts + (size_t)G * E + e) : 0;
    const int pre_e = owns ? __ldcg(counts + (size_t)c * E + e) : 0;
    int q = 0;
    const int nt_e = owns ? expert_tile_count(total_e, aux.nt, q) : 0;
    int2 tot;
    const int2 ex = block_exclusive_scan2(make_int2(total_e, nt_e), sums2, tot);  // ends with a barrier
    if (owns) {
        hist[e] = ex.x + pre_e;
        if (e % G == c) {  // this CTA publishes expert e
            offsets[e] = ex.x;
            write_expert_tiles(e, total_e, ex.x, nt_e, q, ex.y, aux);
        }
    }
    if (c == 0 && threadIdx.x == 0) {
        offsets[E] = tot.x;
        *aux.num_tiles = kDebugChecks ? min(tot.y, aux.max_tiles) : tot.y;
    }
    __syncthreads();
    if (STAGED) {
        warp_scatter(StagedIds{ids_s}, r0, r1, c0, hist, table + warp * E, rows_out, nbits);
    } else {
        warp_scatter(GlobalIds{ids + c0, E, aux.err}, r0, r1, c0, hist, table + warp * E,
                     rows_out, nbits);
    }
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

cudaError_t launch_large_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                                 int32_t* rows, const PermuteAux& aux, cudaStream_t st)
{
    const long long R = (long long)T * k;
    int gmax = device_sms();
    if (gmax > aux.max_chunks) gmax = aux.max_chunks;
    if (gmax > kPermMaxChunks) gmax = kPermMaxChunks;
    if (gmax < 1) return cudaErrorInvalidValue;
    // rows per chunk: a multiple of 32, and as few chunks as that leaves
    const long long S = (((R + gmax - 1) / gmax) + 31) & ~31LL;
    const int G = (int)((R + S - 1) / S);
    const bool staged = S <= kPermStageRows;
    const size_t smem =
        sizeof(int) * ((((size_t)kPermRankWarps * E + E + 3) & ~(size_t)3) + (staged ? (size_t)S : 0));
    auto go = [&](auto kern) {
        cudaError_t err =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        return launch(kern, dim3(G), dim3(kPermWarps * 32), smem, st, ids, (int)R, E, (int)S,
                      offsets, rows, aux);
    };
    return staged ? go(grid_permute_kernel<true>) : go(grid_permute_kernel<false>);
}

cudaError_t launch_build_tiles(const int32_t* offsets, int E, int R, const PermuteAux& aux,
                               cudaStream_t st)
{
    return launch(build_tiles_kernel, dim3(1), dim3(1024), 0, st, offsets, E, R, aux);
}

}  // namespace moe
