// route_permute.cu -- top-k routing of fp32 router logits and the stable
// per-expert permutation of the expanded rows.
//
// Routing ("softmax_sum", FlashInfer PR #3751 page "Optimizing TRTLLM-Gen MoE
// routing", sections "1. dynamic thread-block size" and "performance numbers"):
// one warp owns one token; each lane keeps E/32 logits in registers, the k
// winners are taken one by one with a warp arg-max over (logit desc, expert asc)
// keys, and the k weights are a softmax over the selected logits, summed in
// selection order.  The pages size the routing CTA by token count to keep
// register pressure down; here the register footprint is fixed by the
// per-lane value count V (a template), and the grid scales with T.
//
// Permutation: count -> exclusive scan -> stable scatter.  Ranks inside a warp
// come from __match_any_sync peer masks, ranks across warps from a per-warp
// count table and a column scan, ranks across CTAs from a per-chunk count table
// scanned by one CTA, so the result (ascending expanded id inside every expert)
// never depends on atomic ordering.  No kernel waits on another CTA.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kNoIndex = 0x7fffffff;

// (va, ia) ranks before (vb, ib)?
__device__ __forceinline__ bool key_before(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// Routes one token with the calling warp.  row: E logits.  Writes ids/weights
// (k each) to global memory and, if ids_s != nullptr, the ids to shared memory.
template <int V>
__device__ __forceinline__ void warp_route_token(const float* __restrict__ row, int E, int k,
                                                 int lane, int32_t* __restrict__ ids,
                                                 float* __restrict__ weights, int* ids_s)
{
    float v[V];
#pragma unroll
    for (int m = 0; m < V; ++m) {
        const int e = m * 32 + lane;
        v[m] = (e < E) ? __ldg(row + e) : -INFINITY;
    }
    uint32_t taken = 0;

    // best not-yet-taken value of this lane; m ascending = expert ascending, so a
    // strict '>' keeps the lower expert on equal values
    auto lane_best = [&](float& bv, int& bi) {
        bv = -INFINITY;
        bi = kNoIndex;
#pragma unroll
        for (int m = 0; m < V; ++m) {
            const int e = m * 32 + lane;
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
    float my_l = 0.f;
    int my_id = 0;
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
        if ((wi & 31) == lane) {  // the owner drops the winner and finds its next best
            taken |= 1u << (wi >> 5);
            lane_best(bv, bi);
        }
    }
    // softmax over the selected logits; l_0 is the largest
    const float l0 = __shfl_sync(kFull, my_l, 0);
    const float ex = (lane < k) ? expf(my_l - l0) : 0.f;
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(kFull, ex, j);  // fixed order j = 0..k-1
    if (lane < k) {
        ids[lane] = my_id;
        weights[lane] = ex / sum;
        if (ids_s) ids_s[lane] = my_id;
    }
}

// Exclusive scan of one int per thread over the whole CTA (blockDim.x a
// multiple of 32, <= 1024).  `sums` is shared scratch of 32 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sums, int& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += n;
    }
    if (lane == 31) sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = (lane < nw) ? sums[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(kFull, s, off);
            if (lane >= off) s += n;
        }
        sums[lane] = s;
    }
    __syncthreads();
    const int prefix = (warp > 0) ? sums[warp - 1] : 0;
    total = sums[nw - 1];
    __syncthreads();
    return prefix + incl - v;
}

// Thread e (< E) owns expert e with `count` rows at permuted offset `off` and
// writes its tiles: as few as ceil(count / nt) allows, of near-equal size rounded
// to the MMA's 16-column granule (so no tile is a short tail that streams a whole
// weight block for a few rows), the last one taking the remainder.
// Also zeroes the split-K counters.
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
    for (int i = threadIdx.x; i < aux.n_counters; i += blockDim.x) aux.counters[i] = 0;
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

template <int V>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E,
                                                    int k, int32_t* __restrict__ ids,
                                                    float* __restrict__ weights)
{
    pdl_wait();
    pdl_launch_dependents();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    warp_route_token<V>(logits + (size_t)t * E, E, k, threadIdx.x & 31, ids + (size_t)t * k,
                        weights + (size_t)t * k, nullptr);
}

// One CTA: (route) + count + scan + stable scatter + tile list, for T*k <= kSmallRows.
template <int V>
__global__ void __launch_bounds__(1024, 1)
    small_route_permute_kernel(const float* __restrict__ logits, int T, int E, int k,
                               int32_t* __restrict__ ids, float* __restrict__ weights,
                               int32_t* __restrict__ offsets, int32_t* __restrict__ rows_out,
                               PermuteAux aux)
{
    extern __shared__ int smem[];
    __shared__ int sums[32];
    const int R = T * k;
    int* ids_s = smem;
    int* table = smem + ((R + 3) & ~3);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    pdl_wait();
    pdl_launch_dependents();

    if (logits) {
        for (int t = warp; t < T; t += 32)
            warp_route_token<V>(logits + (size_t)t * E, E, k, lane, ids + (size_t)t * k,
                                weights + (size_t)t * k, ids_s + t * k);
    } else {
        for (int r = threadIdx.x; r < R; r += blockDim.x) ids_s[r] = ids[r];
    }
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) table[i] = 0;
    __syncthreads();

    const int per_warp = (R + 31) / 32;
    const int r0 = min(R, warp * per_warp), r1 = min(R, r0 + per_warp);
    warp_count(ids_s, r0, r1, table + warp * E);
    __syncthreads();

    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    int cnt = 0;
    if (owns)
        for (int w = 0; w < 32; ++w) {
            const int c = table[w * E + e];
            table[w * E + e] = cnt;
            cnt += c;
        }
    int total;
    const int off = block_exclusive_scan(owns ? cnt : 0, sums, total);
    if (owns) {
        offsets[e] = off;
        for (int w = 0; w < 32; ++w) table[w * E + e] += off;
    }
    if (threadIdx.x == 0) offsets[E] = total;
    write_tiles_and_reset(owns, e, cnt, off, aux, sums);
    __syncthreads();

    warp_scatter(ids_s, r0, r1, 0, table + warp * E, rows_out);
}

__global__ void __launch_bounds__(1024) chunk_count_kernel(const int32_t* __restrict__ ids, int R,
                                                           int E, int32_t* __restrict__ counts)
{
    extern __shared__ int hist[];
    pdl_wait();
    pdl_launch_dependents();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int r0 = blockIdx.x * kChunkRows, r1 = min(R, r0 + kChunkRows);
    for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) atomicAdd(&hist[ids[r]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// counts[c][e] -> absolute position of chunk c's first row of expert e.
__global__ void __launch_bounds__(1024) chunk_scan_kernel(int32_t* __restrict__ counts,
                                                          int n_chunks, int E, int32_t* offsets,
                                                          PermuteAux aux)
{
    __shared__ int sums[32];
    pdl_wait();
    pdl_launch_dependents();
    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    int cnt = 0;
    if (owns)
        for (int c = 0; c < n_chunks; ++c) {
            const int v = counts[(size_t)c * E + e];
            counts[(size_t)c * E + e] = cnt;
            cnt += v;
        }
    int total;
    const int off = block_exclusive_scan(owns ? cnt : 0, sums, total);
    if (owns) {
        offsets[e] = off;
        for (int c = 0; c < n_chunks; ++c) counts[(size_t)c * E + e] += off;
    }
    if (threadIdx.x == 0) offsets[E] = total;
    write_tiles_and_reset(owns, e, cnt, off, aux, sums);
}

__global__ void __launch_bounds__(1024, 1)
    chunk_scatter_kernel(const int32_t* __restrict__ ids, int R, int E,
                         const int32_t* __restrict__ base, int32_t* __restrict__ rows_out)
{
    extern __shared__ int smem[];
    int* ids_s = smem;                 // kChunkRows
    int* table = smem + kChunkRows;    // [32][E]
    const int warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_launch_dependents();
    const int c0 = blockIdx.x * kChunkRows, n = min(kChunkRows, R - c0);
    for (int i = threadIdx.x; i < n; i += blockDim.x) ids_s[i] = ids[c0 + i];
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) table[i] = 0;
    __syncthreads();
    constexpr int per_warp = kChunkRows / 32;
    const int r0 = min(n, warp * per_warp), r1 = min(n, r0 + per_warp);
    warp_count(ids_s, r0, r1, table + warp * E);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = base[(size_t)blockIdx.x * E + e];
        for (int w = 0; w < 32; ++w) {
            const int v = table[w * E + e];
            table[w * E + e] = run;
            run += v;
        }
    }
    __syncthreads();
    warp_scatter(ids_s, r0, r1, c0, table + warp * E, rows_out);
}

__global__ void __launch_bounds__(1024) build_tiles_kernel(const int32_t* __restrict__ offsets,
                                                           int E, PermuteAux aux)
{
    __shared__ int sums[32];
    pdl_wait();
    pdl_launch_dependents();
    const bool owns = threadIdx.x < E;
    const int e = threadIdx.x;
    const int off = owns ? offsets[e] : 0;
    const int cnt = owns ? offsets[e + 1] - off : 0;
    write_tiles_and_reset(owns, e, cnt, off, aux, sums);
}

template <typename Kern, typename... Args>
cudaError_t launch(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args)
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

int values_per_lane(int E)
{
    const int v = (E + 31) / 32;
    return v <= 1 ? 1 : v <= 2 ? 2 : v <= 4 ? 4 : v <= 8 ? 8 : v <= 16 ? 16 : 32;
}

}  // namespace

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* weights,
                         cudaStream_t st)
{
    const dim3 grid((T + 7) / 8), block(256);
    switch (values_per_lane(E)) {
    case 1: return launch(route_kernel<1>, grid, block, 0, st, logits, T, E, k, ids, weights);
    case 2: return launch(route_kernel<2>, grid, block, 0, st, logits, T, E, k, ids, weights);
    case 4: return launch(route_kernel<4>, grid, block, 0, st, logits, T, E, k, ids, weights);
    case 8: return launch(route_kernel<8>, grid, block, 0, st, logits, T, E, k, ids, weights);
    case 16: return launch(route_kernel<16>, grid, block, 0, st, logits, T, E, k, ids, weights);
    default: return launch(route_kernel<32>, grid, block, 0, st, logits, T, E, k, ids, weights);
    }
}

template <int V>
static cudaError_t launch_small_v(const float* logits, int T, int E, int k, int32_t* ids,
                                  float* weights, int32_t* offsets, int32_t* rows,
                                  const PermuteAux& aux, cudaStream_t st)
{
    const int R = T * k;
    const size_t smem = sizeof(int) * (size_t)(((R + 3) & ~3) + 32 * E);
    cudaError_t err = cudaFuncSetAttribute(small_route_permute_kernel<V>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch(small_route_permute_kernel<V>, dim3(1), dim3(1024), smem, st, logits, T, E, k,
                  ids, weights, offsets, rows, aux);
}

cudaError_t launch_small_route_permute(const float* logits, int T, int E, int k, int32_t* ids,
                                       float* weights, int32_t* offsets, int32_t* rows,
                                       const PermuteAux& aux, cudaStream_t st)
{
    switch (logits ? values_per_lane(E) : 1) {
    case 1: return launch_small_v<1>(logits, T, E, k, ids, weights, offsets, rows, aux, st);
    case 2: return launch_small_v<2>(logits, T, E, k, ids, weights, offsets, rows, aux, st);
    case 4: return launch_small_v<4>(logits, T, E, k, ids, weights, offsets, rows, aux, st);
    case 8: return launch_small_v<8>(logits, T, E, k, ids, weights, offsets, rows, aux, st);
    case 16: return launch_small_v<16>(logits, T, E, k, ids, weights, offsets, rows, aux, st);
    default: return launch_small_v<32>(logits, T, E, k, ids, weights, offsets, rows, aux, st);
    }
}

size_t large_permute_smem(int E) { return sizeof(int) * (size_t)(kChunkRows + 32 * E); }

cudaError_t launch_large_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                                 int32_t* rows, const PermuteAux& aux, cudaStream_t st)
{
    const int R = T * k;
    const int n_chunks = (R + kChunkRows - 1) / kChunkRows;
    cudaError_t err = launch(chunk_count_kernel, dim3(n_chunks), dim3(1024), sizeof(int) * E, st,
                             ids, R, E, aux.chunk_counts);
    if (err != cudaSuccess) return err;
    err = launch(chunk_scan_kernel, dim3(1), dim3(1024), 0, st, aux.chunk_counts, n_chunks, E,
                 offsets, aux);
    if (err != cudaSuccess) return err;
    const size_t smem = large_permute_smem(E);
    err = cudaFuncSetAttribute(chunk_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (err != cudaSuccess) return err;
    return launch(chunk_scatter_kernel, dim3(n_chunks), dim3(1024), smem, st, ids, R, E,
                  (const int32_t*)aux.chunk_counts, rows);
}

cudaError_t launch_build_tiles(const int32_t* offsets, int E, const PermuteAux& aux,
                               cudaStream_t st)
{
    return launch(build_tiles_kernel, dim3(1), dim3(1024), 0, st, offsets, E, aux);
}

}  // namespace moe
