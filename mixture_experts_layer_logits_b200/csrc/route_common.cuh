// route_common.cuh -- device pieces shared by the routing kernels
// (route_permute.cu) and the one-launch FFN, which routes its tokens itself
// (fused_ffn.cu): the expert order and the softmax over the selected logits, so
// that both produce the same ids and bit-identical routing weights.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

namespace moe {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kNoIndex = 0x7fffffff;

// (va, ia) ranks before (vb, ib)?  Larger logit first, then the lower expert
// index (-0.0 and +0.0 compare equal, so they tie).
__device__ __forceinline__ bool key_before(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// Sorts one (value, index) key per lane across groups of W lanes (W = 8 or 16:
// each group on its own; W = 32: the warp) so that the group's first lane holds
// the key that ranks first (larger value, then lower index).  Bitonic network with
// the "ranks before" relation as the order; keys must be distinct (they are:
// indices are unique).
template <int W>
__device__ __forceinline__ void warp_sort_keys(float& v, int& i, int lane)
{
#pragma unroll
    for (int size = 2; size <= W; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const float ov = __shfl_xor_sync(kFull, v, stride);
            const int oi = __shfl_xor_sync(kFull, i, stride);
            const bool take_first = ((lane & stride) == 0) == ((lane & size) == 0);
            if (take_first == key_before(ov, oi, v, i)) {
                v = ov;
                i = oi;
            }
        }
    }
}

// Float -> unsigned key with the same order (-0.0 and +0.0 map to one key), and
// back.  Key 0 stands below every non-NaN value.
__device__ __forceinline__ uint32_t ordered_key(float f)
{
    const uint32_t b = __float_as_uint(f + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// The k-th largest (k >= 1, duplicates counted) of the warp's 32 values: at most
// k rounds of a warp max reduction, each removing the lanes that hold the max.
__device__ __forceinline__ float warp_kth_largest(float x, int k)
{
    uint32_t key = ordered_key(x);
    int left = k;
    for (;;) {
        const uint32_t m = __reduce_max_sync(kFull, key);
        left -= __popc(__ballot_sync(kFull, key == m));
        if (left <= 0) return key_value(m);
        if (key == m) key = 0;
    }
}

// Sorts the candidates cand[0 .. total) (total <= 32, distinct experts) by (logit
// desc, expert asc) and leaves the j-th in lane j: (my_l, my_id).
__device__ __forceinline__ void sort_candidates(int total, int lane, const float2* cand,
                                                float& my_l, int& my_id)
{
    float cv = -INFINITY;
    int ci = kNoIndex - lane;  // distinct sentinels rank after every expert
    if (lane < total) {
        const float2 cc = cand[lane];
        cv = cc.x;
        ci = __float_as_int(cc.y);
    }
    __syncwarp();  // cand may be rewritten by this warp's next token
    // usually about k candidates: then lanes 0..7 or 0..15 hold all of them and a
    // network over 8 or 16 lanes (6 or 10 stages instead of 15) orders them the
    // same way
    if (total <= 8)
        warp_sort_keys<8>(cv, ci, lane);
    else if (total <= 16)
        warp_sort_keys<16>(cv, ci, lane);
    else
        warp_sort_keys<32>(cv, ci, lane);
    my_l = cv;
    my_id = ci;
}

// Softmax over the selected logits (lane j holds the j-th; l_0 is the largest)
// and the outputs.  The sum is a fixed xor-tree over lanes 0..15 (lanes >= k
// contribute 0), so it is deterministic.
// The routing weight of lane j's selection (lanes >= k get 0; all 32 lanes call).
__device__ __forceinline__ float softmax_weight(float my_l, int k, int lane)
{
    const float l0 = __shfl_sync(kFull, my_l, 0);
    const float ex = (lane < k) ? expf(my_l - l0) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) sum += __shfl_xor_sync(kFull, sum, off);
    sum = __shfl_sync(kFull, sum, 0);
    return ex / sum;
}

__device__ __forceinline__ void write_selection(float my_l, int my_id, int k, int lane,
                                                int32_t* __restrict__ ids,
                                                float* __restrict__ weights, int* ids_s)
{
    const float w = softmax_weight(my_l, k, lane);
    if (lane < k) {
        if (ids) {
            ids[lane] = my_id;
            weights[lane] = w;
        }
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

// block_exclusive_scan of a pair of ints (both members scanned at once).
// `sums` is shared scratch of 32 int2.
__device__ __forceinline__ int2 block_exclusive_scan2(int2 v, int2* sums, int2& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int2 incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int nx = __shfl_up_sync(kFull, incl.x, off);
        const int ny = __shfl_up_sync(kFull, incl.y, off);
        if (lane >= off) {
            incl.x += nx;
            incl.y += ny;
        }
    }
    if (lane == 31) sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int2 s = (lane < nw) ? sums[lane] : make_int2(0, 0);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int nx = __shfl_up_sync(kFull, s.x, off);
            const int ny = __shfl_up_sync(kFull, s.y, off);
            if (lane >= off) {
                s.x += nx;
                s.y += ny;
            }
        }
        sums[lane] = s;
    }
    __syncthreads();
    const int2 prefix = (warp > 0) ? sums[warp - 1] : make_int2(0, 0);
    total = sums[nw - 1];
    __syncthreads();
    return make_int2(prefix.x + incl.x - v.x, prefix.y + incl.y - v.y);
}

}  // namespace moe
