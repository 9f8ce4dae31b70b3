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

}  // namespace moe
