// combine.cu -- the HBM-bound element-wise stages around the grouped GEMMs.
//
//   combine          out[t] = sum_{j=0..k-1} w[t, j] * y[t*k + j], fp32, j ascending,
//                    rounded once to bf16 (the fixed-order fp32 merge principle of the
//                    "FP32 partials" section of the FlashInfer PR #5586 page, applied
//                    to the top-k combine).
//   swiglu finalize  act[p, f] = bf16(silu(sum_s gate_s) * sum_s up_s) for a split w13.
//   reduce y         y[r, h] = bf16(sum_s partial_s[r, h]) for a split w2 whose y is
//                    wanted on its own (moe_grouped_ffn).
//   combine from partials   the two above in one kernel, for moe_forward.
//
// Each thread moves 16-byte vectors and issues all of its loads before using any
// (these kernels are short and latency-bound at decode sizes); the split count
// is read on the device.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gemm_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

using gemm::silu_mul;  // the GEMM epilogue's SwiGLU, bit for bit

constexpr int kMaxK = 16;
constexpr int kMaxSplits = 8;

// One thread per (token, 8 hidden elements): the k rows are all loaded before
// any is used, so a thread keeps up to 16 loads in flight.
template <int KMAX>
__global__ void __launch_bounds__(256)
    combine_kernel(const uint4* __restrict__ y, const float* __restrict__ w, int T, int k, int H8,
                   uint4* __restrict__ out)
{
    pdl_launch_dependents();  // dependents wait for this grid's completion themselves
    pdl_wait();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)T * H8) return;
    const int t = (int)(idx / H8), h8 = (int)(idx % H8);
    uint4 v[KMAX];
    float wj[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
            const long r = (long)t * k + j;
            v[j] = __ldcs(y + r * H8 + h8);  // read once: stream
            wj[j] = __ldg(w + r);
        }
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {  // j ascending: the fixed summation order
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(p[i]);
                acc[2 * i] = fmaf(wj[j], f.x, acc[2 * i]);
                acc[2 * i + 1] = fmaf(wj[j], f.y, acc[2 * i + 1]);
            }
        }
    }
    uint4 o;
    __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    out[idx] = o;
}

// Combine straight from w2's split-K partials.  Block = one token t and 256
// consecutive hidden elements, 64 threads per selected expert j: thread (j, c)
// rebuilds 4 elements of y[t*k + j] as bf16(sum_s partial_s), every slice's load
// in flight (or reads them from y when w2 ran unsplit); then, per element, the
// k rows are accumulated in j order with the same fma chain as combine_kernel.
// The result is bit-identical to reduce_y followed by combine_kernel.
__global__ void __launch_bounds__(1024)
    combine_partials_kernel(const float4* __restrict__ partials, const int32_t* __restrict__ splits,
                            const uint2* __restrict__ y, const float* __restrict__ w, int T,
                            int k, int H4, uint2* __restrict__ out)
{
    __shared__ float4 yrow[kMaxK][64];
    __shared__ float wrow[kMaxK];
    pdl_launch_dependents();
    pdl_wait();
    const int S = *splits;
    const int t = blockIdx.x;
    const int c = threadIdx.x & 63, j = threadIdx.x >> 6;  // blockDim = 64 * k
    const int h4 = blockIdx.y * 64 + c;
    const long R = (long)T * k;
    const long r = (long)t * k + j;
    if (c == 0) wrow[j] = __ldg(w + r);
    if (h4 < H4) {
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (S > 1) {
            float4 pv[kMaxSplits];
#pragma unroll
            for (int s = 0; s < kMaxSplits; ++s)
                if (s < S) pv[s] = __ldcs(partials + ((size_t)s * R + r) * H4 + h4);
#pragma unroll
            for (int s = 0; s < kMaxSplits; ++s) {  // slice order
                if (s < S) {
                    a[0] += pv[s].x; a[1] += pv[s].y; a[2] += pv[s].z; a[3] += pv[s].w;
                }
            }
            a[0] = __bfloat162float(__float2bfloat16_rn(a[0]));
            a[1] = __bfloat162float(__float2bfloat16_rn(a[1]));
            a[2] = __bfloat162float(__float2bfloat16_rn(a[2]));
            a[3] = __bfloat162float(__float2bfloat16_rn(a[3]));
        } else {
            const uint2 v = __ldcs(y + r * H4 + h4);
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
            const float2 f0 = __bfloat1622float2(p[0]), f1 = __bfloat1622float2(p[1]);
            a[0] = f0.x; a[1] = f0.y; a[2] = f1.x; a[3] = f1.y;
        }
        yrow[j][c] = make_float4(a[0], a[1], a[2], a[3]);
    }
    __syncthreads();
    if (j == 0 && h4 < H4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int jj = 0; jj < k; ++jj) {  // j ascending: the fixed summation order
            const float4 v = yrow[jj][c];
            const float wj = wrow[jj];
            acc[0] = fmaf(wj, v.x, acc[0]);
            acc[1] = fmaf(wj, v.y, acc[1]);
            acc[2] = fmaf(wj, v.z, acc[2]);
            acc[3] = fmaf(wj, v.w, acc[3]);
        }
        uint2 o;
        __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
        q[0] = __floats2bfloat162_rn(acc[0], acc[1]);
        q[1] = __floats2bfloat162_rn(acc[2], acc[3]);
        out[(size_t)t * H4 + h4] = o;
    }
}

// partials: [S, R, 2I] fp32 (gate columns [0, I), up columns [I, 2I)); 4 features per thread
__global__ void __launch_bounds__(256)
    swiglu_finalize_kernel(const float4* __restrict__ partials, const int32_t* __restrict__ splits,
                           int R, int I4, uint2* __restrict__ act)
{
    pdl_launch_dependents();  // dependents wait for this grid's completion themselves
    pdl_wait();
    const int S = *splits;
    if (S <= 1) return;  // the GEMM wrote act itself
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)R * I4) return;
    const long p = idx / I4;
    const int f4 = (int)(idx % I4);
    float4 pa[kMaxSplits], pb[kMaxSplits];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {  // every slice's loads in flight at once
        if (s < S) {
            const float4* row = partials + ((size_t)s * R + p) * (2 * I4);
            pa[s] = __ldcs(row + f4);
            pb[s] = __ldcs(row + I4 + f4);
        }
    }
    float g[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {  // slice order
        if (s < S) {
            g[0] += pa[s].x; g[1] += pa[s].y; g[2] += pa[s].z; g[3] += pa[s].w;
            u[0] += pb[s].x; u[1] += pb[s].y; u[2] += pb[s].z; u[3] += pb[s].w;
        }
    }
    uint2 o;
    __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
    q[0] = __floats2bfloat162_rn(silu_mul(g[0], u[0]), silu_mul(g[1], u[1]));
    q[1] = __floats2bfloat162_rn(silu_mul(g[2], u[2]), silu_mul(g[3], u[3]));
    act[idx] = o;
}

// partials: [S, R, H] fp32 by expanded id; 4 elements per thread
__global__ void __launch_bounds__(256)
    reduce_y_kernel(const float4* __restrict__ partials, const int32_t* __restrict__ splits,
                    int R, int H4, uint2* __restrict__ y)
{
    pdl_launch_dependents();  // dependents wait for this grid's completion themselves
    pdl_wait();
    const int S = *splits;
    if (S <= 1) return;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)R * H4) return;
    float4 pv[kMaxSplits];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s)
        if (s < S) pv[s] = __ldcs(partials + (size_t)s * R * H4 + idx);
    float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {  // slice order
        if (s < S) {
            a[0] += pv[s].x; a[1] += pv[s].y; a[2] += pv[s].z; a[3] += pv[s].w;
        }
    }
    uint2 o;
    __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
    q[0] = __floats2bfloat162_rn(a[0], a[1]);
    q[1] = __floats2bfloat162_rn(a[2], a[3]);
    y[idx] = o;
}

template <typename Kern, typename... Args>
cudaError_t launch_1d(Kern kern, long n, cudaStream_t st, Args... args)
{
    return launch_pdl(kern, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, args...);
}

}  // namespace

cudaError_t launch_combine(const void* y, const float* weights, int T, int k, int H, void* out,
                           cudaStream_t st)
{
    const int H8 = H / 8;
    // the k rows' loads are unrolled up to a bound: registers for 16 rows would
    // halve the resident threads at k = 8
    auto go = [&](auto kern) {
        return launch_1d(kern, (long)T * H8, st, static_cast<const uint4*>(y), weights, T, k, H8,
                         static_cast<uint4*>(out));
    };
    if (k <= 2) return go(combine_kernel<2>);
    if (k <= 4) return go(combine_kernel<4>);
    if (k <= 8) return go(combine_kernel<8>);
    return go(combine_kernel<kMaxK>);
}

cudaError_t launch_combine_partials(const float* partials, const int32_t* splits, const void* y,
                                   const float* weights, int T, int k, int H, void* out,
                                   cudaStream_t st)
{
    if (T == 0) return cudaSuccess;
    const int H4 = H / 4;
    return launch_pdl(combine_partials_kernel, dim3((unsigned)T, (unsigned)((H4 + 63) / 64)),
                      dim3((unsigned)(64 * k)), 0, st, reinterpret_cast<const float4*>(partials),
                      splits, static_cast<const uint2*>(y), weights, T, k, H4,
                      static_cast<uint2*>(out));
}

cudaError_t launch_swiglu_finalize(const float* partials, const int32_t* splits, int R, int I,
                                   void* act, cudaStream_t st)
{
    const int I4 = I / 4;
    return launch_1d(swiglu_finalize_kernel, (long)R * I4, st,
                     reinterpret_cast<const float4*>(partials), splits, R, I4,
                     static_cast<uint2*>(act));
}

cudaError_t launch_reduce_y(const float* partials, const int32_t* splits, int R, int H, void* y,
                            cudaStream_t st)
{
    const int H4 = H / 4;
    return launch_1d(reduce_y_kernel, (long)R * H4, st, reinterpret_cast<const float4*>(partials),
                     splits, R, H4, static_cast<uint2*>(y));
}

}  // namespace moe
