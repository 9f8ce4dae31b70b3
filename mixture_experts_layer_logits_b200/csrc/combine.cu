// combine.cu -- the HBM-bound element-wise stages around the grouped GEMMs.
//
//   combine          out[t] = sum_{j=0..k-1} w[t, j] * y[t*k + j], fp32, j ascending,
//                    rounded once to bf16 (the fixed-order fp32 merge principle of the
//                    "FP32 partials" section of the FlashInfer PR #5586 page, applied
//                    to the top-k combine).  When the w2 GEMM ran split-K, y[r] is
//                    first rebuilt as bf16(sum_s partial_s[r]) in slice order, so the
//                    result is the same as combining a materialised y.
//   swiglu finalize  act[p, f] = bf16(silu(sum_s gate_s) * sum_s up_s) for a split w13.
//   reduce y         y[r, h] = bf16(sum_s partial_s[r, h]) for a split w2 whose y is
//                    wanted on its own (moe_grouped_ffn).
//
// Each thread moves 16-byte vectors; the split count is read on the device.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

// silu(g) * u with the same fast exponential and reciprocal as the GEMM epilogue
// (the product is rounded to bf16).
__device__ __forceinline__ float silu_mul(float g, float u)
{
    return g * __frcp_rn(1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ void add4(float (&a)[8], int o, float4 v)
{
    a[o] += v.x;
    a[o + 1] += v.y;
    a[o + 2] += v.z;
    a[o + 3] += v.w;
}

__global__ void __launch_bounds__(256)
    combine_kernel(const uint4* __restrict__ y, const float4* __restrict__ partials,
                   const int32_t* __restrict__ splits, const float* __restrict__ w, int T, int k,
                   int H8, uint4* __restrict__ out)
{
    pdl_wait();
    pdl_launch_dependents();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)T * H8) return;
    const int S = splits ? *splits : 1;
    const int t = (int)(idx / H8), h8 = (int)(idx % H8);
    const long R = (long)T * k;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
        const long r = (long)t * k + j;
        const float wj = __ldg(w + r);
        float yv[8];
        if (S > 1) {
            float s8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) s8[i] = 0.f;
            for (int s = 0; s < S; ++s) {  // slice order
                const float4* pr = partials + ((size_t)s * R + r) * (H8 * 2) + h8 * 2;
                add4(s8, 0, __ldcs(pr));
                add4(s8, 4, __ldcs(pr + 1));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) yv[i] = __bfloat162float(__float2bfloat16_rn(s8[i]));
        } else {
            const uint4 v = __ldcs(y + r * H8 + h8);  // read once: stream (the j loop is
                                                     // unrolled so the k loads overlap)
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(p[i]);
                yv[2 * i] = f.x;
                yv[2 * i + 1] = f.y;
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, yv[i], acc[i]);
    }
    uint4 o;
    __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    out[idx] = o;
}

// partials: [S, R, 2I] fp32 (gate columns [0, I), up columns [I, 2I)); 4 features per thread
__global__ void __launch_bounds__(256)
    swiglu_finalize_kernel(const float4* __restrict__ partials, const int32_t* __restrict__ splits,
                           int R, int I4, uint2* __restrict__ act)
{
    pdl_wait();
    pdl_launch_dependents();
    const int S = *splits;
    if (S <= 1) return;  // the GEMM wrote act itself
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)R * I4) return;
    const long p = idx / I4;
    const int f4 = (int)(idx % I4);
    float g[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
        const float4* row = partials + ((size_t)s * R + p) * (2 * I4);
        const float4 a = __ldcs(row + f4), b = __ldcs(row + I4 + f4);
        g[0] += a.x; g[1] += a.y; g[2] += a.z; g[3] += a.w;
        u[0] += b.x; u[1] += b.y; u[2] += b.z; u[3] += b.w;
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
    pdl_wait();
    pdl_launch_dependents();
    const int S = *splits;
    if (S <= 1) return;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)R * H4) return;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
        const float4 v = __ldcs(partials + (size_t)s * R * H4 + idx);
        a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

cudaError_t launch_combine(const void* y, const float* partials, const int32_t* splits,
                           const float* weights, int T, int k, int H, void* out, cudaStream_t st)
{
    const int H8 = H / 8;
    return launch_1d(combine_kernel, (long)T * H8, st, static_cast<const uint4*>(y),
                     reinterpret_cast<const float4*>(partials), splits, weights, T, k, H8,
                     static_cast<uint4*>(out));
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
