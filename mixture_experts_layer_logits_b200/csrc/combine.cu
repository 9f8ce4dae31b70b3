// combine.cu -- out[t] = sum_{j=0..k-1} w[t, j] * y[t*k + j], fp32, j ascending,
// rounded once to bf16 (the fixed-order fp32 merge principle of the "FP32
// partials" section of the FlashInfer PR #5586 page, applied to the top-k
// combine).  HBM-bound: each thread owns 8 consecutive hidden elements of one
// token and moves them with 16-byte loads/stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y,
                                                      const float* __restrict__ w, int T, int k,
                                                      int H8, uint4* __restrict__ out)
{
    pdl_wait();
    pdl_launch_dependents();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)T * H8) return;
    const int t = (int)(idx / H8), h8 = (int)(idx % H8);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < k; ++j) {
        const float wj = __ldg(w + (size_t)t * k + j);
        const uint4 v = __ldcs(y + ((size_t)t * k + j) * H8 + h8);  // read once: stream
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            acc[2 * i] = fmaf(wj, f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj, f.y, acc[2 * i + 1]);
        }
    }
    uint4 o;
    __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    out[idx] = o;
}

}  // namespace

cudaError_t launch_combine(const void* y, const float* weights, int T, int k, int H, void* out,
                           cudaStream_t st)
{
    const int H8 = H / 8;
    const long n = (long)T * H8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel, static_cast<const uint4*>(y), weights, T, k,
                              H8, static_cast<uint4*>(out));
}

}  // namespace moe
