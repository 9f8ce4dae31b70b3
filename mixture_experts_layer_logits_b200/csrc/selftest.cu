// selftest.cu -- failure detection without a GPU fault.
//
// The layer's kernels never wait without a limit: every mbarrier wait and every
// cross-CTA counter wait gives up after a bounded time, records kDeviceErrorMagic
// in the workspace's error word, drains what it issued and returns, so the host
// learns of the failure through moe_device_status while the CUDA context stays
// usable.  This kernel exercises that path on purpose, with the same primitives
// (mbar_wait; acquire loads against globaltimer) and two waits that nothing can
// satisfy, so tests can check the reporting without a fault or a hang.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(64)
    wait_timeout_kernel(int32_t* err, const int32_t* flag, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none ever comes
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    bool gave_up = false;
    if (threadIdx.x == 0) {
        gave_up = !mbar_wait(&bar, 0, &abort_flag, limit_ns);
    } else if (threadIdx.x == 32) {  // a flag that nothing sets
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(flag) < 1) {
            if (globaltimer_ns() - t0 > limit_ns) {
                gave_up = true;
                break;
            }
            __nanosleep(256);
        }
    }
    if (gave_up) atomicExch(err, kDeviceErrorMagic);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(void* ws, unsigned limit_us, cudaStream_t st)
{
    int32_t* err = static_cast<int32_t*>(ws);
    int32_t* flag = err + 1;
    cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    wait_timeout_kernel<<<1, 64, 0, st>>>(err, flag, (uint64_t)limit_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace moe
