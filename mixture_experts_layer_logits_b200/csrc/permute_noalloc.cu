// permute_noalloc.cu -- moe_permute_noalloc: the stable per-expert permutation
// without a caller-supplied workspace, for callers that cannot allocate device
// memory.
//
// The scratch the permutation kernels need (the per-chunk expert count table and
// the grid barrier of the multi-CTA path, and the per-expert tile list they also
// emit) lives in one file-scope device array of fixed size.  Host code cannot use the array's name
// as a device address, so its address is looked up with cudaGetSymbolAddress
// once per device, with that device current, and handed to the kernels like any
// other pointer.  Nothing here allocates.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"
#include "moe.h"

namespace moe {
namespace {

// chunk count table for up to 256 chunks (the multi-CTA path's grid bound) x 1024
// experts plus its row of expert totals, then up to 1024 tiles (one per expert),
// then a 256-byte tail: the tile count at +0, the error word at +16, the grid
// barrier at +64
constexpr int kMaxChunks = 256;
constexpr size_t kCountBytes = (size_t)(kMaxChunks + 1) * 1024 * sizeof(int32_t);
constexpr size_t kTileBytes = 1024 * sizeof(Tile);
constexpr size_t kScratchBytes = kCountBytes + kTileBytes + 256;
static_assert(64 + sizeof(GridBar) <= 256, "tail layout");
static_assert(kScratchBytes == MOE_PERMUTE_NOALLOC_SCRATCH_BYTES, "header and file disagree");

static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_permute_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_ids, moe_shape_t s,
                                            int32_t* expert_offsets, int32_t* permuted_rows,
                                            moe_stream_t stream)
{
    using namespace moe;
    if (!topk_ids || !expert_offsets || !permuted_rows) return MOE_ERR_INVALID_ARG;
    if (!routing_shape_ok(s)) return MOE_ERR_UNSUPPORTED_SHAPE;  // moe_permute's rules
    const long long R = (long long)s.T * s.top_k;
    if (R > MOE_PERMUTE_NOALLOC_MAX_ROWS) return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(topk_ids) | reinterpret_cast<uintptr_t>(expert_offsets) |
         reinterpret_cast<uintptr_t>(permuted_rows)) & 15u)
        return MOE_ERR_MISALIGNED;

    void* base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e == cudaSuccess) {
        char* p = static_cast<char*>(base);
        PermuteAux aux;
        aux.chunk_counts = reinterpret_cast<int32_t*>(p);
        aux.tiles = reinterpret_cast<Tile*>(p + kCountBytes);
        aux.num_tiles = reinterpret_cast<int32_t*>(p + kCountBytes + kTileBytes);
        // bounded-wait timeouts and debug-build index faults are recorded here
        // (nothing reports them)
        aux.err = reinterpret_cast<int32_t*>(p + kCountBytes + kTileBytes + 16);
        aux.nt = 1 << 30;  // one tile per expert: the tile list stays within 1024 entries
        aux.max_tiles = 1024;
        aux.max_chunks = kMaxChunks;
        aux.bar = reinterpret_cast<GridBar*>(p + kCountBytes + kTileBytes + 64);
        aux.gen = next_generation();
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        int32_t* ids = const_cast<int32_t*>(topk_ids);
        if (R <= kSmallRows)
            e = launch_small_route_permute(nullptr, s.T, s.E, s.top_k, ids, nullptr,
                                           expert_offsets, permuted_rows, aux, st);
        else
            e = launch_large_permute(ids, s.T, s.E, s.top_k, expert_offsets, permuted_rows, aux,
                                     st);
    }
    if (e != cudaSuccess) {
        set_last_cuda_error((int)e);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
