// grouped_ffn_pair.cu -- the grouped expert FFN for large batches on CTA pairs
// (tcgen05 cta_group::2).
//
// Same layer step as grouped_ffn.cu (gathered w13 + SwiGLU, then w2 with a
// scatter to expanded-id order) for the tensor-bound shapes: 256-token tiles and
// no split-K.  A cluster of two CTAs on neighbouring SMs computes one 256 x 256
// accumulator per unit with one MMA instruction per 16-wide K step issued by
// the first CTA: M = 256 weight rows split 128 / 128 between the two CTAs'
// shared memory, N = the tile's token rows split N/2 / N/2.  Each CTA loads only
// its halves, so a 64-deep K stage is 32 KB per CTA: six stages fit, and each
// CTA's 128 x 256 fp32 accumulator takes 256 TMEM columns, so two are in flight
// (the epilogue of one unit overlaps the main loop of the next).
//
// w13 (MODE 0): CTA r of the pair holds gate rows f0 + 64r .. +64 and the up rows
// of the same features as its 128 A rows, so after the MMA its TMEM lanes 0-63
// are gate and 64-127 are up of the same 64 features; the epilogue pairs them
// through shared memory and writes silu(gate) * up.
// w2 (MODE 1): CTA r holds output rows f0 + 128r .. +128.
//
// Synchronisation across the pair (no multicast loads anywhere):
//   full[s]   lives in CTA 0: CTA 0's producer posts the byte count of both CTAs'
//             TMA loads, both CTAs' loads complete on it (.cta_group::2), and the
//             gather warps of both CTAs arrive on it remotely;
//   empty[s], tfull[b]  in each CTA, signalled by CTA 0's MMA commit to both;
//   tempty[b] lives in CTA 0: the epilogue warps of both CTAs arrive on it.
// Every mbarrier wait is bounded; on a timeout the kernel records the error word,
// stops, drains and frees TMEM.  Both CTAs meet at a cluster barrier before
// freeing TMEM, so neither leaves while the pair's MMAs may still use it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kGatherWarps = 6;   // warps 2..7
constexpr int kEpiWarp0 = 8;      // warps 8..15: two epilogue groups of four
constexpr int kN = 256;           // tokens per tile (pair)
constexpr int kHalf = 128;        // B rows per CTA (at most)
constexpr int kBK = 64;
constexpr int kUmmaK = 16;
constexpr int kATile = 128 * kBK * 2;      // this CTA's 128 A rows
constexpr int kBTile = kHalf * kBK * 2;    // this CTA's B rows
constexpr int kStageBytes = kATile + kBTile;
constexpr int kAccCols = kN;
constexpr int kNBuf = 2;
constexpr int kTmemCols = 512;
constexpr int kStageRows = 8;              // epilogue staging: token rows per chunk
constexpr int kStageRowBytes = 256;        // up to 128 bf16 outputs per row
constexpr int kStagingBytes = 2 * 2 * kStageRows * kStageRowBytes;
constexpr int kXBytes = 2 * 64 * kStageRows * 4;  // MODE 0 gate/up exchange, per group
constexpr int kAuxBytes = 1024 + kGatherWarps * kHalf * 4;
constexpr int kMaxSmem = 232448;
constexpr int kStages =
    (kMaxSmem - 1024 - kStagingBytes - kXBytes - kAuxBytes) / kStageBytes > 8
        ? 8
        : (kMaxSmem - 1024 - kStagingBytes - kXBytes - kAuxBytes) / kStageBytes;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kStagingBytes + kXBytes + kAuxBytes;
constexpr int kG = kGatherWarps < kStages ? kGatherWarps : kStages;  // gather groups
constexpr int kW = kGatherWarps / kG;                                 // warps per group
static_assert(kStages >= 4, "pipeline depth");

struct PairArgs {
    const __nv_bfloat16* x;
    const int32_t* permuted_rows;
    const Tile* tiles;
    const int32_t* num_tiles;
    __nv_bfloat16* out;  // MODE 0: act [R, I]; MODE 1: y [R, H]
    int32_t* err;
    int k, H, I, R;
    int num_kt;
    int fb_count;        // MODE 0: I / 128; MODE 1: ceil(H / 256)
};

struct Aux {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ Tile load_tile(const Tile* p)
{
    const int4 lo = __ldcg(reinterpret_cast<const int4*>(p));
    const int4 hi = __ldcg(reinterpret_cast<const int4*>(p) + 1);
    Tile t;
    t.expert = lo.x;
    t.row_start = lo.y;
    t.rows = lo.z;
    t.first = lo.w;
    t.count = hi.x;
    t.pad[0] = hi.y;
    t.pad[1] = hi.z;
    t.pad[2] = hi.w;
    return t;
}

__device__ __forceinline__ float silu_mul(float g, float u)
{
    return g * __frcp_rn(1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ void named_bar_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                             const __grid_constant__ CUtensorMap tm_act, const PairArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* ring = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* staging = ring + kStages * kStageBytes;
    float* xbuf = reinterpret_cast<float*>(staging + kStagingBytes);
    Aux* aux = reinterpret_cast<Aux*>(reinterpret_cast<uint8_t*>(xbuf) + kXBytes);
    int* tok_off = reinterpret_cast<int*>(aux + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: issues the pair MMAs
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&aux->full[s], MODE == 0 ? 1 + 2 * kW : 1);
            mbar_init(&aux->empty[s], 1);
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(&aux->tfull[b], 1);
            mbar_init(&aux->tempty[b], 16);
        }
        mbar_init(&aux->drain, 1);
        aux->abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_w);
        if (MODE == 1) tma_prefetch_desc(&tm_act);
    }
    if (warp == 1) {
        tmem_alloc_pair(&aux->tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;

    // (programmatic dependent launch: as in grouped_ffn.cu)
    if (MODE == 0) pdl_wait();
    pdl_launch_dependents();

    const int ntiles = __ldcg(a.num_tiles);
    const int units = ntiles * a.fb_count;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    volatile int* abort_flag = &aux->abort;
    auto flag_error = [&]() {
        atomicExch(a.err, kDeviceErrorMagic);
        aux->abort = 1;
    };
    // remote (rank 0) addresses of the barriers that live in the first CTA
    const uint32_t full0 = mapa_shared(smem_u32(&aux->full[0]), 0);
    const uint32_t tempty0 = mapa_shared(smem_u32(&aux->tempty[0]), 0);

    auto decode = [&](int u, int& tile, int& fb) {
        const Tile probe = load_tile(a.tiles + u / a.fb_count);
        const int local = u - a.fb_count * probe.first;
        fb = local / probe.count;
        tile = probe.first + local % probe.count;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_normal();
            constexpr uint32_t kTx = 2 * (kATile + (MODE == 1 ? kBTile : 0));
            int stage = 0;
            uint32_t phase = 0;
            int issued[8];
            for (int s = 0; s < kStages; ++s) issued[s] = 0;
            bool ok = true;
            bool dep_ready = MODE == 0;
            for (int u = pair; u < units && ok; u += npairs) {
                int tile, fb;
                decode(u, tile, fb);
                const Tile t = load_tile(a.tiles + tile);
                const int half = ((t.rows + 15) & ~15) >> 1;  // B rows per CTA
                for (int kt = 0; kt < a.num_kt; ++kt) {
                    if (!mbar_wait_cluster(&aux->empty[stage], phase ^ 1u, abort_flag)) {
                        flag_error();
                        ok = false;
                        break;
                    }
                    uint8_t* st = ring + stage * kStageBytes;
                    const uint32_t fbar = full0 + stage * 8;
                    if (leader) mbar_arrive_expect_tx(&aux->full[stage], kTx);
                    if (MODE == 0) {
                        const int row = t.expert * 2 * a.I + fb * 128 + 64 * rank;
                        tma_load_2d_pair(st, &tm_w, fbar, kt * kBK, row, pol);
                        tma_load_2d_pair(st + kATile / 2, &tm_w, fbar, kt * kBK, row + a.I, pol);
                    } else {
                        // when H is an odd number of 128-row blocks the second CTA of the
                        // last block pair reads the next expert's rows (or zero fill past
                        // the tensor) and its outputs are not stored
                        const int row = t.expert * a.H + fb * 256 + 128 * rank;
                        tma_load_2d_pair(st, &tm_w, fbar, kt * kBK, row, pol);
                        if (!dep_ready) {  // act comes from the previous kernel
                            pdl_wait();
                            dep_ready = true;
                        }
                        tma_load_2d_pair(st + kATile, &tm_act, fbar, kt * kBK,
                                         t.row_start + half * (int)rank, pol);
                    }
                    if (kt + 4 < a.num_kt) {  // weight tiles 4 stages ahead to L2
                        const int row = MODE == 0 ? t.expert * 2 * a.I + fb * 128 + 64 * rank
                                                  : t.expert * a.H + fb * 256 + 128 * rank;
                        tma_prefetch_l2_2d(&tm_w, (kt + 4) * kBK, row);
                        if (MODE == 0) tma_prefetch_l2_2d(&tm_w, (kt + 4) * kBK, row + a.I);
                    }
                    issued[stage] += 1;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!dep_ready) pdl_wait();
            if (!ok || *abort_flag) {
                // this CTA's loads complete on the first CTA's barrier; give them time
                // to land before leaving (the first CTA drains its own)
                volatile int never = 0;
                if (leader)
                    for (int s = 0; s < kStages; ++s)
                        if (issued[s] > 0)
                            mbar_wait_cluster(&aux->full[s], (uint32_t)((issued[s] - 1) & 1),
                                              &never, 500000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (CTA 0)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int lu = 0;
            bool ok = true;
            for (int u = pair; u < units && ok; u += npairs, ++lu) {
                int tile, fb;
                decode(u, tile, fb);
                const Tile t = load_tile(a.tiles + tile);
                const int b = lu & 1;
                const uint32_t aphase = (uint32_t)((lu >> 1) & 1);
                if (!mbar_wait_cluster(&aux->tempty[b], aphase ^ 1u, abort_flag)) {
                    flag_error();
                    break;
                }
                tc_fence_after();
                const int n = (t.rows + 15) & ~15;
                const uint32_t idesc = umma_idesc_bf16(256, n);
                const uint32_t d = tmem_base + (uint32_t)(b * kAccCols);
                for (int kt = 0; kt < a.num_kt; ++kt) {
                    if (!mbar_wait_cluster(&aux->full[stage], phase, abort_flag)) {
                        flag_error();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(ring + stage * kStageBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk)
                        umma_bf16_pair(d, umma_desc_sw128(st + kk * 32),
                                       umma_desc_sw128(st + kATile + kk * 32), idesc,
                                       (kt > 0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair(&aux->empty[stage]);  // frees the stage in both CTAs
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit_pair(&aux->tfull[b]);
            }
            umma_commit_pair(&aux->drain);
            volatile int never = 0;
            if (!mbar_wait(&aux->drain, 0, &never, 500000000ull)) atomicExch(a.err, kDeviceErrorMagic);
        }
    } else if (warp < 2 + kG * kW) {
        // ------------------------------------------------------------ gather (MODE 0)
        if (MODE == 0) {
            const int g = (warp - 2) / kW, wi = (warp - 2) % kW;
            int* my_off = tok_off + (warp - 2) * kHalf;
            const uint64_t x_policy = l2_policy_evict_last();
            int q = 0;
            int cur_tile = -1;
            bool ok = true;
            for (int u = pair; u < units && ok; u += npairs) {
                int tile, fb;
                decode(u, tile, fb);
                int kt = ((g - q % kG) + kG) % kG;
                const int q_unit0 = q;
                q += a.num_kt;
                if (kt >= a.num_kt) continue;
                const Tile t = load_tile(a.tiles + tile);
                const int half = ((t.rows + 15) & ~15) >> 1;
                const int j0 = half * (int)rank;                 // this CTA's first tile row
                const int rows = max(0, min(half, t.rows - j0));  // rows it holds
                if (tile != cur_tile) {
                    __syncwarp();
                    for (int j = lane; j < rows; j += 32)
                        my_off[j] = (a.permuted_rows[t.row_start + j0 + j] / a.k) * a.H;
                    __syncwarp();
                    cur_tile = tile;
                }
                const int chunks = rows * 8;
                for (; kt < a.num_kt; kt += kG) {
                    const int qq = q_unit0 + kt;
                    const int stage = qq % kStages;
                    const uint32_t phase = (uint32_t)((qq / kStages) & 1);
                    if (!__all_sync(0xffffffffu, mbar_wait_cluster(&aux->empty[stage], phase ^ 1u,
                                                                   abort_flag))) {
                        if (lane == 0) flag_error();
                        ok = false;
                        break;
                    }
                    const uint32_t bt = smem_u32(ring + stage * kStageBytes + kATile);
                    const __nv_bfloat16* src0 = a.x + kt * kBK;
                    for (int c8 = lane + 32 * wi; c8 < chunks; c8 += 32 * kW) {
                        const int j = c8 >> 3, c = c8 & 7;
                        cp_async_16_hint(bt + j * 128 + ((c ^ (j & 7)) << 4),
                                         src0 + my_off[j] + c * 8, x_policy);
                    }
                    cp_async_commit();
                    cp_async_wait<0>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(full0 + stage * 8);
                }
            }
            cp_async_wait<0>();
        }
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        if (MODE == 1) pdl_wait();
        const int grp = (warp - kEpiWarp0) >> 2;  // token-column half of the tile
        const int q = warp & 3;                 // TMEM lane quarter
        const int gt = q * 32 + lane;           // 0..127 within the group
        float* xg = xbuf + grp * 64 * kStageRows;
        int chunk = 0;
        int lu = 0;
        for (int u = pair; u < units; u += npairs, ++lu) {
            int tile, fb;
            decode(u, tile, fb);
            const Tile t = load_tile(a.tiles + tile);
            const int b = lu & 1;
            const uint32_t aphase = (uint32_t)((lu >> 1) & 1);
            const bool got = mbar_wait_cluster(&aux->tfull[b], aphase, abort_flag);
            if (!got) flag_error();
            if (named_bar_or(1 + grp, 128, !got || *abort_flag)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kAccCols);
            const int jbeg = grp * (kN / 2), jend = min(t.rows, (grp + 1) * (kN / 2));
            // this CTA's output features: MODE 0: 64 act features; MODE 1: 128 y features
            const int fbase = MODE == 0 ? fb * 128 + 64 * (int)rank : fb * 256 + 128 * (int)rank;
            const int nfeat = MODE == 0 ? 64 : (fbase < a.H ? 128 : 0);
            const int vec_per_row = nfeat * 2 / 16;
            for (int j0 = jbeg; j0 < jend; j0 += kStageRows) {
                uint32_t v[8];
                tmem_ld8(tacc + j0, v);
                tmem_ld_wait();
                if (j0 + kStageRows >= jend) {  // accumulator drained
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(tempty0 + b * 8);
                }
                uint8_t* buf = staging + (grp * 2 + (chunk & 1)) * (kStageRows * kStageRowBytes);
                if (MODE == 0) {
                    // lanes 64-127 (warps q = 2, 3) hold up, lanes 0-63 gate, same features
                    if (q >= 2)
#pragma unroll
                        for (int jj = 0; jj < kStageRows; ++jj)
                            xg[(gt - 64) * kStageRows + jj] = __uint_as_float(v[jj]);
                    named_bar_sync(1 + grp, 128);
                    if (q < 2)
#pragma unroll
                        for (int jj = 0; jj < kStageRows; ++jj) {
                            __nv_bfloat16* row =
                                reinterpret_cast<__nv_bfloat16*>(buf + jj * kStageRowBytes);
                            row[gt] = __float2bfloat16_rn(
                                silu_mul(__uint_as_float(v[jj]), xg[gt * kStageRows + jj]));
                        }
                } else {
#pragma unroll
                    for (int jj = 0; jj < kStageRows; ++jj) {
                        __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(buf + jj * kStageRowBytes);
                        row[gt] = __float2bfloat16_rn(__uint_as_float(v[jj]));
                    }
                }
                named_bar_sync(1 + grp, 128);  // staged (and the gate/up buffer read)
                const int n = min(kStageRows, jend - j0);
                for (int i = gt; i < n * vec_per_row; i += 128) {
                    const int jj = i / vec_per_row, c = i % vec_per_row;
                    const int p = t.row_start + j0 + jj;
                    const uint4 val = *reinterpret_cast<const uint4*>(buf + jj * kStageRowBytes + c * 16);
                    __nv_bfloat16* dst = MODE == 0
                        ? a.out + (size_t)p * a.I + fbase
                        : a.out + (size_t)a.permuted_rows[p] * a.H + fbase;
                    *reinterpret_cast<uint4*>(dst + c * 8) = val;
                }
                ++chunk;
            }
            if (jbeg >= jend) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tempty0 + b * 8);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the pair's MMAs and remote arrivals are all done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <int MODE>
cudaError_t launch_pair_mode(const CUtensorMap& tw, const CUtensorMap& ta, const PairArgs& a,
                             int pairs, cudaStream_t st)
{
    auto kern = grouped_gemm_pair_kernel<MODE>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    (void)err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tw, ta, a);
}

}  // namespace

int pair_kernel_max_pairs(int num_sms)
{
    static int cached = -1;
    if (cached >= 0) return cached;
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = grouped_gemm_pair_kernel<0>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
        n = 0;
    cudaGetLastError();
    cached = n;
    return n;
}

cudaError_t launch_grouped_ffn_pair(const FfnBuffers& b, const CUtensorMap& tw13_half,
                                    const CUtensorMap& tw2, const CUtensorMap& tact, int T, int k,
                                    int H, int I, int pairs, cudaStream_t st,
                                    cudaEvent_t between_gemms)
{
    PairArgs a = {};
    a.x = static_cast<const __nv_bfloat16*>(b.x);
    a.permuted_rows = b.permuted_rows;
    a.tiles = b.tiles;
    a.num_tiles = b.num_tiles;
    a.err = b.err;
    a.k = k;
    a.H = H;
    a.I = I;
    a.R = T * k;

    a.out = static_cast<__nv_bfloat16*>(b.act);
    a.num_kt = H / kBK;
    a.fb_count = I / 128;
    cudaError_t err = launch_pair_mode<0>(tw13_half, tw13_half, a, pairs, st);
    if (err != cudaSuccess) return err;
    if (between_gemms) {
        err = cudaEventRecord(between_gemms, st);
        if (err != cudaSuccess) return err;
    }
    a.out = static_cast<__nv_bfloat16*>(b.y);
    a.num_kt = I / kBK;
    a.fb_count = (H / 128 + 1) / 2;
    return launch_pair_mode<1>(tw2, tact, a, pairs, st);
}

}  // namespace moe
