// fused_ffn.cu -- w13 + SwiGLU, w2 and the weighted combine of a weight-streaming
// MoE layer in ONE persistent launch (moe_forward, at most 64 tokens).
//
// With few tokens per expert the layer is a stream of the touched experts'
// weights.  As separate launches (grouped_ffn.cu, then the SwiGLU finalize, w2
// and the combine) every boundary costs a ramp, a tail and a dependency hop on
// the critical path while HBM idles.  Here one CTA per SM walks a single unit
// list -- every w13 unit, then every w2 unit -- so the w2 weight stream starts as
// soon as a CTA has issued its last w13 tile; the steps that need other CTAs'
// results wait on arrival counters instead of a kernel boundary:
//
//   w13 runs unsplit (one unit = a whole K range), so its epilogue finishes act
//   itself: bf16(silu(gate) * up).  w2 tile t reads the act rows of tile t,
//   complete once all fb13 w13 units of tile t have stored them.  Each w13
//   unit's two epilogue groups publish their stores (named barrier, then
//   red.release on tile_ready[t]); the gather warp that fills w2's B operand for
//   tile t waits (acquire loads, bounded) for tile_ready[t] == 2 * fb13, then
//   loads each act tile with one TMA.  The w2 weight TMA never waits.
//
//   out[t, block b] needs y rows t*k + j (every j) of 256-column block b from
//   all S2 slices: each w2 epilogue group adds one release arrival per row to
//   token_ready[t, b].  After its units, each CTA's epilogue warps take (token,
//   block) tasks round-robin, wait for k * S2 arrivals, and combine: y =
//   bf16(sum_s partial_s) per row, then sum_j w[t, j] * y in j order with the
//   combine kernel's fma chain.
//
// act is stored K-blocked ([I / 64][R][64]) so the 64-column slab a w2 stage
// reads is one contiguous run of rows (one TMA box).
//
// Load balance: one w13 unit streams a whole [128 x H] gate block and up block,
// so w13 alone would leave some CTAs a unit behind; the CTAs with one w13 unit
// fewer take that many K tiles of w2 units first (see the schedule below).
//
// w2 and the combine use the multi-launch path's arithmetic (same w2 split
// count, roundings and summation orders); w13's sum over K is one fp32 chain
// where the multi-launch path may add split-K slices, so act -- and out -- can
// differ from that path's by a bf16 rounding.  Deadlock freedom: every CTA runs all
// of its w13 units before any w2 unit and all of its units before any combine
// task; a w13 unit depends on nothing but the routing, a w2 unit only on w13
// units, a combine task only on w2 units, and within a CTA the epilogue finishes
// each unit without waiting for a later one.  The grid is one CTA per SM, so
// every CTA is resident.  Every wait is bounded (2 s) and also gives up when
// another CTA has recorded an error.
//
// Roles (512 threads) as in grouped_ffn.cu: warp 0 TMA producer (w13 or w2
// weight tiles, evict-first), warp 1 TMEM allocator + MMA issuer, warps 2-7
// gather (x rows for w13, act tiles for w2), warps 8-15 two epilogue groups,
// then together the combine.
#include "gemm_common.cuh"

namespace moe {

namespace {

using namespace gemm;

constexpr int kMaxK = 16;       // combine: selected experts per token
constexpr int kMaxSplits = 8;   // split-K slices per GEMM

struct FusedArgs {
    const __nv_bfloat16* x;       // [T, H]
    const int32_t* permuted_rows; // [R]
    const Tile* tiles;
    const int32_t* num_tiles;
    const float* topk_weights;    // [R]
    __nv_bfloat16* act;           // [I / 64, R, 64] (K-blocked)
    float* part2;                 // [S2, R, H] when the w2 split is > 1
    __nv_bfloat16* y;             // [R, H] when the w2 split is 1
    __nv_bfloat16* out;           // [T, H]
    int32_t* tile_ready;          // [max_tiles] w13 arrivals, zero at entry
    int32_t* token_ready;         // [T * fb2] w2 row arrivals, zero at entry
    int32_t* w2_next;             // w2 units handed out at run time, zero at entry
    int32_t* split_out;           // [2] 1, S2 (CTA 0)
    int32_t* err;
    int k, H, I, R;
    int kt13, kt2;                // K tiles: H / 64, I / 64
    int fb13, fb2;                // I / 128 gate/up block pairs; ceil(H / 256) w2 block pairs
    int s2_max;
    int min_kt_per_split;
};

struct Unit {
    int ph;      // 0: w13, 1: w2
    int split;
    int tile;
    int fb;
    int kt0, kt1;
    int expert, row_start, rows;  // of the tile
};

// Each CTA keeps its unit list in shared memory: the static part decoded once
// (two dependent L2 loads per unit, all units at once) instead of once per unit
// in every role -- a single-threaded TMA producer would otherwise stall on them
// between units -- and the dynamic part published by the producer as it claims
// units.  32 bytes per entry plus a sequence word.
constexpr int kUnitTable = 128;
constexpr int kUnitTableBytes = kUnitTable * (32 + 4);
constexpr int kUnitEnd = 2;    // Unit::ph of the list's terminator
constexpr int kUnitAbort = 3;  // Unit::ph when waiting for an entry gave up

// The combine's routing weights, in shared memory right after Aux.
struct ComboScratch {
    float w[kMaxK];
};

__device__ __forceinline__ void flag_error(int32_t* err, Aux* aux)
{
    atomicExch(err, kDeviceErrorMagic);
    aux->abort = 1;
}

// Bounded wait until *ctr >= target, every lane of the warp polling with acquire
// loads (so each lane's later loads are ordered after the arrivals it saw).
// False on a timeout, a local abort or another CTA's recorded error.
__device__ __forceinline__ bool warp_wait_count(const int32_t* ctr, int target,
                                                volatile int* abort, const int32_t* err)
{
    if (__all_sync(0xffffffffu, ld_acquire_gpu(ctr) >= target)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        __nanosleep(64);
        if (__all_sync(0xffffffffu, ld_acquire_gpu(ctr) >= target)) return true;
        const bool stop = *abort || *reinterpret_cast<const volatile int32_t*>(err) ==
                                        kDeviceErrorMagic ||
                          globaltimer_ns() - t0 > 2000000000ull;
        if (__any_sync(0xffffffffu, stop)) return false;
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    fused_ffn_kernel(const __grid_constant__ CUtensorMap tm_w13,
                     const __grid_constant__ CUtensorMap tm_w2,
                     const __grid_constant__ CUtensorMap tm_act, const FusedArgs a)
{
    using C = Cfg<0, NT>;
    static_assert(NT <= 64, "weight-streaming tiles");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* ring = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* staging = ring + C::kStages * C::kStageBytes;
    Aux* aux = reinterpret_cast<Aux*>(staging + C::kStagingBytes);
    ComboScratch* combo = reinterpret_cast<ComboScratch*>(aux + 1);
    int* tok_off = reinterpret_cast<int*>(combo + 1);
    int4* unit_tab = reinterpret_cast<int4*>(reinterpret_cast<uint8_t*>(aux) + C::kAuxBytes);
    int* tab_seq = reinterpret_cast<int*>(unit_tab + 2 * kUnitTable);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&aux->full[s], 1 + C::kW);
            mbar_init(&aux->empty[s], 1);
        }
        for (int b = 0; b < C::kNBuf; ++b) {
            mbar_init(&aux->tfull[b], 1);
            mbar_init(&aux->tempty[b], 8);
        }
        mbar_init(&aux->drain, 1);
        aux->abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_w13);
        tma_prefetch_desc(&tm_w2);
        tma_prefetch_desc(&tm_act);
    }
    if (warp == 1) {
        tmem_alloc(&aux->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;

    // the tile list, permuted rows, routing weights and zeroed counters come from
    // the permutation kernel right before
    pdl_wait();
    pdl_launch_dependents();

    const int ntiles = __ldcg(a.num_tiles);
    // w13 is not split here: its epilogue writes bf16 act directly, which each w2
    // stage then loads with one TMA.  w2 is split only as far as ~4 waves of units
    // need: the run-time hand-out already balances the tail, and every extra
    // slice adds epilogue publishes and combine reads (same-B200 A/B: 16 waves
    // 101.4 us decode / 360.7 us skewed decode, 4 waves 98.2 / 341.8).
    const int s2w = split_count(ntiles * a.fb2, a.s2_max, a.kt2, a.min_kt_per_split, 4);
    const int ktps2 = (a.kt2 + s2w - 1) / s2w;
    const int S2 = (a.kt2 + ktps2 - 1) / ktps2;  // every slice non-empty
    const int U13 = ntiles * a.fb13;
    const int U2 = ntiles * a.fb2 * S2;
    const int tile_target = 2 * a.fb13;  // two epilogue groups per w13 unit
    const int token_target = a.k * S2;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        a.split_out[0] = 1;
        a.split_out[1] = S2;
    }
    volatile int* abort_flag = &aux->abort;

    // Schedule.  CTA b first runs w13 units b, b + G, ...  When U13 is not a
    // multiple of G, the CTAs with one unit fewer ("light", b >= U13 % G) next
    // take `fill` w2 units each -- about one w13 unit's worth of K tiles, the
    // lowest w2 indices.  Those lists are static.  The w2 units left are handed
    // out in increasing order at run time: a CTA's producer claims the next one
    // with an atomic on a workspace counter when it is ready for more, so CTAs
    // that stream faster take more and all of them finish together.
    const int G = gridDim.x, bid = blockIdx.x;
    const int r13 = U13 % G;
    const int n13 = U13 / G + (bid < r13 ? 1 : 0);
    const int nlight = r13 ? G - r13 : 0;
    const int fill = nlight ? min((a.kt13 + ktps2 / 2) / ktps2, U2 / nlight) : 0;
    const int nf = (nlight && bid >= r13) ? fill : 0;
    const int rest0 = nlight * fill;  // the first w2 unit handed out at run time
    const int n_static = n13 + nf;
    auto unit_of = [&](int i) {  // global unit of static entry i: [0, U13) w13, then w2
        return i < n13 ? bid + i * G : U13 + (bid - r13) + (i - n13) * nlight;
    };

    // unit u -> (phase, slice, tile, feature block), each phase in grouped_ffn.cu's
    // expert-grouped order (slice fastest, then tile, then feature block within an
    // expert).
    auto decode = [&](int u) {
        Unit un;
        un.ph = u >= U13;
        const int v = un.ph ? u - U13 : u;
        const int S = un.ph ? S2 : 1, fbc = un.ph ? a.fb2 : a.fb13;
        const int ktps = un.ph ? ktps2 : a.kt13, nkt = un.ph ? a.kt2 : a.kt13;
        un.split = v % S;
        const int rest = v / S;
        const Tile probe = load_tile(a.tiles + rest / fbc);
        const int local = rest - fbc * probe.first;
        un.fb = local / probe.count;
        un.tile = probe.first + local % probe.count;
        un.kt0 = un.split * ktps;
        un.kt1 = min(nkt, un.kt0 + ktps);
        const Tile t = load_tile(a.tiles + un.tile);
        un.expert = t.expert;
        un.row_start = t.row_start;
        un.rows = t.rows;
        return un;
    };
    auto put = [&](int slot, const Unit& un) {
        unit_tab[2 * slot] = make_int4(un.ph | (un.split << 8), un.tile, un.fb, un.kt0 | (un.kt1 << 16));
        unit_tab[2 * slot + 1] = make_int4(un.expert, un.row_start, un.rows, 0);
    };
    auto read = [&](int slot) {
        const int4 e0 = unit_tab[2 * slot], e1 = unit_tab[2 * slot + 1];
        Unit un;
        un.ph = e0.x & 0xff;
        un.split = e0.x >> 8;
        un.tile = e0.y;
        un.fb = e0.z;
        un.kt0 = e0.w & 0xffff;
        un.kt1 = e0.w >> 16;
        un.expert = e1.x;
        un.row_start = e1.y;
        un.rows = e1.z;
        return un;
    };
    for (int i = threadIdx.x; i < kUnitTable; i += blockDim.x) tab_seq[i] = 0;
    for (int i = threadIdx.x; i < min(n_static, kUnitTable); i += blockDim.x)
        put(i, decode(unit_of(i)));
    __syncthreads();
    // The CTA's i-th unit.  Dynamic entries live in the table as a ring with
    // tab_seq[slot] = i + 1 once published; no role trails the producer by more
    // than kStages + kNBuf units, far below the ring's length.
    auto get = [&](int i) {
        if (i < n_static) return i < kUnitTable ? read(i) : decode(unit_of(i));
        const int slot = i % kUnitTable;
        const volatile int* sq = tab_seq + slot;
        if (*sq != i + 1) {
            const uint64_t t0 = globaltimer_ns();
            while (*sq != i + 1) {
                __nanosleep(32);
                if (*abort_flag || globaltimer_ns() - t0 > 2000000000ull) {
                    flag_error(a.err, aux);
                    Unit un;
                    un.ph = kUnitAbort;
                    return un;
                }
            }
        }
        __threadfence_block();
        return read(slot);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();  // each weight block is read once
            int stage = 0;
            uint32_t phase = 0;
            int issued[16];
            for (int s = 0; s < C::kStages; ++s) issued[s] = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                Unit un;
                if (i < n_static) {
                    un = get(i);
                } else {  // claim the next w2 unit and publish it to the other roles
                    const int v = rest0 + atomicAdd(a.w2_next, 1);
                    if (v < U2) {
                        un = decode(U13 + v);
                    } else {
                        un.ph = kUnitEnd;
                        un.split = un.tile = un.fb = un.kt0 = un.kt1 = 0;
                        un.expert = un.row_start = un.rows = 0;
                    }
                    put(i % kUnitTable, un);
                    __threadfence_block();
                    *reinterpret_cast<volatile int*>(tab_seq + i % kUnitTable) = i + 1;
                    if (un.ph == kUnitEnd) break;
                }
                const Unit& t = un;
                const CUtensorMap* tm = un.ph ? &tm_w2 : &tm_w13;
                // w13: the gate block and the up block of feature block fb; w2: two
                // consecutive 128-row blocks of w2[e] (the second may belong to the
                // next expert or lie past the tensor; its accumulator is not stored)
                const int row0 = un.ph ? t.expert * a.H + un.fb * 2 * kBM
                                       : t.expert * 2 * a.I + un.fb * kBM;
                const int row1 = un.ph ? row0 + kBM : row0 + a.I;
                for (int kt = un.kt0; kt < un.kt1; ++kt) {
                    if (!mbar_wait(&aux->empty[stage], phase ^ 1u, abort_flag)) {
                        flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    uint8_t* st = ring + stage * C::kStageBytes;
                    mbar_arrive_expect_tx(&aux->full[stage], C::kTxBytes);
                    tma_load_2d(st, tm, &aux->full[stage], kt * kBK, row0, pol);
                    tma_load_2d(st + kATileBytes, tm, &aux->full[stage], kt * kBK, row1, pol);
                    issued[stage] += 1;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok || *abort_flag) {
                // let every TMA load already issued land before the CTA can exit
                for (int s = 0; s < C::kStages; ++s)
                    if (issued[s] > 0) {
                        volatile int never = 0;
                        mbar_wait(&aux->full[s], (uint32_t)((issued[s] - 1) & 1), &never,
                                  500000000ull);
                    }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int lu = 0; ok; ++lu) {
                const Unit un = get(lu);
                if (un.ph >= kUnitEnd) break;
                const Unit& t = un;
                const int b = lu % C::kNBuf;
                const uint32_t aphase = (uint32_t)((lu / C::kNBuf) & 1);
                if (!mbar_wait(&aux->tempty[b], aphase ^ 1u, abort_flag)) {
                    flag_error(a.err, aux);
                    break;
                }
                tc_fence_after();
                const int n = (t.rows + 15) & ~15;
                const uint32_t idesc = umma_idesc_bf16(kBM, n);
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::kAccCols);
                for (int kt = un.kt0; kt < un.kt1; ++kt) {
                    if (!mbar_wait(&aux->full[stage], phase, abort_flag)) {
                        flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(ring + stage * C::kStageBytes);
                    const uint32_t bt = st + C::kNA * kATileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        const uint32_t acc = (kt > un.kt0 || kk > 0) ? 1u : 0u;
                        const uint64_t bdesc = umma_desc_sw128(bt + kk * 32);
                        umma_bf16(d0, umma_desc_sw128(st + kk * 32), bdesc, idesc, acc);
                        umma_bf16(d0 + NT, umma_desc_sw128(st + kATileBytes + kk * 32), bdesc,
                                  idesc, acc);
                    }
                    umma_commit(&aux->empty[stage]);  // frees the smem stage when read
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit(&aux->tfull[b]);
            }
            // all MMAs issued by this thread are complete before TMEM is freed
            umma_commit(&aux->drain);
            volatile int never = 0;
            if (!mbar_wait(&aux->drain, 0, &never, 500000000ull)) atomicExch(a.err, kDeviceErrorMagic);
        }
    } else if (warp < 2 + kGatherWarps) {
        // ------------------------------------------------------------ gather
        if (warp - 2 < C::kG * C::kW) {
            constexpr int G = C::kG, W = C::kW;
            const int g = (warp - 2) / W, wi = (warp - 2) % W;
            int* my_off = tok_off + (warp - 2) * NT;
            const uint64_t keep = l2_policy_evict_last();  // x / act rows are re-read per block
            int q = 0;  // global stage sequence number (same as the producer's)
            int cur_tile = -1, cur_ph = -1, ready_tile = -1;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const Unit un = get(i);
                if (__any_sync(0xffffffffu, un.ph >= kUnitEnd)) break;
                // first stage of this unit that this warp's group owns
                int kt = un.kt0 + ((g - q % G) + G) % G;
                const int q_unit0 = q;
                q += un.kt1 - un.kt0;
                if (kt >= un.kt1) continue;
                const Unit& t = un;
                if (un.ph == 1 && un.tile != ready_tile) {
                    // every w13 unit of this tile has stored its act rows or slices
                    if (!warp_wait_count(a.tile_ready + un.tile, tile_target, abort_flag, a.err)) {
                        if (lane == 0) flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();  // the act TMA reads after the acquire
                    ready_tile = un.tile;
                }
                if (un.tile != cur_tile || un.ph != cur_ph) {
                    __syncwarp();  // earlier copies' addresses are all issued
                    if (un.ph == 0)
                        for (int j = lane; j < t.rows; j += 32)
                            my_off[j] = (a.permuted_rows[t.row_start + j] / a.k) * a.H;
                    __syncwarp();
                    cur_tile = un.tile;
                    cur_ph = un.ph;
                }
                for (; kt < un.kt1; kt += G) {
                    const int qq = q_unit0 + (kt - un.kt0);
                    const int stage = qq % C::kStages;
                    const uint32_t phase = (uint32_t)((qq / C::kStages) & 1);
                    // warp-uniform decision, so no lane is left behind at __syncwarp
                    if (!__all_sync(0xffffffffu, mbar_wait(&aux->empty[stage], phase ^ 1u,
                                                           abort_flag))) {
                        if (lane == 0) flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    uint8_t* btile = ring + stage * C::kStageBytes + C::kNA * kATileBytes;
                    const uint32_t bt = smem_u32(btile);
                    if (un.ph == 1) {
                        // the act tile: NT consecutive rows of K block kt, one TMA (rows
                        // past the tile belong to other tiles or lie past the tensor and
                        // are zero-filled; their accumulator columns are not stored)
                        if (lane == 0) {
                            if (wi == 0) {
                                mbar_arrive_expect_tx(&aux->full[stage], C::kBTileBytes);
                                tma_load_2d_nohint(btile, &tm_act, &aux->full[stage], 0,
                                                   kt * a.R + t.row_start);
                            } else {
                                mbar_arrive(&aux->full[stage]);
                            }
                        }
                        continue;
                    }
                    // 16-byte copies of the x rows into the 128-byte-swizzled B tile
                    const __nv_bfloat16* src0 = a.x + kt * kBK;
                    for (int c8 = lane + 32 * wi; c8 < t.rows * 8; c8 += 32 * W) {
                        const int j = c8 >> 3, c = c8 & 7;
                        cp_async_16_hint(bt + j * 128 + ((c ^ (j & 7)) << 4),
                                         src0 + my_off[j] + c * 8, keep);
                    }
                    cp_async_commit();
                    cp_async_wait<0>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&aux->full[stage]);
                }
            }
            cp_async_wait<0>();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int grp = (warp - kEpiWarp0) >> 2;  // token-column half
        const int qw = warp & 3;                  // TMEM lane quarter
        const int gt = qw * 32 + lane;            // 0..127 within the group
        const int f_local = qw * 32 + lane;       // feature inside the 128-row block
        uint8_t* gstage = staging + grp * 2 * (kStageRows * kStageRowBytes);
        int chunk = 0;  // staging chunks issued by this group (buffer parity)
        for (int lu = 0;; ++lu) {
            const Unit un = get(lu);
            const Unit& t = un;
            const int b = lu % C::kNBuf;
            const uint32_t aphase = (uint32_t)((lu / C::kNBuf) & 1);
            bool got = false;
            if (un.ph < kUnitEnd) {
                got = mbar_wait(&aux->tfull[b], aphase, abort_flag);
                if (!got) flag_error(a.err, aux);
            }
            // the end of the list, or a failure: the same decision in all 4 warps
            if (named_bar_or(1 + grp, 128, un.ph >= kUnitEnd || !got || *abort_flag)) break;
            tc_fence_after();
            const int ph = un.ph;
            const int S = ph ? S2 : 1;
            // w13: feature f of the gate block (accumulator 0) and of the up block
            // (accumulator 1); w2: output features f and f + 128
            const int f = (ph == 0 ? un.fb * kBM : un.fb * 2 * kBM) + f_local;
            const bool f1_ok = ph == 0 || f + kBM < a.H;
            const uint32_t tacc = tmem_base + ((uint32_t)(qw * 32) << 16) + (uint32_t)(b * C::kAccCols);
            const int jbeg = grp * (NT / 2), jend = min(t.rows, (grp + 1) * (NT / 2));
            if (jbeg >= jend) {  // this group had no columns of the unit
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aux->tempty[b]);
            } else if (S == 1) {
                // staged bf16 rows, copied out whole with 16-byte stores (act by
                // permuted row, or y by expanded id)
                const int row_bytes = ph == 0 ? 2 * kBM
                                    : ((un.fb * 2 + 1) * kBM < a.H ? 4 * kBM : 2 * kBM);
                const int vec_per_row = row_bytes / 16;
                for (int j0 = jbeg; j0 < jend; j0 += kStageRows) {
                    uint32_t gv[8], vv[8];
                    tmem_ld8(tacc + j0, gv);
                    tmem_ld8(tacc + NT + j0, vv);
                    tmem_ld_wait();
                    if (j0 + kStageRows >= jend) {  // accumulator drained: let the MMA go on
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&aux->tempty[b]);
                    }
                    uint8_t* buf = gstage + (chunk & 1) * (kStageRows * kStageRowBytes);
#pragma unroll
                    for (int jj = 0; jj < kStageRows; ++jj) {
                        __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(buf + jj * kStageRowBytes);
                        if (ph == 0) {
                            row[f_local] = __float2bfloat16_rn(
                                silu_mul(__uint_as_float(gv[jj]), __uint_as_float(vv[jj])));
                        } else {
                            row[f_local] = __float2bfloat16_rn(__uint_as_float(gv[jj]));
                            row[kBM + f_local] = __float2bfloat16_rn(__uint_as_float(vv[jj]));
                        }
                    }
                    named_bar_sync(1 + grp, 128);  // staged; the other buffer is free again
                    const int n = min(kStageRows, jend - j0);
                    for (int i = gt; i < n * vec_per_row; i += 128) {
                        const int jj = i / vec_per_row, c = i % vec_per_row;
                        const int p = t.row_start + j0 + jj;
                        const uint4 val = *reinterpret_cast<const uint4*>(buf + jj * kStageRowBytes + c * 16);
                        // act: K block 2 fb + c / 8 of row p; y: expanded-id row
                        __nv_bfloat16* dst = ph == 0
                            ? a.act + ((size_t)(2 * un.fb + (c >> 3)) * a.R + p) * kBK + (c & 7) * 8
                            : a.y + (size_t)a.permuted_rows[p] * a.H + un.fb * 2 * kBM + c * 8;
                        *reinterpret_cast<uint4*>(dst) = val;
                    }
                    ++chunk;
                }
            } else {
                constexpr int kCols = kEpiCols<NT>;
                for (int j0 = jbeg; j0 < jend; j0 += kCols) {
                    uint32_t gv[kCols], vv[kCols];
                    tmem_ld_cols(tacc + j0, gv);
                    tmem_ld_cols(tacc + NT + j0, vv);
                    tmem_ld_wait();
#pragma unroll
                    for (int jj = 0; jj < kCols; ++jj) {
                        const int j = j0 + jj;
                        if (j >= jend) break;
                        const int p = t.row_start + j;
                        {  // w2 slice: fp32 by expanded id
                            const int r = a.permuted_rows[p];
                            float* prow = a.part2 + ((size_t)un.split * a.R + r) * a.H;
                            prow[f] = __uint_as_float(gv[jj]);
                            if (f1_ok) prow[f + kBM] = __uint_as_float(vv[jj]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aux->tempty[b]);
            }

            // ---- publish this group's stores (the barrier orders every thread's
            // stores before the releasing thread's increment)
            if (ph == 0) fence_proxy_async_global();  // act is read by TMA
            named_bar_sync(1 + grp, 128);
            if (ph == 0) {
                if (gt == 0) red_release_gpu_add(a.tile_ready + un.tile, 1);
            } else if (gt < jend - jbeg) {
                const int tok = a.permuted_rows[t.row_start + jbeg + gt] / a.k;
                red_release_gpu_add(a.token_ready + (size_t)tok * a.fb2 + un.fb, 1);
            }
        }

        // ---- combine: (token, 256-column block) tasks, round-robin over the CTAs,
        // by all eight epilogue warps of the CTA once both groups are done
        const int et = threadIdx.x - kEpiWarp0 * 32;     // 0..255
        float4* ysm = reinterpret_cast<float4*>(staging);  // k * 64 float4 <= 16 KB
        const int H4 = a.H / 4;
        const int ntask = (a.R / a.k) * a.fb2;
        for (int task = blockIdx.x; task < ntask; task += gridDim.x) {
            const int tok = task / a.fb2, fb = task % a.fb2;
            bool ready = true;
            if (warp == kEpiWarp0) {
                ready = warp_wait_count(a.token_ready + task, token_target, abort_flag, a.err);
                if (!ready && lane == 0) flag_error(a.err, aux);
                if (ready && lane < a.k) combo->w[lane] = a.topk_weights[(size_t)tok * a.k + lane];
            }
            if (named_bar_or(3, 256, !ready || *abort_flag)) break;  // uniform over the 8 warps
            const int c0 = fb * 2 * kBM;
            const int n4 = min(2 * kBM, a.H - c0) / 4;  // float4 columns of the block
            for (int it = et; it < a.k * n4; it += 256) {
                const int j = it / n4, c4 = c0 / 4 + it % n4;
                const size_t r = (size_t)tok * a.k + j;
                float v[4];
                if (S2 > 1) {  // y = bf16(sum_s partial_s), slice order
                    const float4* src = reinterpret_cast<const float4*>(a.part2) + r * H4 + c4;
                    float4 pv[kMaxSplits];
#pragma unroll
                    for (int s = 0; s < kMaxSplits; ++s)
                        if (s < S2) pv[s] = __ldcg(src + (size_t)s * a.R * H4);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int s = 0; s < kMaxSplits; ++s) {
                        if (s < S2) {
                            acc[0] += pv[s].x; acc[1] += pv[s].y;
                            acc[2] += pv[s].z; acc[3] += pv[s].w;
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[e] = __bfloat162float(__float2bfloat16_rn(acc[e]));
                } else {
                    const uint2 yv = __ldcg(reinterpret_cast<const uint2*>(a.y) + r * H4 + c4);
                    const __nv_bfloat162* yp = reinterpret_cast<const __nv_bfloat162*>(&yv);
                    const float2 f0 = __bfloat1622float2(yp[0]), f1 = __bfloat1622float2(yp[1]);
                    v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
                }
                ysm[it] = make_float4(v[0], v[1], v[2], v[3]);
            }
            named_bar_sync(3, 256);
            if (et < n4) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int j = 0; j < a.k; ++j) {  // j ascending: the fixed summation order
                    const float wj = combo->w[j];
                    const float4 yv = ysm[j * n4 + et];
                    acc[0] = fmaf(wj, yv.x, acc[0]);
                    acc[1] = fmaf(wj, yv.y, acc[1]);
                    acc[2] = fmaf(wj, yv.z, acc[2]);
                    acc[3] = fmaf(wj, yv.w, acc[3]);
                }
                uint2 o;
                __nv_bfloat162* oq = reinterpret_cast<__nv_bfloat162*>(&o);
                oq[0] = __floats2bfloat162_rn(acc[0], acc[1]);
                oq[1] = __floats2bfloat162_rn(acc[2], acc[3]);
                reinterpret_cast<uint2*>(a.out)[(size_t)tok * H4 + c0 / 4 + et] = o;
            }
            named_bar_sync(3, 256);  // ysm and the weights are free again
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

template <int NT>
cudaError_t launch_fused_nt(const CUtensorMap& t13, const CUtensorMap& t2, const CUtensorMap& ta,
                            const FusedArgs& a, int grid, cudaStream_t st)
{
    using C = Cfg<0, NT>;
    // the combine's weights sit in the slack Cfg reserves next to Aux; the unit
    // table follows the aux area
    static_assert(sizeof(Aux) + sizeof(ComboScratch) <= 1024, "aux area");
    static_assert(C::kAuxBytes % 16 == 0, "unit table alignment");
    constexpr int smem = C::kSmemBytes + kUnitTableBytes;
    static_assert(smem <= C::kMaxSmem, "shared memory");
    auto kern = fused_ffn_kernel<NT>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, t13, t2, ta, a);
}

}  // namespace

bool fused_ffn_eligible(int T, int E, int k, int H, int I, const FfnPlan& plan)
{
    (void)E;
    (void)H;
    (void)I;
    return plan.nt <= 64 && (long)T * k <= kSmallRows && k <= kMaxK && plan.s2_max <= kMaxSplits;
}

int fused_ffn_counters(int T, int H, const FfnPlan& plan)
{
    return plan.max_tiles + T * ((H / kBM + 1) / 2) + 1;
}

cudaError_t launch_fused_ffn(const FusedBuffers& b, int T, int E, int k, int H, int I,
                             const FfnPlan& plan, cudaStream_t st)
{
    const int R = T * k;
    CUtensorMap t13, t2, ta;
    cudaError_t err = make_tmap(&t13, b.w13, (uint64_t)E * 2 * I, (uint64_t)H, kBM);
    if (err == cudaSuccess) err = make_tmap(&t2, b.w2, (uint64_t)E * H, (uint64_t)I, kBM);
    // act, K-blocked: (I / 64) * R rows of 64 columns, NT-row boxes
    if (err == cudaSuccess)
        err = make_tmap(&ta, b.act, (uint64_t)(I / kBK) * R, (uint64_t)kBK, (uint32_t)plan.nt);
    if (err != cudaSuccess) return err;
    FusedArgs a = {};
    a.x = static_cast<const __nv_bfloat16*>(b.x);
    a.permuted_rows = b.permuted_rows;
    a.tiles = b.tiles;
    a.num_tiles = b.num_tiles;
    a.topk_weights = b.topk_weights;
    a.act = static_cast<__nv_bfloat16*>(b.act);
    a.part2 = b.part2;
    a.y = static_cast<__nv_bfloat16*>(b.y);
    a.out = static_cast<__nv_bfloat16*>(b.out);
    a.tile_ready = b.counters;
    a.token_ready = b.counters + plan.max_tiles;
    a.w2_next = a.token_ready + (size_t)T * ((H / kBM + 1) / 2);
    a.split_out = b.splits;
    a.err = b.err;
    a.k = k;
    a.H = H;
    a.I = I;
    a.R = R;
    a.kt13 = H / kBK;
    a.kt2 = I / kBK;
    a.fb13 = I / kBM;
    a.fb2 = (H / kBM + 1) / 2;
    a.s2_max = plan.s2_max;
    a.min_kt_per_split = 4;
    switch (plan.nt) {
    case 16: return launch_fused_nt<16>(t13, t2, ta, a, plan.grid, st);
    case 32: return launch_fused_nt<32>(t13, t2, ta, a, plan.grid, st);
    case 64: return launch_fused_nt<64>(t13, t2, ta, a, plan.grid, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
