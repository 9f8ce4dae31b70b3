// fused_ffn.cu -- w13 + SwiGLU, w2 and the weighted combine of a weight-streaming
// MoE layer in ONE persistent launch (moe_forward, at most 64 tokens).
//
// With few tokens per expert the layer is a stream of the touched experts'
// weights.  As separate launches (grouped_ffn.cu, then the SwiGLU finalize, w2
// and the combine) every boundary costs a ramp, a tail and a dependency hop on
// the critical path while HBM idles.  Here one CTA per SM (fewer for small
// layers) walks a single unit list -- every w13 unit, then every w2 unit -- so
// the w2 weight stream starts as soon as a CTA has issued its last w13 tile; the
// steps that need other CTAs' results wait on arrival counters instead of a
// kernel boundary:
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
// each unit without waiting for a later one.  The grid is at most one CTA per SM, so
// every CTA is resident.  Every wait is bounded (2 s) and also gives up when
// another CTA has recorded an error.
//
// Roles (512 threads) as in grouped_ffn.cu: warp 0 TMA producer (w13 or w2
// weight tiles, evict-first), warp 1 TMEM allocator + MMA issuer, warps 2-7
// gather (x rows for w13, act tiles for w2), warps 8-15 two epilogue groups,
// then together the combine.
//
// FP8 weights (F8): w13 and w2 arrive as E4M3 codes with one fp32 scale per
// weight row (weight = e4m3(q) * scale).  The producer streams the codes -- half
// the bytes -- two K tiles (128 codes of each weight row) per ring stage, and the
// tensor cores take them as they are: kind::f8f6f4 MMAs (K = 32 per instruction,
// so half as many MMAs per weight byte as bf16 MMAs on widened codes would need)
// with the token operand in E4M3 too.  The gather warps build that operand
// exactly: each token row (x for w13, act for w2) is scaled by a power of two
// from its largest magnitude and split into two E4M3 terms whose sum is the
// scaled bf16 row; the terms of the tile's rows are the MMA's 2 n columns (n =
// rows rounded up to 16).  E4M3 products are exact in fp32, so the accumulators
// hold the bf16 products; the epilogue adds each row's two columns, undoes the
// power of two and multiplies by the weight row's scale.  The x maxima are
// published per call by the CTAs' epilogue warps before their first unit (token
// t by CTA t mod G); w13's epilogue folds each act row's largest magnitude into
// a counter word (atomic max) before its tile_ready arrival, so w2's operand,
// which waits for that arrival anyway, finds the maxima complete.
#include <cuda_fp16.h>

#include "gemm_common.cuh"
#include "route_common.cuh"

namespace moe {

namespace {

using namespace gemm;

constexpr int kMaxK = 16;       // combine: selected experts per token
constexpr int kMaxSplits = 8;   // split-K slices per GEMM

// The routing every CTA does for itself (one-launch FFN: at most 64 tokens, so at
// most 1024 expanded rows, and at most 1024 experts): permuted rows, routing
// weights by expanded row, expert offsets, and the expert of each tile (every
// expert's rows fit one tile, so tile j is the j-th touched expert).  After the
// unit table in shared memory.
constexpr int kMaxRows = kMaxK * 64;
constexpr int kMaxExperts = 1024;
struct alignas(16) RouteSmem {
    int16_t rows[kMaxRows];
    int16_t tile_expert[kMaxExperts];
    int16_t off[kMaxExperts + 8];
    float w[kMaxRows];
    int n_tiles;
};

struct FusedArgs {
    const __nv_bfloat16* x;       // [T, H]
    const float* logits;          // [T, E]
    int32_t* ids_out;             // [R]     routing outputs, written by CTA 0
    float* weights_out;           // [R]
    int32_t* offsets_out;         // [E + 1]
    int32_t* rows_out;            // [R]
    __nv_bfloat16* act;           // [I / 64, R, 64] (K-blocked)
    float* part2;                 // [S2, R, H] when the w2 split is > 1
    __nv_bfloat16* y;             // [R, H] when the w2 split is 1
    __nv_bfloat16* out;           // [T, H]
    int32_t* tile_ready;          // [max_tiles] w13 arrivals
    int32_t* token_ready;         // [T * fb2] w2 row arrivals
    int32_t* w2_next;             // w2 units handed out at run time
    int n_counters;               // the three above, contiguous: zeroed by CTA 0 every call
    unsigned long long* ready;    // = gen once CTA 0 has zeroed them
    unsigned long long gen;       // unique to this call
    int32_t* split_out;           // [2] 1, S2 (CTA 0)
    int32_t* err;
    const float* s13;             // F8: [E, 2I] w13 row scales
    const float* s2;              // F8: [E, H] w2 row scales
    uint32_t* act_max;            // F8: [R] largest |act| per permuted row (fp32 bits), a counter
    struct XMax* xmax;            // F8: [T] largest |x| per token, tagged with the call's gen
    int T, E, k, H, I, R;
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

constexpr int kFusedReserve = kUnitTableBytes + (int)sizeof(RouteSmem);

template <int NT>
using FCfg = Cfg<0, NT, kFusedReserve>;

// The FP8-weight kernel with E4M3 MMAs (F8).  One ring, as in the bf16 kernel, each
// stage two [128 x 128]-byte E4M3 code boxes (TMA; K tiles kt and kt + 1) and
// the E4M3 token operand of the same 128 K elements: up to 2 NT rows of 128
// bytes in the 128-byte swizzle, rows [0, n) the hi terms and [n, 2n) the lo
// terms of the tile's rows (n = rows rounded up to 16), written by the gather
// warps.  Tensor memory: kNBuf accumulators of 4 NT columns, box 0 (gate block,
// or the first w2 row block) at column 0 (hi terms in [0, n), lo in [n, 2n)),
// box 1 at column 2 NT.  After the routing tables, one fp32 row scale per row
// of the tile for each gather warp, then the T token maxima (64 words).
template <int NT>
struct F8Cfg {
    using C = FCfg<NT>;
    static constexpr int kBoxBytes = kBM * 2 * kBK;  // [128 rows x 128 codes]
    static constexpr int kABytes = 2 * kBoxBytes;
    static constexpr int kBBytes = 2 * NT * 2 * kBK;  // 2 NT rows x 128 codes
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kScaleBytes = kGatherWarps * NT * 4 + 64 * 4;  // + the x maxima
    static constexpr int kFixed = 1024 + C::kStagingBytes + C::kAuxBytes + kFusedReserve + kScaleBytes;
    static constexpr int kStagesRaw = (C::kMaxSmem - kFixed) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kG = kGatherWarps < kStages ? kGatherWarps : kStages;
    static constexpr int kW = kGatherWarps / kG;
    static constexpr int kAccCols = 4 * NT;
    static constexpr int kNBufRaw = 512 / kAccCols;
    static constexpr int kNBuf = kNBufRaw > 8 ? 8 : kNBufRaw;
    static constexpr int kTmemCols = 512;
    static constexpr uint32_t kTxBytes = kABytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kSmemBytes = kFixed + kRingBytes;
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kStages >= 3 && kStages <= kBarSlots, "pipeline depth");
    static_assert(kSmemBytes <= C::kMaxSmem, "shared memory");
    static_assert(kNBuf * kAccCols <= kTmemCols && kNBuf >= 2, "TMEM");
};

// The largest |x| of one token, published once per call by one CTA for all the
// others: `m` first, then `gen` (release).
struct XMax {
    unsigned long long gen;
    uint32_t m;
    uint32_t pad;
};

// ---- E4M3 token operand (F8).  A bf16 row v (x rows for w13, act rows for w2)
// is multiplied by 2^s, s chosen from the row's largest magnitude so that it
// lands in [128, 256), and written as two E4M3 terms: hi = e4m3(v 2^s) and
// lo = e4m3(v 2^s - hi), both rounded to nearest.  A bf16 value has 8
// significant bits and hi keeps the leading 4, so the remainder fits lo's 4
// significant bits: hi + lo is v 2^s exactly unless lo falls below E4M3's
// subnormal step 2^-9, which only entries under 2^-9 of the row's maximum can
// reach (error at most 2^-10 of the scaled unit, 2^-17 of the row maximum).
// The product of two E4M3 values is exact in fp32, so the MMA forms the bf16
// products and the epilogue multiplies (hi + lo) accumulators by 2^-s.

// s for a row whose largest |value| has fp32 bits m (a bf16 value): 7 - its
// exponent, within [-126, 126] so that 2^s and 2^-s are normal floats; 0 for a
// zero or non-finite row.
__device__ __forceinline__ int row_scale_exp(uint32_t m)
{
    if (m == 0u || m >= 0x7f800000u) return 0;
    const int e = (int)(m >> 23) - 127;
    return min(126, max(-126, 7 - e));
}
__device__ __forceinline__ float pow2f(int s) { return __int_as_float((s + 127) << 23); }
// 2^s, or NaN for a row holding inf or NaN: such a row's outputs are NaN.
__device__ __forceinline__ float row_scale(uint32_t m)
{
    return m >= 0x7f800000u ? __int_as_float(0x7fc00000) : pow2f(row_scale_exp(m));
}
__device__ __forceinline__ float row_descale(uint32_t m) { return pow2f(-row_scale_exp(m)); }

// e4m3(a) in the low byte, e4m3(b) in the high byte (round to nearest, finite).
__device__ __forceinline__ uint32_t e4m3x2_pack(float a, float b)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}
// The two E4M3 values of the low 16 bits of w (low byte first) as floats.
__device__ __forceinline__ float2 e4m3x2_unpack(uint32_t w)
{
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(w));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
// Four bf16 values (two words, element 0 in the low half of w0) times sc ->
// their E4M3 hi and lo terms, four codes per word (element 0 in the low byte).
__device__ __forceinline__ void split4(uint32_t w0, uint32_t w1, float sc, uint32_t& hi,
                                       uint32_t& lo)
{
    const float v0 = __uint_as_float(w0 << 16) * sc, v1 = __uint_as_float(w0 & 0xffff0000u) * sc;
    const float v2 = __uint_as_float(w1 << 16) * sc, v3 = __uint_as_float(w1 & 0xffff0000u) * sc;
    const uint32_t h01 = e4m3x2_pack(v0, v1), h23 = e4m3x2_pack(v2, v3);
    const float2 f01 = e4m3x2_unpack(h01), f23 = e4m3x2_unpack(h23);
    hi = h01 | (h23 << 16);
    lo = e4m3x2_pack(v0 - f01.x, v1 - f01.y) | (e4m3x2_pack(v2 - f23.x, v3 - f23.y) << 16);
}
// 16 bf16 values (K order) -> 16 hi codes and 16 lo codes.
__device__ __forceinline__ void split16(const uint4& a, const uint4& b, float sc, uint4& hi,
                                        uint4& lo)
{
    split4(a.x, a.y, sc, hi.x, lo.x);
    split4(a.z, a.w, sc, hi.y, lo.y);
    split4(b.x, b.y, sc, hi.z, lo.z);
    split4(b.z, b.w, sc, hi.w, lo.w);
}
// fp32 bits of the largest |value| among the 8 bf16 values of v, folded into m2
// (two 16-bit lanes).
__device__ __forceinline__ uint32_t absmax8(uint32_t m2, const uint4& v)
{
    m2 = __vmaxu2(m2, v.x & 0x7fff7fffu);
    m2 = __vmaxu2(m2, v.y & 0x7fff7fffu);
    m2 = __vmaxu2(m2, v.z & 0x7fff7fffu);
    return __vmaxu2(m2, v.w & 0x7fff7fffu);
}

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

// Bounded wait until CTA 0 has zeroed this call's arrival counters (*ready ==
// gen, read with acquire).  False on a timeout, a local abort or another CTA's
// recorded error.
__device__ __forceinline__ bool wait_counters(const FusedArgs& a, volatile int* abort)
{
    if (ld_acquire_gpu_u64(a.ready) == a.gen) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        __nanosleep(64);
        if (ld_acquire_gpu_u64(a.ready) == a.gen) return true;
        if (*abort || *reinterpret_cast<const volatile int32_t*>(a.err) == kDeviceErrorMagic ||
            globaltimer_ns() - t0 > 2000000000ull)
            return false;
    }
}

// F8: the largest |x| of token t published this call (fp32 bits, into m): a
// bounded wait for its generation word (acquire), then the value.  False on a
// timeout, a local abort or another CTA's recorded error.
__device__ __forceinline__ bool token_xmax(const FusedArgs& a, int t, volatile int* abort,
                                           uint32_t& m)
{
    const unsigned long long* g = &a.xmax[t].gen;
    if (ld_acquire_gpu_u64(g) != a.gen) {
        const uint64_t t0 = globaltimer_ns();
        for (;;) {
            __nanosleep(64);
            if (ld_acquire_gpu_u64(g) == a.gen) break;
            if (*abort || *reinterpret_cast<const volatile int32_t*>(a.err) == kDeviceErrorMagic ||
                globaltimer_ns() - t0 > 2000000000ull)
                return false;
        }
    }
    m = __ldcg(&a.xmax[t].m);
    return true;
}

// Routes the T tokens in this CTA (every thread calls; ends with a barrier).
// scratch: shared memory unused until the producer starts, at least
// kRouteScratchBytes.  The logits are staged in shared memory -- all T rows with
// one cooperative load when they fit in kStagedLogitBytes, else one row per warp
// at a time -- and each token is selected by one warp in two passes, as in the
// routing kernels: tau = the k-th largest of the 32 lanes' maxima; the experts
// whose logit reaches tau (usually about a dozen) are sorted by (logit desc,
// expert asc) and the first k kept, lane j holding the j-th (more than 32 such
// experts, from ties, or a small k over few experts: k rounds of warp arg-max
// instead).  The weights are those
// kernels' softmax, bit for bit.  Each selection sets bit t of its expert's
// 64-bit token mask (T <= 64).  Then one block scan gives the expert offsets and
// the tiles (touched experts in order), and every expanded row r = t k + j of
// expert e goes to offsets[e] + popc(mask[e] & (2^t - 1)): the stable order
// (ascending r within an expert, because an expert appears at most once per
// token), each row placed independently.  CTA 0 also writes the user-visible
// routing outputs.
constexpr int kStagedLogitBytes = 128 * 1024;
constexpr int kRouteScratchBytes =
    kStagedLogitBytes + kMaxExperts * 8 + (kMaxRows + 32) * 4 + 20 * 32 * 8;

// The two-pass selection; false (nothing selected) when more than 32 experts
// reach tau.
__device__ __forceinline__ bool select_by_threshold(const float* row, int E, int k, int lane,
                                                    float2* cand, float& my_l, int& my_e)
{
    const int M = (E + 31) / 32;  // slot m of lane l: expert 32 m + l
    float mv = -INFINITY;
    for (int m = 0; m < M; ++m) {
        const int e = m * 32 + lane;
        if (e < E) mv = fmaxf(mv, row[e]);
    }
    const float tau = warp_kth_largest(mv, k);
    uint32_t mask = 0;
    for (int m = 0; m < M; ++m) {
        const int e = m * 32 + lane;
        if (e < E && row[e] >= tau) mask |= 1u << m;
    }
    const int c = __popc(mask);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += n;
    }
    const int total = __shfl_sync(kFull, incl, 31);
    if (total > 32) return false;
    int pos = incl - c;
    while (mask) {
        const int m = __ffs(mask) - 1;
        mask &= mask - 1;
        const int e = m * 32 + lane;
        cand[pos++] = make_float2(row[e], __int_as_float(e));
    }
    __syncwarp();
    sort_candidates(total, lane, cand, my_l, my_e);
    return true;
}

__device__ __forceinline__ void select_token(const float* row, int E, int k, int lane,
                                             float2* cand, float& my_l, int& my_e)
{
    const int M = (E + 31) / 32;  // slot m of lane l: expert 32 m + l
    // few rounds over few slots (tiny layers): the k rounds of arg-max below are
    // the shorter dependency chain
    const bool rounds = k * (M + 10) <= 2 * M + 25;
    if (!rounds && select_by_threshold(row, E, k, lane, cand, my_l, my_e)) return;
    // k rounds of warp arg-max over the experts not yet taken (also the exact
    // fallback when more than 32 experts reach tau)
    uint32_t taken = 0;  // bit m: expert 32 m + lane already selected
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = kNoIndex;
        for (int m = 0; m < M; ++m) {  // experts ascend, so '>' keeps the lower one
            const int e = m * 32 + lane;
            if (e < E && !((taken >> m) & 1u)) {
                const float v = row[e];
                if (be == kNoIndex || v > bv) {
                    bv = v;
                    be = e;
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, off);
            const int oi = __shfl_xor_sync(kFull, be, off);
            if (key_before(ov, oi, bv, be)) {
                bv = ov;
                be = oi;
            }
        }
        if (lane == j) {
            my_l = bv;
            my_e = be;
        }
        if (be != kNoIndex && (be & 31) == lane) taken |= 1u << (be >> 5);
    }
}

__device__ __forceinline__ void route_tokens(const FusedArgs& a, RouteSmem* rs, uint8_t* scratch)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    float* logits_s = reinterpret_cast<float*>(scratch);
    unsigned long long* tmask =
        reinterpret_cast<unsigned long long*>(scratch + kStagedLogitBytes);  // [E]
    int* ids_s = reinterpret_cast<int*>(tmask + kMaxExperts);               // [R]
    int* sums = ids_s + kMaxRows;                                           // [32]
    float2* cand = reinterpret_cast<float2*>(sums + 32) + warp * 32;        // [warps][32]
    const int E = a.E, k = a.k;
    const bool all_rows = (long)a.T * E * 4 <= kStagedLogitBytes;
    for (int e = threadIdx.x; e < E; e += blockDim.x) tmask[e] = 0ull;
    if (all_rows) {
        const long n = (long)a.T * E;
        if ((E & 3) == 0) {
            for (long i = threadIdx.x; i < n / 4; i += blockDim.x)
                reinterpret_cast<float4*>(logits_s)[i] =
                    __ldg(reinterpret_cast<const float4*>(a.logits) + i);
        } else {
            for (long i = threadIdx.x; i < n; i += blockDim.x) logits_s[i] = __ldg(a.logits + i);
        }
    }
    __syncthreads();
    for (int t = warp; t < a.T; t += nwarps) {
        const float* row = logits_s + (size_t)t * E;
        if (!all_rows) {  // this warp's row buffer (E <= 1024 floats each)
            float* myrow = logits_s + (size_t)warp * kMaxExperts;
            const float* src = a.logits + (size_t)t * E;
            for (int e = lane; e < E; e += 32) myrow[e] = __ldg(src + e);
            __syncwarp();
            row = myrow;
        }
        float my_l = -INFINITY;
        int my_e = 0;
        select_token(row, E, k, lane, cand, my_l, my_e);
    const float w = softmax_weight(my_l, k, lane);
        if (lane < k) {
            const int r = t * k + lane;
            ids_s[r] = my_e;
            rs->w[r] = w;
            atomicOr(&tmask[my_e], 1ull << t);
            if (blockIdx.x == 0) {
                a.ids_out[r] = my_e;
                a.weights_out[r] = w;
            }
        }
        __syncwarp();  // the row buffer and cand are rewritten for the warp's next token
    }
    __syncthreads();
    // offsets and tiles in one scan: thread i owns experts 2 i and 2 i + 1
    // (blockDim >= E / 2); the low 16 bits count rows, the high ones tiles
    const int e0 = 2 * threadIdx.x, e1 = e0 + 1;
    const int c0 = e0 < E ? __popcll(tmask[e0]) : 0, c1 = e1 < E ? __popcll(tmask[e1]) : 0;
    int packed_total;
    const int packed = block_exclusive_scan((c0 + c1) | (((c0 > 0) + (c1 > 0)) << 16), sums,
                                            packed_total);
    const int base = packed & 0xffff, tbase = packed >> 16;
    if (e0 < E) {
        rs->off[e0] = (int16_t)base;
        if (c0) rs->tile_expert[tbase] = (int16_t)e0;
        if (blockIdx.x == 0) a.offsets_out[e0] = base;
    }
    if (e1 < E) {
        rs->off[e1] = (int16_t)(base + c0);
        if (c1) rs->tile_expert[tbase + (c0 > 0)] = (int16_t)e1;
        if (blockIdx.x == 0) a.offsets_out[e1] = base + c0;
    }
    if (threadIdx.x == 0) {
        rs->off[E] = (int16_t)(packed_total & 0xffff);
        rs->n_tiles = packed_total >> 16;
        if (blockIdx.x == 0) a.offsets_out[E] = packed_total & 0xffff;
    }
    __syncthreads();
    for (int r = threadIdx.x; r < a.R; r += blockDim.x) {
        const int e = ids_s[r], t = r / k;
        const int pos = rs->off[e] + __popcll(tmask[e] & ((1ull << t) - 1ull));
        rs->rows[pos] = (int16_t)r;
        if (blockIdx.x == 0) a.rows_out[pos] = r;
    }
    __syncthreads();
}

// F8: E4M3 weights (kind::f8f6f4 MMAs against the split E4M3 token operand);
// tm_w13 / tm_w2 then map E4M3 codes ([128 x 128]-byte boxes, 128-byte swizzle).
template <int NT, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    fused_ffn_kernel(const __grid_constant__ CUtensorMap tm_w13,
                     const __grid_constant__ CUtensorMap tm_w2,
                     const __grid_constant__ CUtensorMap tm_act, const FusedArgs a)
{
    using C = FCfg<NT>;
    using F8C = F8Cfg<NT>;
    static_assert(NT <= 64, "weight-streaming tiles");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* ring = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    // the ring (bf16: one 64-element K tile per stage; F8: two)
    constexpr int kStagesM = F8 ? F8C::kStages : C::kStages;
    constexpr int kStageBytesM = F8 ? F8C::kStageBytes : C::kStageBytes;
    constexpr int kGM = F8 ? F8C::kG : C::kG;  // gather groups and warps per group
    constexpr int kWM = F8 ? F8C::kW : C::kW;
    constexpr int kAccColsM = F8 ? F8C::kAccCols : C::kAccCols;  // per accumulator buffer
    constexpr int kRingBytes = kStagesM * kStageBytesM;
    constexpr int NBUF = F8 ? F8C::kNBuf : C::kNBuf;  // accumulator buffers
    constexpr int kTmemCols = F8 ? F8C::kTmemCols : C::kTmemCols;
    uint8_t* staging = ring + kRingBytes;
    Aux* aux = reinterpret_cast<Aux*>(staging + C::kStagingBytes);
    ComboScratch* combo = reinterpret_cast<ComboScratch*>(aux + 1);
    int* tok_off = reinterpret_cast<int*>(combo + 1);
    int4* unit_tab = reinterpret_cast<int4*>(reinterpret_cast<uint8_t*>(aux) + C::kAuxBytes);
    int* tab_seq = reinterpret_cast<int*>(unit_tab + 2 * kUnitTable);
    RouteSmem* rs = reinterpret_cast<RouteSmem*>(tab_seq + kUnitTable);
    float* cscale = reinterpret_cast<float*>(rs + 1);  // F8: [gather warps][NT] row scales
    uint32_t* xtab = reinterpret_cast<uint32_t*>(cscale + kGatherWarps * NT);  // F8: [T] max|x|
    // the routing scratch may run on into the epilogue staging that follows the ring
    static_assert(kRouteScratchBytes <= kRingBytes + C::kStagingBytes &&
                      kThreads / 32 * kMaxExperts * 4 <= kStagedLogitBytes && kThreads / 32 <= 20,
                  "routing scratch");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        {
            for (int s = 0; s < kStagesM; ++s) {
                mbar_init(&aux->full[s], 1 + kWM);
                mbar_init(&aux->empty[s], 1);
            }
        }
        for (int b = 0; b < NBUF; ++b) {
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
        tmem_alloc(&aux->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;

    // the inputs, and the workspace, once whatever ran before on the stream is done
    pdl_wait();
    pdl_launch_dependents();
    volatile int* abort_flag = &aux->abort;
    // CTA 0 zeroes the arrival counters and publishes this call's generation; every
    // role waits for it (wait_counters) before its first counter access, which
    // comes after at least one unit of work
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < a.n_counters; i += blockDim.x) a.tile_ready[i] = 0;
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            st_release_gpu_u64(a.ready, a.gen);
        }
    }
    route_tokens(a, rs, ring);  // ring and staging are free until the first load / unit

    const int ntiles = rs->n_tiles;
    // w13 is not split here: its epilogue writes bf16 act directly, which each w2
    // stage then loads with one TMA.  w2 is split only as far as ~4 waves of units
    // need: the run-time hand-out already balances the tail, and every extra
    // slice adds epilogue publishes and combine reads (same-B200 A/B: 16 waves
    // 101.4 us decode / 360.7 us skewed decode, 4 waves 98.2 / 341.8).  E4M3
    // units stream half the bytes, so ~2 waves (decode with E4M3 weights: 4 waves
    // 68.9 us, 2 waves 66.5 us, 1 wave 66.4 us; skewed decode unchanged); bf16 units
    // keep 4 (2 waves: decode 100.6 -> 101.8 us).
    const int s2w = split_count(ntiles * a.fb2, a.s2_max, a.kt2, a.min_kt_per_split, F8 ? 2 : 4);
    int ktps2 = (a.kt2 + s2w - 1) / s2w;
    if (F8) ktps2 = (ktps2 + 1) & ~1;  // whole pair stages
    const int S2 = (a.kt2 + ktps2 - 1) / ktps2;  // every slice non-empty
    const int U13 = ntiles * a.fb13;
    const int U2 = ntiles * a.fb2 * S2;
    const int tile_target = 2 * a.fb13;  // two epilogue groups per w13 unit
    const int token_target = a.k * S2;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        a.split_out[0] = 1;
        a.split_out[1] = S2;
    }

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
        // one tile per expert: tile-major, feature block minor
        un.tile = rest / fbc;
        un.fb = rest % fbc;
        un.kt0 = un.split * ktps;
        un.kt1 = min(nkt, un.kt0 + ktps);
        un.expert = rs->tile_expert[un.tile];
        un.row_start = rs->off[un.expert];
        un.rows = rs->off[un.expert + 1] - un.row_start;
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
    // than its ring stages plus the accumulator buffers in units, far below the
    // ring's length.
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
            // F8: the single ring, two E4M3 boxes per stage
            constexpr int NS = kStagesM;
            constexpr int kStBytes = kStageBytesM;
            constexpr int kBox1 = F8 ? kBM * 2 * kBK : kATileBytes;  // second box
            constexpr int kKtStep = F8 ? 2 : 1;  // K tiles per ring stage
            constexpr uint32_t kTx = F8 ? F8C::kTxBytes : C::kTxBytes;
            uint8_t* const pring = ring;
            int stage = 0;
            uint32_t phase = 0;
            int fills = 0;  // ring stage fills so far (fill q went to stage q % stages)
            bool ok = true;
            bool counters = false;  // this call's counters are zeroed (wait_counters)
            for (int i = 0; ok; ++i) {
                Unit un;
                if (i < n_static) {
                    un = get(i);
                } else {  // claim the next w2 unit and publish it to the other roles
                    if (!counters && !(counters = wait_counters(a, abort_flag))) {
                        flag_error(a.err, aux);
                        break;
                    }
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
                for (int kt = un.kt0; kt < un.kt1; kt += kKtStep) {
                    if (!mbar_wait(&aux->empty[stage], phase ^ 1u, abort_flag)) {
                        flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    uint8_t* st = pring + stage * kStBytes;
                    mbar_arrive_expect_tx(&aux->full[stage], kTx);
                    tma_load_2d(st, tm, &aux->full[stage], kt * kBK, row0, pol);
                    tma_load_2d(st + kBox1, tm, &aux->full[stage], kt * kBK, row1, pol);
                    ++fills;
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok || *abort_flag) {
                // let every TMA load already issued land before the CTA can exit
                for (int s = 0; s < NS; ++s) {
                    const int n_s = fills > s ? (fills - s + NS - 1) / NS : 0;  // fills of stage s
                    if (n_s > 0) {
                        volatile int never = 0;
                        mbar_wait(&aux->full[s], (uint32_t)((n_s - 1) & 1), &never,
                                  500000000ull);
                    }
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
                const int b = lu % NBUF;
                const uint32_t aphase = (uint32_t)((lu / NBUF) & 1);
                if (!mbar_wait(&aux->tempty[b], aphase ^ 1u, abort_flag)) {
                    flag_error(a.err, aux);
                    break;
                }
                tc_fence_after();
                const int n = (t.rows + 15) & ~15;
                // F8: hi and lo terms of the n token rows make the MMA's 2 n columns
                const uint32_t idesc = F8 ? umma_idesc_e4m3(kBM, 2 * n) : umma_idesc_bf16(kBM, n);
                const uint32_t d0 = tmem_base + (uint32_t)(b * kAccColsM);
                for (int kt = un.kt0; kt < un.kt1; kt += (F8 ? 2 : 1)) {
                    uint32_t st, bt;
                    {
                        if (!mbar_wait(&aux->full[stage], phase, abort_flag)) {
                            flag_error(a.err, aux);
                            ok = false;
                            break;
                        }
                        st = smem_u32(ring + stage * kStageBytesM);
                        bt = st + (F8 ? F8C::kABytes : C::kNA * kATileBytes);
                    }
                    tc_fence_after();
                    if constexpr (F8) {
                        // 128 K codes per stage, 32 per MMA: both boxes against the
                        // same token operand
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (kt > un.kt0 || kk > 0) ? 1u : 0u;
                            const uint64_t bdesc = umma_desc_sw128(bt + kk * 32);
                            umma_e4m3(d0, umma_desc_sw128(st + kk * 32), bdesc, idesc, acc);
                            umma_e4m3(d0 + 2 * NT, umma_desc_sw128(st + F8C::kBoxBytes + kk * 32),
                                      bdesc, idesc, acc);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                            const uint32_t acc = (kt > un.kt0 || kk > 0) ? 1u : 0u;
                            const uint64_t bdesc = umma_desc_sw128(bt + kk * 32);
                            umma_bf16(d0, umma_desc_sw128(st + kk * 32), bdesc, idesc, acc);
                            umma_bf16(d0 + NT, umma_desc_sw128(st + kATileBytes + kk * 32), bdesc,
                                      idesc, acc);
                        }
                    }
                    umma_commit(&aux->empty[stage]);  // frees the smem stage when read
                    if (++stage == kStagesM) {
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
        if (F8 && warp - 2 < kGM * kWM) {
            // F8: the E4M3 token operand.  Group g (W warps) fills stages g, g + G,
            // ... of the ring: per stage, each row's 128 bf16 values (x for w13,
            // act for w2) scaled by its row's 2^s and split into hi and lo codes,
            // stored into the stage's B rows j and n + j (128-byte swizzle); then
            // a proxy fence and one arrival per warp.
            constexpr int G = kGM, W = kWM;
            const int g = (warp - 2) / W, wi = (warp - 2) % W;
            int* my_off = tok_off + (warp - 2) * NT;   // w13: element offset of each x row
            float* my_sc = cscale + (warp - 2) * NT;   // 2^s of each row
            // x and act rows are re-read by every feature block's unit: keep them in
            // L2 while the weight stream (evict-first) passes through
            const uint64_t keep = l2_policy_evict_last();
            int q = 0;  // global stage sequence number (same as the producer's)
            int cur_tile = -1, cur_ph = -1, ready_tile = -1;
            bool ok = true;
            bool counters = false;
            bool have_x = false;  // xtab filled (at the first w13 tile)
            for (int i = 0; ok; ++i) {
                const Unit un = get(i);
                if (__any_sync(0xffffffffu, un.ph >= kUnitEnd)) break;
                const int nst = (un.kt1 - un.kt0) >> 1;  // pair stages of the unit
                int sidx = ((g - q % G) + G) % G;       // first one this group owns
                const int q_unit0 = q;
                q += nst;
                if (sidx >= nst) continue;
                const Unit& t = un;
                if (un.ph == 1 && un.tile != ready_tile) {
                    // every w13 unit of this tile has stored its act rows and maxima
                    if ((!counters &&
                         !(counters = __all_sync(0xffffffffu, wait_counters(a, abort_flag)))) ||
                        !warp_wait_count(a.tile_ready + un.tile, tile_target, abort_flag, a.err)) {
                        if (lane == 0) flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    ready_tile = un.tile;
                }
                if (un.ph == 0 && !have_x) {
                    // every token's published max|x|, all at once, into a table in
                    // shared memory (each gather warp writes the same values, and
                    // reads only after its own writes)
                    bool got = true;
                    for (int tk = lane; tk < a.T; tk += 32) {
                        uint32_t m = 0;
                        got = token_xmax(a, tk, abort_flag, m) && got;
                        xtab[tk] = m;
                    }
                    if (__any_sync(0xffffffffu, !got)) {
                        if (lane == 0) flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    have_x = true;
                }
                if (un.tile != cur_tile || un.ph != cur_ph) {
                    __syncwarp();  // the previous tile's rows are all converted
                    bool got = true;
                    for (int j = lane; j < t.rows; j += 32) {
                        uint32_t m = 0;
                        if (un.ph == 0) {
                            const int tok = rs->rows[t.row_start + j] / a.k;
                            my_off[j] = tok * a.H;
                            m = xtab[tok];
                        } else {
                            m = (uint32_t)ld_acquire_gpu(
                                reinterpret_cast<const int*>(a.act_max) + t.row_start + j);
                        }
                        my_sc[j] = row_scale(m);
                    }
                    if (__any_sync(0xffffffffu, !got)) {
                        if (lane == 0) flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    cur_tile = un.tile;
                    cur_ph = un.ph;
                }
                const int n = (t.rows + 15) & ~15;
                const int ntask = t.rows * 8;  // (row, 16-element chunk) pairs
                for (; sidx < nst; sidx += G) {
                    const int qq = q_unit0 + sidx;
                    const int stage = qq % kStagesM;
                    const uint32_t phase = (uint32_t)((qq / kStagesM) & 1);
                    if (!__all_sync(0xffffffffu, mbar_wait(&aux->empty[stage], phase ^ 1u,
                                                           abort_flag))) {
                        if (lane == 0) flag_error(a.err, aux);
                        ok = false;
                        break;
                    }
                    uint8_t* btile = ring + stage * kStageBytesM + F8C::kABytes;
                    const int kt = un.kt0 + 2 * sidx;  // the stage's first K tile
                    // four tasks per lane in flight: loads first, then the splits
                    for (int base = lane + 32 * wi; base < ntask; base += 4 * 32 * W) {
                        uint4 v[4][2];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int c8 = base + u * 32 * W;
                            if (c8 < ntask) {
                                const int j = c8 >> 3, c = c8 & 7;
                                const uint4* src =
                                    un.ph == 0
                                        ? reinterpret_cast<const uint4*>(a.x + my_off[j] + kt * kBK +
                                                                         c * 16)
                                        // act, K-blocked: block kt + c / 4, elements (c % 4) * 16 ..
                                        : reinterpret_cast<const uint4*>(
                                              a.act + ((size_t)(kt + (c >> 2)) * a.R + t.row_start + j) *
                                                          kBK +
                                              (c & 3) * 16);
                                v[u][0] = ldcg_hint_v4(src, keep);
                                v[u][1] = ldcg_hint_v4(src + 1, keep);
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int c8 = base + u * 32 * W;
                            if (c8 < ntask) {
                                const int j = c8 >> 3, c = c8 & 7, jl = n + j;
                                uint4 hi, lo;
                                split16(v[u][0], v[u][1], my_sc[j], hi, lo);
                                *reinterpret_cast<uint4*>(btile + j * 128 + ((c ^ (j & 7)) << 4)) = hi;
                                *reinterpret_cast<uint4*>(btile + jl * 128 + ((c ^ (jl & 7)) << 4)) = lo;
                            }
                        }
                    }
                    fence_proxy_async_smem();  // generic stores, read by the MMA
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&aux->full[stage]);
                }
            }
        } else if (!F8 && warp - 2 < C::kG * C::kW) {
            constexpr int G = C::kG, W = C::kW;
            const int g = (warp - 2) / W, wi = (warp - 2) % W;
            int* my_off = tok_off + (warp - 2) * NT;
            const uint64_t keep = l2_policy_evict_last();  // x / act rows are re-read per block
            int q = 0;  // global stage sequence number (same as the producer's)
            int cur_tile = -1, cur_ph = -1, ready_tile = -1;
            bool ok = true;
            bool counters = false;
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
                    if ((!counters &&
                         !(counters = __all_sync(0xffffffffu, wait_counters(a, abort_flag)))) ||
                        !warp_wait_count(a.tile_ready + un.tile, tile_target, abort_flag, a.err)) {
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
                            my_off[j] = (rs->rows[t.row_start + j] / a.k) * a.H;
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
        if constexpr (F8) {
            // publish the largest |x| of tokens b, b + G, ... for every CTA's token
            // operand (first thing, so no CTA waits long for it): all eight warps
            // read the row, reduce, and one thread writes the value, then the
            // call's generation with release
            const int et = threadIdx.x - kEpiWarp0 * 32;  // 0..255
            uint32_t* red = reinterpret_cast<uint32_t*>(staging);
            const uint64_t keep = l2_policy_evict_last();  // the gather re-reads x from L2
            for (int tk = blockIdx.x; tk < a.T; tk += gridDim.x) {
                const uint4* row = reinterpret_cast<const uint4*>(a.x + (size_t)tk * a.H);
                uint32_t m2 = 0;
                for (int i = et; i < a.H / 8; i += 256) m2 = absmax8(m2, ldcg_hint_v4(row + i, keep));
                const uint32_t m = __reduce_max_sync(0xffffffffu, max(m2 & 0xffffu, m2 >> 16) << 16);
                if (lane == 0) red[warp - kEpiWarp0] = m;
                named_bar_sync(3, 256);
                if (et == 0) {
                    uint32_t mm = 0;
                    for (int w = 0; w < 8; ++w) mm = max(mm, red[w]);
                    a.xmax[tk].m = mm;
                    st_release_gpu_u64(&a.xmax[tk].gen, a.gen);
                }
                named_bar_sync(3, 256);  // red is rewritten for the next token
            }
        }
        // every epilogue thread publishes to (or waits on) the counters: before its
        // first unit's accumulator is even ready, CTA 0 has long zeroed them (the
        // outcome is made the same in all four warps of the group)
        const bool counters = !named_bar_or(1 + grp, 128, !wait_counters(a, abort_flag));
        if (!counters) flag_error(a.err, aux);
        for (int lu = 0; counters; ++lu) {
            const Unit un = get(lu);
            const Unit& t = un;
            const int b = lu % NBUF;
            const uint32_t aphase = (uint32_t)((lu / NBUF) & 1);
            // F8: this thread's two weight-row scales (gate and up rows, or output
            // features f and f + 128), loaded before the accumulator wait
            float sc0 = 1.f, sc1 = 1.f;
            if constexpr (F8) {
                if (un.ph == 0) {
                    const float* sp = a.s13 + (size_t)un.expert * 2 * a.I + un.fb * kBM + f_local;
                    sc0 = __ldg(sp);
                    sc1 = __ldg(sp + a.I);
                } else if (un.ph == 1) {
                    const int f2 = un.fb * 2 * kBM + f_local;
                    const float* sp = a.s2 + (size_t)un.expert * a.H + f2;
                    sc0 = __ldg(sp);
                    if (f2 + kBM < a.H) sc1 = __ldg(sp + kBM);
                }
            }
            // F8: 2^-s of the token column jbeg + lane of this group, each lane
            // loading one column's maximum (all at once; the chunks below take
            // theirs by shuffle).  w13: the tokens' published x maxima, fetched
            // while the MMAs run; w2: the act maxima, complete once this unit's
            // operand was built, so fetched after the accumulator wait.
            float my_ds = 1.f;
            auto load_ds = [&](int ph_) {
                const int j = grp * (NT / 2) + lane;
                uint32_t m = 0;
                if (j < min(t.rows, (grp + 1) * (NT / 2))) {
                    if (ph_ == 0) {
                        if (!token_xmax(a, rs->rows[t.row_start + j] / a.k, abort_flag, m))
                            flag_error(a.err, aux);
                    } else {
                        m = (uint32_t)ld_acquire_gpu(reinterpret_cast<const int*>(a.act_max) +
                                                     t.row_start + j);
                    }
                }
                my_ds = row_descale(m);
            };
            if (F8 && un.ph == 0) load_ds(0);
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
            const uint32_t tacc = tmem_base + ((uint32_t)(qw * 32) << 16) + (uint32_t)(b * kAccColsM);
            const int jbeg = grp * (NT / 2), jend = min(t.rows, (grp + 1) * (NT / 2));
            // F8: the lo terms' columns start at n; the second box's at 2 NT
            const int n8 = (t.rows + 15) & ~15;
            constexpr uint32_t kBox1Col = F8 ? 2 * NT : NT;
            if (F8 && ph == 1) load_ds(1);
            // 2^-s of column j of the group (lanes hold them; all lanes call)
            auto col_descale = [&](int j) -> float {
                return __shfl_sync(0xffffffffu, my_ds, (j - jbeg) & 31);
            };
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
                    if constexpr (F8) {
                        uint32_t gl[8], vl[8];
                        float ds[kStageRows];
#pragma unroll
                        for (int jj = 0; jj < kStageRows; ++jj) ds[jj] = col_descale(j0 + jj);
                        tmem_ld8(tacc + j0, gv);
                        tmem_ld8(tacc + n8 + j0, gl);
                        tmem_ld8(tacc + kBox1Col + j0, vv);
                        tmem_ld8(tacc + kBox1Col + n8 + j0, vl);
                        tmem_ld_wait();
#pragma unroll
                        for (int jj = 0; jj < kStageRows; ++jj) {
                            const float g = __uint_as_float(gv[jj]) + __uint_as_float(gl[jj]);
                            const float u = __uint_as_float(vv[jj]) + __uint_as_float(vl[jj]);
                            gv[jj] = __float_as_uint(g * ds[jj] * sc0);
                            vv[jj] = __float_as_uint(u * ds[jj] * sc1);
                        }
                    } else {
                        tmem_ld8(tacc + j0, gv);
                        tmem_ld8(tacc + NT + j0, vv);
                        tmem_ld_wait();
                    }
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
                            const __nv_bfloat16 av = __float2bfloat16_rn(
                                silu_mul(__uint_as_float(gv[jj]), __uint_as_float(vv[jj])));
                            row[f_local] = av;
                            if constexpr (F8) {  // the row's largest |act|, for w2's operand
                                const uint32_t m = __reduce_max_sync(
                                    0xffffffffu, ((uint32_t)__bfloat16_as_ushort(av) & 0x7fffu) << 16);
                                if (lane == 0 && j0 + jj < jend)
                                    atomicMax(a.act_max + t.row_start + j0 + jj, m);
                            }
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
                            : a.y + (size_t)rs->rows[p] * a.H + un.fb * 2 * kBM + c * 8;
                        *reinterpret_cast<uint4*>(dst) = val;
                    }
                    ++chunk;
                }
            } else {
                constexpr int kCols = kEpiCols<NT>;
                for (int j0 = jbeg; j0 < jend; j0 += kCols) {
                    uint32_t gv[kCols], vv[kCols];
                    if constexpr (F8) {
                        uint32_t gl[kCols], vl[kCols];
                        tmem_ld_cols(tacc + j0, gv);
                        tmem_ld_cols(tacc + n8 + j0, gl);
                        tmem_ld_cols(tacc + kBox1Col + j0, vv);
                        tmem_ld_cols(tacc + kBox1Col + n8 + j0, vl);
                        tmem_ld_wait();
#pragma unroll
                        for (int jj = 0; jj < kCols; ++jj) {
                            const float ds = col_descale(j0 + jj);
                            gv[jj] = __float_as_uint((__uint_as_float(gv[jj]) + __uint_as_float(gl[jj])) * ds);
                            vv[jj] = __float_as_uint((__uint_as_float(vv[jj]) + __uint_as_float(vl[jj])) * ds);
                        }
                    } else {
                        tmem_ld_cols(tacc + j0, gv);
                        tmem_ld_cols(tacc + NT + j0, vv);
                        tmem_ld_wait();
                    }
#pragma unroll
                    for (int jj = 0; jj < kCols; ++jj) {
                        const int j = j0 + jj;
                        if (j >= jend) break;
                        const int p = t.row_start + j;
                        {  // w2 slice: fp32 by expanded id
                            const int r = rs->rows[p];
                            float* prow = a.part2 + ((size_t)un.split * a.R + r) * a.H;
                            float g0 = __uint_as_float(gv[jj]), g1 = __uint_as_float(vv[jj]);
                            if constexpr (F8) {
                                g0 *= sc0;
                                g1 *= sc1;
                            }
                            prow[f] = g0;
                            if (f1_ok) prow[f + kBM] = g1;
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
                const int tok = rs->rows[t.row_start + jbeg + gt] / a.k;
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
                if (ready && lane < a.k) combo->w[lane] = rs->w[tok * a.k + lane];
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
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int NT, bool F8>
cudaError_t launch_fused_nt(const CUtensorMap& t13, const CUtensorMap& t2, const CUtensorMap& ta,
                            const FusedArgs& a, int grid, cudaStream_t st)
{
    using C = FCfg<NT>;
    // the combine's weights sit in the slack Cfg reserves next to Aux; the unit
    // table and the routing tables follow the aux area
    static_assert(sizeof(Aux) + sizeof(ComboScratch) <= 1024, "aux area");
    static_assert(C::kAuxBytes % 16 == 0 && kUnitTableBytes % 16 == 0, "table alignment");
    constexpr int smem = F8 ? F8Cfg<NT>::kSmemBytes : C::kSmemBytes + kFusedReserve;
    static_assert(smem <= C::kMaxSmem, "shared memory");
    auto kern = fused_ffn_kernel<NT, F8>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, t13, t2, ta, a);
}

}  // namespace

bool fused_ffn_eligible(int T, int E, int k, int H, int I, const FfnPlan& plan)
{
    (void)H;
    (void)I;
    // every expert's rows in one tile (plan.nt >= T), and the routing tables fit
    return plan.nt <= 64 && plan.nt >= T && (long)T * k <= kMaxRows && k <= kMaxK &&
           E <= kMaxExperts && plan.s2_max <= kMaxSplits;
}

int fused_ffn_counters(int T, int k, int H, const FfnPlan& plan)
{
    // tile_ready, token_ready, w2_next, then (E4M3 weights) act_max
    return plan.max_tiles + T * ((H / kBM + 1) / 2) + 1 + T * k;
}

cudaError_t launch_fused_ffn(const FusedBuffers& b, int T, int E, int k, int H, int I,
                             const FfnPlan& plan, cudaStream_t st)
{
    const int R = T * k;
    const bool w8 = b.s13 != nullptr;
    CUtensorMap t13, t2, ta;
    // E4M3 codes: [128 rows x 128 bytes] boxes (two K tiles), 128-byte swizzle
    cudaError_t err = w8 ? make_tmap_u8(&t13, b.w13, (uint64_t)E * 2 * I, (uint64_t)H, kBM, 2 * kBK)
                         : make_tmap(&t13, b.w13, (uint64_t)E * 2 * I, (uint64_t)H, kBM);
    if (err == cudaSuccess)
        err = w8 ? make_tmap_u8(&t2, b.w2, (uint64_t)E * H, (uint64_t)I, kBM, 2 * kBK)
                 : make_tmap(&t2, b.w2, (uint64_t)E * H, (uint64_t)I, kBM);
    // act, K-blocked: (I / 64) * R rows of 64 columns, NT-row boxes
    if (err == cudaSuccess)
        err = make_tmap(&ta, b.act, (uint64_t)(I / kBK) * R, (uint64_t)kBK, (uint32_t)plan.nt);
    if (err != cudaSuccess) return err;
    FusedArgs a = {};
    a.x = static_cast<const __nv_bfloat16*>(b.x);
    a.logits = b.logits;
    a.ids_out = b.topk_ids;
    a.weights_out = b.topk_weights;
    a.offsets_out = b.expert_offsets;
    a.rows_out = b.permuted_rows;
    a.act = static_cast<__nv_bfloat16*>(b.act);
    a.part2 = b.part2;
    a.y = static_cast<__nv_bfloat16*>(b.y);
    a.out = static_cast<__nv_bfloat16*>(b.out);
    a.tile_ready = b.counters;
    a.token_ready = b.counters + plan.max_tiles;
    a.w2_next = a.token_ready + (size_t)T * ((H / kBM + 1) / 2);
    a.act_max = reinterpret_cast<uint32_t*>(a.w2_next + 1);
    a.n_counters = fused_ffn_counters(T, k, H, plan);
    a.xmax = static_cast<XMax*>(b.xmax);
    a.ready = b.ready;
    a.gen = b.gen;
    a.split_out = b.splits;
    a.err = b.err;
    a.T = T;
    a.E = E;
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
    a.s13 = b.s13;
    a.s2 = b.s2;
    // no more CTAs than the most units one phase can have: a small layer (tiny: 32
    // w13 units) would otherwise launch idle CTAs that still set up and route
    const long long tiles_max = E < R ? E : R;
    long long units = tiles_max * a.fb13;
    units = units > tiles_max * a.fb2 * plan.s2_max ? units : tiles_max * a.fb2 * plan.s2_max;
    units = units > (long long)T * a.fb2 ? units : (long long)T * a.fb2;
    const int grid = (int)(units < plan.grid ? units : plan.grid);
    switch (plan.nt * 2 + (w8 ? 1 : 0)) {
    case 32: return launch_fused_nt<16, false>(t13, t2, ta, a, grid, st);
    case 64: return launch_fused_nt<32, false>(t13, t2, ta, a, grid, st);
    case 128: return launch_fused_nt<64, false>(t13, t2, ta, a, grid, st);
    case 33: return launch_fused_nt<16, true>(t13, t2, ta, a, grid, st);
    case 65: return launch_fused_nt<32, true>(t13, t2, ta, a, grid, st);
    case 129: return launch_fused_nt<64, true>(t13, t2, ta, a, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
