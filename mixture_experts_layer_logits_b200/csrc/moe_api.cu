// moe_api.cu -- the C ABI declared in include/moe.h: host-side validation,
// workspace layout, the per-shape plan, and the stream-ordered launch chain
//   route (+ permute) -> [permute] -> w13/SwiGLU -> w2 -> combine
// with programmatic dependent launch between consecutive kernels.
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <random>

#include "gemm_common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

bool pdl_enabled()
{
    static const bool on = [] {
        const char* v = getenv("MOE_DISABLE_PDL");
        return !(v && v[0] && v[0] != '0');
    }();
    return on;
}

bool fused_enabled()
{
    static const bool on = [] {
        const char* v = getenv("MOE_DISABLE_FUSED");
        return !(v && v[0] && v[0] != '0');
    }();
    return on;
}

namespace {
thread_local int g_last_cuda_error = 0;
}  // namespace

void set_last_cuda_error(int err) { g_last_cuda_error = err; }

bool routing_shape_ok(const moe_shape_t& s)
{
    if (s.T < 1 || s.E < 1 || s.E > 1024 || s.top_k < 1 || s.top_k > 16 || s.top_k > s.E)
        return false;
    return (long long)s.T * s.top_k <= (1LL << 30);
}

namespace {

// Plans and workspaces are sized for the B200's SM count; the launch grid uses
// the actual device's.
constexpr int kSizingSms = 148;

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ffn_shape_ok(const moe_shape_t& s)
{
    if (!routing_shape_ok(s)) return false;
    if (s.H < 128 || s.I < 128 || s.H % 128 || s.I % 128) return false;
    const long long R = (long long)s.T * s.top_k;
    if ((long long)s.T * s.H > INT_MAX) return false;             // token row offsets
    if ((long long)s.E * 2 * s.I > INT_MAX) return false;         // TMA row coordinates
    if ((long long)s.E * s.H > INT_MAX) return false;
    if (R * (long long)s.H > (1LL << 40) || R * (long long)s.I > (1LL << 40)) return false;
    return true;
}

bool combine_shape_ok(const moe_shape_t& s)
{
    if (s.T < 1 || s.top_k < 1 || s.top_k > 16 || s.H < 128 || s.H % 128) return false;
    return (long long)s.T * s.top_k <= (1LL << 30) && (long long)s.T * s.top_k * s.H <= (1LL << 40);
}

struct Layout {
    size_t err, ids, weights, offsets, rows, tiles, num_tiles, splits, chunks, bar, partials, act,
        y, partials2, counters, ready, xmax, total;
    int max_chunks;  // chunk rows of the multi-CTA permutation's count table
    FfnPlan plan;
    bool ffn;
    bool fused;      // the shape qualifies for the one-launch FFN + combine
    int n_counters;  // its arrival counters (zeroed by its own CTA 0 every call)
};

Layout layout_for(const moe_shape_t& s)
{
    Layout L = {};
    const size_t R = (size_t)s.T * s.top_k;
    L.ffn = s.H > 0 || s.I > 0;
    const int H = L.ffn ? s.H : 128, I = L.ffn ? s.I : 128;
    L.plan = plan_ffn(s.T, s.E, s.top_k, H, I, kSizingSms);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes);
        return at;
    };
    L.err = take(sizeof(int32_t));
    L.ids = take(R * sizeof(int32_t));
    L.weights = take(R * sizeof(float));
    L.offsets = take((size_t)(s.E + 1) * sizeof(int32_t));
    L.rows = take(R * sizeof(int32_t));
    L.tiles = take((size_t)L.plan.max_tiles * sizeof(Tile));
    L.num_tiles = take(sizeof(int32_t));
    L.splits = take(2 * sizeof(int32_t));
    // multi-CTA permutation: per-chunk expert counts (then prefixes over the
    // chunks), one row of expert totals, and its grid barrier
    L.max_chunks = R > (size_t)kSmallRows ? kSizingSms : 0;
    L.chunks = take((size_t)(L.max_chunks + 1) * s.E * sizeof(int32_t));
    L.bar = take(sizeof(GridBar));
    if (L.ffn) {
        size_t p13 = L.plan.s13_max > 1 ? (size_t)L.plan.s13_max * R * 2 * I : 0;
        size_t p2 = L.plan.s2_max > 1 ? (size_t)L.plan.s2_max * R * H : 0;
        L.partials = take((p13 > p2 ? p13 : p2) * sizeof(float));
        const size_t act_rows = R > (size_t)L.plan.nt ? R : (size_t)L.plan.nt;
        L.act = take(act_rows * I * 2);
        L.y = take(R * H * 2);
        // the fused launch keeps w13's and w2's slices live at once
        L.fused = fused_ffn_eligible(s.T, s.E, s.top_k, H, I, L.plan);
        if (L.fused) {
            L.partials2 = take(p2 * sizeof(float));
            L.n_counters = fused_ffn_counters(s.T, s.top_k, H, L.plan);
            L.counters = take((size_t)L.n_counters * sizeof(int32_t));
            L.ready = take(sizeof(unsigned long long));
            L.xmax = take((size_t)s.T * 16);
        }
    }
    L.total = off;
    return L;
}

template <typename T>
T* at(void* ws, size_t off)
{
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace

int device_sms()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kSizingSms;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = kSizingSms;
        cached[dev] = n;
    }
    return cached[dev];
}

namespace {

moe_status_t cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return MOE_OK;
    g_last_cuda_error = (int)e;
    return MOE_ERR_CUDA;
}

}  // namespace

unsigned long long next_generation()
{
    static std::atomic<unsigned long long> counter{[] {
        std::random_device rd;
        return ((unsigned long long)rd() << 32) ^ rd() ^
               (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
    }()};
    return counter.fetch_add(0x9E3779B97F4A7C15ull) + 0x9E3779B97F4A7C15ull;
}

namespace {

PermuteAux make_aux(void* ws, const Layout& L, const moe_shape_t& s)
{
    PermuteAux a;
    a.tiles = at<Tile>(ws, L.tiles);
    a.num_tiles = at<int32_t>(ws, L.num_tiles);
    a.nt = L.plan.nt;
    a.err = at<int32_t>(ws, L.err);
    a.max_tiles = L.plan.max_tiles;
    a.chunk_counts = at<int32_t>(ws, L.chunks);
    a.max_chunks = L.max_chunks;
    a.bar = at<GridBar>(ws, L.bar);
    a.gen = next_generation();
    (void)s;
    return a;
}

moe_status_t run_permute(const float* logits, int32_t* ids, float* weights, const moe_shape_t& s,
                         int32_t* offsets, int32_t* rows, void* ws, const Layout& L,
                         cudaStream_t st)
{
    PermuteAux aux = make_aux(ws, L, s);
    const long R = (long)s.T * s.top_k;
    cudaError_t e;
    if (R <= kSmallRows) {
        e = launch_small_route_permute(logits, s.T, s.E, s.top_k, ids, weights, offsets, rows, aux,
                                       st);
    } else {
        e = cudaSuccess;
        if (logits) e = launch_route(logits, s.T, s.E, s.top_k, ids, weights, st);
        if (e == cudaSuccess) e = launch_large_permute(ids, s.T, s.E, s.top_k, offsets, rows, aux, st);
    }
    return cuda_status(e);
}

moe_status_t run_ffn(const void* x, const void* w13, const void* w2, const int32_t* rows,
                     const moe_shape_t& s, void* y, void* ws, const Layout& L, cudaStream_t st,
                     void* const* mid_event = nullptr, bool reduce_y = true)
{
    FfnBuffers b;
    b.x = x;
    b.w13 = w13;
    b.w2 = w2;
    b.permuted_rows = rows;
    b.tiles = at<Tile>(ws, L.tiles);
    b.num_tiles = at<int32_t>(ws, L.num_tiles);
    b.act = at<void>(ws, L.act);
    b.y = y;
    b.partials = at<float>(ws, L.partials);
    b.splits = at<int32_t>(ws, L.splits);
    b.err = at<int32_t>(ws, L.err);
    FfnPlan plan = L.plan;
    plan.grid = device_sms();
    return cuda_status(launch_grouped_ffn(
        b, s.T, s.E, s.top_k, s.H, s.I, plan, st,
        mid_event ? static_cast<cudaEvent_t>(mid_event[0]) : nullptr, reduce_y));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(moe_shape_t s)
{
    const bool routing_only = s.H == 0 && s.I == 0;
    if (routing_only ? !routing_shape_ok(s) : !ffn_shape_ok(s)) return 0;
    return layout_for(s).total;
}

moe_status_t moe_route(const float* logits, moe_shape_t s, int32_t* topk_ids, float* topk_weights,
                       moe_stream_t stream)
{
    if (!logits || !topk_ids || !topk_weights) return MOE_ERR_INVALID_ARG;
    if (!routing_shape_ok(s)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_weights))
        return MOE_ERR_MISALIGNED;
    return cuda_status(launch_route(logits, s.T, s.E, s.top_k, topk_ids, topk_weights,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_permute(const int32_t* topk_ids, moe_shape_t s, int32_t* expert_offsets,
                         int32_t* permuted_rows, void* ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!topk_ids || !expert_offsets || !permuted_rows || !ws) return MOE_ERR_INVALID_ARG;
    if (!routing_shape_ok(s)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(topk_ids) || !aligned16(expert_offsets) || !aligned16(permuted_rows) ||
        !aligned16(ws))
        return MOE_ERR_MISALIGNED;
    moe_shape_t rs = s;  // H and I play no part in the permutation
    rs.H = rs.I = 0;
    const Layout L = layout_for(rs);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return run_permute(nullptr, const_cast<int32_t*>(topk_ids), nullptr, s, expert_offsets,
                       permuted_rows, ws, L, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_grouped_ffn(const moe_bf16_t* x, const moe_bf16_t* w13, const moe_bf16_t* w2,
                             const int32_t* expert_offsets, const int32_t* permuted_rows,
                             moe_shape_t s, moe_bf16_t* y, void* ws, size_t ws_bytes,
                             moe_stream_t stream)
{
    if (!x || !w13 || !w2 || !expert_offsets || !permuted_rows || !y || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!ffn_shape_ok(s)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(expert_offsets) ||
        !aligned16(permuted_rows) || !aligned16(y) || !aligned16(ws))
        return MOE_ERR_MISALIGNED;
    if (ws_bytes < moe_workspace_size(s)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const Layout L = layout_for(s);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    moe_status_t r = cuda_status(
        launch_build_tiles(expert_offsets, s.E, s.T * s.top_k, make_aux(ws, L, s), st));
    if (r != MOE_OK) return r;
    return run_ffn(x, w13, w2, permuted_rows, s, y, ws, L, st);
}

moe_status_t moe_combine(const moe_bf16_t* y, const float* topk_weights, moe_shape_t s,
                         moe_bf16_t* out, moe_stream_t stream)
{
    if (!y || !topk_weights || !out) return MOE_ERR_INVALID_ARG;
    if (!combine_shape_ok(s)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(y) || !aligned16(topk_weights) || !aligned16(out)) return MOE_ERR_MISALIGNED;
    return cuda_status(launch_combine(y, topk_weights, s.T, s.top_k, s.H, out,
                                      static_cast<cudaStream_t>(stream)));
}

// s13 / s2 set: w13 / w2 are E4M3 codes with those row scales (one-launch path only).
static moe_status_t forward_impl(const moe_bf16_t* x, const float* logits, const void* w13,
                                 const void* w2, const float* s13, const float* s2, moe_shape_t s,
                                 moe_bf16_t* out, int32_t* topk_ids, float* topk_weights,
                                 int32_t* expert_offsets, int32_t* permuted_rows, void* ws,
                                 size_t ws_bytes, moe_stream_t stream, void* const* events)
{
    const bool w8 = s13 || s2;
    if (!x || !logits || !w13 || !w2 || !out || !ws || (w8 && !(s13 && s2)))
        return MOE_ERR_INVALID_ARG;
    if (!ffn_shape_ok(s)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (w8 && (!aligned16(s13) || !aligned16(s2))) return MOE_ERR_MISALIGNED;
    if (!aligned16(x) || !aligned16(logits) || !aligned16(w13) || !aligned16(w2) ||
        !aligned16(out) || !aligned16(ws) || (topk_ids && !aligned16(topk_ids)) ||
        (topk_weights && !aligned16(topk_weights)) ||
        (expert_offsets && !aligned16(expert_offsets)) ||
        (permuted_rows && !aligned16(permuted_rows)))
        return MOE_ERR_MISALIGNED;
    if (ws_bytes < moe_workspace_size(s)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const Layout L = layout_for(s);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* ids = topk_ids ? topk_ids : at<int32_t>(ws, L.ids);
    float* wts = topk_weights ? topk_weights : at<float>(ws, L.weights);
    int32_t* offs = expert_offsets ? expert_offsets : at<int32_t>(ws, L.offsets);
    int32_t* rows = permuted_rows ? permuted_rows : at<int32_t>(ws, L.rows);
    void* y = at<void>(ws, L.y);
    auto mark = [&](int i) -> moe_status_t {
        if (!events) return MOE_OK;
        return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st));
    };

    // E4M3 weights exist only on the one-launch path
    if (w8 && !L.fused) return MOE_ERR_UNSUPPORTED_SHAPE;
    const bool fused = w8 || (L.fused && fused_enabled());
    moe_status_t r = mark(0);
    if (fused) {
        // one launch: routing and the permutation (inside every CTA), w13, w2 and
        // the combine; events [1] .. [4] all mark its end except [1], recorded
        // right after [0]
        if (r == MOE_OK) r = mark(1);
        FusedBuffers b;
        b.x = x;
        b.logits = logits;
        b.w13 = w13;
        b.w2 = w2;
        b.s13 = s13;
        b.s2 = s2;
        b.topk_ids = ids;
        b.topk_weights = wts;
        b.expert_offsets = offs;
        b.permuted_rows = rows;
        b.act = at<void>(ws, L.act);
        b.part2 = at<float>(ws, L.partials2);
        b.y = y;
        b.out = out;
        b.counters = at<int32_t>(ws, L.counters);
        b.ready = at<unsigned long long>(ws, L.ready);
        b.xmax = at<void>(ws, L.xmax);
        b.gen = next_generation();
        b.splits = at<int32_t>(ws, L.splits);
        b.err = at<int32_t>(ws, L.err);
        FfnPlan plan = L.plan;
        plan.grid = device_sms();
        if (r == MOE_OK)
            r = cuda_status(launch_fused_ffn(b, s.T, s.E, s.top_k, s.H, s.I, plan, st));
        for (int i = 2; i <= 4 && r == MOE_OK; ++i) r = mark(i);
        return r;
    }
    if (r == MOE_OK) r = run_permute(logits, ids, wts, s, offs, rows, ws, L, st);
    if (r == MOE_OK) r = mark(1);
    // a split w2 is reduced inside the combine (one launch fewer)
    const bool split2 = L.plan.s2_max > 1;
    if (r == MOE_OK)
        r = run_ffn(x, w13, w2, rows, s, y, ws, L, st, events ? events + 2 : nullptr, !split2);
    if (r == MOE_OK) r = mark(3);
    if (r == MOE_OK)
        r = cuda_status(split2 ? launch_combine_partials(at<float>(ws, L.partials),
                                                         at<int32_t>(ws, L.splits) + 1, y, wts, s.T,
                                                         s.top_k, s.H, out, st)
                               : launch_combine(y, wts, s.T, s.top_k, s.H, out, st));
    if (r == MOE_OK) r = mark(4);
    return r;
}

moe_status_t moe_forward(const moe_bf16_t* x, const float* logits, const moe_bf16_t* w13,
                         const moe_bf16_t* w2, moe_shape_t s, moe_bf16_t* out, int32_t* topk_ids,
                         float* topk_weights, int32_t* expert_offsets, int32_t* permuted_rows,
                         void* ws, size_t ws_bytes, moe_stream_t stream)
{
    return forward_impl(x, logits, w13, w2, nullptr, nullptr, s, out, topk_ids, topk_weights,
                        expert_offsets, permuted_rows, ws, ws_bytes, stream, nullptr);
}

moe_status_t moe_forward_timed(const moe_bf16_t* x, const float* logits, const moe_bf16_t* w13,
                               const moe_bf16_t* w2, moe_shape_t s, moe_bf16_t* out,
                               int32_t* topk_ids, float* topk_weights, int32_t* expert_offsets,
                               int32_t* permuted_rows, void* ws, size_t ws_bytes,
                               moe_stream_t stream, void* const* events, int n_events)
{
    if (!events || n_events != 5) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < 5; ++i)
        if (!events[i]) return MOE_ERR_INVALID_ARG;
    return forward_impl(x, logits, w13, w2, nullptr, nullptr, s, out, topk_ids, topk_weights,
                        expert_offsets, permuted_rows, ws, ws_bytes, stream, events);
}

moe_status_t moe_forward_w8(const moe_bf16_t* x, const float* logits, const uint8_t* w13,
                            const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                            moe_shape_t s, moe_bf16_t* out, int32_t* topk_ids,
                            float* topk_weights, int32_t* expert_offsets, int32_t* permuted_rows,
                            void* ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!w13_scale || !w2_scale) return MOE_ERR_INVALID_ARG;
    return forward_impl(x, logits, w13, w2, w13_scale, w2_scale, s, out, topk_ids, topk_weights,
                        expert_offsets, permuted_rows, ws, ws_bytes, stream, nullptr);
}

moe_status_t moe_forward_w8_timed(const moe_bf16_t* x, const float* logits, const uint8_t* w13,
                                  const float* w13_scale, const uint8_t* w2,
                                  const float* w2_scale, moe_shape_t s, moe_bf16_t* out,
                                  int32_t* topk_ids, float* topk_weights, int32_t* expert_offsets,
                                  int32_t* permuted_rows, void* ws, size_t ws_bytes,
                                  moe_stream_t stream, void* const* events, int n_events)
{
    if (!events || n_events != 5 || !w13_scale || !w2_scale) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < 5; ++i)
        if (!events[i]) return MOE_ERR_INVALID_ARG;
    return forward_impl(x, logits, w13, w2, w13_scale, w2_scale, s, out, topk_ids, topk_weights,
                        expert_offsets, permuted_rows, ws, ws_bytes, stream, events);
}

int moe_forward_w8_supported(moe_shape_t s)
{
    if (!ffn_shape_ok(s)) return 0;
    return layout_for(s).fused ? 1 : 0;
}

int moe_forward_kernel_count(moe_shape_t s)
{
    if (!ffn_shape_ok(s)) return 0;
    const long R = (long)s.T * s.top_k;
    const Layout L = layout_for(s);
    // the one-launch FFN routes and permutes inside its own launch
    if (L.fused && fused_enabled()) return 1;
    // routing and permutation: one kernel, or the route kernel + the one-launch
    // multi-CTA permutation
    const int route_permute = R <= kSmallRows ? 1 : 2;
    // w13, [SwiGLU finalize], w2, combine
    return route_permute + 2 + (L.plan.s13_max > 1 ? 1 : 0) + 1;
}

int moe_forward_fused(moe_shape_t s)
{
    if (!ffn_shape_ok(s)) return 0;
    return layout_for(s).fused && fused_enabled() ? 1 : 0;
}

moe_status_t moe_device_status(void* ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < sizeof(int32_t)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e);
    if (v == 0) return MOE_OK;
    const int32_t zero = 0;  // clear whatever the word held (arbitrary in a fresh workspace)
    e = cudaMemcpyAsync(ws, &zero, sizeof zero, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e);
    return v == kDeviceErrorMagic    ? MOE_ERR_DEVICE_TIMEOUT
           : v == kDeviceBoundsMagic ? MOE_ERR_DEVICE_BOUNDS
                                     : MOE_OK;
}

moe_status_t moe_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned limit_us,
                                       moe_stream_t stream)
{
    if (!ws || limit_us < 1 || limit_us > 2000000u) return MOE_ERR_INVALID_ARG;
    if (!aligned16(ws)) return MOE_ERR_MISALIGNED;
    if (ws_bytes < 2 * sizeof(int32_t)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return cuda_status(launch_wait_timeout_selftest(ws, limit_us, static_cast<cudaStream_t>(stream)));
}

const char* moe_status_string(moe_status_t status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null pointer)";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error (see moe_last_cuda_error)";
    case MOE_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case MOE_ERR_DEVICE_BOUNDS:
        return "a debug-build kernel found an input index out of range (the access was skipped)";
    }
    return "unknown status";
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
