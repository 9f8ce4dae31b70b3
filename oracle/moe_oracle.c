/*
 * moe_oracle.c -- plain, slow, fp64 CPU reference of the MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this code:
 * it is loaded by the test suite, by __graft_entry__.smoke() (as the checker)
 * and by bench.py's cpu_baseline / --impl reference legs.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through the
 * seeded inputs they are both handed.
 *
 * What it computes (the layer forward that the FlashInfer MoE pages turn on):
 *   1. route   : per token, the k experts with the largest raw fp32 router
 *                logit (ties -> lower expert index; -0.0 == +0.0), weights =
 *                softmax over the k selected logits ("softmax_sum" routing,
 *                FlashInfer PR #3751 page, "performance numbers" section: a
 *                softmax followed by division by the sum of the selected
 *                probabilities, which equals a softmax over the selected k).
 *   2. permute : counting sort of the expanded rows r = t*k + j by expert,
 *                ascending r inside an expert (a stable sort).
 *   3. ffn     : for each permuted row p with expert e, token
 *                t = permuted_rows[p] / k (the `members[m] // input_route_divisor`
 *                map of the FlashInfer PR #7368 page, section "1. Ampere",
 *                with the divisor equal to top_k), h = w13[e] . x[t]  (2I),
 *                gate = h[0:I], up = h[I:2I], act = silu(gate) * up,
 *                y[permuted_rows[p]] = w2[e] . act  (H).
 *   4. combine : out[t] = sum_{j=0..k-1} w[t,j] * y[t*k + j], j ascending
 *                (a fixed-order merge, cf. the "FP32 partials" section of the
 *                FlashInfer PR #5586 page).
 *
 * All arithmetic is IEEE double on exactly-upcast bf16/fp32 inputs; nothing is
 * rounded in between unless `round_intermediates` asks for the bf16 rounding of
 * act and y (a diagnostic mode, not the reference).  Every reduction runs in a
 * fixed sequential order per output element, so results do not depend on the
 * number of OpenMP threads.
 *
 * Error behaviour: every entry point returns 0 on success and a negative value
 * on an invalid argument (null pointer, non-positive size, k > E, an expert id
 * out of range); outputs are then left untouched.
 *
 * FP8 weights (the *_w8 entry points): w13 and w2 arrive as E4M3 codes (the
 * OCP "E4M3FN" format: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * subnormals, no infinities, 0x7F / 0xFF are NaN) with one fp32 scale per weight
 * row (per output feature): the weight is e4m3(q) * scale, exact in double.  The
 * layer is otherwise the same four steps.
 *
 * Pinned by tests/test_oracle_pins.py (closed forms of a hand-worked example,
 * rank-count brute force, invariants, reduction to library softmax / a plain
 * SwiGLU MLP, and a dense all-experts masked loop; for the FP8 weights, the
 * E4M3 decoder against a library conversion of every code, bit equality with
 * the bf16 layer when the dequantised weights are bf16 values, and a dense
 * dequantise-then-multiply check; for the diagnostic bf16 rounding, the library
 * float64 -> bfloat16 conversion on ties, subnormals and the overflow boundary,
 * and a dense loop that rounds act and y with it).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Number of OpenMP threads the oracle's parallel loops use. */
int oracle_num_threads(void) { return omp_get_max_threads(); }

/* ---- exact upcasts ------------------------------------------------------ */

/* E4M3 (E4M3FN) code -> double, from the format's definition: exponent field
 * 0 encodes subnormals m * 2^-9; otherwise (1 + m/8) * 2^(e - 7); the all-ones
 * code (exponent 15, mantissa 7) of either sign is NaN; there is no infinity. */
static double e4m3_to_double(uint8_t q)
{
    const int sign = q >> 7, e = (q >> 3) & 15, m = q & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Decodes n E4M3 codes (exported for the pins). */
int oracle_e4m3_to_double(const uint8_t* q, long n, double* out)
{
    if (!q || !out || n < 0) return -1;
    for (long i = 0; i < n; ++i) out[i] = e4m3_to_double(q[i]);
    return 0;
}

/* bf16 bit pattern -> double (exact: bf16 is the top half of an fp32). */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> bf16 via fp32, both steps round-to-nearest-even (ties to the even
 * significand; a finite value past the largest bf16 by half an ulp or more
 * becomes infinity; infinities and NaNs keep their class).  Only used by the
 * diagnostic `round_intermediates` mode. */
static double round_to_bf16(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) != 0x7f800000u) {          /* finite */
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7fffu + lsb;
    }
    u &= 0xffff0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Applies round_to_bf16 to n doubles (exported for the pins). */
int oracle_round_to_bf16(const double* in, long n, double* out)
{
    if (!in || !out || n < 0) return -1;
    for (long i = 0; i < n; ++i) out[i] = round_to_bf16(in[i]);
    return 0;
}

/* ---- 1. route ------------------------------------------------------------ */

/* Sort key of one expert of one token: larger logit first, then lower index. */
typedef struct {
    double logit;
    int32_t expert;
} route_key;

static int route_key_cmp(const void* pa, const void* pb)
{
    const route_key* a = (const route_key*)pa;
    const route_key* b = (const route_key*)pb;
    if (a->logit > b->logit) return -1;
    if (a->logit < b->logit) return 1;
    /* equal values (this includes -0.0 == +0.0): lower expert index first */
    return (a->expert < b->expert) ? -1 : (a->expert > b->expert) ? 1 : 0;
}

/* Route one token: full sort of its E logits, keep the first k, softmax over
 * the kept logits in double, stored as fp32 (round to nearest). */
static void route_one_token(const float* row, int E, int k, route_key* scratch,
                            int32_t* ids, float* weights)
{
    for (int e = 0; e < E; ++e) {
        scratch[e].logit = (double)row[e];
        scratch[e].expert = e;
    }
    qsort(scratch, (size_t)E, sizeof(route_key), route_key_cmp);

    const double lmax = scratch[0].logit;
    double denom = 0.0;
    for (int j = 0; j < k; ++j) denom += exp(scratch[j].logit - lmax);
    for (int j = 0; j < k; ++j) {
        ids[j] = scratch[j].expert;
        weights[j] = (float)(exp(scratch[j].logit - lmax) / denom);
    }
}

int oracle_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_weights)
{
    if (!logits || !topk_ids || !topk_weights || T < 1 || E < 1 || k < 1 || k > E) return -1;
    int bad = 0;
#pragma omp parallel
    {
        route_key* scratch = (route_key*)malloc(sizeof(route_key) * (size_t)E);
        if (!scratch) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int t = 0; t < T; ++t)
                route_one_token(logits + (size_t)t * E, E, k, scratch,
                                topk_ids + (size_t)t * k, topk_weights + (size_t)t * k);
            free(scratch);
        }
    }
    return bad ? -2 : 0;
}

/* ---- 2. permute ---------------------------------------------------------- */

int oracle_permute(const int32_t* topk_ids, int T, int k, int E, int32_t* expert_offsets,
                   int32_t* permuted_rows)
{
    if (!topk_ids || !expert_offsets || !permuted_rows || T < 1 || k < 1 || E < 1) return -1;
    const long R = (long)T * k;
    for (long r = 0; r < R; ++r)
        if (topk_ids[r] < 0 || topk_ids[r] >= E) return -1;

    /* histogram */
    long* count = (long*)calloc((size_t)E, sizeof(long));
    long* cursor = (long*)calloc((size_t)E, sizeof(long));
    if (!count || !cursor) { free(count); free(cursor); return -2; }
    for (long r = 0; r < R; ++r) count[topk_ids[r]] += 1;

    /* exclusive scan */
    expert_offsets[0] = 0;
    for (int e = 0; e < E; ++e) expert_offsets[e + 1] = expert_offsets[e] + (int32_t)count[e];

    /* scatter in ascending r: stable by construction */
    for (int e = 0; e < E; ++e) cursor[e] = expert_offsets[e];
    for (long r = 0; r < R; ++r) permuted_rows[cursor[topk_ids[r]]++] = (int32_t)r;

    free(count);
    free(cursor);
    return 0;
}

/* ---- 3. expert FFN --------------------------------------------------------- */

/* y_row[H] = w2_e . (silu(gate) * up), gate/up = rows [0,I) / [I,2I) of
 * w13_e . x_row.  w13_e is [2I, H] and w2_e is [H, I], both row-major bf16.
 * `act` is caller scratch of I doubles. */
static void expert_ffn_row(const uint16_t* x_row, const uint16_t* w13_e, const uint16_t* w2_e,
                           int H, int I, int round_intermediates, double* act, double* y_row)
{
    for (int c = 0; c < I; ++c) {
        const uint16_t* wg = w13_e + (size_t)c * H;
        const uint16_t* wu = w13_e + (size_t)(I + c) * H;
        double gate = 0.0, up = 0.0;
        for (int i = 0; i < H; ++i) {
            const double xi = bf16_to_double(x_row[i]);
            gate += xi * bf16_to_double(wg[i]);
            up += xi * bf16_to_double(wu[i]);
        }
        const double silu = gate / (1.0 + exp(-gate));
        act[c] = silu * up;
        if (round_intermediates) act[c] = round_to_bf16(act[c]);
    }
    for (int o = 0; o < H; ++o) {
        const uint16_t* w = w2_e + (size_t)o * I;
        double acc = 0.0;
        for (int c = 0; c < I; ++c) acc += act[c] * bf16_to_double(w[c]);
        y_row[o] = round_intermediates ? round_to_bf16(acc) : acc;
    }
}

int oracle_ffn(const uint16_t* x, const uint16_t* w13, const uint16_t* w2,
               const int32_t* expert_offsets, const int32_t* permuted_rows,
               int T, int E, int k, int H, int I, int round_intermediates, double* y)
{
    if (!x || !w13 || !w2 || !expert_offsets || !permuted_rows || !y) return -1;
    if (T < 1 || E < 1 || k < 1 || H < 1 || I < 1) return -1;
    const long R = (long)T * k;
    if (expert_offsets[0] != 0 || expert_offsets[E] != R) return -1;
    int bad = 0;
#pragma omp parallel
    {
        double* act = (double*)malloc(sizeof(double) * (size_t)I);
        if (!act) {
#pragma omp atomic write
            bad = 1;
        } else {
            for (int e = 0; e < E; ++e) {
                const uint16_t* w13_e = w13 + (size_t)e * 2 * I * H;
                const uint16_t* w2_e = w2 + (size_t)e * H * I;
#pragma omp for schedule(dynamic, 1)
                for (long p = expert_offsets[e]; p < expert_offsets[e + 1]; ++p) {
                    const long r = permuted_rows[p];
                    const long t = r / k;                  /* expanded id -> token */
                    expert_ffn_row(x + (size_t)t * H, w13_e, w2_e, H, I, round_intermediates, act,
                                   y + (size_t)r * H);
                }
            }
            free(act);
        }
    }
    return bad ? -2 : 0;
}

/* ---- 4. combine ------------------------------------------------------------ */

int oracle_combine(const double* y, const float* topk_weights, int T, int k, int H, double* out)
{
    if (!y || !topk_weights || !out || T < 1 || k < 1 || H < 1) return -1;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += (double)topk_weights[(size_t)t * k + j] * y[((size_t)t * k + j) * H + h];
            out[(size_t)t * H + h] = acc;
        }
    }
    return 0;
}

/* ---- whole layer ----------------------------------------------------------- */

/* Steps 1-4 in order.  Every output pointer is caller-owned host memory:
 * topk_ids/topk_weights [T*k], expert_offsets [E+1], permuted_rows [T*k],
 * out [T*H] doubles.  y (T*k*H doubles) is allocated here and freed. */
int oracle_forward(const uint16_t* x, const float* logits, const uint16_t* w13, const uint16_t* w2,
                   int T, int E, int k, int H, int I, int round_intermediates, double* out,
                   int32_t* topk_ids, float* topk_weights, int32_t* expert_offsets,
                   int32_t* permuted_rows)
{
    int rc = oracle_route(logits, T, E, k, topk_ids, topk_weights);
    if (rc) return rc;
    rc = oracle_permute(topk_ids, T, k, E, expert_offsets, permuted_rows);
    if (rc) return rc;
    double* y = (double*)malloc(sizeof(double) * (size_t)T * k * H);
    if (!y) return -2;
    rc = oracle_ffn(x, w13, w2, expert_offsets, permuted_rows, T, E, k, H, I, round_intermediates, y);
    if (!rc) rc = oracle_combine(y, topk_weights, T, k, H, out);
    free(y);
    return rc;
}

/* Layer output for a chosen subset of tokens only (for sampled checks at sizes
 * where the full layer is too slow on the CPU).  Each listed token is routed on
 * its own row, its k expert outputs are computed and combined in j order,
 * which is exactly the value oracle_forward gives for that token (the layer
 * output of a token depends only on that token's row of x and of the logits).
 *
 * The expert weights come as per-expert pointer tables (w13_e[e] -> [2I, H],
 * w2_e[e] -> [H, I]) so that a caller may hand over only the experts the
 * listed tokens select; a selected expert with a NULL entry is an error (-3). */
int oracle_forward_tokens(const uint16_t* x, const float* logits,
                          const uint16_t* const* w13_e, const uint16_t* const* w2_e,
                          int T, int E, int k, int H, int I, int round_intermediates,
                          int n_sel, const int32_t* tokens, double* out_sel)
{
    if (!x || !logits || !w13_e || !w2_e || !tokens || !out_sel) return -1;
    if (T < 1 || E < 1 || k < 1 || k > E || H < 1 || I < 1 || n_sel < 0) return -1;
    for (int s = 0; s < n_sel; ++s)
        if (tokens[s] < 0 || tokens[s] >= T) return -1;
    int bad = 0;
#pragma omp parallel
    {
        route_key* scratch = (route_key*)malloc(sizeof(route_key) * (size_t)E);
        double* act = (double*)malloc(sizeof(double) * (size_t)I);
        double* yk = (double*)malloc(sizeof(double) * (size_t)k * H);
        int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
        float* w = (float*)malloc(sizeof(float) * (size_t)k);
        if (!scratch || !act || !yk || !ids || !w) {
#pragma omp atomic write
            bad = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int s = 0; s < n_sel; ++s) {
                const int t = tokens[s];
                route_one_token(logits + (size_t)t * E, E, k, scratch, ids, w);
                int missing = 0;
                for (int j = 0; j < k; ++j) {
                    const int e = ids[j];
                    if (!w13_e[e] || !w2_e[e]) { missing = 1; break; }
                    expert_ffn_row(x + (size_t)t * H, w13_e[e], w2_e[e], H, I,
                                   round_intermediates, act, yk + (size_t)j * H);
                }
                if (missing) {
#pragma omp atomic write
                    bad = -3;
                    continue;
                }
                for (int h = 0; h < H; ++h) {
                    double acc = 0.0;
                    for (int j = 0; j < k; ++j) acc += (double)w[j] * yk[(size_t)j * H + h];
                    out_sel[(size_t)s * H + h] = acc;
                }
            }
        }
        free(scratch);
        free(act);
        free(yk);
        free(ids);
        free(w);
    }
    return bad;
}

/* ---- FP8 weights ------------------------------------------------------------ */

/* dec[q] = e4m3_to_double(q) for all 256 codes: the decoder's values, looked up
 * instead of recomputed for every weight. */
static void e4m3_table(double* dec)
{
    for (int q = 0; q < 256; ++q) dec[q] = e4m3_to_double((uint8_t)q);
}

/* As expert_ffn_row with w13_e = [2I, H] E4M3 codes and s13_e = [2I] row scales,
 * w2_e = [H, I] codes and s2_e = [H] row scales: weight (r, c) = e4m3(q) * s[r],
 * with e4m3(q) = dec[q] (e4m3_table). */
static void expert_ffn_row_w8(const uint16_t* x_row, const uint8_t* q13_e, const float* s13_e,
                              const uint8_t* q2_e, const float* s2_e, int H, int I,
                              const double* dec, double* act, double* y_row)
{
    for (int c = 0; c < I; ++c) {
        const uint8_t* qg = q13_e + (size_t)c * H;
        const uint8_t* qu = q13_e + (size_t)(I + c) * H;
        const double sg = s13_e[c], su = s13_e[I + c];
        double gate = 0.0, up = 0.0;
        for (int i = 0; i < H; ++i) {
            const double xi = bf16_to_double(x_row[i]);
            gate += xi * (dec[qg[i]] * sg);
            up += xi * (dec[qu[i]] * su);
        }
        act[c] = gate / (1.0 + exp(-gate)) * up;
    }
    for (int o = 0; o < H; ++o) {
        const uint8_t* q = q2_e + (size_t)o * I;
        const double so = s2_e[o];
        double acc = 0.0;
        for (int c = 0; c < I; ++c) acc += act[c] * (dec[q[c]] * so);
        y_row[o] = acc;
    }
}

/* The whole layer with FP8 weights: q13 [E, 2I, H] codes + s13 [E, 2I] scales,
 * q2 [E, H, I] codes + s2 [E, H] scales; outputs as oracle_forward. */
int oracle_forward_w8(const uint16_t* x, const float* logits, const uint8_t* q13, const float* s13,
                      const uint8_t* q2, const float* s2, int T, int E, int k, int H, int I,
                      double* out, int32_t* topk_ids, float* topk_weights,
                      int32_t* expert_offsets, int32_t* permuted_rows)
{
    if (!x || !q13 || !s13 || !q2 || !s2 || !out || H < 1 || I < 1) return -1;
    int rc = oracle_route(logits, T, E, k, topk_ids, topk_weights);
    if (rc) return rc;
    rc = oracle_permute(topk_ids, T, k, E, expert_offsets, permuted_rows);
    if (rc) return rc;
    const long R = (long)T * k;
    double* y = (double*)malloc(sizeof(double) * (size_t)R * H);
    if (!y) return -2;
    double dec[256];
    e4m3_table(dec);
    int bad = 0;
#pragma omp parallel
    {
        double* act = (double*)malloc(sizeof(double) * (size_t)I);
        if (!act) {
#pragma omp atomic write
            bad = -2;
        } else {
            for (int e = 0; e < E; ++e) {
#pragma omp for schedule(dynamic, 1)
                for (long p = expert_offsets[e]; p < expert_offsets[e + 1]; ++p) {
                    const long r = permuted_rows[p];
                    expert_ffn_row_w8(x + (size_t)(r / k) * H, q13 + (size_t)e * 2 * I * H,
                                      s13 + (size_t)e * 2 * I, q2 + (size_t)e * H * I,
                                      s2 + (size_t)e * H, H, I, dec, act, y + (size_t)r * H);
                }
            }
            free(act);
        }
    }
    if (!bad) bad = oracle_combine(y, topk_weights, T, k, H, out);
    free(y);
    return bad;
}

/* oracle_forward_tokens with FP8 weights: per-expert pointer tables of codes
 * (q13_e[e] -> [2I, H], q2_e[e] -> [H, I]) and scales (s13_e[e] -> [2I],
 * s2_e[e] -> [H]); a selected expert with a NULL entry is an error (-3). */
int oracle_forward_tokens_w8(const uint16_t* x, const float* logits,
                             const uint8_t* const* q13_e, const float* const* s13_e,
                             const uint8_t* const* q2_e, const float* const* s2_e, int T, int E,
                             int k, int H, int I, int n_sel, const int32_t* tokens,
                             double* out_sel)
{
    if (!x || !logits || !q13_e || !s13_e || !q2_e || !s2_e || !tokens || !out_sel) return -1;
    if (T < 1 || E < 1 || k < 1 || k > E || H < 1 || I < 1 || n_sel < 0) return -1;
    for (int s = 0; s < n_sel; ++s)
        if (tokens[s] < 0 || tokens[s] >= T) return -1;
    double dec[256];
    e4m3_table(dec);
    int bad = 0;
#pragma omp parallel
    {
        route_key* scratch = (route_key*)malloc(sizeof(route_key) * (size_t)E);
        double* act = (double*)malloc(sizeof(double) * (size_t)I);
        double* yk = (double*)malloc(sizeof(double) * (size_t)k * H);
        int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
        float* w = (float*)malloc(sizeof(float) * (size_t)k);
        if (!scratch || !act || !yk || !ids || !w) {
#pragma omp atomic write
            bad = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int s = 0; s < n_sel; ++s) {
                const int t = tokens[s];
                route_one_token(logits + (size_t)t * E, E, k, scratch, ids, w);
                int missing = 0;
                for (int j = 0; j < k; ++j) {
                    const int e = ids[j];
                    if (!q13_e[e] || !s13_e[e] || !q2_e[e] || !s2_e[e]) { missing = 1; break; }
                    expert_ffn_row_w8(x + (size_t)t * H, q13_e[e], s13_e[e], q2_e[e], s2_e[e], H,
                                      I, dec, act, yk + (size_t)j * H);
                }
                if (missing) {
#pragma omp atomic write
                    bad = -3;
                    continue;
                }
                for (int h = 0; h < H; ++h) {
                    double acc = 0.0;
                    for (int j = 0; j < k; ++j) acc += (double)w[j] * yk[(size_t)j * H + h];
                    out_sel[(size_t)s * H + h] = acc;
                }
            }
        }
        free(scratch);
        free(act);
        free(yk);
        free(ids);
        free(w);
    }
    return bad;
}
