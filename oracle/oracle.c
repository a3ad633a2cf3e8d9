/*
 * CPU oracle for paged MQA logits -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this file's library. The product path (the CUDA library and its
 * Python binding) never calls it and shares no code with it.
 *
 * What it computes (plain definition, fp64, single thread, no blocking):
 *
 *   for every batch row b, draft position n < next_n and token t < L:
 *     ctx_bn = clamp(ctx_b - next_n + 1 + n, 0, ctx_b)
 *     out[b,n,t] = sum_h w[b,n,h] * max(0, s_t * (q[b,n,h,:] . k_t[:]))  if t < ctx_bn
 *                = -inf                                                  otherwise
 *   with k_t and s_t read from page block_table[b][t / page_size],
 *   slot t % page_size.
 *
 * Sources: the page "[flashinfer] Blackwell 아키텍처를 위한 고성능 Paged MQA
 * Logits 커널 도입" (an analysis of FlashInfer PR #4365), its introduction
 * (the per-head weighted sum of rectified scores that the DeepSeek MLA
 * sparse-attention indexer computes) and its section 1 (zero-length rows).
 * The page states no formula: the formula above, the draft-row (MTP) masking
 * rule and the FP8/FP4 cache formats are this library's specification.
 *
 * The block-scaled FP4 variant (oracle_logits_nvfp4) takes q in the same
 * format as the FP4 K: per (b, n) row, [H][D/2] packed e2m1 codes then
 * [H][D/16] e4m3 block scales, q[b,n,h,d] = e2m1(code) * e4m3(scale of block
 * d/16). Both operands are decoded to their exact values first; the rest is
 * the FP4 definition.
 *
 * The top-k oracle (oracle_topk) is the selection the indexer makes from
 * these logits (the same page, introduction: the indexer picks the tokens
 * sparse attention will read): per row, the k largest logits of the valid
 * tokens, written out by sorting, nothing more.
 *
 * The schedule oracle follows the same page's section 1 ("스케줄링 알고리즘
 * 개선"), whose "before" algorithm is a linear scan over rows; the GPU uses a
 * binary search, so the two share no search logic.
 *
 * Number formats are decoded here from their definitions:
 *   e4m3 (OCP FP8 E4M3): sign, 4 exponent bits (bias 7), 3 mantissa bits;
 *        exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinity.
 *   e2m1 (OCP MX FP4):   sign, 2 exponent bits (bias 1), 1 mantissa bit;
 *        magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   bf16: the upper 16 bits of an IEEE binary32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

double oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);              /* (m / 8) * 2^(1 - 7) */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

double oracle_e2m1_to_double(uint8_t nibble) {
    int sign = (nibble >> 3) & 1;
    int e = (nibble >> 1) & 0x3;
    int m = nibble & 0x1;
    double v;
    if (e == 0)
        v = 0.5 * m;                            /* (m / 2) * 2^(1 - 1) */
    else
        v = ldexp(1.0 + m / 2.0, e - 1);
    return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * The decoded value of every e4m3 code and every e2m1 code, filled once by the
 * decoders above when the library is loaded. The loops below read these
 * tables instead of calling a decoder per element: the values, and therefore
 * every product and sum, are exactly the decoders'.
 */
static double e4m3_value[256];
static double e2m1_value[16];

__attribute__((constructor)) static void fill_decode_tables(void) {
    for (int c = 0; c < 256; ++c) e4m3_value[c] = oracle_e4m3_to_double((uint8_t)c);
    for (int c = 0; c < 16; ++c) e2m1_value[c] = oracle_e2m1_to_double((uint8_t)c);
}

/* Copies of the two tables (for the tests that pin them to the decoders). */
void oracle_decode_tables(double* e4m3_out, double* e2m1_out) {
    memcpy(e4m3_out, e4m3_value, sizeof e4m3_value);
    memcpy(e2m1_out, e2m1_value, sizeof e2m1_value);
}

static double f32_at(const uint8_t* p) {
    float f;
    memcpy(&f, p, sizeof f);
    return (double)f;
}

static int64_t draft_ctx(int64_t ctx_b, int next_n, int n) {
    int64_t c = ctx_b - next_n + 1 + n;
    if (c < 0) c = 0;
    if (c > ctx_b) c = ctx_b;
    return c;
}

/*
 * Schedule: u_b = ceil(ctx_b / 256); U = sum_b u_b; CTA i starts at global
 * unit start_i = i * floor(U / S) + min(i, U mod S), for i = 0..S. Entry i is
 * (row, unit offset) of the unit with global index start_i, found by walking
 * the rows in order; start_i == U gives the sentinel (B, 0).
 * Output: int32 sched[(S + 1) * 2].
 */
void oracle_schedule(const int32_t* context_lens, int B, int S, int32_t* sched) {
    int64_t U = 0;
    for (int b = 0; b < B; ++b) {
        int64_t c = context_lens[b] > 0 ? context_lens[b] : 0;
        U += (c + 255) / 256;
    }
    for (int i = 0; i <= S; ++i) {
        int64_t start = (int64_t)i * (U / S) + (i < U % S ? i : U % S);
        int row = B, off = 0;
        int64_t before = 0;                     /* units in rows < b */
        for (int b = 0; b < B; ++b) {
            int64_t c = context_lens[b] > 0 ? context_lens[b] : 0;
            int64_t u = (c + 255) / 256;
            if (start < before + u) {           /* unit lies in row b */
                row = b;
                off = (int)(start - before);
                break;
            }
            before += u;
        }
        sched[2 * i] = row;
        sched[2 * i + 1] = off;
    }
}

/*
 * One output element of the FP8 path. q: e4m3 [B][next_n][H][D];
 * kv_cache: pages of [page_size][D] e4m3 K then [page_size] fp32 scales.
 * Returns the fp64 logit and writes the tolerance denominator
 * A = sum_h |w_h| * max(0, s * score_h) to *absw. Requires t < ctx_bn.
 */
static double fp8_point(const uint8_t* q, const uint8_t* kv, const int32_t* bt,
                        const float* w, int next_n, int H, int D, int page_size,
                        int max_pages, int b, int n, int64_t t, double* absw) {
    int64_t page_bytes = (int64_t)page_size * (D + 4);
    int64_t page = bt[(int64_t)b * max_pages + t / page_size];
    int64_t slot = t % page_size;
    const uint8_t* base = kv + page * page_bytes;
    const uint8_t* krow = base + slot * D;
    double s = f32_at(base + (int64_t)page_size * D + slot * 4);
    double sum = 0.0, a = 0.0;
    for (int h = 0; h < H; ++h) {
        const uint8_t* qrow = q + (((int64_t)b * next_n + n) * H + h) * D;
        double score = 0.0;
        for (int d = 0; d < D; ++d)
            score += e4m3_value[qrow[d]] * e4m3_value[krow[d]];
        double r = s * score;
        if (r < 0.0) r = 0.0;
        double wh = (double)w[((int64_t)b * next_n + n) * H + h];
        sum += wh * r;
        a += fabs(wh) * r;
    }
    if (absw) *absw = a;
    return sum;
}

/*
 * One output element of the FP4 path. q: bf16 bits [B][next_n][H][D];
 * kv_cache: pages of [page_size][D/2] packed e2m1 (even element in the low
 * nibble) then [page_size][D/16] e4m3 block scales; k_t[d] =
 * e2m1(code) * e4m3(scale of block d/16). There is no per-token scale (s = 1).
 */
static double fp4_point(const uint16_t* q, const uint8_t* kv, const int32_t* bt,
                        const float* w, int next_n, int H, int D, int page_size,
                        int max_pages, int b, int n, int64_t t, double* absw) {
    int64_t page_bytes = (int64_t)page_size * (D / 2 + D / 16);
    int64_t page = bt[(int64_t)b * max_pages + t / page_size];
    int64_t slot = t % page_size;
    const uint8_t* base = kv + page * page_bytes;
    const uint8_t* krow = base + slot * (D / 2);
    const uint8_t* srow = base + (int64_t)page_size * (D / 2) + slot * (D / 16);
    double sum = 0.0, a = 0.0;
    for (int h = 0; h < H; ++h) {
        const uint16_t* qrow = q + (((int64_t)b * next_n + n) * H + h) * D;
        double score = 0.0;
        for (int d = 0; d < D; ++d) {
            uint8_t byte = krow[d / 2];
            uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double k = e2m1_value[code] * e4m3_value[srow[d / 16]];
            score += oracle_bf16_to_double(qrow[d]) * k;
        }
        double r = score;
        if (r < 0.0) r = 0.0;
        double wh = (double)w[((int64_t)b * next_n + n) * H + h];
        sum += wh * r;
        a += fabs(wh) * r;
    }
    if (absw) *absw = a;
    return sum;
}

/*
 * One output element of the block-scaled FP4 path: q as described in the
 * header (codes then block scales per (b, n) row), K as in fp4_point.
 */
static double nvfp4_point(const uint8_t* q, const uint8_t* kv, const int32_t* bt,
                          const float* w, int next_n, int H, int D, int page_size,
                          int max_pages, int b, int n, int64_t t, double* absw) {
    int64_t page_bytes = (int64_t)page_size * (D / 2 + D / 16);
    int64_t page = bt[(int64_t)b * max_pages + t / page_size];
    int64_t slot = t % page_size;
    const uint8_t* base = kv + page * page_bytes;
    const uint8_t* krow = base + slot * (D / 2);
    const uint8_t* srow = base + (int64_t)page_size * (D / 2) + slot * (D / 16);
    const uint8_t* qbase = q + ((int64_t)b * next_n + n) * ((int64_t)H * (D / 2 + D / 16));
    double sum = 0.0, a = 0.0;
    for (int h = 0; h < H; ++h) {
        const uint8_t* qrow = qbase + (int64_t)h * (D / 2);
        const uint8_t* qsc = qbase + (int64_t)H * (D / 2) + (int64_t)h * (D / 16);
        double score = 0.0;
        for (int d = 0; d < D; ++d) {
            uint8_t kb = krow[d / 2];
            uint8_t kc = (d % 2 == 0) ? (kb & 0xF) : (kb >> 4);
            double k = e2m1_value[kc] * e4m3_value[srow[d / 16]];
            uint8_t qb = qrow[d / 2];
            uint8_t qc = (d % 2 == 0) ? (qb & 0xF) : (qb >> 4);
            double qv = e2m1_value[qc] * e4m3_value[qsc[d / 16]];
            score += qv * k;
        }
        double r = score;
        if (r < 0.0) r = 0.0;
        double wh = (double)w[((int64_t)b * next_n + n) * H + h];
        sum += wh * r;
        a += fabs(wh) * r;
    }
    if (absw) *absw = a;
    return sum;
}

typedef double (*point_fn)(const void*, const uint8_t*, const int32_t*, const float*,
                           int, int, int, int, int, int, int, int64_t, double*);

static void full(point_fn f, const void* q, const uint8_t* kv, const int32_t* bt,
                 const int32_t* ctx, const float* w, int B, int next_n, int H, int D,
                 int page_size, int max_pages, int64_t L, double* out, double* absw) {
    for (int b = 0; b < B; ++b) {
        for (int n = 0; n < next_n; ++n) {
            int64_t c = draft_ctx(ctx[b] > 0 ? ctx[b] : 0, next_n, n);
            double* o = out + ((int64_t)b * next_n + n) * L;
            double* a = absw ? absw + ((int64_t)b * next_n + n) * L : 0;
            for (int64_t t = 0; t < L; ++t) {
                if (t < c) {
                    o[t] = f(q, kv, bt, w, next_n, H, D, page_size, max_pages, b, n, t,
                             a ? &a[t] : 0);
                } else {
                    o[t] = -INFINITY;
                    if (a) a[t] = 0.0;
                }
            }
        }
    }
}

static void points(point_fn f, const void* q, const uint8_t* kv, const int32_t* bt,
                   const int32_t* ctx, const float* w, int next_n, int H, int D,
                   int page_size, int max_pages, const int64_t* idx, int64_t count,
                   double* out, double* absw) {
    for (int64_t i = 0; i < count; ++i) {
        int b = (int)idx[3 * i], n = (int)idx[3 * i + 1];
        int64_t t = idx[3 * i + 2];
        int64_t c = draft_ctx(ctx[b] > 0 ? ctx[b] : 0, next_n, n);
        if (t < c) {
            out[i] = f(q, kv, bt, w, next_n, H, D, page_size, max_pages, b, n, t,
                       absw ? &absw[i] : 0);
        } else {
            out[i] = -INFINITY;
            if (absw) absw[i] = 0.0;
        }
    }
}

static double fp8_point_v(const void* q, const uint8_t* kv, const int32_t* bt, const float* w,
                          int nn, int H, int D, int ps, int mp, int b, int n, int64_t t,
                          double* a) {
    return fp8_point((const uint8_t*)q, kv, bt, w, nn, H, D, ps, mp, b, n, t, a);
}

static double fp4_point_v(const void* q, const uint8_t* kv, const int32_t* bt, const float* w,
                          int nn, int H, int D, int ps, int mp, int b, int n, int64_t t,
                          double* a) {
    return fp4_point((const uint16_t*)q, kv, bt, w, nn, H, D, ps, mp, b, n, t, a);
}

static double nvfp4_point_v(const void* q, const uint8_t* kv, const int32_t* bt,
                           const float* w, int nn, int H, int D, int ps, int mp, int b, int n,
                           int64_t t, double* a) {
    return nvfp4_point((const uint8_t*)q, kv, bt, w, nn, H, D, ps, mp, b, n, t, a);
}

/* Whole output [B][next_n][L] (fp64) and, if absw != NULL, the per-element
 * tolerance denominator. */
void oracle_logits_fp8(const uint8_t* q, const uint8_t* kv, const int32_t* bt,
                       const int32_t* ctx, const float* w, int B, int next_n, int H,
                       int D, int page_size, int max_pages, int64_t L, double* out,
                       double* absw) {
    full(fp8_point_v, q, kv, bt, ctx, w, B, next_n, H, D, page_size, max_pages, L, out, absw);
}

void oracle_logits_fp4(const uint16_t* q, const uint8_t* kv, const int32_t* bt,
                       const int32_t* ctx, const float* w, int B, int next_n, int H,
                       int D, int page_size, int max_pages, int64_t L, double* out,
                       double* absw) {
    full(fp4_point_v, q, kv, bt, ctx, w, B, next_n, H, D, page_size, max_pages, L, out, absw);
}

void oracle_logits_nvfp4(const uint8_t* q, const uint8_t* kv, const int32_t* bt,
                         const int32_t* ctx, const float* w, int B, int next_n, int H,
                         int D, int page_size, int max_pages, int64_t L, double* out,
                         double* absw) {
    full(nvfp4_point_v, q, kv, bt, ctx, w, B, next_n, H, D, page_size, max_pages, L, out,
         absw);
}

/* Selected elements: idx holds count (b, n, t) triples. */
void oracle_points_fp8(const uint8_t* q, const uint8_t* kv, const int32_t* bt,
                       const int32_t* ctx, const float* w, int next_n, int H, int D,
                       int page_size, int max_pages, const int64_t* idx, int64_t count,
                       double* out, double* absw) {
    points(fp8_point_v, q, kv, bt, ctx, w, next_n, H, D, page_size, max_pages, idx, count,
           out, absw);
}

void oracle_points_fp4(const uint16_t* q, const uint8_t* kv, const int32_t* bt,
                       const int32_t* ctx, const float* w, int next_n, int H, int D,
                       int page_size, int max_pages, const int64_t* idx, int64_t count,
                       double* out, double* absw) {
    points(fp4_point_v, q, kv, bt, ctx, w, next_n, H, D, page_size, max_pages, idx, count,
           out, absw);
}

void oracle_points_nvfp4(const uint8_t* q, const uint8_t* kv, const int32_t* bt,
                         const int32_t* ctx, const float* w, int next_n, int H, int D,
                         int page_size, int max_pages, const int64_t* idx, int64_t count,
                         double* out, double* absw) {
    points(nvfp4_point_v, q, kv, bt, ctx, w, next_n, H, D, page_size, max_pages, idx, count,
           out, absw);
}

/*
 * Top-k over a logits array out[B][next_n][L] (fp32): for every row (b, n),
 * with c = min(max(ctx_b, 0), L) and ctx_bn = clamp(c - next_n + 1 + n, 0, c),
 * the k tokens t < ctx_bn of largest out[b,n,t], ordered by value descending
 * and, for equal values, by token ascending (-0.0 and +0.0 are equal values);
 * rows with fewer than k such tokens are padded with -1.
 * Output: int32 idx[B][next_n][k].
 */
typedef struct {
    float v;
    int32_t t;
} topk_item;

static int topk_cmp(const void* x, const void* y) {
    const topk_item* a = (const topk_item*)x;
    const topk_item* b = (const topk_item*)y;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->t > b->t) - (a->t < b->t);
}

void oracle_topk(const float* logits, const int32_t* context_lens, int B, int next_n, int L,
                 int k, int32_t* idx) {
    topk_item* items = (topk_item*)malloc(sizeof(topk_item) * (size_t)(L > 0 ? L : 1));
    for (int b = 0; b < B; ++b) {
        int64_t c = context_lens[b];
        if (c < 0) c = 0;
        if (c > L) c = L;
        for (int n = 0; n < next_n; ++n) {
            const int64_t cbn = draft_ctx(c, next_n, n);
            const float* row = logits + ((int64_t)b * next_n + n) * L;
            for (int64_t t = 0; t < cbn; ++t) {
                items[t].v = row[t];
                items[t].t = (int32_t)t;
            }
            qsort(items, (size_t)cbn, sizeof(topk_item), topk_cmp);
            int32_t* o = idx + ((int64_t)b * next_n + n) * k;
            for (int i = 0; i < k; ++i) o[i] = i < cbn ? items[i].t : -1;
        }
    }
    free(items);
}
