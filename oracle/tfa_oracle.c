/*
 * tfa_oracle.c -- plain, slow, fp64 CPU oracle for tiled GQA prefill attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; the only thing the two sides have in common is the seeded
 * input generator, which holds none of the attention arithmetic.
 *
 * What it computes (every function below restates it, with its source):
 *
 *   For batch b, query head h and new query row i (0 <= i < L), with
 *   prefix P = S - L, absolute position p = P + i and KV head
 *   g = floor(h / (Hq / Hkv)):
 *     key j (0 <= j < S) is ALLOWED iff
 *       (causal  => j <= p)                      causal mask aligned to the
 *                                                end of the cached prefix
 *       (causal && window > 0 => j > p - window) sliding window [p-W+1, p]
 *       (key_mask == NULL || key_mask[b,j] > 0.5) length-S key mask
 *     s_j = scale * sum_d q[b,h,i,d] * k[b,g,j,d]       (fp64, exact bf16 upcast)
 *     softcap c > 0   -> s_j := c * tanh(s_j / c)       (after the scale)
 *     no allowed key  -> o[b,h,i,:] = 0
 *     otherwise       -> m = max s_j, w_j = exp(s_j - m),
 *                        o[b,h,i,:] = sum_j w_j v[b,g,j,:] / sum_j w_j
 *     attention sink  -> a per-query-head logit sigma_h joins the softmax
 *       sigma_h           denominator only: m = max(max_j s_j, sigma_h),
 *                        o = sum_j w_j v_j / (sum_j w_j + exp(sigma_h - m));
 *                        a row with no allowed key stays 0
 *
 * Sources (page title, section):
 *   tiny-llm "Week 2 Day 5: Tiled Dense Prefill Attention", Task 1 (layout
 *     Q [B,Hq,L,128], K/V [B,Hkv,S,128]; KV head floor(h/(Hq/Hkv)); the
 *     online-softmax merge equations m', l', a'), Task 2 (causality aligned to
 *     the end of the cached prefix: row i sees positions through S-L+i; a
 *     fully masked row is finite and all zero).
 *   brotensor "include/brotensor/ops/flash_attention.h" coverage page,
 *     flash_attention_windowed_forward and flash_attention_decode comments
 *     (window keeps keys [max(0, p-window+1), p], window <= 0 = unbounded;
 *     FP32 key mask 1 valid / 0 invalid, positions with mask <= 0.5 dropped,
 *     combined multiplicatively with the causal/window mask; Gemma-2
 *     extensions: attn_softcap > 0 replaces each score, after the
 *     1/sqrt(head_dim) scale and before mask and softmax, by
 *     attn_softcap * tanh(score / attn_softcap), 0 disables it).
 *   mlx-lm PR "Add fused prefill SDPA for sliding-window caches",
 *     Correctness (attention sinks among the tested cases; the page names
 *     them without a formula: the sink reading above is the plain one, a
 *     logit with no value row, taken in the same units as the scores and
 *     neither scaled nor capped).
 *   tinygrad "symbolic llm with prefill" compare view, apps/llm.py
 *     (_attention_inner: scaled_dot_product_attention(..., enable_gqa=True)
 *     with the causal mask full(-inf).triu(start_pos+1)).
 *
 * Inputs are bf16 bit patterns (uint16), upcast exactly to double.  Outputs
 * are double.  Layouts: q/o [B,Hq,L,D], k/v [B,Hkv,S,D], key_mask [B,S] fp32,
 * all contiguous row-major.
 *
 * The "mutant" entry point exists only so that tests can plant plausible
 * mistakes in the oracle and show that the pins catch them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Mutations a test may plant (0 = the correct oracle). */
enum {
    MUT_NONE = 0,
    MUT_CAUSAL_SEES_NEXT = 1,    /* j <= p + 1 instead of j <= p            */
    MUT_WINDOW_ONE_WIDER = 2,    /* j >= p - window instead of j > p - W     */
    MUT_HEAD_MODULO = 3,         /* g = h mod Hkv instead of floor(h / G)    */
    MUT_NO_PREFIX_OFFSET = 4,    /* causal triangle as if S were L (P = 0)   */
    MUT_DROP_SCALE = 5,          /* s_j without the scale factor             */
    MUT_KEYMASK_INVERTED = 6,    /* keep mask <= 0.5 instead of > 0.5        */
    MUT_EMPTY_ROW_UNIFORM = 7,   /* fully masked row averages all V rows     */
    MUT_SOFTCAP_BEFORE_SCALE = 8,/* c * tanh(raw / c) * scale                */
    MUT_SINK_SCALED = 9,         /* sink logit multiplied by the scale       */
    MUT_SINK_IN_NUMERATOR = 10,  /* sink weight also added to every output   */
    MUT_RING_SLOT_SHIFTED = 11,  /* key j read from ring row (j + 1) mod R   */
    MUT_VARLEN_PACKED_CAUSAL = 12,/* causal test on packed token indices      */
    MUT_BWD_NO_DELTA = 13,       /* dS = P dP, without the row term          */
    MUT_BWD_DK_NO_SCALE = 14,    /* dK without the softmax scale             */
    MUT_BWD_DQ_USES_V = 15,      /* dQ accumulates dS V instead of dS K      */
};

static double bf16_bits_to_f64(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Visibility of key j for new query row i.  tiny-llm Week 2 Day 5, Task 2
 * (causal offset by the prefix); brotensor flash_attention.h, decode comment
 * (window [p-window+1, p], window <= 0 unbounded) and forward comment
 * (key mask <= 0.5 dropped, combined multiplicatively). */
static int allowed_impl(long L, long S, long i, long j, int causal, long window,
                        const float *key_mask_row, int mutation)
{
    long P = (mutation == MUT_NO_PREFIX_OFFSET) ? 0 : S - L;
    long p = P + i;
    if (j < 0 || j >= S) return 0;
    if (causal) {
        long last = (mutation == MUT_CAUSAL_SEES_NEXT) ? p + 1 : p;
        if (j > last) return 0;
        if (window > 0) {
            long first = (mutation == MUT_WINDOW_ONE_WIDER) ? p - window : p - window + 1;
            if (j < first) return 0;
        }
    }
    if (key_mask_row) {
        int keep = (mutation == MUT_KEYMASK_INVERTED) ? (key_mask_row[j] <= 0.5f)
                                                      : (key_mask_row[j] > 0.5f);
        if (!keep) return 0;
    }
    return 1;
}

int oracle_allowed(long L, long S, long i, long j, int causal, long window,
                   const float *key_mask_row)
{
    return allowed_impl(L, S, i, j, causal, window, key_mask_row, MUT_NONE);
}

/* GQA head mapping: query head h reads KV head floor(h / (Hq / Hkv)).
 * tiny-llm Week 2 Day 5, Task 1; brotensor flash_attention_decode comment
 * (each KV head serves Hq/Hkv consecutive query heads). */
static int kv_head_impl(int h, int Hq, int Hkv, int mutation)
{
    if (mutation == MUT_HEAD_MODULO) return h % Hkv;
    return h / (Hq / Hkv);
}

static int check_args(const void *q, const void *k, const void *v, const void *o,
                      int B, int Hq, int Hkv, int L, int S, int D)
{
    if (!q || !k || !v || !o) return 1;
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || S < L || D < 1) return 2;
    if (Hq % Hkv != 0) return 3;
    return 0;
}

/* Where one output row reads its operands: its query vector, and the K and V
 * rows of its KV head -- key j at row slot(j) of kb / vb, rows kv_stride
 * elements apart.  slot(j) = j, or j mod ring for a rotating cache (the
 * TensorFold PR 3269 page names a ring-slot position for each cached key and
 * value row without giving a formula; j mod ring is the reading taken). */
typedef struct {
    const uint16_t *qr, *kb, *vb;
    size_t kv_stride;
    long ring;          /* 0: no ring */
    const float *mrow;  /* key-mask row, or NULL */
    int has_sink;
    double sigma;       /* sink logit when has_sink */
    long causal_shift;  /* 0; nonzero only in a planted mistake */
} RowOperands;

static long key_slot(const RowOperands *op, long j, int mutation)
{
    if (!op->ring) return j;
    if (mutation == MUT_RING_SLOT_SHIFTED) return (j + 1) % op->ring;
    return j % op->ring;
}

/* One output row, two passes, exact softmax, no tiling. */
static void row_core(const RowOperands *op, double *out, long L, long S, long i, int D,
                     double scale, int causal, int window, double softcap, int mutation,
                     double *s_buf)
{
    double sc = (mutation == MUT_DROP_SCALE) ? 1.0 : scale;
    double m = -INFINITY;
    int any = 0;
    for (long j = 0; j < S; ++j) {
        if (!allowed_impl(L, S, i + op->causal_shift, j, causal, window, op->mrow, mutation)) {
            s_buf[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        const uint16_t *kr = op->kb + (size_t)key_slot(op, j, mutation) * op->kv_stride;
        for (int d = 0; d < D; ++d) acc += bf16_bits_to_f64(op->qr[d]) * bf16_bits_to_f64(kr[d]);
        s_buf[j] = sc * acc;
        if (softcap > 0.0) {
            /* brotensor flash_attention.h, Gemma-2 extensions: cap after the scale */
            if (mutation == MUT_SOFTCAP_BEFORE_SCALE)
                s_buf[j] = softcap * tanh(acc / softcap) * sc;
            else
                s_buf[j] = softcap * tanh(s_buf[j] / softcap);
        }
        if (s_buf[j] > m) m = s_buf[j];
        any = 1;
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (!any) {
        /* tiny-llm Week 2 Day 5, Task 2: no probability mass -> finite zeros. */
        if (mutation == MUT_EMPTY_ROW_UNIFORM) {
            for (long j = 0; j < S; ++j) {
                const uint16_t *vr = op->vb + (size_t)key_slot(op, j, mutation) * op->kv_stride;
                for (int d = 0; d < D; ++d) out[d] += bf16_bits_to_f64(vr[d]) / (double)S;
            }
        }
        return;
    }
    /* attention sink: one more logit in the denominator, with no value row */
    double sigma = -INFINITY;
    if (op->has_sink) {
        sigma = op->sigma;
        if (mutation == MUT_SINK_SCALED) sigma *= scale;
        if (sigma > m) m = sigma;
    }
    double denom = 0.0;
    for (long j = 0; j < S; ++j) {
        if (s_buf[j] == -INFINITY) continue;
        double w = exp(s_buf[j] - m);
        denom += w;
        const uint16_t *vr = op->vb + (size_t)key_slot(op, j, mutation) * op->kv_stride;
        for (int d = 0; d < D; ++d) out[d] += w * bf16_bits_to_f64(vr[d]);
    }
    if (op->has_sink) {
        double ws = exp(sigma - m);
        denom += ws;
        if (mutation == MUT_SINK_IN_NUMERATOR)
            for (int d = 0; d < D; ++d) out[d] += ws;
    }
    for (int d = 0; d < D; ++d) out[d] /= denom;
}

/* Row (b, h, i) of the dense layout: q/o [B,Hq,L,D], k/v [B,Hkv,rows,D] with
 * rows = S, or rows = ring for a rotating cache. */
static void one_row(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *out,
                    int Hq, int Hkv, int L, int S, long ring, int D, double scale,
                    int causal, int window, const float *key_mask, double softcap,
                    const float *sinks, int mutation, long row, double *s_buf)
{
    long i = row % L;
    long bh = row / L;
    int h = (int)(bh % Hq);
    int b = (int)(bh / Hq);
    int g = kv_head_impl(h, Hq, Hkv, mutation);
    size_t rows = ring ? (size_t)ring : (size_t)S;
    RowOperands op;
    op.qr = q + ((size_t)bh * L + i) * D;
    op.kb = k + ((size_t)b * Hkv + g) * rows * D;
    op.vb = v + ((size_t)b * Hkv + g) * rows * D;
    op.kv_stride = (size_t)D;
    op.ring = ring;
    op.mrow = key_mask ? key_mask + (size_t)b * S : NULL;
    op.has_sink = sinks != NULL;
    op.sigma = sinks ? (double)sinks[h] : 0.0;
    op.causal_shift = 0;
    row_core(&op, out, L, S, i, D, scale, causal, window, softcap, mutation, s_buf);
}

static int attention_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                          int B, int Hq, int Hkv, int L, int S, long ring, int D, double scale,
                          int causal, int window, const float *key_mask, double softcap,
                          const float *sinks, const int64_t *rows, int64_t nrows, int nthreads,
                          int mutation)
{
    int rc = check_args(q, k, v, o, B, Hq, Hkv, L, S, D);
    if (rc) return rc;
    if (!(softcap >= 0.0) || isinf(softcap)) return 6;
    /* a rotating cache keeps the last `ring` positions: every key a row may
     * see must still be there, so causal, a window, and ring >= W - 1 + L */
    if (ring < 0 || (ring > 0 && (!causal || window <= 0 || ring < (long)window - 1 + L)))
        return 7;
    int64_t total = rows ? nrows : (int64_t)B * Hq * L;
    if (rows) {
        for (int64_t r = 0; r < nrows; ++r)
            if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq * L) return 4;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        if (!s_buf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < total; ++r) {
            if (!s_buf) continue;
            long row = rows ? (long)rows[r] : (long)r;
            one_row(q, k, v, o + (size_t)r * D, Hq, Hkv, L, S, ring, D, scale, causal, window,
                    key_mask, softcap, sinks, mutation, row, s_buf);
        }
        free(s_buf);
    }
    return failed ? 5 : 0;
}

/* Plain definition.  rows: optional list of flattened (b*Hq + h)*L + i row
 * indices; o then holds nrows x D values in that order.  rows == NULL computes
 * every row and o is [B,Hq,L,D].  Returns 0 on success. */
int oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                     int B, int Hq, int Hkv, int L, int S, int D, double scale,
                     int causal, int window, const float *key_mask,
                     const int64_t *rows, int64_t nrows, int nthreads)
{
    return attention_impl(q, k, v, o, B, Hq, Hkv, L, S, 0, D, scale, causal, window, key_mask,
                          0.0, NULL, rows, nrows, nthreads, MUT_NONE);
}

/* The definition with the score variants: softcap (0 = none) and sinks
 * (fp32 [Hq] logits, NULL = none). */
int oracle_attention_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                        int B, int Hq, int Hkv, int L, int S, int D, double scale,
                        int causal, int window, const float *key_mask, double softcap,
                        const float *sinks, const int64_t *rows, int64_t nrows, int nthreads)
{
    return attention_impl(q, k, v, o, B, Hq, Hkv, L, S, 0, D, scale, causal, window, key_mask,
                          softcap, sinks, rows, nrows, nthreads, MUT_NONE);
}

/* Rotating cache (TensorFold PR 3269, WINDOW and RING): k/v are
 * [B,Hkv,ring,D] and key position j (0 <= j < S, S = prefix + L) lives in row
 * j mod ring.  Causal with a window; ring >= window - 1 + L, so every key a
 * row may see is still in the ring (else returns 7). */
int oracle_attention_ring(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                          int B, int Hq, int Hkv, int L, int S, long ring, int D, double scale,
                          int window, double softcap, const float *sinks, const int64_t *rows,
                          int64_t nrows, int nthreads)
{
    if (ring <= 0) return 7;
    return attention_impl(q, k, v, o, B, Hq, Hkv, L, S, ring, D, scale, 1, window, NULL,
                          softcap, sinks, rows, nrows, nthreads, MUT_NONE);
}

/* The same definition with one planted mistake; for mutation tests only. */
int oracle_attention_mutant(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                            int B, int Hq, int Hkv, int L, int S, long ring, int D, double scale,
                            int causal, int window, const float *key_mask, double softcap,
                            const float *sinks, int mutation)
{
    return attention_impl(q, k, v, o, B, Hq, Hkv, L, S, ring, D, scale, causal, window, key_mask,
                          softcap, sinks, NULL, 0, 1, mutation);
}

/* Packed variable-length attention (brotensor flash_attention.h,
 * flash_attention_varlen_forward comment): sequence b owns query rows
 * [cu_q[b], cu_q[b+1]) and key/value rows [cu_k[b], cu_k[b+1]) of
 * q/o [Tq, Hq, D] and k/v [Tk, Hkv, D]; nothing crosses sequences.  Within a
 * sequence the definition above holds with L = its query count and S = its
 * key count, so the causal offset is S - L (brotensor's rule
 * k - cu_k[b] <= q - cu_q[b] when the two counts match).  A causal sequence
 * needs S >= L (else returns 8). */
static int varlen_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                       const int32_t *cu_q, const int32_t *cu_k, int B, int Hq, int Hkv, int D,
                       double scale, int causal, int window, double softcap, const float *sinks,
                       int nthreads, int mutation)
{
    if (!q || !k || !v || !o || !cu_q || !cu_k) return 1;
    if (B < 1 || Hq < 1 || Hkv < 1 || D < 1) return 2;
    if (Hq % Hkv != 0) return 3;
    if (!(softcap >= 0.0) || isinf(softcap)) return 6;
    if (cu_q[0] != 0 || cu_k[0] != 0) return 8;
    long max_s = 1;
    for (int b = 0; b < B; ++b) {
        long Lb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
        if (Lb < 0 || Sb < 0 || (causal && Sb < Lb)) return 8;
        if (Sb > max_s) max_s = Sb;
    }
    long total = (long)cu_q[B] * Hq;  /* rows, in packed order (t, h) */
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)max_s);
        if (!s_buf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (long r = 0; r < total; ++r) {
            if (!s_buf) continue;
            long t = r / Hq;
            int h = (int)(r % Hq);
            int b = 0;
            while (cu_q[b + 1] <= t) ++b;
            long i = t - cu_q[b];
            long Lb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
            int g = kv_head_impl(h, Hq, Hkv, mutation);
            RowOperands op;
            op.qr = q + ((size_t)t * Hq + h) * D;
            op.kb = k + ((size_t)cu_k[b] * Hkv + g) * D;
            op.vb = v + ((size_t)cu_k[b] * Hkv + g) * D;
            op.kv_stride = (size_t)Hkv * D;
            op.ring = 0;
            op.mrow = NULL;
            op.has_sink = sinks != NULL;
            op.sigma = sinks ? (double)sinks[h] : 0.0;
            op.causal_shift = (mutation == MUT_VARLEN_PACKED_CAUSAL) ? (long)cu_q[b] - cu_k[b] : 0;
            row_core(&op, o + ((size_t)t * Hq + h) * D, Lb, Sb, i, D, scale, causal, window,
                     softcap, mutation, s_buf);
        }
        free(s_buf);
    }
    return failed ? 5 : 0;
}

int oracle_attention_varlen(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                            const int32_t *cu_q, const int32_t *cu_k, int B, int Hq, int Hkv,
                            int D, double scale, int causal, int window, double softcap,
                            const float *sinks, int nthreads)
{
    return varlen_impl(q, k, v, o, cu_q, cu_k, B, Hq, Hkv, D, scale, causal, window, softcap,
                       sinks, nthreads, MUT_NONE);
}

int oracle_attention_varlen_mutant(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                   double *o, const int32_t *cu_q, const int32_t *cu_k, int B,
                                   int Hq, int Hkv, int D, double scale, int causal, int window,
                                   int mutation)
{
    return varlen_impl(q, k, v, o, cu_q, cu_k, B, Hq, Hkv, D, scale, causal, window, 0.0, NULL,
                       1, mutation);
}

/* Row-normalised softmax weights of one (b, h): W is L x S, zero where the
 * key is not allowed, rows of a fully masked query all zero.  Same
 * definition as oracle_attention, stopped before the weighted sum of V. */
int oracle_softmax_weights(const uint16_t *q, const uint16_t *k, double *W,
                           int B, int Hq, int Hkv, int L, int S, int D, double scale,
                           int causal, int window, const float *key_mask, int b, int h,
                           int mutation)
{
    if (!q || !k || !W) return 1;
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || S < L || D < 1 || Hq % Hkv) return 2;
    if (b < 0 || b >= B || h < 0 || h >= Hq) return 4;
    int g = kv_head_impl(h, Hq, Hkv, mutation);
    const float *mrow = key_mask ? key_mask + (size_t)b * S : NULL;
    double sc = (mutation == MUT_DROP_SCALE) ? 1.0 : scale;
    for (long i = 0; i < L; ++i) {
        double *wr = W + (size_t)i * S;
        const uint16_t *qr = q + (((size_t)b * Hq + h) * L + i) * D;
        double m = -INFINITY;
        for (long j = 0; j < S; ++j) {
            wr[j] = -INFINITY;
            if (!allowed_impl(L, S, i, j, causal, window, mrow, mutation)) continue;
            const uint16_t *kr = k + (((size_t)b * Hkv + g) * S + j) * D;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += bf16_bits_to_f64(qr[d]) * bf16_bits_to_f64(kr[d]);
            wr[j] = sc * acc;
            if (wr[j] > m) m = wr[j];
        }
        double denom = 0.0;
        for (long j = 0; j < S; ++j) {
            wr[j] = (wr[j] == -INFINITY) ? 0.0 : exp(wr[j] - m);
            denom += wr[j];
        }
        if (denom > 0.0)
            for (long j = 0; j < S; ++j) wr[j] /= denom;
    }
    return 0;
}

/* Gradients of the plain definition with respect to q, k and v, for an
 * upstream gradient dout of the output (brotensor flash_attention.h,
 * flash_attention_backward and flash_attention_varlen_backward comments: the
 * backward of the bare attention core, recompute-based; causal- and
 * mask-excluded positions contribute nothing to any gradient).  With
 * s = scale q.k over the allowed keys, P the softmax of each row (a row with
 * no allowed key has P = 0 and output 0) and O = P V:
 *   dV[b,g,j]   = sum over the group's heads h and rows i of P[h,i,j] dout[h,i]
 *   dP[h,i,j]   = dout[h,i] . v[g,j]
 *   dS[h,i,j]   = P[h,i,j] (dP[h,i,j] - sum_j' P[h,i,j'] dP[h,i,j'])
 *   dQ[b,h,i]   = scale sum_j dS[h,i,j] k[g,j]
 *   dK[b,g,j]   = scale sum over h, i of dS[h,i,j] q[h,i]
 * (the softmax Jacobian: d softmax_j / d s_j' = P_j (delta_jj' - P_j')).
 * Inputs bf16 bits, upcast exactly; dout likewise; outputs fp64 in the input
 * layouts.  Parallel over (b, g): one thread owns a KV head's dK/dV. */
static int backward_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const uint16_t *dout, double *dq, double *dk, double *dv, int B, int Hq,
                         int Hkv, int L, int S, int D, double scale, int causal, int window,
                         const float *key_mask, int nthreads, int mutation)
{
    int rc = check_args(q, k, v, dq, B, Hq, Hkv, L, S, D);
    if (rc) return rc;
    if (!dout || !dk || !dv) return 1;
    memset(dq, 0, sizeof(double) * (size_t)B * Hq * L * D);
    memset(dk, 0, sizeof(double) * (size_t)B * Hkv * S * D);
    memset(dv, 0, sizeof(double) * (size_t)B * Hkv * S * D);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)S);
        double *dP = (double *)malloc(sizeof(double) * (size_t)S);
        if (!P || !dP) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long bg = 0; bg < (long)B * Hkv; ++bg) {
            if (!P || !dP) continue;
            const int b = (int)(bg / Hkv), g = (int)(bg % Hkv);
            const float *mrow = key_mask ? key_mask + (size_t)b * S : NULL;
            const uint16_t *kb = k + ((size_t)b * Hkv + g) * (size_t)S * D;
            const uint16_t *vb = v + ((size_t)b * Hkv + g) * (size_t)S * D;
            double *dkb = dk + ((size_t)b * Hkv + g) * (size_t)S * D;
            double *dvb = dv + ((size_t)b * Hkv + g) * (size_t)S * D;
            for (int h = 0; h < Hq; ++h) {
                if (kv_head_impl(h, Hq, Hkv, mutation) != g) continue;
                for (long i = 0; i < L; ++i) {
                    const size_t row = (((size_t)b * Hq + h) * L + i) * D;
                    const uint16_t *qr = q + row, *dor = dout + row;
                    double m = -INFINITY;
                    for (long j = 0; j < S; ++j) {
                        P[j] = -INFINITY;
                        if (!allowed_impl(L, S, i, j, causal, window, mrow, mutation)) continue;
                        double acc = 0.0;
                        for (int d = 0; d < D; ++d)
                            acc += bf16_bits_to_f64(qr[d]) * bf16_bits_to_f64(kb[(size_t)j * D + d]);
                        P[j] = scale * acc;
                        if (P[j] > m) m = P[j];
                    }
                    if (m == -INFINITY) continue;  /* no allowed key: no gradient */
                    double denom = 0.0;
                    for (long j = 0; j < S; ++j) {
                        P[j] = (P[j] == -INFINITY) ? 0.0 : exp(P[j] - m);
                        denom += P[j];
                    }
                    double delta = 0.0;  /* sum_j P_j dP_j */
                    for (long j = 0; j < S; ++j) {
                        P[j] /= denom;
                        dP[j] = 0.0;
                        if (P[j] == 0.0) continue;
                        for (int d = 0; d < D; ++d)
                            dP[j] += bf16_bits_to_f64(dor[d]) * bf16_bits_to_f64(vb[(size_t)j * D + d]);
                        delta += P[j] * dP[j];
                    }
                    if (mutation == MUT_BWD_NO_DELTA) delta = 0.0;
                    const double ks = (mutation == MUT_BWD_DK_NO_SCALE) ? 1.0 : scale;
                    const uint16_t *qsrc = (mutation == MUT_BWD_DQ_USES_V) ? vb : kb;
                    for (long j = 0; j < S; ++j) {
                        if (P[j] == 0.0) continue;
                        const double ds = P[j] * (dP[j] - delta);
                        for (int d = 0; d < D; ++d) {
                            dvb[(size_t)j * D + d] += P[j] * bf16_bits_to_f64(dor[d]);
                            dkb[(size_t)j * D + d] += ks * ds * bf16_bits_to_f64(qr[d]);
                            dq[row + d] += scale * ds * bf16_bits_to_f64(qsrc[(size_t)j * D + d]);
                        }
                    }
                }
            }
        }
        free(P);
        free(dP);
    }
    return failed ? 5 : 0;
}

/* dQ of the listed rows only (row = (b*Hq + h)*L + i; dq holds nrows x D):
 * the same per-row arithmetic as backward_impl, which a row's dQ needs alone
 * (its softmax weights, dP and row term), so it scales to any size. */
int oracle_attention_backward_dq_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                      const uint16_t *dout, double *dq, int B, int Hq, int Hkv,
                                      int L, int S, int D, double scale, int causal, int window,
                                      const float *key_mask, const int64_t *rows, int64_t nrows,
                                      int nthreads)
{
    int rc = check_args(q, k, v, dq, B, Hq, Hkv, L, S, D);
    if (rc) return rc;
    if (!dout || !rows) return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq * L) return 4;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)S);
        double *dP = (double *)malloc(sizeof(double) * (size_t)S);
        if (!P || !dP) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!P || !dP) continue;
            const long row = (long)rows[r];
            const long i = row % L;
            const long bh = row / L;
            const int h = (int)(bh % Hq), b = (int)(bh / Hq);
            const int g = kv_head_impl(h, Hq, Hkv, MUT_NONE);
            const float *mrow = key_mask ? key_mask + (size_t)b * S : NULL;
            const uint16_t *kb = k + ((size_t)b * Hkv + g) * (size_t)S * D;
            const uint16_t *vb = v + ((size_t)b * Hkv + g) * (size_t)S * D;
            const uint16_t *qr = q + (size_t)row * D, *dor = dout + (size_t)row * D;
            double *out = dq + (size_t)r * D;
            for (int d = 0; d < D; ++d) out[d] = 0.0;
            double m = -INFINITY;
            for (long j = 0; j < S; ++j) {
                P[j] = -INFINITY;
                if (!allowed_impl(L, S, i, j, causal, window, mrow, MUT_NONE)) continue;
                double acc = 0.0;
                for (int d = 0; d < D; ++d)
                    acc += bf16_bits_to_f64(qr[d]) * bf16_bits_to_f64(kb[(size_t)j * D + d]);
                P[j] = scale * acc;
                if (P[j] > m) m = P[j];
            }
            if (m == -INFINITY) continue;
            double denom = 0.0;
            for (long j = 0; j < S; ++j) {
                P[j] = (P[j] == -INFINITY) ? 0.0 : exp(P[j] - m);
                denom += P[j];
            }
            double delta = 0.0;
            for (long j = 0; j < S; ++j) {
                P[j] /= denom;
                dP[j] = 0.0;
                if (P[j] == 0.0) continue;
                for (int d = 0; d < D; ++d)
                    dP[j] += bf16_bits_to_f64(dor[d]) * bf16_bits_to_f64(vb[(size_t)j * D + d]);
                delta += P[j] * dP[j];
            }
            for (long j = 0; j < S; ++j) {
                if (P[j] == 0.0) continue;
                const double ds = P[j] * (dP[j] - delta);
                for (int d = 0; d < D; ++d) out[d] += scale * ds * bf16_bits_to_f64(kb[(size_t)j * D + d]);
            }
        }
        free(P);
        free(dP);
    }
    return failed ? 5 : 0;
}

/* dK and dV of the listed keys of KV head g of batch b only (dk, dv hold
 * nkeys x D each): every query row of the group's heads still needs its full
 * softmax normalisation and row term, but only the listed keys' products are
 * accumulated.  Same arithmetic as backward_impl; parallel over query rows
 * with per-thread accumulators reduced at the end. */
int oracle_attention_backward_kv_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                      const uint16_t *dout, double *dk, double *dv, int B, int Hq,
                                      int Hkv, int L, int S, int D, double scale, int causal,
                                      int window, const float *key_mask, int b, int g,
                                      const int64_t *keys, int64_t nkeys, int nthreads)
{
    int rc = check_args(q, k, v, dk, B, Hq, Hkv, L, S, D);
    if (rc) return rc;
    if (!dout || !dv || !keys) return 1;
    if (b < 0 || b >= B || g < 0 || g >= Hkv) return 4;
    for (int64_t t = 0; t < nkeys; ++t)
        if (keys[t] < 0 || keys[t] >= S) return 4;
    const int G = Hq / Hkv;
    memset(dk, 0, sizeof(double) * (size_t)nkeys * D);
    memset(dv, 0, sizeof(double) * (size_t)nkeys * D);
    const float *mrow = key_mask ? key_mask + (size_t)b * S : NULL;
    const uint16_t *kb = k + ((size_t)b * Hkv + g) * (size_t)S * D;
    const uint16_t *vb = v + ((size_t)b * Hkv + g) * (size_t)S * D;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)S);
        double *dP = (double *)malloc(sizeof(double) * (size_t)S);
        double *ak = (double *)calloc((size_t)nkeys * D, sizeof(double));
        double *av = (double *)calloc((size_t)nkeys * D, sizeof(double));
        if (!P || !dP || !ak || !av) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (long hi = 0; hi < (long)G * L; ++hi) {
            if (!P || !dP || !ak || !av) continue;
            const int h = g * G + (int)(hi / L);
            const long i = hi % L;
            const size_t row = (((size_t)b * Hq + h) * L + i) * D;
            const uint16_t *qr = q + row, *dor = dout + row;
            double m = -INFINITY;
            for (long j = 0; j < S; ++j) {
                P[j] = -INFINITY;
                if (!allowed_impl(L, S, i, j, causal, window, mrow, MUT_NONE)) continue;
                double acc = 0.0;
                for (int d = 0; d < D; ++d)
                    acc += bf16_bits_to_f64(qr[d]) * bf16_bits_to_f64(kb[(size_t)j * D + d]);
                P[j] = scale * acc;
                if (P[j] > m) m = P[j];
            }
            if (m == -INFINITY) continue;
            double denom = 0.0;
            for (long j = 0; j < S; ++j) {
                P[j] = (P[j] == -INFINITY) ? 0.0 : exp(P[j] - m);
                denom += P[j];
            }
            double delta = 0.0;
            for (long j = 0; j < S; ++j) {
                P[j] /= denom;
                dP[j] = 0.0;
                if (P[j] == 0.0) continue;
                for (int d = 0; d < D; ++d)
                    dP[j] += bf16_bits_to_f64(dor[d]) * bf16_bits_to_f64(vb[(size_t)j * D + d]);
                delta += P[j] * dP[j];
            }
            for (int64_t t = 0; t < nkeys; ++t) {
                const long j = (long)keys[t];
                if (P[j] == 0.0) continue;
                const double ds = P[j] * (dP[j] - delta);
                for (int d = 0; d < D; ++d) {
                    av[(size_t)t * D + d] += P[j] * bf16_bits_to_f64(dor[d]);
                    ak[(size_t)t * D + d] += scale * ds * bf16_bits_to_f64(qr[d]);
                }
            }
        }
#pragma omp critical
        {
            if (ak && av)
                for (size_t e = 0; e < (size_t)nkeys * D; ++e) {
                    dk[e] += ak[e];
                    dv[e] += av[e];
                }
        }
        free(P);
        free(dP);
        free(ak);
        free(av);
    }
    return failed ? 5 : 0;
}

int oracle_attention_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const uint16_t *dout, double *dq, double *dk, double *dv, int B,
                              int Hq, int Hkv, int L, int S, int D, double scale, int causal,
                              int window, const float *key_mask, int nthreads)
{
    return backward_impl(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, D, scale, causal, window,
                         key_mask, nthreads, MUT_NONE);
}

int oracle_attention_backward_mutant(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                     const uint16_t *dout, double *dq, double *dk, double *dv,
                                     int B, int Hq, int Hkv, int L, int S, int D, double scale,
                                     int causal, int window, const float *key_mask, int mutation)
{
    return backward_impl(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, D, scale, causal, window,
                         key_mask, 1, mutation);
}

/* Brute-force count of allowed (b, h, i, j) quadruples: the "unmasked pairs"
 * whose 4*D flops the throughput metric counts. */
int64_t oracle_count_pairs(int B, int Hq, int L, int S, int causal, int window,
                           const float *key_mask)
{
    int64_t n = 0;
    for (int b = 0; b < B; ++b) {
        const float *mrow = key_mask ? key_mask + (size_t)b * S : NULL;
        int64_t nb = 0;
        for (long i = 0; i < L; ++i)
            for (long j = 0; j < S; ++j) nb += allowed_impl(L, S, i, j, causal, window, mrow, MUT_NONE);
        n += nb * Hq;
    }
    return n;
}

/* Tiled online-softmax variant, following the merge of tiny-llm Week 2 Day 5,
 * Task 1: per row keep FP-accumulated running max m, sum l and weighted value
 * accumulator a; for each key tile with tile maximum m_b, tile sum l_b and
 * tile accumulator a_b:
 *     m' = max(m, m_b)
 *     l' = e^(m - m') l + e^(m_b - m') l_b
 *     a' = e^(m - m') a + e^(m_b - m') a_b
 * and finally out = a' / l'.  Key tiles are BK wide; rows are grouped in
 * blocks of BQ, and when skip_empty is set a key tile that has no allowed
 * (row, key) pair for ANY row of the block is skipped without reading K/V
 * (the masked-tile skipping of mlx-lm PR "Skip fully masked key tiles in Flint
 * sliding-window prefill").  A tile with no allowed key for one row contributes
 * nothing to that row: its masked scores add zero weight to the row sum and to
 * the accumulator (tiny-llm Week 2 Day 5, Task 1, the merge with masked cells).
 * Exists so tests can show that tiling, merging and skipping leave the plain
 * definition's result unchanged. */
int oracle_attention_blockwise(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *o,
                               int B, int Hq, int Hkv, int L, int S, int D, double scale,
                               int causal, int window, const float *key_mask,
                               int BQ, int BK, int skip_empty, int64_t *tiles_visited)
{
    int rc = check_args(q, k, v, o, B, Hq, Hkv, L, S, D);
    if (rc) return rc;
    if (BQ < 1 || BK < 1) return 2;
    int64_t visited = 0;
    double *a = (double *)malloc(sizeof(double) * (size_t)D);
    double *ab = (double *)malloc(sizeof(double) * (size_t)D);
    double *sb = (double *)malloc(sizeof(double) * (size_t)BK);
    if (!a || !ab || !sb) { free(a); free(ab); free(sb); return 5; }
    for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
        int g = kv_head_impl(h, Hq, Hkv, MUT_NONE);
        const float *mrow = key_mask ? key_mask + (size_t)b * S : NULL;
        for (long i0 = 0; i0 < L; i0 += BQ) {
            long i1 = (i0 + BQ < L) ? i0 + BQ : L;
            for (long i = i0; i < i1; ++i) {
                const uint16_t *qr = q + (((size_t)b * Hq + h) * L + i) * D;
                double m = -INFINITY, l = 0.0;
                for (int d = 0; d < D; ++d) a[d] = 0.0;
                for (long j0 = 0; j0 < S; j0 += BK) {
                    long j1 = (j0 + BK < S) ? j0 + BK : S;
                    if (skip_empty) {
                        int live = 0;
                        for (long ii = i0; ii < i1 && !live; ++ii)
                            for (long j = j0; j < j1 && !live; ++j)
                                live = allowed_impl(L, S, ii, j, causal, window, mrow, MUT_NONE);
                        if (!live) continue;
                    }
                    if (i == i0) ++visited;
                    double mb = -INFINITY;
                    for (long j = j0; j < j1; ++j) {
                        sb[j - j0] = -INFINITY;
                        if (!allowed_impl(L, S, i, j, causal, window, mrow, MUT_NONE)) continue;
                        const uint16_t *kr = k + (((size_t)b * Hkv + g) * S + j) * D;
                        double acc = 0.0;
                        for (int d = 0; d < D; ++d) acc += bf16_bits_to_f64(qr[d]) * bf16_bits_to_f64(kr[d]);
                        sb[j - j0] = scale * acc;
                        if (sb[j - j0] > mb) mb = sb[j - j0];
                    }
                    if (mb == -INFINITY) continue; /* no mass in this tile for this row */
                    double lb = 0.0;
                    for (int d = 0; d < D; ++d) ab[d] = 0.0;
                    for (long j = j0; j < j1; ++j) {
                        if (sb[j - j0] == -INFINITY) continue;
                        double w = exp(sb[j - j0] - mb);
                        lb += w;
                        const uint16_t *vr = v + (((size_t)b * Hkv + g) * S + j) * D;
                        for (int d = 0; d < D; ++d) ab[d] += w * bf16_bits_to_f64(vr[d]);
                    }
                    double mn = (m > mb) ? m : mb;
                    double fo = (m == -INFINITY) ? 0.0 : exp(m - mn);
                    double fb = exp(mb - mn);
                    l = fo * l + fb * lb;
                    for (int d = 0; d < D; ++d) a[d] = fo * a[d] + fb * ab[d];
                    m = mn;
                }
                double *out = o + (((size_t)b * Hq + h) * L + i) * D;
                for (int d = 0; d < D; ++d) out[d] = (l > 0.0) ? a[d] / l : 0.0;
            }
        }
    }
    free(a); free(ab); free(sb);
    if (tiles_visited) *tiles_visited = visited;
    return 0;
}
