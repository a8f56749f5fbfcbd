/*
 * Exact-attention oracle: a plain, slow, fp64 CPU restatement of what the
 * attention forward pass computes.  TEST INFRASTRUCTURE ONLY: the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it; the product
 * path never does.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it follows (page, section):
 *  - "FlashAttention-3 vs naive attention" (cnblogs), section 1.1: the basic
 *    attention S = QK^T/sqrt(d) + mask, P = softmax(S), O = PV.  This file
 *    writes that definition out literally, one query row at a time: all
 *    scores of the row are materialised, the softmax is taken in two passes
 *    (row max, then exponentials and their sum), and the output is the
 *    P-weighted sum of V rows.  No tiling and no online recurrence: the pages
 *    state that the tiled method is exactly equal to this (gsyq.cn FA vs FIA,
 *    section 1; cnblogs section 1 and section 9).
 *  - "flash-attention" skill page (skillsmp), section 3.2: causal mask and
 *    the default softmax_scale = 1/sqrt(headdim); section 3.4: packed
 *    variable-length batches described by cu_seqlens, with no attention
 *    across sequences; appendix "GQA/MQA": q heads share kv heads without a
 *    manual repeat (read as contiguous groups, kv head = h / (Hq/Hkv));
 *    appendix "PagedAttention": a paged K/V pool [num_blocks, block_size,
 *    kv_heads, head_dim] addressed through block_table[batch, max_blocks]
 *    and cache_seqlens[batch], with one query token per request at the last
 *    position (it sees every cached token).
 *  - The log-sum-exp of each row (natural log, of the scaled logits) is
 *    returned beside O; the pages name the row max m and sum l, and
 *    LSE = m + ln l.
 *  - "flash-attention" skill page, section 3.3 (advanced features): a
 *    sliding window window_size = (left, right) -- key j is visible to query
 *    i when i - left <= j <= i + right, a negative bound meaning no limit on
 *    that side ((4096, 0) looks 4096 tokens to the left); softcapping, which
 *    replaces each logit x by softcap * tanh(x / softcap); and ALiBi slopes of
 *    shape (nheads,) or (batch, nheads), read as the linear distance penalty
 *    -slope * |i - j| added to the logit of query i and key j.  Logit here
 *    means the scaled score scale * <q, k>; the cap is applied first and the
 *    ALiBi penalty is added to the capped value.
 *  - "flash-attention" skill page, section 3.5 (inference KV cache): one new
 *    token per request is appended to the (paged) cache -- k_new and v_new go
 *    to position cache_seqlens[b] -- and its query attends to the cache
 *    including itself; rotary_cos / rotary_sin apply RoPE on the fly to q
 *    and k_new at that position, pairs (x_i, x_{i + rd/2}) by default and
 *    adjacent pairs (x_{2i}, x_{2i+1}) when rotary_interleaved; dimensions
 *    past the rotary dimension rd are left as they are.  The cache holds
 *    bf16, so the rotated key is the exact rotation rounded once to bf16
 *    (nearest, ties to even), and the rotated query likewise (it feeds a
 *    bf16 product).
 *  - FP8 (skill page, comparison tables: FA3/FA4 support FP8): Q, K and V
 *    stored as OCP e4m3 bytes (4 exponent bits, bias 7, 3 mantissa bits, no
 *    infinities) with one descale factor per tensor; the attention is the
 *    plain definition on the exact values descale * e4m3.
 *
 * Precision: every product and sum is in double.  Inputs are read in the
 * caller's element type (bf16 bit patterns, fp32 or fp64) and upcast
 * exactly.  The scale is taken as given (callers pass the fp32 value the GPU
 * receives).
 *
 * Threading: OpenMP over independent (row, head) units only; each unit is
 * computed by one thread in a fixed order, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_BF16 = 0, OR_F32 = 1, OR_F64 = 2 };

/* Exact upcast of one element of an input tensor. */
static double elem(const void *base, size_t i, int dtype)
{
    if (dtype == OR_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    if (dtype == OR_F32)
        return (double)((const float *)base)[i];
    return ((const double *)base)[i];
}

/*
 * The logits of one query row against an explicit list of key rows:
 * s_j = scale * <q, k_j>, then softcap * tanh(s_j / softcap) when
 * softcap > 0, then + bias[j] when bias is not NULL.
 */
static void row_logits_q(const void *q, int qdtype, const void *k, int dtype, size_t qrow,
                         const size_t *krows, size_t n, int d, double scale, double softcap,
                         const double *bias, double *s)
{
    for (size_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += elem(q, qrow + (size_t)c, qdtype) * elem(k, krows[j] + (size_t)c, dtype);
        s[j] = scale * dot;
        if (softcap > 0.0)
            s[j] = softcap * tanh(s[j] / softcap);
        if (bias)
            s[j] += bias[j];
    }
}

static void row_logits(const void *q, const void *k, int dtype, size_t qrow,
                       const size_t *krows, size_t n, int d, double scale, double softcap,
                       const double *bias, double *s)
{
    row_logits_q(q, dtype, k, dtype, qrow, krows, n, d, scale, softcap, bias, s);
}

/*
 * One query row against an explicit list of key/value rows.
 *   qrow: element offset of the query vector (d consecutive elements)
 *   krows/vrows: element offsets of each visible key/value vector
 *   n: number of visible keys (n == 0 gives O = 0, LSE = -inf)
 *   softcap, bias: logit modifiers of row_logits (0 / NULL for none)
 * s and p are caller scratch of length >= n.
 */
static void attend_one_row_q(const void *q, int qdtype, const void *k, const void *v,
                             int dtype, size_t qrow, const size_t *krows, const size_t *vrows,
                             size_t n, int d, double scale, double softcap,
                             const double *bias, double *s, double *p, double *o_out,
                             double *lse_out)
{
    if (n == 0) {
        for (int c = 0; c < d; ++c)
            o_out[c] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    row_logits_q(q, qdtype, k, dtype, qrow, krows, n, d, scale, softcap, bias, s);
    /* softmax, pass 1: the row max */
    double m = s[0];
    for (size_t j = 1; j < n; ++j)
        if (s[j] > m)
            m = s[j];
    /* pass 2: exponentials, their sum, and the normalised probabilities */
    double z = 0.0;
    for (size_t j = 0; j < n; ++j) {
        p[j] = exp(s[j] - m);
        z += p[j];
    }
    for (size_t j = 0; j < n; ++j)
        p[j] = p[j] / z;
    /* O = sum_j P_j v_j */
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (size_t j = 0; j < n; ++j)
            acc += p[j] * elem(v, vrows[j] + (size_t)c, dtype);
        o_out[c] = acc;
    }
    *lse_out = m + log(z);
}

static void attend_one_row(const void *q, const void *k, const void *v, int dtype,
                           size_t qrow, const size_t *krows, const size_t *vrows,
                           size_t n, int d, double scale, double softcap, const double *bias,
                           double *s, double *p, double *o_out, double *lse_out)
{
    attend_one_row_q(q, dtype, k, v, dtype, qrow, krows, vrows, n, d, scale, softcap, bias, s,
                     p, o_out, lse_out);
}

/* Sequence index b such that cu[b] <= t < cu[b+1]; -1 if none. */
static int seq_of_token(const int32_t *cu, int B, int64_t t)
{
    for (int b = 0; b < B; ++b)
        if (t >= cu[b] && t < cu[b + 1])
            return b;
    return -1;
}

/*
 * Whether key j is visible to query i, both local indices in a sequence of L
 * tokens: j in [0, L); causal keeps j <= i; window_left >= 0 keeps
 * j >= i - window_left; window_right >= 0 keeps j <= i + window_right.
 */
static int key_visible(int64_t i, int64_t j, int64_t L, int causal, int window_left,
                       int window_right)
{
    if (j < 0 || j >= L)
        return 0;
    if (causal && j > i)
        return 0;
    if (window_left >= 0 && j < i - window_left)
        return 0;
    if (window_right >= 0 && j > i + window_right)
        return 0;
    return 1;
}

/* The ALiBi slope of (sequence b, query head h): alibi[b * stride + h]
 * (stride 0 for one slope per head, Hq for one per sequence and head). */
static double alibi_slope(const float *alibi, int stride, int b, int h)
{
    return (double)alibi[(size_t)b * (size_t)stride + (size_t)h];
}

/*
 * Prefill for an explicit list of (token, head) rows.
 *   q: [T, Hq, d]; k, v: [T, Hkv, d]; cu_seqlens: [B+1] prefix sums.
 *   rows_t/rows_h: the requested rows (nrows of them).
 *   o: [nrows, d] (double); lse: [nrows] (double).
 * Query token t of sequence b (local index i = t - cu[b]) sees the keys
 * cu[b] + j with key_visible(i, j, ...).  softcap > 0 caps the logits;
 * alibi (fp32, may be NULL) adds -slope * |i - j|.
 * Returns 0, or -1 on an invalid argument.
 */
int oracle_prefill_rows_ex(const void *q, const void *k, const void *v, int dtype,
                           const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d,
                           int causal, double scale, int window_left, int window_right,
                           double softcap, const float *alibi, int alibi_stride,
                           const int64_t *rows_t, const int32_t *rows_h, int64_t nrows,
                           double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || softcap < 0.0 ||
        alibi_stride < 0)
        return -1;
    int64_t T = cu_seqlens[B];
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b) {
        if (cu_seqlens[b + 1] < cu_seqlens[b])
            return -1;
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen)
            maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    }
    for (int64_t r = 0; r < nrows; ++r)
        if (rows_t[r] < 0 || rows_t[r] >= T || rows_h[r] < 0 || rows_h[r] >= Hq)
            return -1;
    const int group = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        size_t cap = (size_t)(maxlen > 0 ? maxlen : 1);
        double *s = (double *)malloc(cap * sizeof(double));
        double *p = (double *)malloc(cap * sizeof(double));
        double *bias = (double *)malloc(cap * sizeof(double));
        size_t *kr = (size_t *)malloc(cap * sizeof(size_t));
        if (!s || !p || !bias || !kr) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t t = rows_t[r];
                int h = rows_h[r];
                int kh = h / group;
                int b = seq_of_token(cu_seqlens, B, t);
                int64_t start = cu_seqlens[b];
                int64_t L = cu_seqlens[b + 1] - start;
                int64_t i = t - start;
                double slope = alibi ? alibi_slope(alibi, alibi_stride, b, h) : 0.0;
                size_t n = 0;
                for (int64_t j = 0; j < L; ++j) {
                    if (!key_visible(i, j, L, causal, window_left, window_right))
                        continue;
                    kr[n] = ((size_t)(start + j) * (size_t)Hkv + (size_t)kh) * (size_t)d;
                    bias[n] = -slope * fabs((double)(i - j));
                    ++n;
                }
                size_t qrow = ((size_t)t * (size_t)Hq + (size_t)h) * (size_t)d;
                attend_one_row(q, k, v, dtype, qrow, kr, kr, n, d, scale, softcap,
                               alibi ? bias : NULL, s, p, o + (size_t)r * (size_t)d, lse + r);
            }
        }
        free(s);
        free(p);
        free(bias);
        free(kr);
    }
    return bad ? -1 : 0;
}

/* oracle_prefill_rows_ex with no window, cap or ALiBi. */
int oracle_prefill_rows(const void *q, const void *k, const void *v, int dtype,
                        const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d,
                        int causal, double scale, const int64_t *rows_t,
                        const int32_t *rows_h, int64_t nrows, double *o, double *lse)
{
    return oracle_prefill_rows_ex(q, k, v, dtype, cu_seqlens, B, Hq, Hkv, d, causal, scale,
                                  -1, -1, 0.0, NULL, 0, rows_t, rows_h, nrows, o, lse);
}

/*
 * Full prefill: every (token, head).  o: [T, Hq, d] double; lse: [Hq, T]
 * double (may be NULL).  Variant arguments as in oracle_prefill_rows_ex.
 */
int oracle_prefill_ex(const void *q, const void *k, const void *v, int dtype,
                      const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                      double scale, int window_left, int window_right, double softcap,
                      const float *alibi, int alibi_stride, double *o, double *lse)
{
    if (B < 0 || Hq <= 0)
        return -1;
    int64_t T = cu_seqlens[B];
    int64_t nrows = T * Hq;
    int64_t *rt = (int64_t *)calloc((size_t)(nrows > 0 ? nrows : 1), sizeof(int64_t));
    int32_t *rh = (int32_t *)calloc((size_t)(nrows > 0 ? nrows : 1), sizeof(int32_t));
    double *l = (double *)calloc((size_t)(nrows > 0 ? nrows : 1), sizeof(double));
    if (!rt || !rh || !l) {
        free(rt);
        free(rh);
        free(l);
        return -1;
    }
    /* row r = t*Hq + h, so o comes out directly in [T, Hq, d] order */
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < Hq; ++h) {
            rt[t * Hq + h] = t;
            rh[t * Hq + h] = h;
        }
    int rc = oracle_prefill_rows_ex(q, k, v, dtype, cu_seqlens, B, Hq, Hkv, d, causal, scale,
                                    window_left, window_right, softcap, alibi, alibi_stride,
                                    rt, rh, nrows, o, l);
    if (rc == 0 && lse)
        for (int64_t t = 0; t < T; ++t)
            for (int h = 0; h < Hq; ++h)
                lse[(size_t)h * (size_t)T + (size_t)t] = l[t * Hq + h];
    free(rt);
    free(rh);
    free(l);
    return rc;
}

/* oracle_prefill_ex with no window, cap or ALiBi. */
int oracle_prefill(const void *q, const void *k, const void *v, int dtype,
                   const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                   double scale, double *o, double *lse)
{
    return oracle_prefill_ex(q, k, v, dtype, cu_seqlens, B, Hq, Hkv, d, causal, scale, -1, -1,
                             0.0, NULL, 0, o, lse);
}

/*
 * The probability matrix P of one (sequence, head) for small cases:
 * P: [L, L] double, row i = query i, column j = key j, zero where masked.
 * Variant arguments as in oracle_prefill_rows_ex.
 */
int oracle_prefill_probs(const void *q, const void *k, int dtype, const int32_t *cu_seqlens,
                         int B, int Hq, int Hkv, int d, int causal, double scale,
                         int window_left, int window_right, double softcap, const float *alibi,
                         int alibi_stride, int b, int h, double *P)
{
    if (b < 0 || b >= B || h < 0 || h >= Hq || Hq % Hkv != 0 || softcap < 0.0)
        return -1;
    int64_t start = cu_seqlens[b];
    int64_t L = cu_seqlens[b + 1] - start;
    int kh = h / (Hq / Hkv);
    size_t cap = (size_t)(L > 0 ? L : 1);
    double *s = (double *)malloc(cap * sizeof(double));
    double *bias = (double *)malloc(cap * sizeof(double));
    size_t *kr = (size_t *)malloc(cap * sizeof(size_t));
    int64_t *col = (int64_t *)malloc(cap * sizeof(int64_t));
    if (!s || !bias || !kr || !col) {
        free(s);
        free(bias);
        free(kr);
        free(col);
        return -1;
    }
    double slope = alibi ? alibi_slope(alibi, alibi_stride, b, h) : 0.0;
    for (int64_t i = 0; i < L; ++i) {
        size_t n = 0;
        for (int64_t j = 0; j < L; ++j) {
            P[(size_t)i * (size_t)L + (size_t)j] = 0.0;
            if (!key_visible(i, j, L, causal, window_left, window_right))
                continue;
            kr[n] = ((size_t)(start + j) * (size_t)Hkv + (size_t)kh) * (size_t)d;
            bias[n] = -slope * fabs((double)(i - j));
            col[n] = j;
            ++n;
        }
        if (n == 0)
            continue;
        size_t qrow = ((size_t)(start + i) * (size_t)Hq + (size_t)h) * (size_t)d;
        row_logits(q, k, dtype, qrow, kr, n, d, scale, softcap, alibi ? bias : NULL, s);
        double m = s[0];
        for (size_t j = 1; j < n; ++j)
            if (s[j] > m)
                m = s[j];
        double z = 0.0;
        for (size_t j = 0; j < n; ++j)
            z += exp(s[j] - m);
        for (size_t j = 0; j < n; ++j)
            P[(size_t)i * (size_t)L + (size_t)col[j]] = exp(s[j] - m) / z;
    }
    free(s);
    free(bias);
    free(kr);
    free(col);
    return 0;
}

/*
 * Paged decode: one query token per request at the last position.
 *   q: [B, Hq, d]; k_pages, v_pages: [num_pages, page_size, Hkv, d]
 *   block_table: [B, max_blocks] int32; seq_lens: [B] int32
 *   o: [B, Hq, d] double; lse: [B, Hq] double (may be NULL)
 * Token t of request b lives in page block_table[b][t / page_size], slot
 * t % page_size.  Computed in one pass over all seq_len tokens, with no
 * split: splitting is what the GPU path does and is checked against this.
 * Returns 0, -1 on an invalid argument, -2 if a used block_table entry is
 * outside [0, num_pages).
 */
int oracle_decode_paged(const void *q, const void *k_pages, const void *v_pages, int dtype,
                        const int32_t *block_table, const int32_t *seq_lens, int B, int Hq,
                        int Hkv, int d, int page_size, int max_blocks, int64_t num_pages,
                        double scale, double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || page_size <= 0)
        return -1;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || (int64_t)seq_lens[b] > (int64_t)max_blocks * page_size)
            return -1;
        if (seq_lens[b] > maxlen)
            maxlen = seq_lens[b];
        int64_t used = ((int64_t)seq_lens[b] + page_size - 1) / page_size;
        for (int64_t i = 0; i < used; ++i) {
            int32_t pg = block_table[(size_t)b * (size_t)max_blocks + (size_t)i];
            if (pg < 0 || pg >= num_pages)
                return -2;
        }
    }
    const int group = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        size_t cap = (size_t)(maxlen > 0 ? maxlen : 1);
        double *s = (double *)malloc(cap * sizeof(double));
        double *p = (double *)malloc(cap * sizeof(double));
        size_t *kr = (size_t *)malloc(cap * sizeof(size_t));
        if (!s || !p || !kr) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)B * Hq; ++r) {
                int b = (int)(r / Hq);
                int h = (int)(r % Hq);
                int kh = h / group;
                int64_t n = seq_lens[b];
                for (int64_t t = 0; t < n; ++t) {
                    int64_t page = block_table[(size_t)b * (size_t)max_blocks + (size_t)(t / page_size)];
                    int64_t slot = t % page_size;
                    kr[t] = (((size_t)page * (size_t)page_size + (size_t)slot) * (size_t)Hkv +
                             (size_t)kh) * (size_t)d;
                }
                double l;
                attend_one_row(q, k_pages, v_pages, dtype, (size_t)r * (size_t)d, kr, kr,
                               (size_t)n, d, scale, 0.0, NULL, s, p, o + (size_t)r * (size_t)d,
                               &l);
                if (lse)
                    lse[r] = l;
            }
        }
        free(s);
        free(p);
        free(kr);
    }
    return bad ? -1 : 0;
}

/*
 * Nearest bf16 value of a double (ties to even), as a double.  bf16 keeps 8
 * significant bits and the fp32 exponent range; the inputs here are far
 * from its overflow and underflow limits.
 */
static double round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x))
        return x;
    int e;
    double m = frexp(x, &e);         /* x = m * 2^e, 0.5 <= |m| < 1 */
    double scaled = ldexp(m, 8);     /* 8 significant bits above the point */
    double r = nearbyint(scaled);    /* default rounding: nearest, ties to even */
    return ldexp(r, e - 8);
}

/* Bit pattern of the bf16 value of a double that round_bf16 already made
 * representable. */
static uint16_t bf16_bits(double x)
{
    float f = (float)x;              /* exact: x has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/*
 * RoPE of one d-vector at table row `row` (cos/sin rows of rd/2 fp32
 * values): pair i is (x_i, x_{i+rd/2}), or (x_{2i}, x_{2i+1}) when
 * interleaved, rotated by the angle whose cosine and sine are cos[i] and
 * sin[i]; dims >= rd are copied.  In and out are double.
 */
static void rope_vec(const double *x, double *out, int d, int rd, int interleaved,
                     const float *cos_row, const float *sin_row)
{
    for (int c = 0; c < d; ++c)
        out[c] = x[c];
    for (int i = 0; i < rd / 2; ++i) {
        int a = interleaved ? 2 * i : i;
        int b = interleaved ? 2 * i + 1 : i + rd / 2;
        double co = (double)cos_row[i], si = (double)sin_row[i];
        out[a] = x[a] * co - x[b] * si;
        out[b] = x[a] * si + x[b] * co;
    }
}

/*
 * RoPE of n rows: x [n, d] (dtype), pos [n], tables cos/sin [max_pos, rd/2]
 * fp32; out [n, d] double, exact (not rounded).  Returns 0, -1 on a bad
 * argument (rd odd or > d, or a position outside [0, max_pos)).
 */
int oracle_rope(const void *x, int dtype, int64_t n, int d, const int32_t *pos,
                const float *cos_tab, const float *sin_tab, int64_t max_pos, int rotary_dim,
                int interleaved, double *out)
{
    if (n < 0 || d <= 0 || rotary_dim < 0 || rotary_dim > d || rotary_dim % 2 != 0)
        return -1;
    double *row = (double *)malloc((size_t)d * sizeof(double));
    if (!row)
        return -1;
    int bad = 0;
    for (int64_t r = 0; r < n && !bad; ++r) {
        if (pos[r] < 0 || pos[r] >= max_pos) {
            bad = 1;
            break;
        }
        for (int c = 0; c < d; ++c)
            row[c] = elem(x, (size_t)r * (size_t)d + (size_t)c, dtype);
        const float *co = cos_tab + (size_t)pos[r] * (size_t)(rotary_dim / 2);
        const float *si = sin_tab + (size_t)pos[r] * (size_t)(rotary_dim / 2);
        rope_vec(row, out + (size_t)r * (size_t)d, d, rotary_dim, interleaved, co, si);
    }
    free(row);
    return bad ? -1 : 0;
}

/*
 * Decode with cache append and optional RoPE, bf16 tensors only.
 *   q [B, Hq, d]; k_new, v_new [B, Hkv, d]; k_pages, v_pages
 *   [num_pages, page_size, Hkv, d] (bf16 bits, MODIFIED: the new token is
 *   written at position cache_seqlens[b]); block_table [B, max_blocks];
 *   cache_seqlens [B] = tokens already cached; cos/sin [max_pos, rd/2] fp32
 *   or NULL (no rotation; rotary_dim ignored).
 *   q_rot (out, may be NULL) [B, Hq, d] double: the bf16 rotated queries.
 *   o [B, Hq, d] double; lse [B, Hq] double (may be NULL).
 * Steps: for every request, rotate (or not) q and k_new at position
 * pos = cache_seqlens[b], round them to bf16, write k and v_new into the
 * page slot of pos; then every query attends to tokens [0, pos] of its
 * request's updated cache.  Returns 0, -1 on a bad argument, -2 if a page
 * the append or the attention needs is outside [0, num_pages).
 */
int oracle_decode_paged_append(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                               uint16_t *k_pages, uint16_t *v_pages,
                               const int32_t *block_table, const int32_t *cache_seqlens, int B,
                               int Hq, int Hkv, int d, int page_size, int max_blocks,
                               int64_t num_pages, double scale, const float *cos_tab,
                               const float *sin_tab, int64_t max_pos, int rotary_dim,
                               int interleaved, double *q_rot, double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || page_size <= 0)
        return -1;
    if (cos_tab && (rotary_dim < 0 || rotary_dim > d || rotary_dim % 2 != 0))
        return -1;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b) {
        int64_t pos = cache_seqlens[b];
        if (pos < 0 || pos + 1 > (int64_t)max_blocks * page_size)
            return -1;
        if (cos_tab && pos >= max_pos)
            return -1;
        if (pos + 1 > maxlen)
            maxlen = pos + 1;
        for (int64_t i = 0; i <= pos / page_size; ++i) {
            int32_t pg = block_table[(size_t)b * (size_t)max_blocks + (size_t)i];
            if (pg < 0 || pg >= num_pages)
                return -2;
        }
    }
    const int group = Hq / Hkv;
    double *qr = (double *)malloc((size_t)B * (size_t)Hq * (size_t)d * sizeof(double));
    double *tmp = (double *)malloc((size_t)d * sizeof(double));
    double *rot = (double *)malloc((size_t)d * sizeof(double));
    if (!qr || !tmp || !rot) {
        free(qr);
        free(tmp);
        free(rot);
        return -1;
    }
    /* 1. rotate, round to bf16, append */
    for (int b = 0; b < B; ++b) {
        int64_t pos = cache_seqlens[b];
        const float *co = cos_tab ? cos_tab + (size_t)pos * (size_t)(rotary_dim / 2) : NULL;
        const float *si = cos_tab ? sin_tab + (size_t)pos * (size_t)(rotary_dim / 2) : NULL;
        for (int h = 0; h < Hq; ++h) {
            size_t off = ((size_t)b * (size_t)Hq + (size_t)h) * (size_t)d;
            for (int c = 0; c < d; ++c)
                tmp[c] = elem(q, off + (size_t)c, OR_BF16);
            if (co)
                rope_vec(tmp, rot, d, rotary_dim, interleaved, co, si);
            else
                memcpy(rot, tmp, (size_t)d * sizeof(double));
            for (int c = 0; c < d; ++c)
                qr[off + (size_t)c] = round_bf16(rot[c]);
        }
        int64_t page = block_table[(size_t)b * (size_t)max_blocks + (size_t)(pos / page_size)];
        int64_t slot = pos % page_size;
        for (int kh = 0; kh < Hkv; ++kh) {
            size_t src = ((size_t)b * (size_t)Hkv + (size_t)kh) * (size_t)d;
            size_t dst = (((size_t)page * (size_t)page_size + (size_t)slot) * (size_t)Hkv +
                          (size_t)kh) * (size_t)d;
            for (int c = 0; c < d; ++c)
                tmp[c] = elem(k_new, src + (size_t)c, OR_BF16);
            if (co)
                rope_vec(tmp, rot, d, rotary_dim, interleaved, co, si);
            else
                memcpy(rot, tmp, (size_t)d * sizeof(double));
            for (int c = 0; c < d; ++c) {
                k_pages[dst + (size_t)c] = bf16_bits(round_bf16(rot[c]));
                v_pages[dst + (size_t)c] = v_new[src + (size_t)c];
            }
        }
    }
    if (q_rot)
        memcpy(q_rot, qr, (size_t)B * (size_t)Hq * (size_t)d * sizeof(double));
    /* 2. attend over [0, pos] of the updated cache */
    int bad = 0;
#pragma omp parallel
    {
        size_t cap = (size_t)(maxlen > 0 ? maxlen : 1);
        double *s = (double *)malloc(cap * sizeof(double));
        double *p = (double *)malloc(cap * sizeof(double));
        size_t *kr = (size_t *)malloc(cap * sizeof(size_t));
        if (!s || !p || !kr) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < (int64_t)B * Hq; ++r) {
                int b = (int)(r / Hq);
                int h = (int)(r % Hq);
                int kh = h / group;
                int64_t n = (int64_t)cache_seqlens[b] + 1;
                for (int64_t t = 0; t < n; ++t) {
                    int64_t page = block_table[(size_t)b * (size_t)max_blocks + (size_t)(t / page_size)];
                    kr[t] = (((size_t)page * (size_t)page_size + (size_t)(t % page_size)) *
                             (size_t)Hkv + (size_t)kh) * (size_t)d;
                }
                double l;
                attend_one_row_q(qr, OR_F64, k_pages, v_pages, OR_BF16, (size_t)r * (size_t)d,
                                 kr, kr, (size_t)n, d, scale, 0.0, NULL, s, p,
                                 o + (size_t)r * (size_t)d, &l);
                if (lse)
                    lse[r] = l;
            }
        }
        free(s);
        free(p);
        free(kr);
    }
    free(qr);
    free(tmp);
    free(rot);
    return bad ? -1 : 0;
}

/* Exact value of an OCP e4m3 byte: sign, 4-bit exponent (bias 7), 3-bit
 * mantissa; exponent 0 is subnormal (m/8 * 2^-6); 0x7F/0xFF are NaN. */
double oracle_e4m3_value(uint8_t b)
{
    int sign = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/*
 * FP8 prefill: q [T, Hq, d], k, v [T, Hkv, d] as e4m3 bytes with per-tensor
 * descale factors; the attention of the exact values descale * e4m3 (fp64),
 * with the masks of oracle_prefill.  o [T, Hq, d] double, lse [Hq, T].
 */
int oracle_prefill_fp8(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                       const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                       double scale, double q_descale, double k_descale, double v_descale,
                       double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0)
        return -1;
    size_t T = (size_t)cu_seqlens[B];
    size_t nq = T * (size_t)Hq * (size_t)d, nk = T * (size_t)Hkv * (size_t)d;
    double *qd = (double *)malloc((nq ? nq : 1) * sizeof(double));
    double *kd = (double *)malloc((nk ? nk : 1) * sizeof(double));
    double *vd = (double *)malloc((nk ? nk : 1) * sizeof(double));
    if (!qd || !kd || !vd) {
        free(qd);
        free(kd);
        free(vd);
        return -1;
    }
    for (size_t i = 0; i < nq; ++i)
        qd[i] = q_descale * oracle_e4m3_value(q[i]);
    for (size_t i = 0; i < nk; ++i) {
        kd[i] = k_descale * oracle_e4m3_value(k[i]);
        vd[i] = v_descale * oracle_e4m3_value(v[i]);
    }
    int rc = oracle_prefill(qd, kd, vd, OR_F64, cu_seqlens, B, Hq, Hkv, d, causal, scale, o, lse);
    free(qd);
    free(kd);
    free(vd);
    return rc;
}

/* Threads the OpenMP runtime will use (for reporting). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
