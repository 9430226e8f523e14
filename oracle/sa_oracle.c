/*
 * sa_oracle.c -- plain fp64 CPU oracle for indexed sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the CPU
 * baseline leg of the benchmark load this library; the product path never
 * does.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes, step by step, in the order the pages describe the path:
 *
 *  1. Relevance scoring with head weighting ("Optimizing Next-Gen LLM
 *     Inference", §3.1; "Inference Acceleration for New Large Model
 *     Architectures", §3.1 steps 1-2).  The pages name the two steps but print
 *     no formula; the reading used here is the lightning-indexer score
 *         I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:])
 *     over every visible position s <= pos_t, with q_I and k_I dequantised
 *     exactly (e4m3 code times its fp32 scale) before any arithmetic.
 *  2. Top-K selection (same sections, step 3): the K positions with the
 *     largest score, ties broken towards the lower position, all of them when
 *     fewer than K are visible; emitted in ascending position order and padded
 *     with -1.
 *  3. Sparse attention on the selected rows of the MLA latent cache
 *     ("Optimizing Next-Gen LLM Inference", §3.3; "Inference Acceleration for
 *     New Large Model Architectures", §3.2): per head, softmax over
 *     z_s = sm_scale * q[t,h,:] . kv[s,:] (latent + rope), output
 *     sum_s p_s * kv[s, 0:d_latent] and the log-sum-exp.  An FP8 latent is
 *     dequantised with its page-tile scale ("Optimizing Next-Gen LLM
 *     Inference", §4, block-wise quantised KV cache).
 *
 * Every value is widened to double first; sums run in index order.  Threads
 * split the work over disjoint outputs only, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };
enum { OR_OK = 0, OR_BAD_ARG = -1, OR_BAD_PAGE = -2, OR_BAD_INDEX = -3,
       OR_NAN = -4, OR_NO_MEMORY = -5 };

/* ---------------------------------------------------------------------------
 * Storage formats
 * ------------------------------------------------------------------------- */

/* OCP e4m3fn: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Exponent
 * field 0 holds subnormals (m/8) * 2^-6; S.1111.111 is NaN; no infinities. */
static double e4m3_value(uint8_t code)
{
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double element(int dtype, const void *base, int64_t i)
{
    switch (dtype) {
    case OR_F32: return (double)((const float *)base)[i];
    case OR_BF16: return bf16_value(((const uint16_t *)base)[i]);
    case OR_E4M3: return e4m3_value(((const uint8_t *)base)[i]);
    }
    return NAN;
}

void oracle_decode(int dtype, const void *src, double *dst, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        dst[i] = element(dtype, src, i);
}

/* ---------------------------------------------------------------------------
 * Paged cache addressing: logical position s of sequence b lives in physical
 * row page_table[b][s / page_size] * page_size + s % page_size.
 * ------------------------------------------------------------------------- */

typedef struct {
    const int32_t *page_table;
    int32_t max_pages, page_size, num_pages;
} pages_t;

static int64_t phys_row(const pages_t *pg, int32_t seq, int64_t s)
{
    int64_t slot = s / pg->page_size;
    if (slot >= pg->max_pages)
        return -1;
    int32_t page = pg->page_table[(int64_t)seq * pg->max_pages + slot];
    if (page < 0 || page >= pg->num_pages)
        return -1;
    return (int64_t)page * pg->page_size + s % pg->page_size;
}

/* ---------------------------------------------------------------------------
 * A tiny work pool: items are claimed one at a time under a mutex.
 * ------------------------------------------------------------------------- */

typedef struct pool pool_t;
typedef int (*item_fn)(pool_t *, int64_t item);
struct pool {
    pthread_mutex_t mu;
    int64_t next, count;
    int status;
    item_fn fn;
    const void *ctx;
};

static void *pool_worker(void *arg)
{
    pool_t *p = (pool_t *)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        int64_t it = p->status == OR_OK ? p->next++ : p->count;
        pthread_mutex_unlock(&p->mu);
        if (it >= p->count)
            return NULL;
        int rc = p->fn(p, it);
        if (rc != OR_OK) {
            pthread_mutex_lock(&p->mu);
            if (p->status == OR_OK)
                p->status = rc;
            pthread_mutex_unlock(&p->mu);
        }
    }
}

static int pool_run(item_fn fn, const void *ctx, int64_t count, int nthreads)
{
    pool_t p;
    pthread_mutex_init(&p.mu, NULL);
    p.next = 0;
    p.count = count;
    p.status = OR_OK;
    p.fn = fn;
    p.ctx = ctx;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < nthreads; i++)
        if (pthread_create(&th[started], NULL, pool_worker, &p) == 0)
            started++;
    pool_worker(&p);
    for (int i = 0; i < started; i++)
        pthread_join(th[i], NULL);
    pthread_mutex_destroy(&p.mu);
    return p.status;
}

/* ---------------------------------------------------------------------------
 * 1. Indexer scores
 * ------------------------------------------------------------------------- */

typedef struct {
    int32_t n_q;
    const int32_t *q_seq, *q_pos;
    int32_t h_index, d_index;
    int32_t scale_group;       /* e4m3 scale granularity: 0 = one per row, g = one per g values */
    int32_t q_dtype;           /* OR_F32, OR_BF16 or OR_E4M3 */
    const void *q_index;       /* [n_q, h_index, d_index] */
    const float *q_index_scale;/* [n_q, h_index, d_index / g] (g = d_index when 0) for e4m3 */
    const float *w;            /* [n_q, h_index] */
    int32_t k_dtype;           /* OR_F32, OR_BF16 or OR_E4M3 */
    const void *k_index;       /* [rows, d_index] */
    const float *k_index_scale;/* [rows, d_index / g] for e4m3 */
    pages_t pg;
    double *scores;
    int64_t ld;
    int64_t chunk;             /* positions per work item */
    int64_t chunks_per_query;
} score_ctx;

static int score_item(pool_t *p, int64_t item)
{
    const score_ctx *c = (const score_ctx *)p->ctx;
    int64_t t = item / c->chunks_per_query;
    int64_t s0 = (item % c->chunks_per_query) * c->chunk;
    int64_t V = (int64_t)c->q_pos[t] + 1;
    int64_t s1 = s0 + c->chunk < V ? s0 + c->chunk : V;
    if (s0 >= s1)
        return OR_OK;
    const int H = c->h_index, d = c->d_index;
    const int g = c->scale_group > 0 ? c->scale_group : d;   /* values per scale */
    const int ng = d / g;                                     /* scales per row */
    double *q = malloc(sizeof(double) * (size_t)H * d);
    double *k = malloc(sizeof(double) * (size_t)d);
    if (!q || !k) {
        free(q);
        free(k);
        return OR_NO_MEMORY;
    }
    /* dequantised indexer query q_I[t] */
    for (int j = 0; j < H; j++)
        for (int i = 0; i < d; i++) {
            double qs = c->q_dtype == OR_E4M3
                            ? (double)c->q_index_scale[(t * H + j) * (int64_t)ng + i / g] : 1.0;
            q[j * d + i] = element(c->q_dtype, c->q_index, (t * H + j) * (int64_t)d + i) * qs;
        }
    int rc = OR_OK;
    for (int64_t s = s0; s < s1 && rc == OR_OK; s++) {
        int64_t row = phys_row(&c->pg, c->q_seq[t], s);
        if (row < 0) {
            rc = OR_BAD_PAGE;
            break;
        }
        for (int i = 0; i < d; i++) {
            double ks = c->k_dtype == OR_E4M3 ? (double)c->k_index_scale[row * ng + i / g] : 1.0;
            k[i] = element(c->k_dtype, c->k_index, row * d + i) * ks;
            if (isnan(k[i]))
                rc = OR_NAN;     /* a poisoned (never written) slot was read */
        }
        double I = 0.0;
        for (int j = 0; j < H; j++) {
            double dot = 0.0;
            for (int i = 0; i < d; i++)
                dot += q[j * d + i] * k[i];
            I += (double)c->w[t * H + j] * (dot > 0.0 ? dot : 0.0);
        }
        if (isnan(I))
            rc = OR_NAN;
        c->scores[t * c->ld + s] = I;
    }
    free(q);
    free(k);
    return rc;
}

int oracle_index_scores(int32_t n_q, const int32_t *q_seq, const int32_t *q_pos,
                        int32_t h_index, int32_t d_index, int32_t scale_group,
                        int32_t q_dtype, const void *q_index, const float *q_index_scale,
                        const float *w,
                        int32_t k_dtype, const void *k_index, const float *k_index_scale,
                        const int32_t *page_table, int32_t max_pages, int32_t page_size,
                        int32_t num_pages, double *scores, int64_t ld, int nthreads)
{
    if (n_q < 0 || h_index <= 0 || d_index <= 0 || page_size <= 0 || !scores)
        return OR_BAD_ARG;
    /* one scale per key row and per (query, head) row, or one per group of scale_group
     * values (the pages' group-32 scales, "Inference Acceleration for New Large
     * Model Architectures" §4.1; "Optimizing Next-Gen LLM Inference" §4 table) */
    if (scale_group < 0 || (scale_group > 0 && d_index % scale_group != 0))
        return OR_BAD_ARG;
    /* the indexer's BF16 path ("Optimizing Next-Gen LLM Inference" §3.1: a BF16
     * path next to the quantised one) reads unscaled bf16 values */
    if ((q_dtype != OR_F32 && q_dtype != OR_BF16 && q_dtype != OR_E4M3) ||
        (k_dtype != OR_F32 && k_dtype != OR_BF16 && k_dtype != OR_E4M3))
        return OR_BAD_ARG;
    int64_t maxV = 0;
    for (int32_t t = 0; t < n_q; t++) {
        int64_t V = (int64_t)q_pos[t] + 1;
        if (V < 1 || V > ld)
            return OR_BAD_ARG;
        if (V > maxV)
            maxV = V;
    }
    score_ctx c = { n_q, q_seq, q_pos, h_index, d_index, scale_group, q_dtype, q_index,
                    q_index_scale, w,
                    k_dtype, k_index, k_index_scale,
                    { page_table, max_pages, page_size, num_pages }, scores, ld, 4096, 0 };
    c.chunks_per_query = (maxV + c.chunk - 1) / c.chunk;
    if (c.chunks_per_query == 0)
        return OR_OK;
    return pool_run(score_item, &c, (int64_t)n_q * c.chunks_per_query, nthreads);
}

/* ---------------------------------------------------------------------------
 * 2. Top-K: order by (score descending, position ascending), keep the first
 *    min(K, V), emit ascending positions, pad with -1.
 * ------------------------------------------------------------------------- */

typedef struct {
    double score;
    int64_t pos;
} ranked_t;

static int by_rank(const void *a, const void *b)
{
    const ranked_t *x = (const ranked_t *)a, *y = (const ranked_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos > y->pos) - (x->pos < y->pos);
}

static int by_value(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

int oracle_topk(int32_t n_q, const double *scores, int64_t ld, const int32_t *valid,
                int32_t K, int32_t *idx)
{
    if (n_q < 0 || K <= 0 || !scores || !valid || !idx)
        return OR_BAD_ARG;
    for (int32_t t = 0; t < n_q; t++) {
        int64_t V = valid[t];
        if (V < 0 || V > ld)
            return OR_BAD_ARG;
        ranked_t *r = malloc(sizeof(ranked_t) * (size_t)(V > 0 ? V : 1));
        if (!r)
            return OR_NO_MEMORY;
        for (int64_t s = 0; s < V; s++) {
            r[s].score = scores[t * ld + s];
            r[s].pos = s;
            if (isnan(r[s].score)) {
                free(r);
                return OR_NAN;
            }
        }
        qsort(r, (size_t)V, sizeof(ranked_t), by_rank);
        int64_t n = V < K ? V : K;
        int32_t *out = idx + (int64_t)t * K;
        for (int64_t i = 0; i < n; i++)
            out[i] = (int32_t)r[i].pos;
        qsort(out, (size_t)n, sizeof(int32_t), by_value);
        for (int64_t i = n; i < K; i++)
            out[i] = -1;
        free(r);
    }
    return OR_OK;
}

/* ---------------------------------------------------------------------------
 * 3. Sparse attention over the given rows
 * ------------------------------------------------------------------------- */

typedef struct {
    int32_t n_q;
    const int32_t *q_seq, *q_pos;
    int32_t heads, d_latent, d_rope;
    int32_t q_dtype;           /* OR_F32 or OR_BF16 */
    const void *q;             /* [n_q, heads, d_latent + d_rope] */
    double sm_scale;
    int32_t kv_dtype;          /* OR_F32, OR_BF16 or OR_E4M3 */
    const void *kv;            /* f32/bf16: [rows, d_latent + d_rope]; e4m3: [rows, d_latent] */
    const void *kv_rope;       /* e4m3 cache: bf16 [rows, d_rope] */
    const float *kv_scale;     /* e4m3 cache: [num_pages, page_size / scale_tokens,
                                *   d_latent / scale_dims], one per tile */
    int32_t scale_tokens;      /* tokens of a page per scale tile */
    int32_t scale_dims;        /* latent dims per scale tile */
    pages_t pg;
    const int32_t *idx;
    int32_t K;
    double *out, *lse;
} attn_ctx;

static int attn_item(pool_t *p, int64_t t)
{
    const attn_ctx *c = (const attn_ctx *)p->ctx;
    const int32_t dl = c->d_latent, dr = c->d_rope, D = dl + dr;
    const int32_t *sel = c->idx + t * (int64_t)c->K;
    int64_t V = (int64_t)c->q_pos[t] + 1;
    int32_t n = 0;
    for (int32_t k = 0; k < c->K; k++) {
        if (sel[k] < 0)
            continue;
        if (sel[k] >= V)
            return OR_BAD_INDEX;
        n++;
    }
    if (n == 0) {
        for (int32_t h = 0; h < c->heads; h++) {
            for (int32_t i = 0; i < dl; i++)
                c->out[(t * c->heads + h) * (int64_t)dl + i] = 0.0;
            c->lse[t * c->heads + h] = -INFINITY;
        }
        return OR_OK;
    }
    double *rows = malloc(sizeof(double) * (size_t)n * D);
    double *z = malloc(sizeof(double) * (size_t)n);
    double *qh = malloc(sizeof(double) * (size_t)D);
    if (!rows || !z || !qh) {
        free(rows);
        free(z);
        free(qh);
        return OR_NO_MEMORY;
    }
    int rc = OR_OK;
    int32_t r = 0;
    for (int32_t k = 0; k < c->K && rc == OR_OK; k++) {
        if (sel[k] < 0)
            continue;
        int64_t row = phys_row(&c->pg, c->q_seq[t], sel[k]);
        if (row < 0) {
            rc = OR_BAD_PAGE;
            break;
        }
        double *dst = rows + (int64_t)r * D;
        if (c->kv_dtype == OR_E4M3) {
            /* the scale of (token, dim) is that of its tile within its page */
            const int64_t page = row / c->pg.page_size;
            const int32_t tok = (int32_t)(row % c->pg.page_size);
            const int32_t tiles_t = c->pg.page_size / c->scale_tokens;
            const int32_t tiles_d = dl / c->scale_dims;
            const float *ps = c->kv_scale + (page * tiles_t + tok / c->scale_tokens) * tiles_d;
            for (int32_t i = 0; i < dl; i++)
                dst[i] = e4m3_value(((const uint8_t *)c->kv)[row * dl + i]) *
                         (double)ps[i / c->scale_dims];
            for (int32_t i = 0; i < dr; i++)
                dst[dl + i] = bf16_value(((const uint16_t *)c->kv_rope)[row * dr + i]);
        } else {
            for (int32_t i = 0; i < D; i++)
                dst[i] = element(c->kv_dtype, c->kv, row * D + i);
        }
        for (int32_t i = 0; i < D; i++)
            if (isnan(dst[i]))
                rc = OR_NAN;     /* a poisoned (never written) slot was read */
        r++;
    }
    for (int32_t h = 0; h < c->heads && rc == OR_OK; h++) {
        for (int32_t i = 0; i < D; i++)
            qh[i] = element(c->q_dtype, c->q, (t * c->heads + h) * (int64_t)D + i);
        double m = -INFINITY;
        for (int32_t j = 0; j < n; j++) {
            double dot = 0.0;
            for (int32_t i = 0; i < D; i++)
                dot += qh[i] * rows[(int64_t)j * D + i];
            z[j] = c->sm_scale * dot;
            if (z[j] > m)
                m = z[j];
        }
        double l = 0.0;
        for (int32_t j = 0; j < n; j++)
            l += exp(z[j] - m);
        double *o = c->out + (t * c->heads + h) * (int64_t)dl;
        for (int32_t i = 0; i < dl; i++)
            o[i] = 0.0;
        for (int32_t j = 0; j < n; j++) {
            double pj = exp(z[j] - m) / l;
            for (int32_t i = 0; i < dl; i++)
                o[i] += pj * rows[(int64_t)j * D + i];
        }
        c->lse[t * c->heads + h] = m + log(l);
        if (isnan(c->lse[t * c->heads + h]))
            rc = OR_NAN;
    }
    free(rows);
    free(z);
    free(qh);
    return rc;
}

int oracle_sparse_attn(int32_t n_q, const int32_t *q_seq, const int32_t *q_pos,
                       int32_t heads, int32_t d_latent, int32_t d_rope,
                       int32_t q_dtype, const void *q, double sm_scale,
                       int32_t kv_dtype, const void *kv, const void *kv_rope,
                       const float *kv_scale, int32_t scale_tokens, int32_t scale_dims,
                       const int32_t *page_table, int32_t max_pages, int32_t page_size,
                       int32_t num_pages, const int32_t *idx, int32_t K,
                       double *out, double *lse, int nthreads)
{
    if (n_q < 0 || heads <= 0 || d_latent <= 0 || d_rope < 0 || K <= 0 || !out || !lse)
        return OR_BAD_ARG;
    if (q_dtype != OR_F32 && q_dtype != OR_BF16)
        return OR_BAD_ARG;
    if (kv_dtype == OR_E4M3 && (!kv_rope || !kv_scale))
        return OR_BAD_ARG;
    if (kv_dtype == OR_E4M3 &&
        (scale_tokens <= 0 || page_size % scale_tokens != 0 || scale_dims <= 0 ||
         d_latent % scale_dims != 0))
        return OR_BAD_ARG;
    attn_ctx c = { n_q, q_seq, q_pos, heads, d_latent, d_rope, q_dtype, q, sm_scale,
                   kv_dtype, kv, kv_rope, kv_scale, scale_tokens, scale_dims,
                   { page_table, max_pages, page_size, num_pages }, idx, K, out, lse };
    return pool_run(attn_item, &c, n_q, nthreads);
}

/* ---------------------------------------------------------------------------
 * Input preparation ("Optimizing Next-Gen LLM Inference", §3.2 and the §4
 * table; "Inference Acceleration for New Large Model Architectures", §3.3 and
 * §4.1-4.2): dynamic FP8 quantisation of the indexer query and of new index
 * keys, and block-quantised rows appended to the latent cache.
 *
 * The pages fix the format (8-bit float, one scale per group) but not the
 * arithmetic.  The reading used here: per group of values, in fp32,
 *     amax  = max |x|,   scale = amax / 448   (1 when amax is 0),
 *     code  = e4m3(x / scale), rounded to nearest, ties to even, saturated
 *             to +-448,
 * so that the largest magnitude lands on e4m3's largest finite value.  The
 * scale and the quotient are fp32 operations (what the kernel does), because
 * they decide an integer code; the rounding to e4m3 is then taken exactly,
 * in double, from that fp32 value.
 * ------------------------------------------------------------------------- */

/* Exact fp32 value -> OCP e4m3fn code.  e4m3 values are integers times
 * 2^(e-3) for the binade [2^e, 2^(e+1)), e >= -6; below 2^-6 the spacing
 * stays 2^-9 (subnormals).  The value must not be NaN. */
static uint8_t e4m3_code(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0)
        return sign | 0x7E;                  /* saturate: S.1111.110 = 448 */
    if (a == 0.0)
        return sign;
    int e2;
    frexp(a, &e2);                           /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                          /* a in [2^e, 2^(e+1)) */
    if (e < -6)
        e = -6;
    double step = ldexp(1.0, e - 3);
    double q = nearbyint(a / step) * step;   /* a / step is exact; ties to even */
    if (q < ldexp(1.0, -6))                  /* subnormal: m * 2^-9, m in 0..7 */
        return sign | (uint8_t)(q / ldexp(1.0, -9));
    frexp(q, &e2);
    e = e2 - 1;                              /* rounding may have moved q up a binade */
    int m = (int)((q / ldexp(1.0, e) - 1.0) * 8.0);
    return sign | (uint8_t)((e + 7) << 3) | (uint8_t)m;
}

/* Exact fp32 value -> bf16 bits, round to nearest, ties to even (finite
 * values; bf16 keeps fp32's exponent and the top 7 fraction bits). */
static uint16_t bf16_code(float xf)
{
    double x = (double)xf;
    double a = fabs(x);
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    if (a == 0.0)
        return sign;
    int e2;
    frexp(a, &e2);
    int e = e2 - 1;
    if (e < -126)
        e = -126;                            /* bf16 subnormals share fp32's range */
    double step = ldexp(1.0, e - 7);
    double q = nearbyint(a / step) * step;
    if (q >= ldexp(1.0, 128))
        return sign | 0x7F80;                /* overflow rounds to infinity */
    if (q < ldexp(1.0, -126))
        return sign | (uint16_t)(q / ldexp(1.0, -133));
    frexp(q, &e2);
    e = e2 - 1;
    int m = (int)((q / ldexp(1.0, e) - 1.0) * 128.0);
    return sign | (uint16_t)((e + 127) << 7) | (uint16_t)m;
}

/* n_groups groups of `group` consecutive fp32 values -> e4m3 codes and one
 * fp32 scale per group (rule above). */
int oracle_quantize_e4m3(int64_t n_groups, int32_t group, const float *x, uint8_t *codes,
                         float *scales)
{
    if (n_groups < 0 || group <= 0 || (n_groups > 0 && (!x || !codes || !scales)))
        return OR_BAD_ARG;
    for (int64_t g = 0; g < n_groups; g++) {
        const float *v = x + g * group;
        float amax = 0.0f;
        for (int32_t i = 0; i < group; i++) {
            if (isnan(v[i]))
                return OR_NAN;
            if (fabsf(v[i]) > amax)
                amax = fabsf(v[i]);
        }
        float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
        scales[g] = scale;
        for (int32_t i = 0; i < group; i++) {
            float r = v[i] / scale;
            codes[g * group + i] = e4m3_code(r);
        }
    }
    return OR_OK;
}

/* n fp32 values -> bf16 bits. */
int oracle_to_bf16(int64_t n, const float *x, uint16_t *bits)
{
    if (n < 0 || (n > 0 && (!x || !bits)))
        return OR_BAD_ARG;
    for (int64_t i = 0; i < n; i++) {
        if (isnan(x[i]))
            return OR_NAN;
        bits[i] = bf16_code(x[i]);
    }
    return OR_OK;
}

/* n fp32 values -> e4m3 codes directly (no scale), for pinning the encoder. */
int oracle_e4m3_encode(int64_t n, const float *x, uint8_t *codes)
{
    if (n < 0 || (n > 0 && (!x || !codes)))
        return OR_BAD_ARG;
    for (int64_t i = 0; i < n; i++) {
        if (isnan(x[i]))
            return OR_NAN;
        codes[i] = e4m3_code(x[i]);
    }
    return OR_OK;
}

/* E8M0 scale bytes (the shared scale of the OCP MX formats, which "Long-Context
 * LLM Inference Optimization" names for the index query and keys: MXFP8, one
 * scale per group of 32 values) -> their values as fp32: byte b stands for
 * 2^(b - 127), exactly representable for every b in [0, 254]; 255 is NaN. */
int oracle_e8m0_decode(int64_t n, const uint8_t *bytes, float *out)
{
    if (n < 0 || (n > 0 && (!bytes || !out)))
        return OR_BAD_ARG;
    for (int64_t i = 0; i < n; i++)
        out[i] = bytes[i] == 255 ? (float)NAN : (float)ldexp(1.0, (int)bytes[i] - 127);
    return OR_OK;
}
