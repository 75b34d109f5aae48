/*
 * QSA MQA indexer score: CPU oracle in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header or table with the CUDA path.
 *
 * What it computes, written out plainly (no tiling, no reordering):
 *
 *   score(t, n) = scale * sum_{h<4} max(0, sum_{c<128} q[t,h,c] * k[n,c])
 *
 * (QSA docs, MATE, section "MQA score": four query heads share one
 * compressed key of dimension 128, the score sums the four head-wise ReLU
 * dot products and scales by 1/sqrt(128), passed here as a multiplier.)
 * bf16 inputs widen exactly to double and every sum runs in double, in index
 * order.
 *
 * Masking (vLLM qsa_cache.py, "_logical_positions" and the metadata kernel's
 * "visible_blocks"): a query token at logical position
 *     pos = seq_len - query_len + i
 * sees compressed keys n < visible = max(0, min((pos + 1) // 4, seq_len // 4));
 * every other column is -inf.  Decode reads key n of request b from page
 * page_table[b, n // page_size], row n % page_size (vLLM qsa_cache.py,
 * "_logical_to_physical_qsa_slots"); an entry that is -1 or not a valid page
 * gives -inf (QSA docs, "MQA score": missing or out-of-range pages are
 * masked to -inf).  Prefill row t sees keys in its interval [ks[t], ke[t])
 * clipped to [0, Nk); column j of the row holds key ks[t] + j.
 *
 * Parity status: every function here is pinned by the CPU tests (closed
 * forms, invariants, exact integer brute force, the cache writer's rule and
 * the FLOP counts printed in the vLLM PR's prefill table).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define QSA_HEADS 4
#define QSA_DIM 128
#define QSA_RATIO 4

/* ---------------------------------------------------------------- helpers */

static double bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Value of an IEEE binary16 (fp16) bit pattern: 1 sign bit, 5 exponent bits
 * with bias 15, 10 mantissa bits; exponent 0 holds zero and the subnormals
 * m * 2^-24, exponent 31 holds the infinities and NaNs. */
static double f16_to_double(uint16_t bits) {
    int sign = bits >> 15, ex = (bits >> 10) & 31, man = bits & 1023;
    double mag;
    if (ex == 31) mag = man ? NAN : INFINITY;
    else if (ex == 0) mag = ldexp((double)man, -24);
    else mag = ldexp(1.0 + man / 1024.0, ex - 15);
    return sign ? -mag : mag;
}

double qsa_oracle_f16_to_double(uint16_t bits) { return f16_to_double(bits); }

/* A 16-bit input element: bf16 or (f16 != 0) fp16. */
static double elem_to_double(uint16_t bits, int f16) {
    return f16 ? f16_to_double(bits) : bf16_to_double(bits);
}

static int64_t floor_div(int64_t a, int64_t b) {
    int64_t q = a / b;
    if ((a % b != 0) && ((a < 0) != (b < 0))) q -= 1;
    return q;
}

/* A simple static split of [0, n) over threads. */
typedef void (*range_fn)(void *ctx, int64_t begin, int64_t end);
typedef struct { range_fn fn; void *ctx; int64_t begin, end; } range_job;

static void *range_thread(void *arg) {
    range_job *j = (range_job *)arg;
    j->fn(j->ctx, j->begin, j->end);
    return NULL;
}

int qsa_oracle_default_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void *ctx) {
    if (nthreads <= 0) nthreads = qsa_oracle_default_threads();
    if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
    if (nthreads <= 1) { fn(ctx, 0, n); return; }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    range_job *jobs = (range_job *)malloc(sizeof(range_job) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) {
        jobs[i].fn = fn; jobs[i].ctx = ctx;
        jobs[i].begin = n * i / nthreads;
        jobs[i].end = n * (i + 1) / nthreads;
        pthread_create(&th[i], NULL, range_thread, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    free(jobs);
}

/* ------------------------------------------------------------- the mask */

int64_t qsa_oracle_logical_position(int64_t seq_len, int64_t query_len, int64_t i) {
    return seq_len - query_len + i;
}

int64_t qsa_oracle_visible_blocks(int64_t pos, int64_t seq_len) {
    int64_t by_pos = floor_div(pos + 1, QSA_RATIO);
    int64_t by_len = floor_div(seq_len, QSA_RATIO);
    int64_t v = by_pos < by_len ? by_pos : by_len;
    return v > 0 ? v : 0;
}

/* visible[b * Q + i] for every decode row. */
void qsa_oracle_decode_visible(const int32_t *seq_lens, int64_t B, int64_t Q, int32_t *visible) {
    for (int64_t b = 0; b < B; ++b)
        for (int64_t i = 0; i < Q; ++i) {
            int64_t pos = qsa_oracle_logical_position(seq_lens[b], Q, i);
            visible[b * Q + i] = (int32_t)qsa_oracle_visible_blocks(pos, seq_lens[b]);
        }
}

/* Per-row key intervals of a packed prefill batch: sequence s has query rows
 * cu_seqlens_q[s] .. cu_seqlens_q[s+1], seq_lens[s] tokens in all, and its
 * keys start at key_offsets[s]. */
void qsa_oracle_prefill_intervals(const int32_t *cu_seqlens_q, const int32_t *seq_lens,
                                  const int32_t *key_offsets, int64_t S,
                                  int32_t *ks, int32_t *ke) {
    for (int64_t s = 0; s < S; ++s) {
        int64_t qlen = (int64_t)cu_seqlens_q[s + 1] - cu_seqlens_q[s];
        for (int64_t i = 0; i < qlen; ++i) {
            int64_t t = cu_seqlens_q[s] + i;
            int64_t pos = qsa_oracle_logical_position(seq_lens[s], qlen, i);
            ks[t] = key_offsets[s];
            ke[t] = (int32_t)(key_offsets[s] + qsa_oracle_visible_blocks(pos, seq_lens[s]));
        }
    }
}

/* ------------------------------------------------------------- the score */

/* Value of an fp8 E4M3 code (the e4m3 format with no infinities: 1 sign
 * bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 holds the
 * subnormals m * 2^-9; the codes with all exponent and mantissa bits set are
 * NaN; the largest finite magnitude is 1.75 * 2^8 = 448). */
double qsa_oracle_e4m3_to_double(uint8_t code) {
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* A key row as exact doubles: bf16 elements, or fp8 E4M3 elements times the
 * cache's dequantisation scale k_scale (the cache stores e4m3(bf16(k) /
 * k_scale): vLLM qsa_prepare.py, "_to_dst_dtype", rounds to bf16 first, then
 * scales for an fp8 destination). */
static void key_row_16(const uint16_t *k_row, int f16, double *k) {
    for (int e = 0; e < QSA_DIM; ++e) k[e] = elem_to_double(k_row[e], f16);
}

static void key_row_e4m3(const uint8_t *k_row, double k_scale, double *k) {
    for (int e = 0; e < QSA_DIM; ++e) k[e] = qsa_oracle_e4m3_to_double(k_row[e]) * k_scale;
}

/* scale * sum_h max(0, q_h . k) for one query row (4 heads) and one key. */
static double head_sum_score(const uint16_t *q_row, int64_t q_stride_h, int f16,
                             const double *k, double scale) {
    double s = 0.0;
    for (int h = 0; h < QSA_HEADS; ++h) {
        const uint16_t *qh = q_row + h * q_stride_h;
        double d = 0.0;
        for (int c = 0; c < QSA_DIM; ++c) d += elem_to_double(qh[c], f16) * k[c];
        s += d > 0.0 ? d : 0.0;
    }
    return scale * s;
}

typedef struct {
    const uint16_t *q; int64_t q_sb, q_st, q_sh;
    const uint16_t *k_cache; int64_t num_pages, page_size, k_page_stride, k_row_stride;
    const int32_t *page_table; int64_t pt_stride, max_pages;
    const int32_t *seq_lens; int64_t B, Q;
    double scale;
    const uint8_t *k8; double k_scale;   /* fp8 cache when k8 != NULL (then k_cache is unused) */
    int f16;                             /* q (and a 16-bit cache) hold fp16 instead of bf16 */
} decode_args;

/* Score of decode row (b, i) against compressed key n, or -inf when masked. */
static double decode_entry(const decode_args *a, int64_t b, int64_t i, int64_t n) {
    int64_t pos = qsa_oracle_logical_position(a->seq_lens[b], a->Q, i);
    int64_t visible = qsa_oracle_visible_blocks(pos, a->seq_lens[b]);
    if (n < 0 || n >= visible) return -INFINITY;
    int64_t logical_page = n / a->page_size;
    if (logical_page >= a->max_pages) return -INFINITY;
    int64_t page = a->page_table[b * a->pt_stride + logical_page];
    if (page < 0 || page >= a->num_pages) return -INFINITY;
    const uint16_t *q_row = a->q + b * a->q_sb + i * a->q_st;
    int64_t row_off = page * a->k_page_stride + (n % a->page_size) * a->k_row_stride;
    double k[QSA_DIM];
    if (a->k8) key_row_e4m3(a->k8 + row_off, a->k_scale, k);
    else key_row_16(a->k_cache + row_off, a->f16, k);
    return head_sum_score(q_row, a->q_sh, a->f16, k, a->scale);
}

typedef struct { decode_args a; double *out; int64_t W; } decode_full_ctx;

static void decode_rows(void *vctx, int64_t begin, int64_t end) {
    decode_full_ctx *c = (decode_full_ctx *)vctx;
    for (int64_t r = begin; r < end; ++r) {
        int64_t b = r / c->a.Q, i = r % c->a.Q;
        for (int64_t n = 0; n < c->W; ++n) c->out[r * c->W + n] = decode_entry(&c->a, b, i, n);
    }
}

/* out[(b * Q + i) * W + n] for every row and every n < W; q and k_cache
 * hold bf16, or fp16 when f16 != 0. */
void qsa_oracle_decode(const uint16_t *q, int64_t q_sb, int64_t q_st, int64_t q_sh,
                       const uint16_t *k_cache, int64_t num_pages, int64_t page_size,
                       int64_t k_page_stride, int64_t k_row_stride,
                       const int32_t *page_table, int64_t pt_stride, int64_t max_pages,
                       const int32_t *seq_lens, int64_t B, int64_t Q, double scale,
                       double *out, int64_t W, int nthreads, int f16) {
    decode_full_ctx c = {{q, q_sb, q_st, q_sh, k_cache, num_pages, page_size, k_page_stride,
                          k_row_stride, page_table, pt_stride, max_pages, seq_lens, B, Q, scale,
                          NULL, 0.0, f16},
                         out, W};
    parallel_for(B * Q, nthreads, decode_rows, &c);
}

/* qsa_oracle_decode over an fp8 E4M3 key cache (strides in bytes = elements)
 * with dequantisation scale k_scale. */
void qsa_oracle_decode_fp8(const uint16_t *q, int64_t q_sb, int64_t q_st, int64_t q_sh,
                           const uint8_t *k8, double k_scale, int64_t num_pages, int64_t page_size,
                           int64_t k_page_stride, int64_t k_row_stride,
                           const int32_t *page_table, int64_t pt_stride, int64_t max_pages,
                           const int32_t *seq_lens, int64_t B, int64_t Q, double scale,
                           double *out, int64_t W, int nthreads) {
    decode_full_ctx c = {{q, q_sb, q_st, q_sh, NULL, num_pages, page_size, k_page_stride,
                          k_row_stride, page_table, pt_stride, max_pages, seq_lens, B, Q, scale,
                          k8, k_scale, 0},
                         out, W};
    parallel_for(B * Q, nthreads, decode_rows, &c);
}

typedef struct {
    const uint16_t *q; int64_t q_st, q_sh;
    const uint16_t *k; int64_t k_stride, Nk;
    const int32_t *ks, *ke;
    double scale;
    int f16;   /* q and k hold fp16 instead of bf16 */
} prefill_args;

/* Score of prefill row t at column j (key ks[t] + j), or -inf when masked. */
static double prefill_entry(const prefill_args *a, int64_t t, int64_t j) {
    int64_t lo = a->ks[t] > 0 ? a->ks[t] : 0;
    int64_t hi = a->ke[t] < a->Nk ? a->ke[t] : a->Nk;
    int64_t n = (int64_t)a->ks[t] + j;
    if (j < 0 || n < lo || n >= hi) return -INFINITY;
    double k[QSA_DIM];
    key_row_16(a->k + n * a->k_stride, a->f16, k);
    return head_sum_score(a->q + t * a->q_st, a->q_sh, a->f16, k, a->scale);
}

typedef struct { prefill_args a; double *out; int64_t W; } prefill_full_ctx;

static void prefill_rows(void *vctx, int64_t begin, int64_t end) {
    prefill_full_ctx *c = (prefill_full_ctx *)vctx;
    for (int64_t t = begin; t < end; ++t)
        for (int64_t j = 0; j < c->W; ++j) c->out[t * c->W + j] = prefill_entry(&c->a, t, j);
}

/* out[t * W + j] for every row t < T and column j < W; q and k hold bf16,
 * or fp16 when f16 != 0. */
void qsa_oracle_prefill(const uint16_t *q, int64_t q_st, int64_t q_sh,
                        const uint16_t *k, int64_t k_stride, int64_t Nk,
                        const int32_t *ks, const int32_t *ke, int64_t T, double scale,
                        double *out, int64_t W, int nthreads, int f16) {
    prefill_full_ctx c = {{q, q_st, q_sh, k, k_stride, Nk, ks, ke, scale, f16}, out, W};
    parallel_for(T, nthreads, prefill_rows, &c);
}

typedef struct { prefill_args a; const int64_t *tt, *jj; double *out; } prefill_entries_ctx;

static void prefill_entries_range(void *vctx, int64_t begin, int64_t end) {
    prefill_entries_ctx *c = (prefill_entries_ctx *)vctx;
    for (int64_t e = begin; e < end; ++e) c->out[e] = prefill_entry(&c->a, c->tt[e], c->jj[e]);
}

/* out[e] = score of prefill row tt[e] at column jj[e]. */
void qsa_oracle_prefill_entries(const uint16_t *q, int64_t q_st, int64_t q_sh,
                                const uint16_t *k, int64_t k_stride, int64_t Nk,
                                const int32_t *ks, const int32_t *ke, double scale,
                                const int64_t *tt, const int64_t *jj, int64_t count,
                                double *out, int nthreads, int f16) {
    prefill_entries_ctx c = {{q, q_st, q_sh, k, k_stride, Nk, ks, ke, scale, f16}, tt, jj, out};
    parallel_for(count, nthreads, prefill_entries_range, &c);
}

/* ------------------------------------------------------------- top-k */

/* Per-row top-k (the caller's selection step in the QSA docs' pipeline;
 * widths 512 / 1024 / 2048 in the vLLM PR's top-k discussion).  The
 * candidates of row r are its first lengths[r] columns whose score is not
 * masked: a -inf (or NaN) score marks a block the row cannot see, and the
 * selection runs over visible blocks only.  Take the min(k, #candidates)
 * largest scores, ties going to the lower column; write their column
 * indices in ascending order and pad the rest of the k slots with -1.
 * -0.0 and +0.0 compare equal.  The ordering is done by the C library's
 * qsort. */

typedef struct { double v; int64_t j; } scored_col;

static int by_score_desc_then_col(const void *pa, const void *pb) {
    const scored_col *a = (const scored_col *)pa, *b = (const scored_col *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_col(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

typedef struct {
    const double *scores; int64_t stride;
    const int32_t *lengths; int64_t k;
    int32_t *idx; int64_t idx_stride;
} topk_ctx;

static void topk_rows(void *vctx, int64_t begin, int64_t end) {
    topk_ctx *c = (topk_ctx *)vctx;
    for (int64_t r = begin; r < end; ++r) {
        int64_t len = c->lengths[r] > 0 ? c->lengths[r] : 0;
        int32_t *dst = c->idx + r * c->idx_stride;
        int64_t ncand = 0, take = 0;
        if (len > 0) {
            scored_col *cols = (scored_col *)malloc(sizeof(scored_col) * (size_t)len);
            for (int64_t j = 0; j < len; ++j) {
                double v = c->scores[r * c->stride + j];
                if (!(v > -INFINITY)) continue;  /* masked block (or NaN) */
                cols[ncand].v = v;
                cols[ncand].j = j;
                ++ncand;
            }
            take = ncand < c->k ? ncand : c->k;
            qsort(cols, (size_t)ncand, sizeof(scored_col), by_score_desc_then_col);
            for (int64_t s = 0; s < take; ++s) dst[s] = (int32_t)cols[s].j;
            free(cols);
            qsort(dst, (size_t)take, sizeof(int32_t), by_col);
        }
        for (int64_t s = take; s < c->k; ++s) dst[s] = -1;
    }
}

void qsa_oracle_topk(const double *scores, int64_t stride, const int32_t *lengths, int64_t rows,
                     int64_t k, int32_t *idx, int64_t idx_stride, int nthreads) {
    topk_ctx c = {scores, stride, lengths, k, idx, idx_stride};
    parallel_for(rows, nthreads, topk_rows, &c);
}

/* ====================================================== core attention
 *
 * The stage after the indexer (QSA docs, MATE, section "Core Attention"):
 * the caller keeps the top-scoring compressed blocks, expands them to token
 * indices, and sparse attention runs over those tokens.
 */

/* Block -> token index expansion.  Row t (logical position pos[t]) keeps the
 * blocks blk[t, 0..k); block b stands for tokens 4b .. 4b + 3.  The docs tie
 * the widths as tokens = 4 * blocks + 3: the 3 extra slots hold the tokens of
 * the row's open group, the tokens after its last complete group, which no
 * compressed key covers yet: positions 4 * visible .. pos with visible =
 * visible_blocks(pos, seq_len) (at most 3 of them).  Output row t lists, in
 * order, the four tokens of each non-negative block index (in the order the
 * blocks are given), then the open-group tokens ascending, then -1 up to the
 * width 4k + 3.  A row whose position is negative keeps no open group. */
void qsa_oracle_expand_indices(const int32_t *blk, int64_t blk_stride, const int32_t *pos,
                               const int32_t *seq_len_of_row, int64_t rows, int64_t k,
                               int32_t *tok, int64_t tok_stride) {
    int64_t width = 4 * k + 3;
    for (int64_t t = 0; t < rows; ++t) {
        int32_t *dst = tok + t * tok_stride;
        int64_t n = 0;
        for (int64_t i = 0; i < k; ++i) {
            int64_t b = blk[t * blk_stride + i];
            if (b < 0) continue;
            for (int64_t r = 0; r < 4; ++r) dst[n++] = (int32_t)(4 * b + r);
        }
        int64_t p = pos[t];
        if (p >= 0) {
            int64_t vis = qsa_oracle_visible_blocks(p, seq_len_of_row[t]);
            for (int64_t j = 4 * vis; j <= p && n < width; ++j) dst[n++] = (int32_t)j;
        }
        while (n < width) dst[n++] = -1;
    }
}

typedef struct {
    const uint16_t *q; int64_t q_st, q_sh, Hq;
    const uint16_t *k_cache, *v_cache;
    int64_t num_pages, page_size, kv_page_stride, kv_row_stride, kv_head_stride, Hkv;
    const int32_t *page_table; int64_t pt_stride, max_pages;
    const int32_t *row_req, *row_pos, *seq_lens;
    const int32_t *tok; int64_t tok_stride, width;
    const double *gate;   /* [T, Hq] or NULL */
    double scale;
    double *out;          /* [T, Hq, 256] */
    double *lse;          /* [T, Hq] */
} sparse_attn_ctx;

#define QSA_ATTN_DIM 256

/* Row of token j of request r in the paged K/V pool for KV head g, or NULL
 * when the token is outside the request or its page is missing. */
static const uint16_t *kv_row(const sparse_attn_ctx *c, const uint16_t *cache, int64_t r, int64_t j, int64_t g) {
    int64_t logical = j / c->page_size;
    if (logical >= c->max_pages) return NULL;
    int64_t page = c->page_table[r * c->pt_stride + logical];
    if (page < 0 || page >= c->num_pages) return NULL;
    return cache + page * c->kv_page_stride + (j % c->page_size) * c->kv_row_stride + g * c->kv_head_stride;
}

/* Softmax attention of query row t, head h, over the listed tokens that the
 * row may see: index j >= 0, j <= pos (no future token), j < seq_len of the
 * row's request, page present.  Each listed token counts once per listing.
 * Scores s_i = scale * q . k_i; out = sum_i softmax(s)_i * v_i, times
 * sigmoid(gate) when a gate is given; lse = log(sum_i exp(s_i)) (natural
 * log).  A row with no such token gives zero output and lse = -inf.  Query
 * heads share KV head h / (Hq / Hkv). */
static void sparse_attn_rows(void *vctx, int64_t begin, int64_t end) {
    sparse_attn_ctx *c = (sparse_attn_ctx *)vctx;
    int64_t group = c->Hq / c->Hkv;
    double *s = (double *)malloc(sizeof(double) * (size_t)(c->width > 0 ? c->width : 1));
    const uint16_t **vrow = (const uint16_t **)malloc(sizeof(uint16_t *) * (size_t)(c->width > 0 ? c->width : 1));
    for (int64_t th = begin; th < end; ++th) {
        int64_t t = th / c->Hq, h = th % c->Hq, g = h / group;
        int64_t r = c->row_req[t], pos = c->row_pos[t];
        double *o = c->out + th * QSA_ATTN_DIM;
        for (int d = 0; d < QSA_ATTN_DIM; ++d) o[d] = 0.0;
        int64_t n = 0;
        if (r >= 0) {
            const uint16_t *qh = c->q + t * c->q_st + h * c->q_sh;
            for (int64_t i = 0; i < c->width; ++i) {
                int64_t j = c->tok[t * c->tok_stride + i];
                if (j < 0 || j > pos || j >= c->seq_lens[r]) continue;
                const uint16_t *kr = kv_row(c, c->k_cache, r, j, g);
                const uint16_t *vr = kv_row(c, c->v_cache, r, j, g);
                if (!kr || !vr) continue;
                double dot = 0.0;
                for (int d = 0; d < QSA_ATTN_DIM; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(kr[d]);
                s[n] = c->scale * dot;
                vrow[n] = vr;
                ++n;
            }
        }
        if (n == 0) {
            c->lse[th] = -INFINITY;
            continue;
        }
        double m = s[0];
        for (int64_t i = 1; i < n; ++i) m = s[i] > m ? s[i] : m;
        double denom = 0.0;
        for (int64_t i = 0; i < n; ++i) denom += exp(s[i] - m);
        double lse = m + log(denom);
        for (int64_t i = 0; i < n; ++i) {
            double p = exp(s[i] - lse);
            for (int d = 0; d < QSA_ATTN_DIM; ++d) o[d] += p * bf16_to_double(vrow[i][d]);
        }
        if (c->gate) {
            double gt = 1.0 / (1.0 + exp(-c->gate[th]));
            for (int d = 0; d < QSA_ATTN_DIM; ++d) o[d] *= gt;
        }
        c->lse[th] = lse;
    }
    free(s);
    free(vrow);
}

/* Sparse core attention over paged K/V: q bf16 [T, Hq, 256] (row stride
 * q_st, head stride q_sh), K and V bf16 [pages, page_size, Hkv, 256] with the
 * given page, row and head strides, row t belonging to request row_req[t]
 * (negative: a padding row) at logical position row_pos[t], token list
 * tok[t, 0..width).  out [T, Hq, 256] and lse [T, Hq] in fp64. */
void qsa_oracle_sparse_attention(const uint16_t *q, int64_t q_st, int64_t q_sh, int64_t Hq,
                                 const uint16_t *k_cache, const uint16_t *v_cache, int64_t num_pages,
                                 int64_t page_size, int64_t kv_page_stride, int64_t kv_row_stride,
                                 int64_t kv_head_stride, int64_t Hkv,
                                 const int32_t *page_table, int64_t pt_stride, int64_t max_pages,
                                 const int32_t *row_req, const int32_t *row_pos, const int32_t *seq_lens,
                                 const int32_t *tok, int64_t tok_stride, int64_t width, int64_t T,
                                 const double *gate, double scale, double *out, double *lse, int nthreads) {
    sparse_attn_ctx c = {q, q_st, q_sh, Hq, k_cache, v_cache, num_pages, page_size, kv_page_stride,
                         kv_row_stride, kv_head_stride, Hkv, page_table, pt_stride, max_pages,
                         row_req, row_pos, seq_lens, tok, tok_stride, width, gate, scale, out, lse};
    parallel_for(T * Hq, nthreads, sparse_attn_rows, &c);
}
