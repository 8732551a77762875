/*
 * fp64 CPU oracle for the speculative-decoding attention / acceptance path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this file;
 * only the tests, the smoke check and the benchmark's CPU-baseline leg use it.  It shares no
 * code, header, table or helper with the CUDA library: the only thing both sides share is the
 * bytes of the seeded inputs.
 *
 * Every routine is the plain definition written out in double precision: no tiling, no
 * splitting, no online softmax.  bf16 inputs are widened exactly (bits << 16) and fp32 inputs
 * are widened exactly to double.  OpenMP only spreads independent output rows over threads;
 * the arithmetic of each row is sequential and identical for any thread count.
 *
 * Sources (the pages print no formulas or code; each routine states the reading it takes):
 *  [StD]  "Sparse-to-Dense: A Free Lunch for Lossless Acceleration of Video Understanding in
 *         LLMs" (gist.science, pt), technical summary: "Procedimento de Decodificacao" (dense
 *         parallel verification in one pass over the full KV, longest matching prefix plus one
 *         bonus token), "Selecao de Cache KV" (top-K KV per layer and head), "Principais
 *         Contribuicoes" (lossless: output distribution unchanged).
 *  [SPW]  "Sparrow: Text-Anchored Window Attention with Visual-Semantic Glimpsing for
 *         Speculative Decoding in Video LLMs" (gist.science zh, section 3.1 HSR-VATA; pt,
 *         section 3.A): the draft drops the visual KV and attends only to text-anchored
 *         positions; an FC maps [text embedding ; reused target hidden state] to the draft input.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "sd_oracle.h"

/* ---------------------------------------------------------------- element access ---------- */

static double orc_widen(const void *base, int dtype, int64_t off)
{
    if (dtype == ORC_F32)
        return (double)((const float *)base)[off];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[off]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Element offset of row (sequence b, KV head h, position j) of the cache.  Returns -1 when a
 * paged cache has no valid page for j. */
static int64_t orc_kv_row(const orc_cache *c, int b, int h, int64_t j)
{
    if (c->page_size == 0)
        return (int64_t)b * c->stride_b + (int64_t)h * c->stride_h + j * c->stride_pos;
    int32_t page = c->block_table[(int64_t)b * c->max_pages + j / c->page_size];
    if (page < 0 || page >= c->num_pages)
        return -1;
    return (((int64_t)page * c->h_kv + h) * c->page_size + (j % c->page_size)) * c->head_dim;
}

static double orc_scale(const orc_query *q, int head_dim)
{
    return q->softmax_scale > 0.0 ? q->softmax_scale : 1.0 / sqrt((double)head_dim);
}

/* ---------------------------------------------------------------- attention over a set --- */

/* O = sum_{j in P} exp(s_j - max s) v_j / sum_{j in P} exp(s_j - max s),
 * s_j = scale * (q . k_j).  P is given as an explicit list of positions.  An empty P gives
 * O = 0.  Two plain passes: all scores first, then the weighted sum. */
static int orc_attend_set(const orc_cache *c, int b, int g, const double *q, double scale,
                          const int64_t *pos, int64_t n, double *scratch, double *out)
{
    const int d = c->head_dim;
    for (int i = 0; i < d; ++i)
        out[i] = 0.0;
    if (n == 0)
        return ORC_OK;
    double mx = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        int64_t kr = orc_kv_row(c, b, g, pos[t]);
        if (kr < 0)
            return ORC_ERR_ARG;
        double s = 0.0;
        for (int i = 0; i < d; ++i)
            s += q[i] * orc_widen(c->k, c->dtype, kr + i);
        s *= scale;
        scratch[t] = s;
        if (s > mx)
            mx = s;
    }
    double den = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        double w = exp(scratch[t] - mx);
        int64_t vr = orc_kv_row(c, b, g, pos[t]);
        den += w;
        for (int i = 0; i < d; ++i)
            out[i] += w * orc_widen(c->v, c->dtype, vr + i);
    }
    for (int i = 0; i < d; ++i)
        out[i] /= den;
    return ORC_OK;
}

/* Shared driver: for every (sequence, query row, query head) build the allowed position set
 * with `build` and attend over it.  Query head h reads KV head h / (h_q / h_kv). */
typedef int64_t (*orc_set_builder)(const void *ctx, int b, int64_t kv_len, int n_q, int i,
                                   int g, int64_t *pos);

static int orc_attention_driver(const orc_query *q, const void *qdata, const orc_cache *c,
                                int batch, orc_set_builder build, const void *ctx, double *out)
{
    if (q->h_q <= 0 || c->h_kv <= 0 || q->h_q % c->h_kv != 0 || c->head_dim <= 0)
        return ORC_ERR_ARG;
    const int d = c->head_dim, hq = q->h_q, G = q->h_q / c->h_kv;
    const double scale = orc_scale(q, d);
    int64_t max_kv = 0;
    for (int b = 0; b < batch; ++b) {
        int n_q = q->q_start[b + 1] - q->q_start[b];
        if (n_q < 0 || c->kv_len[b] < n_q)
            return ORC_ERR_ARG;
        if (c->kv_len[b] > max_kv)
            max_kv = c->kv_len[b];
    }
    const int64_t total_rows = q->q_start[batch];
    int err = ORC_OK;
#pragma omp parallel
    {
        int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(max_kv + 1));
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(max_kv + 1));
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t w = 0; w < total_rows * hq; ++w) {
            int64_t row = w / hq;
            int h = (int)(w % hq);
            int b = 0;
            while (q->q_start[b + 1] <= row)
                ++b;
            int n_q = q->q_start[b + 1] - q->q_start[b];
            int i = (int)(row - q->q_start[b]);
            int g = h / G;
            for (int e = 0; e < d; ++e)
                qv[e] = orc_widen(qdata, c->dtype, (row * hq + h) * d + e);
            int64_t n = build(ctx, b, c->kv_len[b], n_q, i, g, pos);
            int rc = orc_attend_set(c, b, g, qv, scale, pos, n, scratch,
                                    out + (row * hq + h) * d);
            if (rc != ORC_OK) {
#pragma omp atomic write
                err = rc;
            }
        }
        free(pos);
        free(scratch);
        free(qv);
    }
    return err;
}

/* Dense verification [StD "Procedimento de Decodificacao"]: the n_q = gamma + 1 new rows were
 * appended at positions [kv_len - n_q, kv_len); row i sees every position up to its own,
 * j <= kv_len - n_q + i (bottom-right aligned causal mask). */
static int64_t orc_build_verify(const void *ctx, int b, int64_t kv_len, int n_q, int i, int g,
                                int64_t *pos)
{
    (void)ctx; (void)b; (void)g;
    int64_t limit = kv_len - n_q + i;
    for (int64_t j = 0; j <= limit; ++j)
        pos[j] = j;
    return limit + 1;
}

int orc_verify_attention(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                         double *out)
{
    return orc_attention_driver(q, qdata, c, batch, orc_build_verify, NULL, out);
}

/* Single-token decode, written independently of the routines above: one query row per
 * sequence (row b), attending to all kv_len positions.  The softmax vector is formed first
 * and then applied to V. */
int orc_decode_attention(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                         double *out)
{
    if (q->h_q <= 0 || c->h_kv <= 0 || q->h_q % c->h_kv != 0)
        return ORC_ERR_ARG;
    const int d = c->head_dim, hq = q->h_q, G = hq / c->h_kv;
    const double scale = orc_scale(q, d);
    int err = ORC_OK;
    for (int b = 0; b < batch; ++b) {
        const int64_t L = c->kv_len[b];
        double *p = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        for (int h = 0; h < hq; ++h) {
            const int g = h / G;
            double *o = out + ((int64_t)b * hq + h) * d;
            for (int e = 0; e < d; ++e)
                o[e] = 0.0;
            if (L == 0)
                continue;
            for (int64_t j = 0; j < L; ++j) {
                int64_t kr = orc_kv_row(c, b, g, j);
                if (kr < 0) {
                    err = ORC_ERR_ARG;
                    p[j] = -INFINITY;
                    continue;
                }
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += orc_widen(qdata, c->dtype, ((int64_t)b * hq + h) * d + e) *
                           orc_widen(c->k, c->dtype, kr + e);
                p[j] = dot * scale;
            }
            double mx = p[0];
            for (int64_t j = 1; j < L; ++j)
                mx = p[j] > mx ? p[j] : mx;
            double z = 0.0;
            for (int64_t j = 0; j < L; ++j) {
                p[j] = exp(p[j] - mx);
                z += p[j];
            }
            for (int64_t j = 0; j < L; ++j) {
                int64_t vr = orc_kv_row(c, b, g, j);
                if (vr < 0)
                    continue;
                for (int e = 0; e < d; ++e)
                    o[e] += (p[j] / z) * orc_widen(c->v, c->dtype, vr + e);
            }
        }
        free(p);
    }
    return err;
}

/* Text-anchored window attention [SPW 3.1 / 3.A]: the visual span [vis_begin, vis_end) is
 * dropped entirely; of the remaining positions at or before the row's causal limit, only the
 * last `window` are kept (the window counts non-visual positions and ends at the row's own
 * position). */
typedef struct {
    const int32_t *vis_begin, *vis_end, *window;
} orc_ta_ctx;

static int64_t orc_build_text_anchored(const void *ctx, int b, int64_t kv_len, int n_q, int i,
                                       int g, int64_t *pos)
{
    (void)g;
    const orc_ta_ctx *t = (const orc_ta_ctx *)ctx;
    int64_t limit = kv_len - n_q + i;
    int64_t vb = t->vis_begin[b], ve = t->vis_end[b], W = t->window[b];
    int64_t n = 0;
    for (int64_t j = limit; j >= 0 && n < W; --j) {
        if (j >= vb && j < ve)
            continue;
        pos[n++] = j;
    }
    for (int64_t a = 0, z = n - 1; a < z; ++a, --z) { /* ascending order */
        int64_t tmp = pos[a];
        pos[a] = pos[z];
        pos[z] = tmp;
    }
    return n;
}

int orc_text_anchored_attention(const orc_query *q, const void *qdata, const orc_cache *c,
                                int batch, const int32_t *vis_begin, const int32_t *vis_end,
                                const int32_t *window, double *out)
{
    for (int b = 0; b < batch; ++b)
        if (window[b] < 1 || vis_begin[b] > vis_end[b])
            return ORC_ERR_ARG;
    orc_ta_ctx ctx = {vis_begin, vis_end, window};
    return orc_attention_driver(q, qdata, c, batch, orc_build_text_anchored, &ctx, out);
}

/* Sparse draft attention [StD "Metodologia": the sparse model M_s attends only to the top-K
 * KV entries]: the allowed set of row i is ({idx[b][g][0..k)} U [tail_begin, limit]) restricted
 * to [0, limit], limit = kv_len - n_q + i, taken as a set (an index listed twice, or also in the
 * tail, counts once).  Negative idx entries are padding and are ignored. */
typedef struct {
    const int32_t *idx;
    int k;
    int h_kv;
    const int32_t *tail_begin;
} orc_sp_ctx;

static int64_t orc_build_sparse(const void *ctx, int b, int64_t kv_len, int n_q, int i, int g,
                                int64_t *pos)
{
    const orc_sp_ctx *t = (const orc_sp_ctx *)ctx;
    int64_t limit = kv_len - n_q + i;
    unsigned char *mark = (unsigned char *)calloc((size_t)(limit + 1), 1);
    const int32_t *sel = t->idx + ((int64_t)b * t->h_kv + g) * t->k;
    for (int e = 0; e < t->k; ++e)
        if (sel[e] >= 0 && sel[e] <= limit)
            mark[sel[e]] = 1;
    int64_t tb = t->tail_begin[b] < 0 ? 0 : t->tail_begin[b];
    for (int64_t j = tb; j <= limit; ++j)
        mark[j] = 1;
    int64_t n = 0;
    for (int64_t j = 0; j <= limit; ++j)
        if (mark[j])
            pos[n++] = j;
    free(mark);
    return n;
}

int orc_sparse_attention(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                         const int32_t *idx, int k, const int32_t *tail_begin, double *out)
{
    if (k < 0)
        return ORC_ERR_ARG;
    orc_sp_ctx ctx = {idx, k, c->h_kv, tail_begin};
    return orc_attention_driver(q, qdata, c, batch, orc_build_sparse, &ctx, out);
}

/* ---------------------------------------------------------------- top-K selection -------- */

typedef struct {
    double s;
    int64_t j;
} orc_scored;

/* Larger score first; equal scores: lower position first. */
static int orc_cmp_scored(const void *a, const void *b)
{
    const orc_scored *x = (const orc_scored *)a, *y = (const orc_scored *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int orc_cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Top-K KV selection [StD "Selecao de Cache KV": keep the top-K KV entries, chosen per layer
 * and per head].  Score of candidate j for KV head g: the sum over the group's query heads of
 * the last query row's dot product with k_j (scaling by 1/sqrt(d) or by 1/G changes no rank, so
 * the unscaled sum is used).  The k best are taken, equal scores going to the lower position,
 * and written in ascending position order; unused slots get -1.  gap[b*h_kv+g] receives
 * (s_(k) - s_(k+1)) / max|s| (the margin at the selection boundary), or +inf when every
 * candidate is selected. */
int orc_topk_select(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                    const int32_t *cand_begin, const int32_t *cand_end, int k, int32_t *idx_out,
                    double *gap)
{
    if (k < 1 || q->h_q % c->h_kv != 0)
        return ORC_ERR_ARG;
    const int d = c->head_dim, hq = q->h_q, hk = c->h_kv, G = hq / hk;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < batch * hk; ++w) {
        int b = w / hk, g = w % hk;
        int64_t cb = cand_begin[b], ce = cand_end[b];
        int32_t *dst = idx_out + (int64_t)w * k;
        for (int e = 0; e < k; ++e)
            dst[e] = -1;
        if (ce <= cb) {
            if (gap) gap[w] = INFINITY;
            continue;
        }
        int64_t n = ce - cb;
        int64_t last_row = q->q_start[b + 1] - 1;
        orc_scored *sc = (orc_scored *)malloc(sizeof(orc_scored) * (size_t)n);
        double smax = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            int64_t j = cb + t;
            int64_t kr = orc_kv_row(c, b, g, j);
            double s = 0.0;
            if (kr < 0) {
#pragma omp atomic write
                err = ORC_ERR_ARG;
            } else {
                for (int h = g * G; h < (g + 1) * G; ++h)
                    for (int e = 0; e < d; ++e)
                        s += orc_widen(qdata, c->dtype, (last_row * hq + h) * d + e) *
                             orc_widen(c->k, c->dtype, kr + e);
            }
            sc[t].s = s;
            sc[t].j = j;
            if (fabs(s) > smax)
                smax = fabs(s);
        }
        qsort(sc, (size_t)n, sizeof(orc_scored), orc_cmp_scored);
        int64_t take = n < k ? n : k;
        for (int64_t e = 0; e < take; ++e)
            dst[e] = (int32_t)sc[e].j;
        qsort(dst, (size_t)take, sizeof(int32_t), orc_cmp_i32);
        if (gap) {
            if (n <= k)
                gap[w] = INFINITY;
            else
                gap[w] = smax > 0.0 ? (sc[k - 1].s - sc[k].s) / smax : 0.0;
        }
        free(sc);
    }
    return err;
}

/* The same scores as orc_topk_select, written out: scores[(b*h_kv+g)*row_width + t] is the
 * score of candidate cand_begin[b] + t. */
int orc_topk_scores(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                    const int32_t *cand_begin, const int32_t *cand_end, int64_t row_width,
                    double *scores)
{
    const int d = c->head_dim, hq = q->h_q, hk = c->h_kv, G = hq / hk;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < batch * hk; ++w) {
        int b = w / hk, g = w % hk;
        int64_t last_row = q->q_start[b + 1] - 1;
        for (int64_t j = cand_begin[b]; j < cand_end[b] && j - cand_begin[b] < row_width; ++j) {
            int64_t kr = orc_kv_row(c, b, g, j);
            double s = 0.0;
            if (kr < 0) {
#pragma omp atomic write
                err = ORC_ERR_ARG;
            } else {
                for (int h = g * G; h < (g + 1) * G; ++h)
                    for (int e = 0; e < d; ++e)
                        s += orc_widen(qdata, c->dtype, (last_row * hq + h) * d + e) *
                             orc_widen(c->k, c->dtype, kr + e);
            }
            scores[(int64_t)w * row_width + (j - cand_begin[b])] = s;
        }
    }
    return err;
}

/* ---------------------------------------------------------------- mean text attention -- */

/* Sparse-to-Dense's own selection score [StD "Selecao de Cache KV": the top-K visual KV
 * entries are chosen at prefill from the mean attention scores that the text tokens direct to
 * the visual tokens, separately for every layer and head].  The query rows of sequence b are
 * its prefill text tokens: the last n_q positions of its cache, row i at position
 * kv_len - n_q + i, attending causally (j <= limit_i = kv_len - n_q + i) with its own softmax
 * over every position it sees.  For KV head g and candidate j, with the G query heads h of the
 * group:
 *     a_{h,i}(j) = exp(s_{h,i,j} - m_{h,i}) / sum_{j' <= limit_i} exp(s_{h,i,j'} - m_{h,i})
 *                  (0 when j > limit_i),   s = scale * q_{h,i} . k_j,   m = max over j' <= limit_i
 *     score_j    = 1 / (G * n_q) * sum_h sum_i a_{h,i}(j)
 * (the mean over the group's heads as well as the text rows: one KV entry serves the whole
 * group).  scores[(b*h_kv+g)*row_width + t] receives the score of candidate cand_begin[b] + t. */
int orc_topk_attention_scores(const orc_query *q, const void *qdata, const orc_cache *c,
                              int batch, const int32_t *cand_begin, const int32_t *cand_end,
                              int64_t row_width, double *scores)
{
    if (q->h_q % c->h_kv != 0)
        return ORC_ERR_ARG;
    const int d = c->head_dim, hq = q->h_q, hk = c->h_kv, G = hq / hk;
    const double scale = orc_scale(q, d);
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < batch * hk; ++w) {
        int b = w / hk, g = w % hk;
        int64_t kv_len = c->kv_len[b];
        int64_t r0 = q->q_start[b], n_q = q->q_start[b + 1] - r0;
        int64_t cb = cand_begin[b], ce = cand_end[b];
        double *dst = scores + (int64_t)w * row_width;
        for (int64_t t = 0; t < row_width; ++t)
            dst[t] = (t < ce - cb) ? 0.0 : NAN;
        if (n_q < 1 || kv_len < n_q)
            continue;
        double *s = (double *)malloc(sizeof(double) * (size_t)kv_len);
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        for (int h = g * G; h < (g + 1) * G; ++h) {
            for (int64_t i = 0; i < n_q; ++i) {
                int64_t limit = kv_len - n_q + i;
                for (int e = 0; e < d; ++e)
                    qv[e] = orc_widen(qdata, c->dtype, ((r0 + i) * hq + h) * d + e);
                /* every score the row sees, then its softmax denominator */
                double m = -INFINITY;
                for (int64_t j = 0; j <= limit; ++j) {
                    int64_t kr = orc_kv_row(c, b, g, j);
                    double dot = 0.0;
                    if (kr < 0) {
#pragma omp atomic write
                        err = ORC_ERR_ARG;
                    } else {
                        for (int e = 0; e < d; ++e)
                            dot += qv[e] * orc_widen(c->k, c->dtype, kr + e);
                    }
                    s[j] = scale * dot;
                    if (s[j] > m)
                        m = s[j];
                }
                double den = 0.0;
                for (int64_t j = 0; j <= limit; ++j)
                    den += exp(s[j] - m);
                /* this row's weights of the candidates it sees */
                for (int64_t j = cb; j < ce && j <= limit && j - cb < row_width; ++j)
                    if (j >= 0)
                        dst[j - cb] += exp(s[j] - m) / den;
            }
        }
        for (int64_t t = 0; t < ce - cb && t < row_width; ++t)
            dst[t] /= (double)G * (double)n_q;
        free(qv);
        free(s);
    }
    return err;
}

/* Top-K selection by the mean text attention above: the k highest scores of every
 * (sequence, KV head), equal scores going to the lower position, written in ascending position
 * order with -1 in unused slots (the same selection rule as orc_topk_select).  gap[b*h_kv+g]
 * receives (score_(k) - score_(k+1)) / score_(1), or +inf when every candidate is selected. */
int orc_topk_select_attention(const orc_query *q, const void *qdata, const orc_cache *c,
                              int batch, const int32_t *cand_begin, const int32_t *cand_end,
                              int k, int32_t *idx_out, double *gap)
{
    if (k < 1 || q->h_q % c->h_kv != 0)
        return ORC_ERR_ARG;
    const int hk = c->h_kv;
    int64_t width = 1;
    for (int b = 0; b < batch; ++b)
        if ((int64_t)cand_end[b] - cand_begin[b] > width)
            width = (int64_t)cand_end[b] - cand_begin[b];
    double *all = (double *)malloc(sizeof(double) * (size_t)(batch * hk) * (size_t)width);
    int err = orc_topk_attention_scores(q, qdata, c, batch, cand_begin, cand_end, width, all);
    for (int w = 0; w < batch * hk; ++w) {
        int b = w / hk;
        int64_t cb = cand_begin[b], n = (int64_t)cand_end[b] - cb;
        int32_t *dst = idx_out + (int64_t)w * k;
        for (int e = 0; e < k; ++e)
            dst[e] = -1;
        if (n <= 0) {
            if (gap) gap[w] = INFINITY;
            continue;
        }
        orc_scored *sc = (orc_scored *)malloc(sizeof(orc_scored) * (size_t)n);
        for (int64_t t = 0; t < n; ++t) {
            sc[t].s = all[(int64_t)w * width + t];
            sc[t].j = cb + t;
        }
        qsort(sc, (size_t)n, sizeof(orc_scored), orc_cmp_scored);
        int64_t take = n < k ? n : k;
        for (int64_t e = 0; e < take; ++e)
            dst[e] = (int32_t)sc[e].j;
        qsort(dst, (size_t)take, sizeof(int32_t), orc_cmp_i32);
        if (gap) {
            if (n <= k)
                gap[w] = INFINITY;
            else
                gap[w] = sc[0].s > 0.0 ? (sc[k - 1].s - sc[k].s) / sc[0].s : 0.0;
        }
        free(sc);
    }
    free(all);
    return err;
}

/* ---------------------------------------------------------------- HSR projection --------- */

/* Hidden-state reuse [SPW 3.1]: the draft input is an FC over the concatenation
 * [current text embedding ; reused target hidden state]:
 *   y[r][o] = sum_{i<D} W[o][i] e[r][i] + sum_{i<D} W[o][D+i] h[r][i] (+ bias[o]).
 * W is row-major [D][2D] (out x in); all operands are bf16 bits. */
int orc_hsr_project(const uint16_t *emb, const uint16_t *hid, int n, int d_model,
                    const uint16_t *w, const uint16_t *bias, double *y)
{
    if (n < 0 || d_model <= 0)
        return ORC_ERR_ARG;
    const int64_t D = d_model;
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < D; ++o) {
        for (int r = 0; r < n; ++r) {
            double acc = 0.0;
            for (int64_t i = 0; i < D; ++i)
                acc += orc_widen(w, ORC_BF16, o * 2 * D + i) * orc_widen(emb, ORC_BF16, r * D + i);
            for (int64_t i = 0; i < D; ++i)
                acc += orc_widen(w, ORC_BF16, o * 2 * D + D + i) *
                       orc_widen(hid, ORC_BF16, r * D + i);
            if (bias)
                acc += orc_widen(bias, ORC_BF16, o);
            y[(int64_t)r * D + o] = acc;
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------- draft layer ----------- */

/* Sparrow's draft layer [SPW 3.1 HSR-VATA: the draft takes an FC over [text embedding ; reused
 * target hidden state] and attends only to text-anchored positions].  The pages name no layer
 * internals; the reading taken is one pre-norm decoder layer of the target's shapes:
 *   x  = W_hsr [e ; h]
 *   a  = RMSNorm(x) * ln1,       [q ; k ; v] = W_qkv a + b_qkv
 *   q, k rotated by RoPE at the row's position (rotate-half pairs (i, i + d/2),
 *        angle = pos * theta^(-2i/d))
 *   k, v stored in the draft's own cache at the row's position (the cache's bf16 type), q
 *        rounded to bf16 (the attention call's query type)
 *   o  = text-anchored attention of the rows over the cache (window W, no visual span)
 *   x2 = x + W_o o
 *   m  = RMSNorm(x2) * ln2,      y = x2 + W_down (silu(W_gate m) * (W_up m))
 * with RMSNorm(x)_i = x_i / sqrt(mean_j x_j^2 + eps) and silu(t) = t / (1 + exp(-t)).  All
 * arithmetic in double; weights and caches are bf16 bits. */

static void orc_rmsnorm(const double *x, int n, const uint16_t *gamma, double eps, double *y)
{
    double ss = 0.0;
    for (int i = 0; i < n; ++i)
        ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss / (double)n + eps);
    for (int i = 0; i < n; ++i)
        y[i] = x[i] * r * orc_widen(gamma, ORC_BF16, i);
}

static void orc_rope(double *v, int d, double pos, double theta)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double ang = pos * pow(theta, -2.0 * (double)i / (double)d);
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

/* y[o] = sum_i W[o][i] x[i] (+ bias[o]); W bf16 [m][k] row-major. */
static void orc_linear(const uint16_t *W, const uint16_t *bias, const double *x, int64_t m,
                       int64_t k, double *y)
{
    for (int64_t o = 0; o < m; ++o) {
        double acc = 0.0;
        for (int64_t i = 0; i < k; ++i)
            acc += orc_widen(W, ORC_BF16, o * k + i) * x[i];
        if (bias)
            acc += orc_widen(bias, ORC_BF16, o);
        y[o] = acc;
    }
}

/* Nearest bf16 (ties to even) of a double, through float. */
static uint16_t orc_to_bf16(double x)
{
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

int orc_rmsnorm_rows(const double *x, int rows, int n, const uint16_t *gamma, double eps,
                     double *y)
{
    for (int r = 0; r < rows; ++r)
        orc_rmsnorm(x + (int64_t)r * n, n, gamma, eps, y + (int64_t)r * n);
    return ORC_OK;
}

int orc_rope_rows(double *v, int rows, int d, const double *pos, double theta)
{
    for (int r = 0; r < rows; ++r)
        orc_rope(v + (int64_t)r * d, d, pos[r], theta);
    return ORC_OK;
}

/* The n rows are the last n positions of the cache (row r at position kv_len - n + r); the
 * caller's cache arrays receive the rows' k and v.  inter (may be NULL) receives, per row,
 * x [D], q [h_q d] (after RoPE, before rounding), o [h_q d], x2 [D] (in that order). */
int orc_draft_layer(const orc_draft_weights *w, const uint16_t *emb, const uint16_t *hid, int n,
                    const orc_cache *c, int window, double *y, double *inter)
{
    const int D = w->d_model, d = w->head_dim, hq = w->h_q, hk = w->h_kv, F = w->d_ff;
    const int nqkv = (hq + 2 * hk) * d;
    if (n < 1 || c->h_kv != hk || c->head_dim != d || c->dtype != ORC_BF16 || hq % hk)
        return ORC_ERR_ARG;
    const int64_t kv_len = c->kv_len[0];
    if (kv_len < n || window < 1)
        return ORC_ERR_ARG;
    double *x = malloc(sizeof(double) * (size_t)n * D);
    double *a = malloc(sizeof(double) * (size_t)D);
    double *qkv = malloc(sizeof(double) * (size_t)nqkv);
    double *q = malloc(sizeof(double) * (size_t)n * hq * d);
    uint16_t *qb = malloc(sizeof(uint16_t) * (size_t)n * hq * d);
    double *o = malloc(sizeof(double) * (size_t)n * hq * d);
    double *x2 = malloc(sizeof(double) * (size_t)D);
    double *gu = malloc(sizeof(double) * (size_t)2 * F);
    double *sv = malloc(sizeof(double) * (size_t)F);
    double *cat = malloc(sizeof(double) * (size_t)2 * D);
    uint16_t *kc = (uint16_t *)c->k, *vc = (uint16_t *)c->v;
    int err = ORC_OK;
    for (int r = 0; r < n; ++r) {
        for (int i = 0; i < D; ++i) {
            cat[i] = orc_widen(emb, ORC_BF16, (int64_t)r * D + i);
            cat[D + i] = orc_widen(hid, ORC_BF16, (int64_t)r * D + i);
        }
        orc_linear(w->w_hsr, NULL, cat, D, 2 * D, x + (int64_t)r * D);
        orc_rmsnorm(x + (int64_t)r * D, D, w->ln1, w->rms_eps, a);
        orc_linear(w->w_qkv, w->b_qkv, a, nqkv, D, qkv);
        const int64_t pos = kv_len - n + r;
        for (int h = 0; h < hq + hk; ++h)
            orc_rope(qkv + (int64_t)h * d, d, (double)pos, w->rope_theta);
        for (int i = 0; i < hq * d; ++i) {
            q[(int64_t)r * hq * d + i] = qkv[i];
            qb[(int64_t)r * hq * d + i] = orc_to_bf16(qkv[i]);
        }
        for (int g = 0; g < hk; ++g) {
            int64_t row = orc_kv_row(c, 0, g, pos);
            if (row < 0) {
                err = ORC_ERR_ARG;
                continue;
            }
            for (int e = 0; e < d; ++e) {
                kc[row + e] = orc_to_bf16(qkv[(int64_t)(hq + g) * d + e]);
                vc[row + e] = orc_to_bf16(qkv[(int64_t)(hq + hk + g) * d + e]);
            }
        }
    }
    if (err == ORC_OK) {
        int32_t qs[2] = {0, n}, vb = 0, ve = 0, win = window;
        orc_query qd = {hq, 0.0, qs};
        err = orc_text_anchored_attention(&qd, qb, c, 1, &vb, &ve, &win, o);
    }
    for (int r = 0; err == ORC_OK && r < n; ++r) {
        orc_linear(w->w_o, NULL, o + (int64_t)r * hq * d, D, (int64_t)hq * d, x2);
        for (int i = 0; i < D; ++i)
            x2[i] += x[(int64_t)r * D + i];
        orc_rmsnorm(x2, D, w->ln2, w->rms_eps, a);
        orc_linear(w->w_gate_up, NULL, a, 2 * (int64_t)F, D, gu);
        for (int i = 0; i < F; ++i)
            sv[i] = gu[i] / (1.0 + exp(-gu[i])) * gu[F + i];
        orc_linear(w->w_down, NULL, sv, D, F, y + (int64_t)r * D);
        for (int i = 0; i < D; ++i)
            y[(int64_t)r * D + i] += x2[i];
        if (inter) {
            double *dst = inter + (int64_t)r * (2 * D + 2 * hq * d);
            memcpy(dst, x + (int64_t)r * D, sizeof(double) * (size_t)D);
            memcpy(dst + D, q + (int64_t)r * hq * d, sizeof(double) * (size_t)hq * d);
            memcpy(dst + D + hq * d, o + (int64_t)r * hq * d, sizeof(double) * (size_t)hq * d);
            memcpy(dst + D + 2 * hq * d, x2, sizeof(double) * (size_t)D);
        }
    }
    free(x); free(a); free(qkv); free(q); free(qb); free(o); free(x2); free(gu); free(sv);
    free(cat);
    return err;
}

/* ---------------------------------------------------------------- acceptance ------------- */

/* Index of the largest entry; equal values go to the lower index; NaN ranks below -inf. */
static int64_t orc_argmax(const float *z, int64_t n)
{
    int64_t best = 0;
    for (int64_t x = 1; x < n; ++x) {
        if (isnan(z[x]))
            continue;
        if (isnan(z[best]) || z[x] > z[best])
            best = x;
    }
    return best;
}

/* Greedy verification [StD "Procedimento de Decodificacao"]: t_i = argmax of target row i
 * (i = 0..gamma); the longest prefix n with d_{i+1} == t_i for i < n is accepted, and the
 * target's own token t_n is appended as the bonus.  Output: d_1..d_n, t_n; n_acc[b] = n. */
int orc_accept_greedy(const float *tgt, const int32_t *draft, const int32_t *gamma, int batch,
                      int vocab, int32_t *n_acc, int32_t *out_tok, int out_stride)
{
    int64_t off_t = 0, off_d = 0;
    for (int b = 0; b < batch; ++b) {
        const int gm = gamma[b];
        if (gm < 0 || out_stride < gm + 1)
            return ORC_ERR_ARG;
        int n = 0;
        int64_t t_n = orc_argmax(tgt + off_t * vocab, vocab);
        while (n < gm && draft[off_d + n] == t_n) {
            ++n;
            t_n = orc_argmax(tgt + (off_t + n) * vocab, vocab);
        }
        for (int e = 0; e < n; ++e)
            out_tok[(int64_t)b * out_stride + e] = draft[off_d + e];
        out_tok[(int64_t)b * out_stride + n] = (int32_t)t_n;
        n_acc[b] = n;
        off_t += gm + 1;
        off_d += gm;
    }
    return ORC_OK;
}

/* log sum exp with the max shift. */
static double orc_lse(const float *z, int64_t n)
{
    double m = -INFINITY;
    for (int64_t x = 0; x < n; ++x)
        if ((double)z[x] > m)
            m = (double)z[x];
    double s = 0.0;
    for (int64_t x = 0; x < n; ++x)
        s += exp((double)z[x] - m);
    return m + log(s);
}

/* Smallest x with sum_{y<=x} w_y > v * Z (Z = sum of all w); if rounding leaves no such x,
 * the last x with w_x > 0.  *margin receives min(v Z - C(x-1), C(x) - v Z) / Z. */
static int64_t orc_draw(const double *w, int64_t n, double v, double *margin)
{
    double Z = 0.0;
    for (int64_t x = 0; x < n; ++x)
        Z += w[x];
    double target = v * Z, c = 0.0;
    int64_t last_pos = 0;
    for (int64_t x = 0; x < n; ++x) {
        double prev = c;
        c += w[x];
        if (w[x] > 0.0)
            last_pos = x;
        if (c > target) {
            double a = target - prev, bnd = c - target;
            *margin = (a < bnd ? a : bnd) / Z;
            return x;
        }
    }
    *margin = 0.0;
    return last_pos;
}

/* Speculative sampling with residual resampling [StD "Principais Contribuicoes": acceleration
 * without changing the output distribution; the rule itself is the standard one]:
 * p_i = softmax(target row i), q_i = softmax(draft row i).  For i = 1..gamma the drafted token
 * d_i is accepted iff u_i <= p_{i-1}(d_i) / q_{i-1}(d_i).  At the first rejection (i = n+1) a
 * token is drawn from norm(max(0, p_n - q_n)) with v_n (from p_n when that residual is all
 * zero); when all gamma are accepted the bonus is drawn from p_gamma with v_gamma.
 * accept_margin[k] = u_k - ratio_k for every evaluated draft position (NaN otherwise);
 * draw_margin[b] = the drawn token's distance to its CDF bucket edges, divided by Z. */
int orc_accept_sample(const float *tgt, const float *drf, const int32_t *draft, const float *u,
                      const float *v, const int32_t *gamma, int batch, int vocab, int32_t *n_acc,
                      int32_t *out_tok, int out_stride, double *accept_margin,
                      double *draw_margin)
{
    int64_t off_t = 0, off_d = 0;
    double *w = (double *)malloc(sizeof(double) * (size_t)vocab);
    for (int b = 0; b < batch; ++b) {
        const int gm = gamma[b];
        if (gm < 0 || out_stride < gm + 1) {
            free(w);
            return ORC_ERR_ARG;
        }
        for (int e = 0; e < gm; ++e)
            if (accept_margin)
                accept_margin[off_d + e] = NAN;
        int n = 0;
        int rejected = 0;
        for (int i = 1; i <= gm; ++i) {
            const float *zp = tgt + (off_t + i - 1) * vocab;
            const float *zq = drf + (off_d + i - 1) * vocab;
            int32_t x = draft[off_d + i - 1];
            double r = 0.0;
            if (x >= 0 && x < vocab)
                r = exp(((double)zp[x] - orc_lse(zp, vocab)) - ((double)zq[x] - orc_lse(zq, vocab)));
            if (accept_margin)
                accept_margin[off_d + i - 1] = (double)u[off_d + i - 1] - r;
            if ((double)u[off_d + i - 1] <= r) {
                ++n;
            } else {
                rejected = 1;
                break;
            }
        }
        const float *zp = tgt + (off_t + n) * vocab;
        double lp = orc_lse(zp, vocab);
        double Z = 0.0;
        if (rejected) {
            const float *zq = drf + (off_d + n) * vocab;
            double lq = orc_lse(zq, vocab);
            for (int64_t x = 0; x < vocab; ++x) {
                double diff = exp((double)zp[x] - lp) - exp((double)zq[x] - lq);
                w[x] = diff > 0.0 ? diff : 0.0;
                Z += w[x];
            }
        }
        if (!rejected || Z == 0.0)
            for (int64_t x = 0; x < vocab; ++x)
                w[x] = exp((double)zp[x] - lp);
        double margin = 0.0;
        int64_t tok = orc_draw(w, vocab, (double)v[off_t + n], &margin);
        if (draw_margin)
            draw_margin[b] = margin;
        for (int e = 0; e < n; ++e)
            out_tok[(int64_t)b * out_stride + e] = draft[off_d + e];
        out_tok[(int64_t)b * out_stride + n] = (int32_t)tok;
        n_acc[b] = n;
        off_t += gm + 1;
        off_d += gm;
    }
    free(w);
    return ORC_OK;
}

/* ---------------------------------------------------------------- threads ---------------- */

int orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
