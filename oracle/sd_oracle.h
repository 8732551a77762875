/*
 * fp64 CPU oracle: declarations.  TEST INFRASTRUCTURE ONLY (see sd_oracle.c).
 * This header belongs to the oracle alone; the CUDA library has its own, unrelated header.
 */
#ifndef SD_ORACLE_H
#define SD_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_OK = 0, ORC_ERR_ARG = 1 };
enum { ORC_F32 = 0, ORC_BF16 = 1 };

/* KV cache (host memory).  Contiguous when page_size == 0: element (b, h, j, e) is at
 * b*stride_b + h*stride_h + j*stride_pos + e.  Paged otherwise: page p = block_table[b][j/ps]
 * holds [h_kv][page_size][head_dim]. */
typedef struct {
    int32_t dtype;
    int32_t h_kv;
    int32_t head_dim;
    int32_t page_size;
    const void *k;
    const void *v;
    int64_t stride_b, stride_h, stride_pos;
    const int32_t *block_table;
    int32_t max_pages;
    int32_t num_pages;
    const int32_t *kv_len; /* [batch] */
} orc_cache;

/* Query rows [q_start[batch]][h_q][head_dim] in the cache's dtype; sequence b owns rows
 * [q_start[b], q_start[b+1]). */
typedef struct {
    int32_t h_q;
    double softmax_scale; /* <= 0 selects 1/sqrt(head_dim) */
    const int32_t *q_start;
} orc_query;

int orc_verify_attention(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                         double *out);
int orc_decode_attention(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                         double *out);
int orc_text_anchored_attention(const orc_query *q, const void *qdata, const orc_cache *c,
                                int batch, const int32_t *vis_begin, const int32_t *vis_end,
                                const int32_t *window, double *out);
int orc_sparse_attention(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                         const int32_t *idx, int k, const int32_t *tail_begin, double *out);
int orc_topk_select(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                    const int32_t *cand_begin, const int32_t *cand_end, int k, int32_t *idx_out,
                    double *gap);
int orc_topk_scores(const orc_query *q, const void *qdata, const orc_cache *c, int batch,
                    const int32_t *cand_begin, const int32_t *cand_end, int64_t row_width,
                    double *scores);
int orc_topk_attention_scores(const orc_query *q, const void *qdata, const orc_cache *c,
                              int batch, const int32_t *cand_begin, const int32_t *cand_end,
                              int64_t row_width, double *scores);
int orc_topk_select_attention(const orc_query *q, const void *qdata, const orc_cache *c,
                              int batch, const int32_t *cand_begin, const int32_t *cand_end,
                              int k, int32_t *idx_out, double *gap);
int orc_hsr_project(const uint16_t *emb, const uint16_t *hid, int n, int d_model,
                    const uint16_t *w, const uint16_t *bias, double *y);
int orc_accept_greedy(const float *tgt, const int32_t *draft, const int32_t *gamma, int batch,
                      int vocab, int32_t *n_acc, int32_t *out_tok, int out_stride);
int orc_accept_sample(const float *tgt, const float *drf, const int32_t *draft, const float *u,
                      const float *v, const int32_t *gamma, int batch, int vocab, int32_t *n_acc,
                      int32_t *out_tok, int out_stride, double *accept_margin,
                      double *draw_margin);
/* Weights of one draft layer (all bf16 bits; b_qkv may be NULL). */
typedef struct {
    int32_t d_model, h_q, h_kv, head_dim, d_ff;
    double rms_eps, rope_theta;
    const uint16_t *w_hsr;     /* [d_model][2 d_model] */
    const uint16_t *ln1;       /* [d_model] */
    const uint16_t *w_qkv;     /* [(h_q + 2 h_kv) head_dim][d_model] */
    const uint16_t *b_qkv;     /* [(h_q + 2 h_kv) head_dim] */
    const uint16_t *w_o;       /* [d_model][h_q head_dim] */
    const uint16_t *ln2;       /* [d_model] */
    const uint16_t *w_gate_up; /* [2 d_ff][d_model]: the gate rows, then the up rows */
    const uint16_t *w_down;    /* [d_model][d_ff] */
} orc_draft_weights;

int orc_rmsnorm_rows(const double *x, int rows, int n, const uint16_t *gamma, double eps,
                     double *y);
int orc_rope_rows(double *v, int rows, int d, const double *pos, double theta);
int orc_draft_layer(const orc_draft_weights *w, const uint16_t *emb, const uint16_t *hid, int n,
                    const orc_cache *c, int window, double *y, double *inter);
int orc_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
