/*
 * sd_attn.h -- C interface of libsdattn.so: the attention and acceptance hot path of
 * speculative decoding in video LLMs, as hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * Sources, by page title and section (the pages give the method, not formulas or code):
 *  [StD] "Sparse-to-Dense: A Free Lunch for Lossless Acceleration of Video Understanding in
 *        LLMs" (gist.science, pt), technical summary:
 *        - "Procedimento de Decodificacao": the sparse model drafts gamma tokens; the dense
 *          model verifies them in parallel with one read of the full KV cache; the longest
 *          matching prefix (n tokens) is accepted plus one extra bonus token.
 *        - "Metodologia": the sparse draft attends only to the top-K KV entries.
 *        - "Selecao de Cache KV": the top-K selection is per layer and per head.
 *        - "Principais Contribuicoes": lossless, the output distribution is unchanged.
 *  [SPW] "Sparrow: Text-Anchored Window Attention with Visual-Semantic Glimpsing for
 *        Speculative Decoding in Video LLMs" (gist.science zh section 3.1 HSR-VATA; pt
 *        section 3.A): hidden-state reuse (an FC over [text embedding ; reused target hidden
 *        state]) and text-anchored window attention that drops the visual KV cache.
 *
 * Conventions shared by every call
 *  - Every pointer argument is DEVICE memory owned by the caller unless stated otherwise;
 *    descriptor structs themselves are read on the host during the call and may be freed
 *    after it returns.  The library allocates no device memory and keeps no global state
 *    (except the wait bound of sd_set_wait_timeout_ns and the fixed scratch of
 *    sd_verify_attention_noalloc);
 *    scratch memory ("workspace") is passed in by the caller, sized by the *_workspace_size
 *    queries.  Calls on different streams with different workspaces may run concurrently.
 *  - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t; NULL means the
 *    legacy default stream).  No call synchronises the device.
 *  - Host-side validation runs before anything is launched.  An invalid argument returns a
 *    status != SD_OK and launches nothing.  A launch failure returns SD_ERR_CUDA.
 *  - Problems only visible on the device (an out-of-range page index, a bad sparse index,
 *    an out-of-range drafted token, a length exceeding a host hint) are OR-ed as
 *    SD_DEVERR_* bits into the optional int32 flag `dev_err` (device memory, may be NULL);
 *    the offending element is skipped, nothing is read or written out of bounds.
 *  - Tensors are row-major.  bf16 tensors hold IEEE bfloat16 bit patterns.
 */
#ifndef SD_ATTN_H
#define SD_ATTN_H

#include <stddef.h>
#include <stdint.h>

/* Exported symbols keep default visibility even when the library is built hidden-by-default. */
#if defined(__GNUC__)
#define SD_API __attribute__((visibility("default")))
#else
#define SD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SD_OK = 0,
    SD_ERR_INVALID_ARG = 1, /* a host-checkable argument is wrong; nothing launched */
    SD_ERR_UNSUPPORTED = 2, /* valid, but not a supported configuration (dtype, head_dim) */
    SD_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the size query returned */
    SD_ERR_CUDA = 4         /* a CUDA launch or runtime call failed */
} sd_status;

typedef enum { SD_F32 = 0, SD_BF16 = 1 } sd_dtype;

/* Attention kinds, for sd_attention_workspace_size. */
typedef enum {
    SD_ATTN_VERIFY = 0,
    SD_ATTN_TEXT_ANCHORED = 1,
    SD_ATTN_SPARSE = 2
} sd_attn_kind;

/* Device error bits (OR-ed into *dev_err). */
#define SD_DEVERR_PAGE 1u     /* block_table entry outside [0, num_pages) */
#define SD_DEVERR_INDEX 2u    /* sparse index not strictly ascending, or candidate range bad */
#define SD_DEVERR_TOKEN 4u    /* drafted token outside [0, vocab) */
#define SD_DEVERR_NUMERIC 8u  /* non-finite softmax statistics during sampling */
#define SD_DEVERR_SHAPE 16u   /* a device length exceeds its host hint (rows, kv_len) */
#define SD_DEVERR_TIMEOUT 32u /* a bounded wait inside a kernel expired; its outputs are undefined */

/*
 * KV cache of a batch of independent sequences.  A multi-layer problem is a batch whose
 * entries are layers (each entry has its own cache, found through stride_b or block_table).
 * Each sequence holds kv_len[b] positions: the context (visual span, then text), then the
 * positions appended for the current draft / verify step.
 *
 *  dtype      SD_F32 or SD_BF16; Q and O of the attention calls use the same type.
 *  h_kv       KV heads; query head h uses KV head h / (h_q / h_kv).
 *  head_dim   64 or 128.
 *  k, v       base pointers (device).
 *  Contiguous layout (page_size == 0): element (b, h, j, e) of K is at
 *             k[b*stride_b + h*stride_h + j*stride_pos + e]; strides in elements, e contiguous.
 *             stride_pos must equal head_dim (rows are dense); for the tensor-core verify path
 *             the base must be 16-byte aligned and stride_h, stride_b multiples of 8 elements.
 *  Paged layout (page_size == 16): page p holds [h_kv][16][head_dim] elements at
 *             k + p*h_kv*16*head_dim; position j of sequence b lives in page
 *             block_table[b*max_pages_per_seq + j/16] at slot j%16.  num_pages bounds entries.
 *  kv_len     device int32 [batch].
 */
typedef struct {
    int32_t dtype;
    int32_t h_kv;
    int32_t head_dim;
    int32_t page_size;
    const void *k;
    const void *v;
    int64_t stride_b;
    int64_t stride_h;
    int64_t stride_pos;
    const int32_t *block_table;
    int32_t max_pages_per_seq;
    int32_t num_pages;
    const int32_t *kv_len;
} sd_kv_desc;

/*
 * Query rows.  Q (and the output O) are [total_rows][h_q][head_dim]; sequence b owns rows
 * [q_start[b], q_start[b+1]) (device int32 [batch+1], q_start[0] == 0).  Its n_q rows are the
 * LAST n_q positions of its cache (the caller appended their K/V before the call), so row i
 * sees positions j <= kv_len - n_q + i (bottom-right aligned causal mask).
 *
 *  max_q_rows     host hint: an upper bound of q_start[b+1] - q_start[b] (sizes grid/workspace).
 *  max_kv_len     host hint: an upper bound of kv_len[b] (sizes the split-KV decomposition).
 *  softmax_scale  scale of q.k; 0 selects 1/sqrt(head_dim).
 */
typedef struct {
    int32_t h_q;
    int32_t max_q_rows;
    int32_t max_kv_len;
    float softmax_scale;
    const int32_t *q_start;
} sd_q_desc;

/* Human-readable name of a status. */
SD_API const char *sd_status_string(sd_status s);

/* Library version, major*10000 + minor*100 + patch. */
SD_API int32_t sd_version(void);

/*
 * Bound of every wait inside the library's tensor-core kernels (a pipeline stage waiting for a
 * copy or an MMA that another warp of the same CTA issues).  A wait that runs out sets
 * SD_DEVERR_TIMEOUT in the call's dev_err; the CTA then waits (at most 1 s more) for the copies
 * and MMAs it has already issued, frees its tensor memory and exits, so the device stays usable
 * and the call's outputs are undefined.  Process-wide, for the calls launched after it returns;
 * ns = 0 restores the default of 1 s (1e9 ns).  Returns the previous bound.  Meant for failure
 * detection and its tests: a bound of 1 ns makes a call's waits run out at once.
 */
SD_API uint64_t sd_set_wait_timeout_ns(uint64_t ns);

/*
 * Workspace bytes a verify or text-anchored call needs for these descriptors (host hints only;
 * device arrays are not read).  A call may be given more.  *bytes may be 0.  SD_ATTN_SPARSE is
 * rejected (SD_ERR_INVALID_ARG): its size depends on k, see sd_sparse_workspace_size.
 */
SD_API sd_status sd_attention_workspace_size(sd_attn_kind kind, const sd_q_desc *q,
                                      const sd_kv_desc *kv, int32_t batch, size_t *bytes);

/*
 * How an attention call with these host hints is decomposed (host values only; device arrays
 * are not read; nothing is launched).  *engine: SD_ENGINE_CUDA_CORE, SD_ENGINE_TC (tcgen05, one
 * CTA per split of every (sequence, KV head) unit) or SD_ENGINE_TC_PERSISTENT (tcgen05, one CTA
 * per SM over an even share of all units' tiles, long streams); *parts: the split count, or the
 * persistent plan's partial slots per unit.  extent: a text-anchored call's max_window or a
 * sparse call's k (ignored for verify); max_tail: a sparse call's hint (ignored otherwise).  The
 * tensor-core engines also need 16-byte aligned q and out at the call (else CUDA cores run it).
 * Returns SD_ERR_INVALID_ARG for invalid descriptors, SD_ERR_UNSUPPORTED for a head_dim other
 * than 64 or 128.
 */
typedef enum {
    SD_ENGINE_CUDA_CORE = 0,
    SD_ENGINE_TC = 1,
    SD_ENGINE_TC_PERSISTENT = 2
} sd_attn_engine;

SD_API sd_status sd_attention_plan(sd_attn_kind kind, const sd_q_desc *q, const sd_kv_desc *kv,
                                   int32_t batch, int32_t extent, int32_t max_tail,
                                   int32_t *engine, int32_t *parts);

/*
 * Dense verification attention [StD "Procedimento de Decodificacao"]: the target scores the
 * gamma+1 new positions of every sequence in one pass over its full cache.  For every row i
 * of sequence b and query head h:
 *     O = softmax(scale * q . k_j  over j <= kv_len[b] - n_q + i) . V
 * computed as split-KV flash-decoding (each split keeps an online softmax; the splits are
 * merged by their log-sum-exp).  q: [rows][h_q][d], out: [rows][h_q][d] (kv dtype).
 * Tensor cores (tcgen05) serve bf16 caches with d = 64 or 128 and at most 128 planned rows
 * per KV head (G * max_q_rows), when q_data and out are 16-byte aligned and the cache layout
 * can be described to the copy engine (16-byte aligned base and strides); CUDA cores serve the
 * rest (fp32 caches, more rows, other layouts).
 */
SD_API sd_status sd_verify_attention(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv,
                              int32_t batch, void *out, void *workspace, size_t workspace_bytes,
                              int32_t *dev_err, void *stream);

/*
 * Text-anchored window attention [SPW 3.1 / 3.A]: Sparrow's draft drops the visual KV cache
 * and attends only inside a text-anchored window.  For row i of sequence b the allowed
 * positions are the last window[b] positions j <= kv_len[b] - n_q + i that lie outside the
 * visual span [vis_begin[b], vis_end[b]) (the window counts non-visual positions and ends at
 * the row's own position; it may reach below the visual span).  vis_begin, vis_end, window:
 * device int32 [batch]; window >= 1; vis_begin <= vis_end (else the span is taken as empty
 * and SD_DEVERR_INDEX is set).  max_window: host hint >= every window[b].
 * A row with no allowed position outputs zeros.
 */
SD_API sd_status sd_text_anchored_attention(const sd_q_desc *q, const void *q_data,
                                     const sd_kv_desc *kv, int32_t batch,
                                     const int32_t *vis_begin, const int32_t *vis_end,
                                     const int32_t *window, int32_t max_window, void *out,
                                     void *workspace, size_t workspace_bytes, int32_t *dev_err,
                                     void *stream);

/*
 * Workspace bytes of sd_sparse_attention with these descriptors, k list entries and the
 * max_tail hint (host values only).  For bf16 caches it includes the staging of the selected
 * rows: batch * h_kv * k * head_dim * 2 bytes for K and as much for V, plus their positions.
 */
SD_API sd_status sd_sparse_workspace_size(const sd_q_desc *q, const sd_kv_desc *kv,
                                          int32_t batch, int32_t k, int32_t max_tail,
                                          size_t *bytes);

/*
 * Sparse draft attention [StD "Metodologia"]: the sparse model attends only to the selected
 * top-K KV entries plus the dense tail.  For row i of sequence b and KV head g the allowed
 * set is ({idx[b][g][0..k)} U [tail_begin[b], limit]) restricted to j <= limit,
 * limit = kv_len[b] - n_q + i.  idx: device int32 [batch][h_kv][k], ascending; negative
 * entries are padding and ignored; entries >= tail_begin are covered by the tail; a
 * non-ascending list sets SD_DEVERR_INDEX and repeated entries are skipped.
 * tail_begin: device int32 [batch].  max_tail: host hint >= kv_len[b] - tail_begin[b].
 * bf16 caches: the kept entries' K and V rows are first copied, in list order, into the
 * workspace, and the tensor-core kernel streams that compact run and the tail.  The workspace
 * (sd_sparse_workspace_size) must not be shared with a call in flight.
 */
SD_API sd_status sd_sparse_attention(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv,
                              int32_t batch, const int32_t *idx, int32_t k,
                              const int32_t *tail_begin, int32_t max_tail, void *out,
                              void *workspace, size_t workspace_bytes, int32_t *dev_err,
                              void *stream);

/*
 * Staged sparse selection [StD "Metodologia": the top-K KV entries are chosen once and reused
 * by every draft step].  sd_sparse_stage copies, for every (sequence, KV head), the K and V
 * rows of the entries of idx that sd_sparse_attention would use (0 <= x < tail_begin[b], not
 * equal to the entry before; a non-ascending list sets SD_DEVERR_INDEX) into `selection`,
 * in list order, with their positions and counts.  sd_sparse_attention_staged then computes
 * exactly what sd_sparse_attention computes for that idx, reading the staged rows instead of
 * gathering them again; the selection stays valid while idx, tail_begin and the selected cache
 * rows are unchanged (the draft steps of one cycle append only to the tail).
 *
 * selection: device memory of sd_sparse_selection_size bytes, 256-byte aligned, owned by the
 * caller.  k must be the same in the three calls.  bf16 caches, head_dim 64 or 128 and at most
 * 128 rows per KV head; otherwise SD_ERR_UNSUPPORTED (use sd_sparse_attention).  The staged
 * attention's workspace: sd_attention_workspace_size is not used; pass
 * sd_sparse_workspace_size(...) bytes or more.
 */
SD_API sd_status sd_sparse_selection_size(const sd_kv_desc *kv, int32_t batch, int32_t k,
                                          size_t *bytes);

SD_API sd_status sd_sparse_stage(const sd_kv_desc *kv, int32_t batch, const int32_t *idx,
                                 int32_t k, const int32_t *tail_begin, void *selection,
                                 size_t selection_bytes, int32_t *dev_err, void *stream);

SD_API sd_status sd_sparse_attention_staged(const sd_q_desc *q, const void *q_data,
                                            const sd_kv_desc *kv, int32_t batch,
                                            const void *selection, int32_t k,
                                            const int32_t *tail_begin, int32_t max_tail,
                                            void *out, void *workspace, size_t workspace_bytes,
                                            int32_t *dev_err, void *stream);

/*
 * Workspace for sd_topk_select.  max_cand: host hint >= cand_end[b] - cand_begin[b].
 */
SD_API sd_status sd_topk_workspace_size(const sd_kv_desc *kv, int32_t batch, int32_t max_cand,
                                 int32_t k, size_t *bytes);

/*
 * Top-K KV selection [StD "Selecao de Cache KV": top-K KV entries per layer and per head].
 * For sequence b and KV head g, candidate j in [cand_begin[b], cand_end[b]) scores
 *     s_j = sum over the group's query heads h of  q_last[h] . k_j
 * where q_last is the LAST query row of the sequence (row q_start[b+1]-1 of q_data).  The
 * scale 1/sqrt(d) changes no rank and is not applied.  Scores are accumulated in fp64.  The k
 * highest scores are selected, equal scores going to the lower position, and written in
 * ascending position order to idx_out [batch][h_kv][k] (device int32); when fewer than k
 * candidates exist all of them are written and the rest is -1.  A key with an infinite or NaN
 * element scores +inf, -inf or NaN as that sum does (NaN ranks below every other score).
 */
SD_API sd_status sd_topk_select(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv,
                         int32_t batch, const int32_t *cand_begin, const int32_t *cand_end,
                         int32_t max_cand, int32_t k, int32_t *idx_out, void *workspace,
                         size_t workspace_bytes, int32_t *dev_err, void *stream);

/*
 * Score modes of the top-K selection.
 *  SD_TOPK_LAST_QUERY            the score of sd_topk_select: the sum over the KV head's query
 *                                heads of the sequence's last query row dotted with k_j.
 *  SD_TOPK_MEAN_TEXT_ATTENTION   Sparse-to-Dense's own rule [StD "Selecao de Cache KV": the
 *                                top-K visual KV entries are chosen at prefill from the mean
 *                                attention the text tokens direct to the visual tokens, per
 *                                layer and head]: the query rows of sequence b are its n_q
 *                                prefill text rows, the LAST n_q positions of its cache (row i
 *                                at position kv_len[b] - n_q + i), each attending causally with
 *                                its own softmax (scale softmax_scale, 0 = 1/sqrt(d)) over every
 *                                position it sees; the score of candidate j is its attention
 *                                weight averaged over the n_q rows and the G query heads:
 *                                  score_j = 1/(G n_q) sum_h sum_i a_{h,i}(j)
 */
typedef enum { SD_TOPK_LAST_QUERY = 0, SD_TOPK_MEAN_TEXT_ATTENTION = 1 } sd_topk_score;

/*
 * Workspace of sd_topk_select_scored.  Mode SD_TOPK_MEAN_TEXT_ATTENTION also holds one float
 * per (text row, query head): batch * q->max_q_rows * q->h_q * 4 bytes beyond the keys.
 */
SD_API sd_status sd_topk_scored_workspace_size(sd_topk_score mode, const sd_q_desc *q,
                                               const sd_kv_desc *kv, int32_t batch,
                                               int32_t max_cand, int32_t k, size_t *bytes);

/*
 * Top-K selection with a score mode (see sd_topk_score).  SD_TOPK_LAST_QUERY computes exactly
 * what sd_topk_select computes.  The selection rule is the same for both modes: the k highest
 * scores of every (sequence, KV head) among [cand_begin[b], cand_end[b]), equal scores to the
 * lower position, written ascending to idx_out [batch][h_kv][k] (-1 padded).
 * scores_out (device double [batch][h_kv][max_cand], may be NULL) receives every candidate's
 * score (slot t: candidate cand_begin[b] + t); NaN-free inputs give finite scores.
 * SD_TOPK_MEAN_TEXT_ATTENTION: q / q_data hold the prefill text rows (q->max_q_rows bounds the
 * rows of every sequence; q->max_kv_len bounds kv_len); its scores are accumulated in fp32 per
 * 128-row tile and in fp64 across tiles, with the scores themselves from fp32 tensor-core
 * products of the bf16 inputs (CUDA cores for fp32 caches), so two scores closer than about
 * 1e-5 relative may rank in either order.
 */
SD_API sd_status sd_topk_select_scored(sd_topk_score mode, const sd_q_desc *q, const void *q_data,
                                       const sd_kv_desc *kv, int32_t batch,
                                       const int32_t *cand_begin, const int32_t *cand_end,
                                       int32_t max_cand, int32_t k, int32_t *idx_out,
                                       double *scores_out, void *workspace,
                                       size_t workspace_bytes, int32_t *dev_err, void *stream);

/*
 * Hidden-state reuse projection [SPW 3.1]: the draft input is an FC over the concatenation
 * of the current text embedding and the reused target hidden state:
 *     y[r][o] = sum_i W[o][i] emb[r][i] + sum_i W[o][d_model+i] hid[r][i] (+ bias[o])
 * emb, hid: [n_rows][d_model]; W: [d_model][2*d_model] (out x in); bias: [d_model] or NULL;
 * y: [n_rows][d_model].  All bf16; fp32 accumulation.  The concatenation is never
 * materialised.  1 <= n_rows <= 16; d_model a multiple of 16; emb, hid and W 16-byte aligned.
 */
SD_API sd_status sd_hsr_project(const void *emb, const void *hid, int32_t n_rows, int32_t d_model,
                         const void *weight, const void *bias, void *y, void *stream);

/*
 * Sparrow's draft layer [SPW 3.1 HSR-VATA: the draft model takes an FC over [text embedding ;
 * reused target hidden state] and attends only to text-anchored positions].  The pages name no
 * other layer internals; this is one pre-norm decoder layer of the target's shapes:
 *     x  = W_hsr [e ; h]                                   (as sd_hsr_project, kept in fp32)
 *     a  = RMSNorm(x) * ln1,  [q ; k ; v] = W_qkv a + b_qkv
 *     q, k rotated by RoPE at the row's position (rotate-half pairs (i, i + d/2),
 *          angle = pos * rope_theta^(-2i/d))
 *     k, v written into the draft's cache at the row's position; q rounded to bf16
 *     o  = text-anchored attention of the rows over that cache (window, no visual span)
 *     x2 = x + W_o o,  m = RMSNorm(x2) * ln2,  y = x2 + W_down (silu(W_gate m) * (W_up m))
 * with RMSNorm(x)_i = x_i / sqrt(mean_j x_j^2 + rms_eps).  All weights bf16, row-major
 * [out][in]: w_hsr [d_model][2 d_model], ln1 / ln2 [d_model], w_qkv [(h_q + 2 h_kv) head_dim]
 * [d_model] (query heads, then key heads, then value heads), b_qkv [(h_q + 2 h_kv) head_dim] or
 * NULL, w_o [d_model][h_q head_dim], w_gate_up [2 d_ff][d_model] (the gate rows, then the up
 * rows), w_down [d_model][d_ff]; the matrices and the two norm weights 16-byte aligned.
 */
typedef struct {
    int32_t d_model, h_q, h_kv, head_dim, d_ff;
    float rms_eps, rope_theta;
    const void *w_hsr, *ln1, *w_qkv, *b_qkv, *w_o, *ln2, *w_gate_up, *w_down;
} sd_draft_layer_desc;

/*
 * Workspace of sd_draft_layer (fp32 activations of the rows and the attention's workspace).
 */
SD_API sd_status sd_draft_layer_workspace_size(const sd_draft_layer_desc *w, int32_t n_rows,
                                               const sd_kv_desc *cache, int32_t max_kv_len,
                                               int32_t window, size_t *bytes);

/*
 * One draft layer for n_rows (1..4) rows of one sequence: emb, hid [n_rows][d_model] bf16 in,
 * y [n_rows][d_model] bf16 out.  cache: the draft's own bf16 KV cache of that sequence (batch 1,
 * contiguous or paged, head_dim 64 or 128), whose device kv_len[0] already counts the rows: row r
 * is position kv_len[0] - n_rows + r, and the call WRITES its k and v there.  max_kv_len: host
 * hint >= kv_len[0]; window >= 1.  The fp32 accumulation of every projection is exact to about
 * 1e-6 relative; the rows' q, k and v pass through bf16 (the cache's type), the MLP input too.
 * workspace: sd_draft_layer_workspace_size bytes, 256-byte aligned.
 */
SD_API sd_status sd_draft_layer(const sd_draft_layer_desc *w, const void *emb, const void *hid,
                                int32_t n_rows, const sd_kv_desc *cache, int32_t max_kv_len,
                                int32_t window, void *y, void *workspace, size_t workspace_bytes,
                                int32_t *dev_err, void *stream);

/*
 * Workspace for sd_accept_greedy / sd_accept_sample.  max_gamma: host hint >= gamma[b].
 */
SD_API sd_status sd_accept_workspace_size(int32_t batch, int32_t max_gamma, int32_t vocab,
                                   size_t *bytes);

/*
 * Greedy acceptance [StD "Procedimento de Decodificacao"].  Sequence b has gamma[b] drafted
 * tokens and gamma[b]+1 target rows; rows and tokens are packed over the batch:
 * tgt_logits [sum(gamma+1)][vocab] fp32, draft_tok [sum(gamma)] int32, gamma [batch] int32
 * (all device).  t_i = argmax of target row i (equal values: lowest id; NaN ranks lowest);
 * n = the longest prefix with draft_tok_{i} == t_i; the output row b of out_tok
 * [batch][out_stride] receives d_1..d_n followed by the bonus t_n (n+1 tokens) and
 * n_acc[b] = n.  out_stride >= max_gamma + 1.
 */
SD_API sd_status sd_accept_greedy(const float *tgt_logits, const int32_t *draft_tok,
                           const int32_t *gamma, int32_t batch, int32_t max_gamma, int32_t vocab,
                           int32_t *n_acc, int32_t *out_tok, int32_t out_stride, void *workspace,
                           size_t workspace_bytes, int32_t *dev_err, void *stream);

/*
 * Speculative-sampling acceptance with residual resampling [StD "Principais Contribuicoes":
 * lossless].  p_i = softmax(target row i), q_i = softmax(draft row i) (temperature 1).
 * For i = 1..gamma the drafted d_i is accepted iff u_i <= p_{i-1}(d_i) / q_{i-1}(d_i); at the
 * first rejection (n accepted) a token is drawn from norm(max(0, p_n - q_n)) with v_n (from p_n
 * if that residual is all zero); after gamma acceptances the bonus is drawn from p_gamma with
 * v_gamma.  A draw from weights w with uniform v is the smallest x with
 * sum_{y<=x} w_y > v * sum_y w_y.
 * draft_logits [sum(gamma)][vocab] fp32; u [sum(gamma)] fp32; v [sum(gamma+1)] fp32 (caller
 * supplied uniforms in [0,1), so the kernels hold no RNG state).  Softmax statistics use fp32
 * per element and fp64 for the per-row totals and the accept ratio.  near_boundary (device
 * int32 [batch], may be NULL) receives the number of decisions of that sequence whose
 * |u - ratio| < 1e-6 or whose draw fell within 1e-6*Z of a CDF edge.
 */
SD_API sd_status sd_accept_sample(const float *tgt_logits, const float *draft_logits,
                           const int32_t *draft_tok, const float *u, const float *v,
                           const int32_t *gamma, int32_t batch, int32_t max_gamma, int32_t vocab,
                           int32_t *n_acc, int32_t *out_tok, int32_t out_stride,
                           int32_t *near_boundary, void *workspace, size_t workspace_bytes,
                           int32_t *dev_err, void *stream);

/*
 * Verify attention without any allocation (no counterpart in the papers: it exists for callers
 * that cannot allocate device memory at call time, such as a serving engine whose paged KV pool
 * has taken all free HBM, or a host program that only holds device pointers handed to it by
 * another runtime; cudaMalloc there would fail, shrink the pool, or synchronise the device).
 *
 * Computes exactly what sd_verify_attention computes, with the same arguments minus the
 * workspace: the split-KV partials go to a scratch array of SD_VERIFY_NOALLOC_SCRATCH_BYTES
 * that the library holds in device memory of each device it runs on.  A call whose workspace
 * (sd_attention_workspace_size with SD_ATTN_VERIFY) exceeds that size returns
 * SD_ERR_WORKSPACE and launches nothing.  Nothing in the scratch needs to start at zero.
 *
 * The first call on a device looks up the scratch's address (and may load the module that
 * holds it), so make it before any stream capture.  Calls that may overlap on one device
 * (different streams or host threads without ordering between them) share the scratch and
 * race; calls on one stream are safe.  Errors: as sd_verify_attention; SD_ERR_UNSUPPORTED if
 * the current device ordinal is 64 or more; SD_ERR_CUDA if the address lookup fails.
 */
#define SD_VERIFY_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

SD_API sd_status sd_verify_attention_noalloc(const sd_q_desc *q, const void *q_data,
                                      const sd_kv_desc *kv, int32_t batch, void *out,
                                      int32_t *dev_err, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SD_ATTN_H */
