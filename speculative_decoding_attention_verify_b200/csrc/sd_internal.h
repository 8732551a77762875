// Internal interfaces between the C-ABI layer (sd_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sd_attn.h"
#include "sd_common.cuh"

// Profiling ranges.  Built with -DSD_NVTX (SD_NVTX=1 in the environment of the package's
// build), every compute entry point opens an NVTX range named after itself for the duration
// of the host call (validation, planning and the launches; the GPU work itself is timed by
// the profiler).  NVTX 3 is header-only and does nothing unless a tool is attached.  The
// default build defines the macro away.
#ifdef SD_NVTX
#include <nvtx3/nvToolsExt.h>
namespace sd {
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace sd
#define SD_RANGE(name) ::sd::NvtxRange sd_nvtx_range_(name)
#else
#define SD_RANGE(name) ((void)0)
#endif

namespace sd {

// Parameters of one attention launch (all three kinds).
struct AttnParams {
    int kind;  // sd_attn_kind
    KVView kv;
    int batch;
    int h_q;
    int group;       // h_q / h_kv
    int max_q_rows;  // host hint
    int max_kv_len;  // host hint: upper bound of every kv_len
    int rows_cap;    // batch * max_q_rows: rows addressable in the split workspace
    float scale_log2;  // softmax_scale * log2(e)
    const void *q;
    const int32_t *q_start;
    void *out;
    // text-anchored
    const int32_t *vis_begin;
    const int32_t *vis_end;
    const int32_t *window;
    // sparse
    const int32_t *idx;
    int k_sel;
    const int32_t *tail_begin;
    // sparse, tensor-core path: the selected rows compacted per (sequence, KV head)
    void *ck, *cv;     // [batch][h_kv][k_cap][head_dim] bf16
    int32_t *cpos;     // [batch][h_kv][k_cap] their positions
    int32_t *k_eff;    // [batch][h_kv] kept entries
    int k_cap;
    // split-KV decomposition
    int n_splits;
    int n_rowblocks;
    float *ws_o;   // [n_splits][rows_cap][h_q][head_dim] unnormalised partial outputs
    float *ws_ml;  // [n_splits][rows_cap][h_q][2] (running max in log2 units, sum)
    int32_t *dev_err;
    unsigned long long wait_ns;  // bound of every pipeline wait inside the kernel
    // persistent tensor-core decomposition (0: one CTA per (split, KV head, sequence)): every
    // (sequence, KV head) unit is persist_s items (tile slots, unit-local tiles 0..persist_s-1,
    // those past the unit's own tile count empty), and CTA i of persist_g takes the items
    // [i N / persist_g, (i+1) N / persist_g) of all units in (sequence, KV head) order
    // (N = units * persist_s).  A unit covered by one CTA gets its normalised output directly;
    // otherwise the k-th CTA covering it writes partial slot k, merged by attn_merge_kernel.
    int persist_s;
    int persist_g;
};

// Decomposition of an attention call (host side; depends on host hints only).  Both the
// tensor-core and the CUDA-core decompositions are planned; the workspace fits either, so a
// call can fall back to the CUDA-core engine when the tensor-core path cannot be set up.
struct AttnPlan {
    bool tensor_core;  // tcgen05 path preferred
    int tc_splits;
    int tc_persist_s, tc_persist_g, tc_slots;  // persistent tcgen05 decomposition (0: classic)
    int simt_splits;
    int n_rowblocks;     // CUDA-core path
    int rows_per_block;  // CUDA-core path
    int max_kv_len;
    size_t ws_bytes;
};

int device_sm_count();
unsigned long long wait_limit_ns();  // the process-wide bound set by sd_set_wait_timeout_ns
// Plan of an attention call whose streams hold at most max_stream positions.  When the caller's
// workspace was sized for a longer stream (ws_stream > max_stream: a text-anchored call whose
// workspace query knew only max_kv_len), the split counts are capped at those of the ws_stream
// plan, so that the workspace it reported always suffices (the split model is not monotone in
// the stream length).
// tc_tiles: a bound of one unit's tiles on the tensor-core path (0: derived from the stream).
AttnPlan plan_attention(int kind, int dtype, int head_dim, int h_q, int h_kv, int batch,
                        int max_q_rows, long long max_stream, long long ws_stream = 0,
                        bool paged = false, long long tc_tiles = 0);

cudaError_t launch_attention_simt(const AttnParams &p, const AttnPlan &plan, cudaStream_t s);
cudaError_t launch_attention_tc(const AttnParams &p, const AttnPlan &plan, cudaStream_t s);
cudaError_t launch_sparse_compact(const AttnParams &p, cudaStream_t s);
cudaError_t launch_attention_merge(const AttnParams &p, cudaStream_t s);
bool tc_supported(int kind, int dtype, int head_dim, int rows);
bool tc_persistent_fits(int head_dim, int rows);  // shared memory of a persistent launch
int tc_persistent_max_segments();                 // units one persistent CTA may touch

// Top-K.
struct TopkParams {
    KVView kv;
    int batch;
    int h_q;
    int group;
    const void *q;
    const int32_t *q_start;
    const int32_t *cand_begin;
    const int32_t *cand_end;
    int max_cand;
    int k;
    int32_t *idx_out;
    int n_splits;
    unsigned long long *keys;  // [batch][h_kv][max_cand] order-preserving score keys
    int32_t *dev_err;
    // mean text attention mode: the query rows are the prefill text rows (the last rows of
    // each cache); their log-sum-exps (log2 units of the scaled scores) go to lse
    int max_q_rows;     // host hint of the text rows per sequence
    int max_kv_len;     // host hint: an upper bound of every kv_len
    int rows_cap;       // batch * max_q_rows: rows addressable in lse
    float scale_log2;   // softmax scale * log2(e)
    float *lse;         // [rows_cap][h_q]
    double *scores;     // nullable: [batch][h_kv][max_cand] every candidate's score
    unsigned long long wait_ns;  // bound of every pipeline wait inside the kernels
    // fp32 scoring (last-query mode without scores_out): per (unit, split) the largest error
    // sum of the split's candidates (float bits) and whether any score was not finite
    uint2 *parts;       // [batch][h_kv][part_stride]
    int part_stride;    // >= n_splits
};
size_t topk_workspace_bytes(int batch, int h_kv, int max_cand);
int topk_part_stride(int max_cand);  // the largest split count the scoring may use
int topk_score_ctas_per_sm();  // resident scoring CTAs per SM
cudaError_t launch_topk(const TopkParams &p, cudaStream_t s);
// The selection half of top-K (radix select of p.keys, ascending output).
cudaError_t launch_topk_select(const TopkParams &p, cudaStream_t s);
// Mean text attention scores into p.keys (two passes: row log-sum-exps, then column sums).
cudaError_t launch_text_attention_scores(const TopkParams &p, cudaStream_t s);

// HSR projection.
cudaError_t launch_hsr(const void *emb, const void *hid, int n_rows, int d_model, const void *w,
                       const void *bias, void *y, cudaStream_t s);

// Acceptance.
struct AcceptParams {
    const float *tgt;
    const float *drf;
    const int32_t *draft_tok;
    const float *u;
    const float *v;
    const int32_t *gamma;
    int batch;
    int max_gamma;
    int vocab;
    int32_t *n_acc;
    int32_t *out_tok;
    int out_stride;
    int32_t *near_boundary;
    int n_chunks;   // vocabulary chunks per row (statistics, argmax)
    int n_wchunks;  // vocabulary chunks of a sequence's drawing row (draw weights)
    void *ws;
    int32_t *dev_err;
};
size_t accept_workspace_bytes(int batch, int max_gamma, int vocab, int *n_chunks,
                              int *n_wchunks = nullptr);
cudaError_t launch_accept_greedy(const AcceptParams &p, cudaStream_t s);
cudaError_t launch_accept_sample(const AcceptParams &p, cudaStream_t s);

// Verify attention split into validation/plan and launch, for entry points that supply their
// own workspace (defined with the other entry points).
sd_status verify_plan(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv, int batch,
                      const void *out, AttnPlan *plan);
sd_status verify_run(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv, int batch,
                     void *out, const AttnPlan &plan, void *workspace, int32_t *dev_err,
                     void *stream);

}  // namespace sd
