// C-ABI entry points of libsdattn: host-side validation, decomposition and dispatch.
// Every check here runs before any launch; on failure nothing is launched.
#include <math.h>
#include <atomic>
#include <stdint.h>
#include <string.h>

#include "sd_internal.h"

namespace sd {

namespace {
std::atomic<unsigned long long> g_wait_ns{1000000000ull};
}  // namespace

unsigned long long wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // clear the sticky-free error of a failed query
        return 148;
    }
    return n;
}

AttnPlan plan_attention(int kind, int dtype, int head_dim, int h_q, int h_kv, int batch,
                        int max_q_rows, long long max_stream, long long ws_stream, bool paged,
                        long long tc_tiles) {
    AttnPlan plan{};
    const int G = h_q / h_kv;
    const int rows = G * max_q_rows;
    const int sms = device_sm_count();
    const size_t rows_cap = (size_t)batch * max_q_rows;
    if (max_stream < 1) max_stream = 1;
    plan.max_kv_len = (int)(max_stream < (1LL << 30) ? max_stream : (1LL << 30));
    plan.tensor_core = tc_supported(kind, dtype, head_dim, rows);
    // CUDA-core decomposition: 64-position tiles, a 3-stage K/V ring of 3*2*64 rows in
    // shared memory; two CTAs fit per SM when the ring is at most 96 KB.  Modelled time of
    // split count s: waves x (per-CTA set-up and merge share, about two tiles' worth, + tiles
    // per CTA), with at least two tiles per CTA; the smallest wins.
    plan.rows_per_block = rows <= 8 ? 8 : 16;
    plan.n_rowblocks = (rows + plan.rows_per_block - 1) / plan.rows_per_block;
    {
        const int esz = dtype == SD_BF16 ? 2 : 4;
        const long long ring = 3LL * 2 * 64 * head_dim * esz;
        const long long slots = (long long)sms * (ring <= 96 * 1024 ? 2 : 1);
        const long long units = (long long)batch * h_kv * plan.n_rowblocks;
        const long long tiles = (max_stream + 63) / 64;
        long long best = -1;
        plan.simt_splits = 1;
        for (long long s = 1; s <= 256; ++s) {
            if (s > 1 && tiles / s < 2) break;
            const long long ctas = units * s;
            const long long waves = (ctas + slots - 1) / slots;
            const long long t = waves * (2 + (tiles + s - 1) / s);
            if (best < 0 || t < best) {
                best = t;
                plan.simt_splits = (int)s;
            }
        }
    }
    // Tensor-core decompositions, one CTA per SM; the tile count of a unit is bounded by
    // tc_tiles (verify: the stream's tiles; text-anchored: its two runs may each add a tile,
    // and with pages two more; sparse: given by the caller).  Classic, modelled time of split
    // count s: waves x (per-CTA start-up and drain, about three tiles' worth, + tiles per CTA),
    // the smallest wins.  Persistent: every unit's tiles in one list spread evenly over the
    // SMs, about (all tiles / SMs) + three tiles' worth of start-up and drain + two for the
    // split merge + three per switch to another unit inside a CTA (its Q, the epilogue);
    // taken when it models faster.
    plan.tc_splits = 1;
    plan.tc_persist_s = plan.tc_persist_g = plan.tc_slots = 0;
    if (plan.tensor_core) {
        if (tc_tiles < 1)
            tc_tiles = (max_stream + 127) / 128 +
                       (kind == SD_ATTN_TEXT_ANCHORED ? 1 + (paged ? 2 : 0) : 0);
        const long long units = (long long)batch * h_kv;
        const long long tiles = tc_tiles;
        long long best = -1;
        for (long long s = 1; s <= 64; ++s) {
            if (s > 1 && tiles / s < 2) break;
            const long long ctas = units * s;
            const long long waves = (ctas + sms - 1) / sms;
            const long long t = waves * (3 + (tiles + s - 1) / s);
            if (best < 0 || t < best) {
                best = t;
                plan.tc_splits = (int)s;
            }
        }
        const long long n_items = units * tiles;
        if (tiles >= 2 && n_items <= (1LL << 40) && tc_persistent_fits(head_dim, rows)) {
            const long long g = n_items < sms ? n_items : sms;
            const long long q = n_items / g;  // items per CTA, at least
            const long long per_cta = (n_items + g - 1) / g;
            const long long switches = (per_cta + tiles - 1) / tiles;  // (upper estimate)
            const long long t = per_cta + 3 + 2 + 3 * switches;
            // units a CTA's range may touch: its items span at most ceil(per_cta / tiles) + 1
            const bool segs_ok = (per_cta + tiles - 1) / tiles + 1 <= tc_persistent_max_segments();
            if (t < best && segs_ok) {
                plan.tc_persist_s = (int)tiles;
                plan.tc_persist_g = (int)g;
                // CTAs whose item range meets one unit's: a range of at least q items, so at
                // most ceil((tiles - 1) / q) + 1 of them (one spare)
                plan.tc_slots = (int)((tiles - 1 + q - 1) / q + 2);
            }
        }
    }
    if (ws_stream > max_stream) {
        const AttnPlan w = plan_attention(kind, dtype, head_dim, h_q, h_kv, batch, max_q_rows,
                                          ws_stream, 0, paged, 0);
        int cap = w.simt_splits > w.tc_splits ? w.simt_splits : w.tc_splits;
        if (w.tc_slots > cap) cap = w.tc_slots;
        if (plan.simt_splits > cap) plan.simt_splits = cap;
        if (plan.tc_splits > cap) plan.tc_splits = cap;
        if (plan.tc_slots > cap) plan.tc_persist_s = plan.tc_persist_g = plan.tc_slots = 0;
    }
    int splits = plan.simt_splits > plan.tc_splits ? plan.simt_splits : plan.tc_splits;
    if (plan.tc_slots > splits) splits = plan.tc_slots;
    plan.ws_bytes = splits > 1 ? (size_t)splits * rows_cap * h_q * (head_dim + 2) * sizeof(float)
                               : 0;
    return plan;
}

}  // namespace sd

using namespace sd;

namespace {

bool kv_desc_ok(const sd_kv_desc *kv, int batch) {
    if (!kv || batch < 1) return false;
    if (kv->dtype != SD_F32 && kv->dtype != SD_BF16) return false;
    if (kv->h_kv < 1 || !kv->k || !kv->v || !kv->kv_len) return false;
    const int esz = kv->dtype == SD_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(kv->k) | reinterpret_cast<uintptr_t>(kv->v)) & 15) return false;
    if (kv->page_size == 0) {
        if (kv->stride_pos != kv->head_dim) return false;
        if (kv->stride_h < 0 || kv->stride_b < 0) return false;
        if (((kv->stride_h * esz) & 15) || ((kv->stride_b * esz) & 15)) return false;
    } else {
        if (kv->page_size != kPageSize) return false;
        if (!kv->block_table || kv->max_pages_per_seq < 1 || kv->num_pages < 1) return false;
    }
    return true;
}

bool head_dim_supported(int d) { return d == 64 || d == 128; }

KVView make_view(const sd_kv_desc *kv) {
    KVView v;
    v.dtype = kv->dtype;
    v.h_kv = kv->h_kv;
    v.head_dim = kv->head_dim;
    v.page_size = kv->page_size;
    v.k = kv->k;
    v.v = kv->v;
    v.stride_b = kv->stride_b;
    v.stride_h = kv->stride_h;
    v.stride_pos = kv->stride_pos;
    v.block_table = kv->block_table;
    v.max_pages = kv->max_pages_per_seq;
    v.num_pages = kv->num_pages;
    v.kv_len = kv->kv_len;
    return v;
}

sd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SD_OK : SD_ERR_CUDA; }

// Common validation of the attention calls; fills the plan for the kind.
sd_status check_attention(sd_attn_kind kind, const sd_q_desc *q, const sd_kv_desc *kv, int batch,
                          long long max_stream, AttnPlan *plan, long long ws_stream = 0,
                          long long tc_tiles = 0) {
    if (!q || !kv || batch < 1 || batch > 65535) return SD_ERR_INVALID_ARG;
    if (!kv_desc_ok(kv, batch)) return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    if (q->h_q < 1 || q->h_q % kv->h_kv != 0 || q->max_q_rows < 1 || q->max_kv_len < 1 ||
        !q->q_start || !(q->softmax_scale >= 0.f) || isinf(q->softmax_scale))
        return SD_ERR_INVALID_ARG;
    if ((long long)batch * q->max_q_rows > (1LL << 30)) return SD_ERR_INVALID_ARG;
    *plan = plan_attention(kind, kv->dtype, kv->head_dim, q->h_q, kv->h_kv, batch, q->max_q_rows,
                           max_stream, ws_stream, kv->page_size != 0, tc_tiles);
    return SD_OK;
}

AttnParams base_params(sd_attn_kind kind, const sd_q_desc *q, const void *q_data,
                       const sd_kv_desc *kv, int batch, void *out, const AttnPlan &plan,
                       void *ws, int32_t *dev_err) {
    AttnParams p{};
    p.kind = kind;
    p.kv = make_view(kv);
    p.batch = batch;
    p.h_q = q->h_q;
    p.group = q->h_q / kv->h_kv;
    p.max_q_rows = q->max_q_rows;
    p.max_kv_len = q->max_kv_len;
    p.rows_cap = batch * q->max_q_rows;
    const float scale = q->softmax_scale > 0.f ? q->softmax_scale
                                               : (float)(1.0 / sqrt((double)kv->head_dim));
    p.scale_log2 = scale * kLog2e;
    p.q = q_data;
    p.q_start = q->q_start;
    p.out = out;
    p.n_rowblocks = plan.n_rowblocks;
    p.ws_o = reinterpret_cast<float *>(ws);
    p.dev_err = dev_err;
    p.wait_ns = wait_limit_ns();
    return p;
}

// Tiles of one unit of a sparse call on the tensor-core path: the compacted selection, then
// the tail (which, from a page boundary, may start up to 15 positions lower).
long long sparse_tc_tiles(const sd_kv_desc *kv, long long k, long long max_tail) {
    return (k + 127) / 128 + (max_tail + (kv->page_size != 0 ? 15 : 0) + 127) / 128;
}

void set_splits(AttnParams &p, int n_splits) {
    p.n_splits = n_splits;
    p.ws_ml = n_splits > 1 ? p.ws_o + (size_t)n_splits * p.rows_cap * p.h_q * p.kv.head_dim
                           : nullptr;
}

// The plan's tensor-core decomposition: persistent (n_splits = the partial slots) or classic.
void set_tc_decomposition(AttnParams &p, const AttnPlan &plan) {
    p.persist_s = plan.tc_persist_s;
    p.persist_g = plan.tc_persist_g;
    set_splits(p, plan.tc_persist_s ? plan.tc_slots : plan.tc_splits);
}

sd_status run_attention(AttnParams p, const AttnPlan &plan, void *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaErrorNotSupported;
    const bool aligned = ((reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.out)) &
                          15) == 0;
    if (plan.tensor_core && aligned) {
        set_tc_decomposition(p, plan);
        e = launch_attention_tc(p, plan, s);
        if (e != cudaSuccess && e != cudaErrorNotSupported) return SD_ERR_CUDA;
    }
    if (e == cudaErrorNotSupported) {
        p.persist_s = p.persist_g = 0;
        set_splits(p, plan.simt_splits);
        e = launch_attention_simt(p, plan, s);
    }
    if (e != cudaSuccess) return SD_ERR_CUDA;
    if (p.n_splits > 1) e = launch_attention_merge(p, s);
    return cuda_status(e);
}

// A staged sparse selection: K, V [batch][h_kv][k_cap][d] bf16, positions [batch][h_kv][k_cap]
// and per-unit counts, from offset `base`; each region 256-byte aligned.
struct SelLayout {
    size_t ck, cv, cpos, k_eff, end;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

SelLayout sel_layout(size_t base, const sd_kv_desc *kv, int batch, int k) {
    SelLayout l{};
    const size_t units = (size_t)batch * kv->h_kv, kc = (size_t)(k > 0 ? k : 1);
    l.ck = up256(base);
    l.cv = l.ck + up256(units * kc * kv->head_dim * 2);
    l.cpos = l.cv + up256(units * kc * kv->head_dim * 2);
    l.k_eff = l.cpos + up256(units * kc * 4);
    l.end = l.k_eff + up256(units * 4);
    return l;
}

void set_selection(AttnParams &p, void *base, const SelLayout &l, int k) {
    char *w = static_cast<char *>(base);
    p.ck = w + l.ck;
    p.cv = w + l.cv;
    p.cpos = reinterpret_cast<int32_t *>(w + l.cpos);
    p.k_eff = reinterpret_cast<int32_t *>(w + l.k_eff);
    p.k_cap = k > 0 ? k : 1;
}

// Workspace bytes of sd_sparse_attention: the split partials, plus a staged selection when
// the tensor-core path is planned.
size_t sparse_ws_bytes(const AttnPlan &plan, const sd_kv_desc *kv, int batch, int k) {
    return plan.tensor_core ? sel_layout(plan.ws_bytes, kv, batch, k).end : plan.ws_bytes;
}

// Workspace of the mean text attention mode: the score keys, then one log-sum-exp per
// (text row, query head), each region 256-byte aligned.
struct TaLayout {
    size_t keys, lse, end;
};

TaLayout text_attention_ws(int batch, int h_kv, int max_cand, int h_q, int max_q_rows) {
    TaLayout l{};
    l.keys = 0;
    l.lse = up256(topk_workspace_bytes(batch, h_kv, max_cand));
    l.end = l.lse + up256((size_t)batch * max_q_rows * h_q * sizeof(float));
    return l;
}

long long stream_hint(sd_attn_kind kind, const sd_q_desc *q, long long extra) {
    if (kind == SD_ATTN_TEXT_ANCHORED) {
        const long long w = extra + q->max_q_rows - 1;
        return w < q->max_kv_len ? w : q->max_kv_len;
    }
    if (kind == SD_ATTN_SPARSE) {
        const long long w = extra;
        return w < q->max_kv_len ? w : q->max_kv_len;
    }
    return q->max_kv_len;
}

}  // namespace

namespace sd {

// Validation and plan of a verify call, for entry points that supply their own workspace.
sd_status verify_plan(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv, int batch,
                      const void *out, AttnPlan *plan) {
    if (!q_data || !out) return SD_ERR_INVALID_ARG;
    return check_attention(SD_ATTN_VERIFY, q, kv, batch, q ? q->max_kv_len : 0, plan);
}

// Launch of a verify call planned by verify_plan, on a workspace of at least plan.ws_bytes.
sd_status verify_run(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv, int batch,
                     void *out, const AttnPlan &plan, void *workspace, int32_t *dev_err,
                     void *stream) {
    AttnParams p = base_params(SD_ATTN_VERIFY, q, q_data, kv, batch, out, plan, workspace, dev_err);
    return run_attention(p, plan, stream);
}

}  // namespace sd

extern "C" {

const char *sd_status_string(sd_status s) {
    switch (s) {
        case SD_OK: return "SD_OK";
        case SD_ERR_INVALID_ARG: return "SD_ERR_INVALID_ARG: invalid argument";
        case SD_ERR_UNSUPPORTED: return "SD_ERR_UNSUPPORTED: unsupported configuration";
        case SD_ERR_WORKSPACE: return "SD_ERR_WORKSPACE: workspace missing or too small";
        case SD_ERR_CUDA: return "SD_ERR_CUDA: CUDA launch or runtime error";
    }
    return "unknown sd_status";
}

int32_t sd_version(void) { return 200; }

uint64_t sd_set_wait_timeout_ns(uint64_t ns) {
    return g_wait_ns.exchange(ns == 0 ? 1000000000ull : ns, std::memory_order_relaxed);
}

sd_status sd_attention_workspace_size(sd_attn_kind kind, const sd_q_desc *q,
                                      const sd_kv_desc *kv, int32_t batch, size_t *bytes) {
    if (!bytes || !q || !kv) return SD_ERR_INVALID_ARG;
    // (sparse calls also stage the selected rows: see sd_sparse_workspace_size)
    if (kind != SD_ATTN_VERIFY && kind != SD_ATTN_TEXT_ANCHORED) return SD_ERR_INVALID_ARG;
    if (kv->h_kv < 1 || q->h_q < 1 || q->h_q % kv->h_kv || batch < 1 || q->max_q_rows < 1)
        return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    // Worst-case stream for the kind (hints of the specific call are not known here).
    const AttnPlan plan = plan_attention(kind, kv->dtype, kv->head_dim, q->h_q, kv->h_kv, batch,
                                         q->max_q_rows, q->max_kv_len, 0, kv->page_size != 0, 0);
    *bytes = plan.ws_bytes;
    return SD_OK;
}

sd_status sd_attention_plan(sd_attn_kind kind, const sd_q_desc *q, const sd_kv_desc *kv,
                            int32_t batch, int32_t extent, int32_t max_tail, int32_t *engine,
                            int32_t *parts) {
    if (!engine || !parts || !q || !kv) return SD_ERR_INVALID_ARG;
    if (kind != SD_ATTN_VERIFY && kind != SD_ATTN_TEXT_ANCHORED && kind != SD_ATTN_SPARSE)
        return SD_ERR_INVALID_ARG;
    if (kv->h_kv < 1 || q->h_q < 1 || q->h_q % kv->h_kv || batch < 1 || q->max_q_rows < 1 ||
        q->max_kv_len < 1 || extent < 0 || max_tail < 0 || extent > (1 << 30))
        return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    const bool paged = kv->page_size != 0;
    AttnPlan plan;
    if (kind == SD_ATTN_VERIFY) {
        plan = plan_attention(kind, kv->dtype, kv->head_dim, q->h_q, kv->h_kv, batch,
                              q->max_q_rows, q->max_kv_len, 0, paged, 0);
    } else if (kind == SD_ATTN_TEXT_ANCHORED) {
        if (extent < 1) return SD_ERR_INVALID_ARG;
        plan = plan_attention(kind, kv->dtype, kv->head_dim, q->h_q, kv->h_kv, batch,
                              q->max_q_rows, stream_hint(kind, q, extent), q->max_kv_len, paged,
                              0);
    } else {
        if (extent > (1 << 16)) return SD_ERR_INVALID_ARG;
        plan = plan_attention(kind, kv->dtype, kv->head_dim, q->h_q, kv->h_kv, batch,
                              q->max_q_rows, stream_hint(kind, q, (long long)extent + max_tail),
                              0, paged, sparse_tc_tiles(kv, extent, max_tail));
    }
    if (!plan.tensor_core) {
        *engine = SD_ENGINE_CUDA_CORE;
        *parts = plan.simt_splits;
    } else if (plan.tc_persist_s) {
        *engine = SD_ENGINE_TC_PERSISTENT;
        *parts = plan.tc_slots;
    } else {
        *engine = SD_ENGINE_TC;
        *parts = plan.tc_splits;
    }
    return SD_OK;
}

sd_status sd_verify_attention(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv,
                              int32_t batch, void *out, void *workspace, size_t workspace_bytes,
                              int32_t *dev_err, void *stream) {
    SD_RANGE("sd_verify_attention");
    AttnPlan plan;
    if (!q_data || !out) return SD_ERR_INVALID_ARG;
    sd_status st = check_attention(SD_ATTN_VERIFY, q, kv, batch, q ? q->max_kv_len : 0, &plan);
    if (st != SD_OK) return st;
    if (plan.ws_bytes > workspace_bytes || (plan.ws_bytes && !workspace)) return SD_ERR_WORKSPACE;
    AttnParams p = base_params(SD_ATTN_VERIFY, q, q_data, kv, batch, out, plan, workspace, dev_err);
    return run_attention(p, plan, stream);
}

sd_status sd_text_anchored_attention(const sd_q_desc *q, const void *q_data,
                                     const sd_kv_desc *kv, int32_t batch,
                                     const int32_t *vis_begin, const int32_t *vis_end,
                                     const int32_t *window, int32_t max_window, void *out,
                                     void *workspace, size_t workspace_bytes, int32_t *dev_err,
                                     void *stream) {
    SD_RANGE("sd_text_anchored_attention");
    if (!q_data || !out || !vis_begin || !vis_end || !window || max_window < 1)
        return SD_ERR_INVALID_ARG;
    AttnPlan plan;
    if (!q) return SD_ERR_INVALID_ARG;
    // (the workspace query sized the plan of a max_kv_len stream)
    sd_status st = check_attention(SD_ATTN_TEXT_ANCHORED, q, kv, batch,
                                   stream_hint(SD_ATTN_TEXT_ANCHORED, q, max_window), &plan,
                                   q->max_kv_len);
    if (st != SD_OK) return st;
    if (plan.ws_bytes > workspace_bytes || (plan.ws_bytes && !workspace)) return SD_ERR_WORKSPACE;
    AttnParams p = base_params(SD_ATTN_TEXT_ANCHORED, q, q_data, kv, batch, out, plan, workspace,
                               dev_err);
    p.vis_begin = vis_begin;
    p.vis_end = vis_end;
    p.window = window;
    return run_attention(p, plan, stream);
}

sd_status sd_sparse_workspace_size(const sd_q_desc *q, const sd_kv_desc *kv, int32_t batch,
                                   int32_t k, int32_t max_tail, size_t *bytes) {
    if (!bytes || !q || !kv || k < 0 || k > (1 << 16) || max_tail < 0) return SD_ERR_INVALID_ARG;
    if (kv->h_kv < 1 || q->h_q < 1 || q->h_q % kv->h_kv || batch < 1 || q->max_q_rows < 1 ||
        q->max_kv_len < 1)
        return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    const AttnPlan plan = plan_attention(SD_ATTN_SPARSE, kv->dtype, kv->head_dim, q->h_q,
                                         kv->h_kv, batch, q->max_q_rows,
                                         stream_hint(SD_ATTN_SPARSE, q, (long long)k + max_tail),
                                         0, kv->page_size != 0, sparse_tc_tiles(kv, k, max_tail));
    *bytes = sparse_ws_bytes(plan, kv, batch, k);
    return SD_OK;
}

sd_status sd_sparse_attention(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv,
                              int32_t batch, const int32_t *idx, int32_t k,
                              const int32_t *tail_begin, int32_t max_tail, void *out,
                              void *workspace, size_t workspace_bytes, int32_t *dev_err,
                              void *stream) {
    SD_RANGE("sd_sparse_attention");
    if (!q_data || !out || !tail_begin || k < 0 || (k > 0 && !idx) || max_tail < 0 ||
        k > (1 << 16))
        return SD_ERR_INVALID_ARG;
    AttnPlan plan;
    if (!q) return SD_ERR_INVALID_ARG;
    sd_status st = check_attention(SD_ATTN_SPARSE, q, kv, batch,
                                   stream_hint(SD_ATTN_SPARSE, q, (long long)k + max_tail), &plan,
                                   0, sparse_tc_tiles(kv, k, max_tail));
    if (st != SD_OK) return st;
    const size_t need = sparse_ws_bytes(plan, kv, batch, k);
    if (need > workspace_bytes || (need && !workspace)) return SD_ERR_WORKSPACE;
    AttnParams p = base_params(SD_ATTN_SPARSE, q, q_data, kv, batch, out, plan, workspace, dev_err);
    p.idx = idx;
    p.k_sel = k;
    p.tail_begin = tail_begin;
    const bool aligned = ((reinterpret_cast<uintptr_t>(q_data) | reinterpret_cast<uintptr_t>(out)) &
                          15) == 0;
    if (plan.tensor_core && aligned) {
        // tensor-core path: stage the selected rows, then stream [selection ; tail]
        set_selection(p, workspace, sel_layout(plan.ws_bytes, kv, batch, k), k);
        const cudaError_t e = launch_sparse_compact(p, reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return SD_ERR_CUDA;
    } else {
        plan.tensor_core = false;
    }
    return run_attention(p, plan, stream);
}

sd_status sd_sparse_selection_size(const sd_kv_desc *kv, int32_t batch, int32_t k,
                                   size_t *bytes) {
    if (!bytes || !kv || batch < 1 || k < 0 || k > (1 << 16) || kv->h_kv < 1)
        return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    *bytes = sel_layout(0, kv, batch, k).end;
    return SD_OK;
}

sd_status sd_sparse_stage(const sd_kv_desc *kv, int32_t batch, const int32_t *idx, int32_t k,
                          const int32_t *tail_begin, void *selection, size_t selection_bytes,
                          int32_t *dev_err, void *stream) {
    SD_RANGE("sd_sparse_stage");
    if (!tail_begin || k < 0 || (k > 0 && !idx) || k > (1 << 16) || batch < 1 || batch > 65535)
        return SD_ERR_INVALID_ARG;
    if (!kv_desc_ok(kv, batch)) return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    if (kv->dtype != SD_BF16) return SD_ERR_UNSUPPORTED;
    const SelLayout l = sel_layout(0, kv, batch, k);
    if (!selection || l.end > selection_bytes || (reinterpret_cast<uintptr_t>(selection) & 255))
        return SD_ERR_WORKSPACE;
    AttnParams p{};
    p.kind = SD_ATTN_SPARSE;
    p.kv = make_view(kv);
    p.batch = batch;
    p.idx = idx;
    p.k_sel = k;
    p.tail_begin = tail_begin;
    p.dev_err = dev_err;
    set_selection(p, selection, l, k);
    return cuda_status(launch_sparse_compact(p, reinterpret_cast<cudaStream_t>(stream)));
}

sd_status sd_sparse_attention_staged(const sd_q_desc *q, const void *q_data,
                                     const sd_kv_desc *kv, int32_t batch, const void *selection,
                                     int32_t k, const int32_t *tail_begin, int32_t max_tail,
                                     void *out, void *workspace, size_t workspace_bytes,
                                     int32_t *dev_err, void *stream) {
    SD_RANGE("sd_sparse_attention_staged");
    if (!q || !q_data || !out || !tail_begin || !selection || k < 0 || max_tail < 0 ||
        k > (1 << 16))
        return SD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(selection) & 255) ||
        ((reinterpret_cast<uintptr_t>(q_data) | reinterpret_cast<uintptr_t>(out)) & 15))
        return SD_ERR_INVALID_ARG;
    AttnPlan plan;
    sd_status st = check_attention(SD_ATTN_SPARSE, q, kv, batch,
                                   stream_hint(SD_ATTN_SPARSE, q, (long long)k + max_tail), &plan,
                                   0, sparse_tc_tiles(kv, k, max_tail));
    if (st != SD_OK) return st;
    if (!plan.tensor_core) return SD_ERR_UNSUPPORTED;  // bf16, head_dim 64/128, <= 128 rows
    if (plan.ws_bytes > workspace_bytes || (plan.ws_bytes && !workspace)) return SD_ERR_WORKSPACE;
    AttnParams p = base_params(SD_ATTN_SPARSE, q, q_data, kv, batch, out, plan, workspace, dev_err);
    p.k_sel = k;
    p.tail_begin = tail_begin;
    set_selection(p, const_cast<void *>(selection), sel_layout(0, kv, batch, k), k);
    set_tc_decomposition(p, plan);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_attention_tc(p, plan, s);
    if (e == cudaErrorNotSupported) return SD_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return SD_ERR_CUDA;
    if (p.n_splits > 1) e = launch_attention_merge(p, s);
    return cuda_status(e);
}

sd_status sd_topk_workspace_size(const sd_kv_desc *kv, int32_t batch, int32_t max_cand,
                                 int32_t k, size_t *bytes) {
    if (!kv || !bytes || batch < 1 || max_cand < 0 || k < 1 || kv->h_kv < 1)
        return SD_ERR_INVALID_ARG;
    *bytes = topk_workspace_bytes(batch, kv->h_kv, max_cand);
    return SD_OK;
}

sd_status sd_topk_select(const sd_q_desc *q, const void *q_data, const sd_kv_desc *kv,
                         int32_t batch, const int32_t *cand_begin, const int32_t *cand_end,
                         int32_t max_cand, int32_t k, int32_t *idx_out, void *workspace,
                         size_t workspace_bytes, int32_t *dev_err, void *stream) {
    SD_RANGE("sd_topk_select");
    return sd_topk_select_scored(SD_TOPK_LAST_QUERY, q, q_data, kv, batch, cand_begin, cand_end,
                                 max_cand, k, idx_out, nullptr, workspace, workspace_bytes,
                                 dev_err, stream);
}

sd_status sd_topk_scored_workspace_size(sd_topk_score mode, const sd_q_desc *q,
                                        const sd_kv_desc *kv, int32_t batch, int32_t max_cand,
                                        int32_t k, size_t *bytes) {
    if (!kv || !bytes || batch < 1 || max_cand < 0 || k < 1 || kv->h_kv < 1)
        return SD_ERR_INVALID_ARG;
    if (mode == SD_TOPK_LAST_QUERY) {
        *bytes = topk_workspace_bytes(batch, kv->h_kv, max_cand);
        return SD_OK;
    }
    if (mode != SD_TOPK_MEAN_TEXT_ATTENTION || !q || q->h_q < 1 || q->max_q_rows < 1)
        return SD_ERR_INVALID_ARG;
    *bytes = text_attention_ws(batch, kv->h_kv, max_cand, q->h_q, q->max_q_rows).end;
    return SD_OK;
}

sd_status sd_topk_select_scored(sd_topk_score mode, const sd_q_desc *q, const void *q_data,
                                const sd_kv_desc *kv, int32_t batch, const int32_t *cand_begin,
                                const int32_t *cand_end, int32_t max_cand, int32_t k,
                                int32_t *idx_out, double *scores_out, void *workspace,
                                size_t workspace_bytes, int32_t *dev_err, void *stream) {
    SD_RANGE("sd_topk_select_scored");
    if (mode != SD_TOPK_LAST_QUERY && mode != SD_TOPK_MEAN_TEXT_ATTENTION)
        return SD_ERR_INVALID_ARG;
    if (!q || !q_data || !cand_begin || !cand_end || !idx_out || k < 1 || max_cand < 0 ||
        batch > 65535)
        return SD_ERR_INVALID_ARG;
    if (!kv_desc_ok(kv, batch)) return SD_ERR_INVALID_ARG;
    if (!head_dim_supported(kv->head_dim)) return SD_ERR_UNSUPPORTED;
    if (q->h_q < 1 || q->h_q % kv->h_kv != 0 || !q->q_start) return SD_ERR_INVALID_ARG;
    TopkParams p{};
    p.kv = make_view(kv);
    p.batch = batch;
    p.h_q = q->h_q;
    p.group = q->h_q / kv->h_kv;
    p.q = q_data;
    p.q_start = q->q_start;
    p.cand_begin = cand_begin;
    p.cand_end = cand_end;
    p.max_cand = max_cand;
    p.k = k;
    p.idx_out = idx_out;
    p.keys = reinterpret_cast<unsigned long long *>(workspace);
    p.scores = scores_out;
    p.dev_err = dev_err;
    p.wait_ns = wait_limit_ns();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (mode == SD_TOPK_MEAN_TEXT_ATTENTION) {
        if (q->max_q_rows < 1 || q->max_kv_len < 1 || !(q->softmax_scale >= 0.f) ||
            isinf(q->softmax_scale) || (long long)batch * q->max_q_rows > (1LL << 30))
            return SD_ERR_INVALID_ARG;
        const TaLayout l = text_attention_ws(batch, kv->h_kv, max_cand, q->h_q, q->max_q_rows);
        if (l.end > workspace_bytes || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
            return SD_ERR_WORKSPACE;
        p.max_q_rows = q->max_q_rows;
        p.max_kv_len = q->max_kv_len;
        p.rows_cap = batch * q->max_q_rows;
        const float scale = q->softmax_scale > 0.f ? q->softmax_scale
                                                   : (float)(1.0 / sqrt((double)kv->head_dim));
        p.scale_log2 = scale * kLog2e;
        p.lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + l.lse);
        return cuda_status(launch_text_attention_scores(p, s));
    }
    const size_t need = topk_workspace_bytes(batch, kv->h_kv, max_cand);
    if (need > workspace_bytes || (need && !workspace)) return SD_ERR_WORKSPACE;
    // Scoring CTAs stream 128-candidate spans through a shared-memory ring; choose the split
    // count whose CTAs fill whole waves best, with at least four spans per CTA.
    const int sms = device_sm_count();
    const long long units = (long long)batch * kv->h_kv;
    const long long slots = (long long)sms * topk_score_ctas_per_sm();
    const long long tiles = ((long long)max_cand + 127) / 128;
    double best = -1.0;
    p.n_splits = 1;
    const int max_splits = topk_part_stride(max_cand);
    for (long long sp = 1; sp <= max_splits; ++sp) {
        if (sp > 1 && tiles / sp < 4) break;
        const long long ctas = units * sp;
        const long long waves = (ctas + slots - 1) / slots;
        const double score = (double)ctas / (double)(waves * slots) - 0.005 * (double)sp;
        if (score > best) {
            best = score;
            p.n_splits = (int)sp;
        }
    }
    // the scoring's per-split partials follow the keys
    p.part_stride = max_splits;
    p.parts = reinterpret_cast<uint2 *>(static_cast<char *>(workspace) +
                                        (size_t)units * max_cand * sizeof(unsigned long long));
    return cuda_status(launch_topk(p, s));
}

sd_status sd_hsr_project(const void *emb, const void *hid, int32_t n_rows, int32_t d_model,
                         const void *weight, const void *bias, void *y, void *stream) {
    SD_RANGE("sd_hsr_project");
    if (!emb || !hid || !weight || !y || n_rows < 1 || n_rows > 16 || d_model < 16 ||
        d_model % 16 != 0 || d_model > (1 << 20))
        return SD_ERR_INVALID_ARG;
    const uintptr_t a = reinterpret_cast<uintptr_t>(emb) | reinterpret_cast<uintptr_t>(hid) |
                        reinterpret_cast<uintptr_t>(weight);
    if (a & 15) return SD_ERR_INVALID_ARG;
    if ((size_t)4 * 2 * d_model * 2 > 200 * 1024) return SD_ERR_UNSUPPORTED;
    return cuda_status(launch_hsr(emb, hid, n_rows, d_model, weight, bias, y,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

sd_status sd_accept_workspace_size(int32_t batch, int32_t max_gamma, int32_t vocab,
                                   size_t *bytes) {
    if (!bytes || batch < 1 || max_gamma < 0 || vocab < 1) return SD_ERR_INVALID_ARG;
    *bytes = accept_workspace_bytes(batch, max_gamma, vocab, nullptr);
    return SD_OK;
}

static sd_status accept_common(const float *tgt, const int32_t *draft_tok, const int32_t *gamma,
                               int32_t batch, int32_t max_gamma, int32_t vocab, int32_t *n_acc,
                               int32_t *out_tok, int32_t out_stride, void *workspace,
                               size_t workspace_bytes, AcceptParams *p) {
    if (!tgt || !gamma || !n_acc || !out_tok || batch < 1 || batch > 65535 || max_gamma < 0 ||
        vocab < 1 || out_stride < max_gamma + 1 || (max_gamma > 0 && !draft_tok))
        return SD_ERR_INVALID_ARG;
    if ((long long)batch * (2 * max_gamma + 1) > 65535) return SD_ERR_UNSUPPORTED;
    int n_chunks = 1, n_wchunks = 1;
    const size_t need = accept_workspace_bytes(batch, max_gamma, vocab, &n_chunks, &n_wchunks);
    if (need > workspace_bytes || !workspace) return SD_ERR_WORKSPACE;
    *p = AcceptParams{};
    p->tgt = tgt;
    p->draft_tok = draft_tok;
    p->gamma = gamma;
    p->batch = batch;
    p->max_gamma = max_gamma;
    p->vocab = vocab;
    p->n_acc = n_acc;
    p->out_tok = out_tok;
    p->out_stride = out_stride;
    p->n_chunks = n_chunks;
    p->n_wchunks = n_wchunks;
    p->ws = workspace;
    return SD_OK;
}

sd_status sd_accept_greedy(const float *tgt_logits, const int32_t *draft_tok,
                           const int32_t *gamma, int32_t batch, int32_t max_gamma, int32_t vocab,
                           int32_t *n_acc, int32_t *out_tok, int32_t out_stride, void *workspace,
                           size_t workspace_bytes, int32_t *dev_err, void *stream) {
    SD_RANGE("sd_accept_greedy");
    AcceptParams p;
    sd_status st = accept_common(tgt_logits, draft_tok, gamma, batch, max_gamma, vocab, n_acc,
                                 out_tok, out_stride, workspace, workspace_bytes, &p);
    if (st != SD_OK) return st;
    p.dev_err = dev_err;
    return cuda_status(launch_accept_greedy(p, reinterpret_cast<cudaStream_t>(stream)));
}

sd_status sd_accept_sample(const float *tgt_logits, const float *draft_logits,
                           const int32_t *draft_tok, const float *u, const float *v,
                           const int32_t *gamma, int32_t batch, int32_t max_gamma, int32_t vocab,
                           int32_t *n_acc, int32_t *out_tok, int32_t out_stride,
                           int32_t *near_boundary, void *workspace, size_t workspace_bytes,
                           int32_t *dev_err, void *stream) {
    SD_RANGE("sd_accept_sample");
    if (!v || (max_gamma > 0 && (!draft_logits || !u))) return SD_ERR_INVALID_ARG;
    AcceptParams p;
    sd_status st = accept_common(tgt_logits, draft_tok, gamma, batch, max_gamma, vocab, n_acc,
                                 out_tok, out_stride, workspace, workspace_bytes, &p);
    if (st != SD_OK) return st;
    p.drf = draft_logits;
    p.u = u;
    p.v = v;
    p.near_boundary = near_boundary;
    p.dev_err = dev_err;
    return cuda_status(launch_accept_sample(p, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
