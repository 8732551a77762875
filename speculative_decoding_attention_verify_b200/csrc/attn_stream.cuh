// Position streams of the attention kinds, shared by the CUDA-core engines.
//
// Each (sequence, KV head) of an attention call visits an ordered list of cache positions:
//   verify          [0, kv_len)
//   text-anchored   the non-visual positions from the lowest windowed position to kv_len
//   sparse          the selected positions (ascending prefix of idx below the tail), then
//                   [tail_begin, kv_len)
// described as two segments (s0, len0) and (s1, len1); for sparse the first segment is the
// index list itself.  Splits take contiguous chunks of this logical list.
#pragma once

#include "sd_internal.h"

namespace sd {

// Positions of one row's text-anchored window: the last W positions j <= limit outside
// [vb, ve), as up to two ranges [lo1, hi1] and [lo2, hi2] (a range with lo > hi is empty).
__device__ __forceinline__ void window_ranges(int limit, int vb, int ve, int W, int &lo1,
                                              int &hi1, int &lo2, int &hi2) {
    lo2 = 1;
    hi2 = 0;
    if (vb >= ve) vb = ve = 0;
    if (limit < 0 || W <= 0) {
        lo1 = 1;
        hi1 = 0;
        return;
    }
    if (limit >= ve) {  // row above the visual span
        lo1 = max(ve, limit - W + 1);
        hi1 = limit;
        const int rem = W - (hi1 - lo1 + 1);
        if (rem > 0 && vb > 0) {
            hi2 = vb - 1;
            lo2 = max(0, vb - rem);
        }
    } else if (limit >= vb) {  // row inside the span: only positions below it
        hi1 = vb - 1;
        lo1 = max(0, vb - W);
    } else {  // row below the span
        hi1 = limit;
        lo1 = max(0, limit - W + 1);
    }
}

// Per-CTA description of the stream of sequence b / KV head g.
struct StreamInfo {
    int s0, len0, s1, len1;
    int vb, ve, W;        // text-anchored span and window (span clamped; empty if invalid)
    int tail;             // sparse tail start
    const int32_t *sel;   // sparse selected list of this (b, g)
};

// Block-cooperative set-up of the stream (all NT threads must call it; it synchronises).
// s_buf must hold at least 4 + NT/32 ints.
template <int NT>
__device__ __forceinline__ StreamInfo stream_setup(const AttnParams &p, int b, int g, int n_q,
                                                   int kv_len, int *s_buf) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    StreamInfo si{};
    si.vb = si.ve = si.W = 0;
    if (p.kind == SD_ATTN_TEXT_ANCHORED) {
        si.vb = __ldg(p.vis_begin + b);
        si.ve = __ldg(p.vis_end + b);
        si.W = __ldg(p.window + b);
        if (si.vb > si.ve) {
            if (tid == 0) set_dev_err(p.dev_err, SD_DEVERR_INDEX);
            si.vb = si.ve = 0;
        }
        si.vb = min(max(si.vb, 0), kv_len);
        si.ve = min(max(si.ve, 0), kv_len);
    }
    si.tail = 0;
    si.sel = nullptr;
    if (p.kind == SD_ATTN_SPARSE) {
        // The list is ascending with -1 padding; its usable entries (0 <= x < tail) form a
        // prefix, counted in parallel.  Order violations are flagged here; repeated entries
        // are skipped when positions are mapped.
        si.tail = min(max(__ldg(p.tail_begin + b), 0), kv_len);
        si.sel = p.idx + ((int64_t)b * p.kv.h_kv + g) * p.k_sel;
        int cnt = 0;
        for (int e = tid; e < p.k_sel; e += NT) {
            const int x = __ldg(si.sel + e);
            const bool use = x >= 0 && x < si.tail;
            cnt += use ? 1 : 0;
            if (use && e > 0) {
                const int prev = __ldg(si.sel + e - 1);
                if (prev >= x || prev < 0) set_dev_err(p.dev_err, SD_DEVERR_INDEX);
            }
        }
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (lane == 0) s_buf[4 + warp] = cnt;
    } else if (tid == 0) {
        int s0 = 0, len0 = 0, s1 = 0, len1 = 0;
        if (p.kind == SD_ATTN_VERIFY) {
            len0 = kv_len;
        } else {
            // Lowest position any row of this sequence may see (windows slide up with rows).
            int lowest = kv_len;
            for (int i = 0; i < n_q; ++i) {
                int lo1, hi1, lo2, hi2;
                window_ranges(kv_len - n_q + i, si.vb, si.ve, si.W, lo1, hi1, lo2, hi2);
                if (lo2 <= hi2) lowest = min(lowest, lo2);
                if (lo1 <= hi1) lowest = min(lowest, lo1);
            }
            if (si.vb < si.ve && lowest < si.vb) {
                s0 = lowest;
                len0 = si.vb - lowest;
                s1 = si.ve;
            } else {
                s1 = (si.vb < si.ve && lowest >= si.vb) ? max(lowest, si.ve) : lowest;
            }
            len1 = max(0, kv_len - s1);
        }
        s_buf[0] = s0;
        s_buf[1] = len0;
        s_buf[2] = s1;
        s_buf[3] = len1;
    }
    __syncthreads();
    if (p.kind == SD_ATTN_SPARSE && tid == 0) {
        int k_eff = 0;
        for (int w = 0; w < NT / 32; ++w) k_eff += s_buf[4 + w];
        s_buf[0] = 0;
        s_buf[1] = k_eff;
        s_buf[2] = si.tail;
        s_buf[3] = kv_len - si.tail;
    }
    __syncthreads();
    si.s0 = s_buf[0];
    si.len0 = s_buf[1];
    si.s1 = s_buf[2];
    si.len1 = s_buf[3];
    return si;
}

// The stream of sequence b for verify and text-anchored calls, computed by one thread on its
// own (no block synchronisation): the same runs as stream_setup.
__device__ __forceinline__ StreamInfo stream_info_single(const AttnParams &p, int b, int n_q,
                                                         int kv_len) {
    StreamInfo si{};
    si.vb = si.ve = si.W = 0;
    si.tail = 0;
    si.sel = nullptr;
    si.s0 = si.len0 = si.s1 = si.len1 = 0;
    if (p.kind == SD_ATTN_VERIFY) {
        si.len0 = kv_len;
        return si;
    }
    si.vb = __ldg(p.vis_begin + b);
    si.ve = __ldg(p.vis_end + b);
    si.W = __ldg(p.window + b);
    if (si.vb > si.ve) {
        set_dev_err(p.dev_err, SD_DEVERR_INDEX);
        si.vb = si.ve = 0;
    }
    si.vb = min(max(si.vb, 0), kv_len);
    si.ve = min(max(si.ve, 0), kv_len);
    int lowest = kv_len;
    for (int i = 0; i < n_q; ++i) {
        int lo1, hi1, lo2, hi2;
        window_ranges(kv_len - n_q + i, si.vb, si.ve, si.W, lo1, hi1, lo2, hi2);
        if (lo2 <= hi2) lowest = min(lowest, lo2);
        if (lo1 <= hi1) lowest = min(lowest, lo1);
    }
    if (si.vb < si.ve && lowest < si.vb) {
        si.s0 = lowest;
        si.len0 = si.vb - lowest;
        si.s1 = si.ve;
    } else {
        si.s1 = (si.vb < si.ve && lowest >= si.vb) ? max(lowest, si.ve) : lowest;
    }
    si.len1 = max(0, kv_len - si.s1);
    return si;
}

// Allowed ranges of local row lr (query row lr / G) of the stream's sequence.
__device__ __forceinline__ void row_ranges(const AttnParams &p, const StreamInfo &si, int lr,
                                           int R, int n_q, int kv_len, int &lo1, int &hi1,
                                           int &lo2, int &hi2) {
    lo1 = 1;
    hi1 = 0;
    lo2 = 1;
    hi2 = 0;
    if (lr >= R) return;
    const int limit = kv_len - n_q + lr / p.group;
    if (p.kind == SD_ATTN_TEXT_ANCHORED) {
        window_ranges(limit, si.vb, si.ve, si.W, lo1, hi1, lo2, hi2);
    } else {
        lo1 = 0;
        hi1 = limit;
    }
}

// Physical position of logical stream position pl (or -1: repeated sparse entry, or out of
// the sequence).
__device__ __forceinline__ int stream_position(const AttnParams &p, const StreamInfo &si, int pl,
                                               int kv_len) {
    int j;
    if (pl < si.len0) {
        if (p.kind == SD_ATTN_SPARSE) {
            j = __ldg(si.sel + pl);
            if (pl > 0 && __ldg(si.sel + pl - 1) >= j) j = -1;  // repeated: skip
        } else {
            j = si.s0 + pl;
        }
    } else {
        j = si.s1 + (pl - si.len0);
    }
    return (j >= 0 && j < kv_len) ? j : -1;
}

}  // namespace sd
