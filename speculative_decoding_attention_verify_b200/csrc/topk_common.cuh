// Device helpers shared by the two top-K score modes (query-key and mean text attention).
#pragma once

#include "sd_internal.h"

namespace sd {

// Order-preserving 64-bit key of a score: a larger score gives a larger key; -0 == +0; NaN
// ranks below every other score.
__device__ __forceinline__ unsigned long long score_key(double x) {
    if (x != x) return 0ull;  // NaN ranks lowest
    x += 0.0;                 // -0 -> +0
    unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Clamp the candidate range of sequence b to [0, kv_len) and to max_cand entries (a range
// outside those bounds sets SD_DEVERR_INDEX when `report`).
__device__ __forceinline__ void cand_range(const TopkParams &p, int b, int &cb, int &n,
                                           bool report) {
    const int kv_len = __ldg(p.kv.kv_len + b);
    int lo = __ldg(p.cand_begin + b), hi = __ldg(p.cand_end + b);
    const bool bad = lo < 0 || hi > kv_len || hi - lo > p.max_cand ||
                     (p.kv.page_size != 0 && kv_len > p.kv.max_pages * kPageSize);
    lo = max(lo, 0);
    hi = min(hi, kv_len);
    if (p.kv.page_size != 0) hi = min(hi, p.kv.max_pages * kPageSize);
    hi = min(hi, lo + p.max_cand);
    cb = lo;
    n = max(0, hi - lo);
    if (bad && report) set_dev_err(p.dev_err, SD_DEVERR_INDEX);
}

// The same, reported by thread 0 of the CTAs with blockIdx.x == 0.
__device__ __forceinline__ void cand_range(const TopkParams &p, int b, int &cb, int &n) {
    cand_range(p, b, cb, n, threadIdx.x == 0 && blockIdx.x == 0);
}

}  // namespace sd
