// Greedy and speculative-sampling acceptance over the vocabulary.
//
// Rows are packed per sequence: target rows at sum_{b'<b}(gamma+1), draft rows / tokens / u
// at sum_{b'<b} gamma, v alongside the target rows.  Every row is cut into n_chunks
// vocabulary chunks so that a handful of sequences still fill the GPU.
//
// Greedy:   accept_argmax_kernel  (row, chunk) -> best (value, lowest index) as a 64-bit key
//           accept_greedy_kernel  per sequence: reduce the chunks of every row, then the
//                                 longest matching prefix and the bonus token.
// Sampling: accept_stats_kernel   (row, chunk) -> (max, sum exp(z - max)) in fp32
//           accept_decide_kernel  per sequence: log-sum-exp of every row in fp64 (a warp per
//                                 row), then the accept decisions u <= p/q (ratio in fp64),
//                                 which row draws and how
//           accept_wsum_kernel    (sequence, chunk) -> sum of the draw weights (fp64); the
//                                 drawing row has chunks of its own, about two CTAs per SM
//                                 over the batch
//           accept_draw_kernel    per sequence: find the chunk holding v*Z (a warp scans the
//                                 chunk sums), then the token by an in-order prefix sum inside
//                                 it; write the outputs.
#include "sd_internal.h"

namespace sd {
namespace {

constexpr int kThreads = 256;
constexpr double kNearBoundary = 1e-6;

struct Decision {
    double lse_p;   // log-sum-exp of the drawing target row
    double lse_q;   // of the matching draft row (residual mode)
    int n;          // accepted drafts
    int residual;   // 1: draw from max(0, p - q); 0: draw from p
    int near;       // near-boundary count so far
    int pad;
};

// Offsets of sequence b: target rows (sum of gamma+1) and draft rows (sum of gamma).
__device__ __forceinline__ void row_offsets(const int32_t *gamma, int b, int64_t &off_t,
                                            int64_t &off_d) {
    int64_t s = 0;
    for (int i = 0; i < b; ++i) s += __ldg(gamma + i);
    off_d = s;
    off_t = s + b;
}

__device__ __forceinline__ unsigned long long argmax_key(float x, int idx) {
    unsigned int u;
    if (x != x) {
        u = 0u;  // NaN ranks below -inf
    } else {
        x += 0.0f;  // -0 -> +0
        const unsigned int bits = __float_as_uint(x);
        u = (bits >> 31) ? ~bits : (bits | 0x80000000u);
    }
    return ((unsigned long long)u << 32) | (unsigned long long)(0xffffffffu - (unsigned)idx);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
        x = y > x ? y : x;
    }
    return x;
}

__device__ __forceinline__ void chunk_range(int vocab, int n_chunks, int c, int &lo, int &hi) {
    lo = (int)((int64_t)vocab * c / n_chunks);
    hi = (int)((int64_t)vocab * (c + 1) / n_chunks);
}

// ---------------------------------------------------------------- greedy -----------------

__global__ void __launch_bounds__(kThreads) accept_argmax_kernel(const AcceptParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    __shared__ unsigned long long s_red[kThreads / 32];
    const int c = blockIdx.x, slot = blockIdx.y;
    const int b = slot / (p.max_gamma + 1), i = slot % (p.max_gamma + 1);
    const int gm = __ldg(p.gamma + b);
    if (gm < 0 || gm > p.max_gamma || i > gm) return;
    int64_t off_t, off_d;
    row_offsets(p.gamma, b, off_t, off_d);
    const float *row = p.tgt + (off_t + i) * (int64_t)p.vocab;
    int lo, hi;
    chunk_range(p.vocab, p.n_chunks, c, lo, hi);
    unsigned long long best = 0ull;
    for (int x = lo + threadIdx.x; x < hi; x += kThreads) {
        const unsigned long long k = argmax_key(__ldg(row + x), x);
        best = k > best ? k : best;
    }
    best = warp_max_u64(best);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned long long v = threadIdx.x < kThreads / 32 ? s_red[threadIdx.x] : 0ull;
        v = warp_max_u64(v);
        if (threadIdx.x == 0)
            reinterpret_cast<unsigned long long *>(p.ws)[(int64_t)slot * p.n_chunks + c] = v;
    }
}

__global__ void accept_greedy_kernel(const AcceptParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    extern __shared__ int s_t[];  // argmax of every target row of this sequence
    const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gm = __ldg(p.gamma + b);
    if (gm < 0 || gm > p.max_gamma) {
        if (threadIdx.x == 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    const unsigned long long *keys = reinterpret_cast<const unsigned long long *>(p.ws);
    for (int i = warp; i <= gm; i += blockDim.x / 32) {
        const int64_t slot = (int64_t)b * (p.max_gamma + 1) + i;
        unsigned long long best = 0ull;
        for (int c = lane; c < p.n_chunks; c += 32) {
            const unsigned long long k = keys[slot * p.n_chunks + c];
            best = k > best ? k : best;
        }
        best = warp_max_u64(best);
        if (lane == 0) s_t[i] = (int)(0xffffffffu - (unsigned)(best & 0xffffffffull));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t off_t, off_d;
        row_offsets(p.gamma, b, off_t, off_d);
        int n = 0;
        while (n < gm) {
            const int d = __ldg(p.draft_tok + off_d + n);
            if (d < 0 || d >= p.vocab) set_dev_err(p.dev_err, SD_DEVERR_TOKEN);
            if (d != s_t[n]) break;
            ++n;
        }
        int32_t *out = p.out_tok + (int64_t)b * p.out_stride;
        for (int e = 0; e < n; ++e) out[e] = __ldg(p.draft_tok + off_d + e);
        out[n] = s_t[n];
        p.n_acc[b] = n;
    }
}

// ---------------------------------------------------------------- sampling ---------------

// Row slot layout of the statistics: target rows first (batch*(max_gamma+1)), then draft rows.
__global__ void __launch_bounds__(kThreads) accept_stats_kernel(const AcceptParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    __shared__ float s_m[kThreads / 32], s_s[kThreads / 32];
    const int c = blockIdx.x, slot = blockIdx.y;
    const int n_tslots = p.batch * (p.max_gamma + 1);
    const bool target = slot < n_tslots;
    const int b = target ? slot / (p.max_gamma + 1) : (slot - n_tslots) / p.max_gamma;
    const int i = target ? slot % (p.max_gamma + 1) : (slot - n_tslots) % p.max_gamma;
    const int gm = __ldg(p.gamma + b);
    if (gm < 0 || gm > p.max_gamma || (target ? i > gm : i >= gm)) return;
    int64_t off_t, off_d;
    row_offsets(p.gamma, b, off_t, off_d);
    const float *row = target ? p.tgt + (off_t + i) * (int64_t)p.vocab
                              : p.drf + (off_d + i) * (int64_t)p.vocab;
    int lo, hi;
    chunk_range(p.vocab, p.n_chunks, c, lo, hi);
    float m = -INFINITY;
    for (int x = lo + threadIdx.x; x < hi; x += kThreads) m = fmaxf(m, __ldg(row + x));
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
    __syncthreads();
    m = s_m[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, s_m[w]);
    float s = 0.f;
    if (m != -INFINITY)
        for (int x = lo + threadIdx.x; x < hi; x += kThreads) s += expf(__ldg(row + x) - m);
    s = warp_sum(s);
    if ((threadIdx.x & 31) == 0) s_s[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) tot += s_s[w];
        reinterpret_cast<float2 *>(p.ws)[(int64_t)slot * p.n_chunks + c] = make_float2(m, tot);
    }
}

__device__ double row_lse(const AcceptParams &p, int slot, int lane) {
    const float2 *st = reinterpret_cast<const float2 *>(p.ws) + (int64_t)slot * p.n_chunks;
    float M = -INFINITY;
    for (int c = lane; c < p.n_chunks; c += 32) M = fmaxf(M, st[c].x);
    M = warp_max(M);
    double S = 0.0;
    if (M != -INFINITY)
        for (int c = lane; c < p.n_chunks; c += 32)
            if (st[c].x != -INFINITY) S += (double)st[c].y * exp((double)st[c].x - (double)M);
    S = warp_sum_d(S);
    return (double)M + log(S);
}

__device__ __forceinline__ Decision *decisions(const AcceptParams &p) {
    const int n_slots = p.batch * (2 * p.max_gamma + 1);
    char *base = reinterpret_cast<char *>(p.ws) + (size_t)n_slots * p.n_chunks * sizeof(float2);
    return reinterpret_cast<Decision *>(base);
}

__device__ __forceinline__ double *chunk_sums(const AcceptParams &p) {  // [batch][n_wchunks]
    return reinterpret_cast<double *>(decisions(p) + p.batch);
}

constexpr int kDecideWarps = 8;

// One CTA per sequence: the log-sum-exps of its rows (a warp per row) and the draft tokens'
// logits first, in parallel; then the accept decisions in order from shared memory.
__global__ void __launch_bounds__(kDecideWarps * 32) accept_decide_kernel(const AcceptParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    extern __shared__ double s_dec[];  // lse of target rows [gm + 1], draft rows [gm], ratios [gm]
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gm = __ldg(p.gamma + b);
    Decision *dec = decisions(p) + b;
    if (gm < 0 || gm > p.max_gamma) {
        if (tid == 0) {
            set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
            dec->n = -1;
        }
        return;
    }
    int64_t off_t, off_d;
    row_offsets(p.gamma, b, off_t, off_d);
    const int n_tslots = p.batch * (p.max_gamma + 1);
    double *s_lp = s_dec, *s_lq = s_dec + (gm + 1), *s_r = s_lq + gm;
    for (int j = warp; j < 2 * gm + 1; j += kDecideWarps) {
        const bool target = j <= gm;
        const int i = target ? j : j - (gm + 1);
        const double l = row_lse(p, target ? b * (p.max_gamma + 1) + i
                                           : n_tslots + b * p.max_gamma + i, lane);
        if (lane == 0) (target ? s_lp : s_lq)[i] = l;
    }
    __syncthreads();
    // ratio p/q of every draft token (fp64), with the row checks
    for (int i = tid; i < gm; i += kDecideWarps * 32) {
        const double lp = s_lp[i], lq = s_lq[i];
        const int x = __ldg(p.draft_tok + off_d + i);
        double r = 0.0;
        if (x >= 0 && x < p.vocab) {
            const double zp = (double)__ldg(p.tgt + (off_t + i) * (int64_t)p.vocab + x);
            const double zq = (double)__ldg(p.drf + (off_d + i) * (int64_t)p.vocab + x);
            r = exp((zp - lp) - (zq - lq));
        } else {
            set_dev_err(p.dev_err, SD_DEVERR_TOKEN);
        }
        if (!(lp == lp) || !(lq == lq) || isinf(lp) || isinf(lq))
            set_dev_err(p.dev_err, SD_DEVERR_NUMERIC);
        s_r[i] = r;
    }
    __syncthreads();
    if (tid == 0) {
        int n = 0, near = 0;
        bool rejected = false;
        for (int i = 0; i < gm; ++i) {
            const double u = (double)__ldg(p.u + off_d + i);
            const double r = s_r[i];
            if (fabs(u - r) < kNearBoundary) ++near;
            if (u <= r) {
                ++n;
            } else {
                rejected = true;
                break;
            }
        }
        dec->lse_p = s_lp[n];
        dec->lse_q = rejected ? s_lq[n] : 0.0;
        dec->n = n;
        dec->residual = rejected ? 1 : 0;
        dec->near = near;
    }
}

// Draw weight of token x: p_x, or max(0, p_x - q_x) in residual mode.  Evaluated in fp64 from
// the fp64 log-sum-exps: in residual mode p and q nearly cancel, so rounding either exponent to
// fp32 (about 1e-7 relative at |z - lse| ~ 16) could move a prefix sum across a token boundary
// by more than the 1e-6 * Z window that is counted as near-boundary.
__device__ __forceinline__ double draw_weight(const float *zp, const float *zq, double lp,
                                              double lq, bool residual, int x) {
    const double pp = exp((double)__ldg(zp + x) - lp);
    if (!residual) return pp;
    const double d = pp - exp((double)__ldg(zq + x) - lq);
    return d > 0.0 ? d : 0.0;
}

__device__ double block_sum_d(double x, double *s_red) {
    x = warp_sum_d(x);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = x;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) t += s_red[w];
    __syncthreads();
    return t;
}

// (sequence, chunk) -> sum of the draw weights of the chunk.
__global__ void __launch_bounds__(kThreads) accept_wsum_kernel(const AcceptParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    __shared__ double s_red[kThreads / 32];
    const int c = blockIdx.x, b = blockIdx.y;
    const Decision dec = decisions(p)[b];
    if (dec.n < 0) return;
    int64_t off_t, off_d;
    row_offsets(p.gamma, b, off_t, off_d);
    const float *zp = p.tgt + (off_t + dec.n) * (int64_t)p.vocab;
    const float *zq = p.drf + (off_d + dec.n) * (int64_t)p.vocab;
    int lo, hi;
    chunk_range(p.vocab, p.n_wchunks, c, lo, hi);
    double s = 0.0;
    for (int x = lo + threadIdx.x; x < hi; x += kThreads)
        s += draw_weight(zp, zq, dec.lse_p, dec.lse_q, dec.residual != 0, x);
    s = block_sum_d(s, s_red);
    if (threadIdx.x == 0) chunk_sums(p)[(int64_t)b * p.n_wchunks + c] = s;
}

// One CTA per sequence: locate v*Z, finish the outputs.
__global__ void __launch_bounds__(kThreads) accept_draw_kernel(const AcceptParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    __shared__ double s_red[kThreads / 32];
    __shared__ double s_warp_tot[kThreads / 32];
    __shared__ int s_found;
    __shared__ double s_c_before, s_c_at;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Decision dec = decisions(p)[b];
    if (dec.n < 0) return;
    int64_t off_t, off_d;
    row_offsets(p.gamma, b, off_t, off_d);
    const float *zp = p.tgt + (off_t + dec.n) * (int64_t)p.vocab;
    const float *zq = p.drf + (off_d + dec.n) * (int64_t)p.vocab;
    bool residual = dec.residual != 0;
    const int nw = p.n_wchunks;
    const double *cs = chunk_sums(p) + (int64_t)b * nw;
    const double v_draw = (double)__ldg(p.v + off_t + dec.n);
    __shared__ double s_z, s_before;
    __shared__ int s_clo;
    // Z, and the chunk where the running total first exceeds v*Z: warp 0 reads the chunk sums
    // 32 at a time (Z: lane-strided partials, then the warp's tree; a fixed order)
    if (warp == 0) {
        double t = 0.0;
        for (int c = lane; c < nw; c += 32) t += cs[c];
        t = warp_sum_d(t);
        const double tgt = v_draw * t;
        double run = 0.0, bef = 0.0;
        int found = nw - 1;
        for (int c0 = 0; c0 < nw; c0 += 32) {
            const int c = c0 + lane;
            const double x = c < nw ? cs[c] : 0.0;
            double incl = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            // (the last chunk takes whatever rounding leaves past the total)
            const unsigned hit = __ballot_sync(0xffffffffu, c < nw && (c == nw - 1 || run + incl > tgt));
            if (hit) {
                const int l = __ffs(hit) - 1;
                found = c0 + l;
                bef = run + __shfl_sync(0xffffffffu, incl - x, l);
                break;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            s_z = t;
            s_clo = found;
            s_before = bef;
        }
    }
    __syncthreads();
    double Z = s_z;
    int c_lo = 0, c_hi = nw;  // chunks to scan
    double before = 0.0;
    if (residual && !(Z > 0.0)) {  // empty residual: draw from p over the whole vocabulary
        residual = false;
        Z = 0.0;
        for (int c = 0; c < nw; ++c) {
            int lo, hi;
            chunk_range(p.vocab, nw, c, lo, hi);
            double s = 0.0;
            for (int x = lo + tid; x < hi; x += kThreads)
                s += draw_weight(zp, zq, dec.lse_p, 0.0, false, x);
            Z += block_sum_d(s, s_red);
        }
    } else {
        c_lo = s_clo;
        c_hi = c_lo + 1;
        before = s_before;
    }
    const double target = (double)__ldg(p.v + off_t + dec.n) * Z;
    if (tid == 0) s_found = -1;
    __syncthreads();
    int last_pos = -1;  // last x with a positive weight seen (fallback)
    double run = before;
    for (int c = c_lo; c < c_hi; ++c) {
        int lo, hi;
        chunk_range(p.vocab, nw, c, lo, hi);
        for (int base = lo; base < hi; base += kThreads) {
            const int x = base + tid;
            const double w = x < hi ? draw_weight(zp, zq, dec.lse_p, dec.lse_q,
                                                  residual, x)
                                    : 0.0;
            // in-order inclusive prefix sum over the tile
            double incl = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane == 31) s_warp_tot[warp] = incl;
            __syncthreads();
            double wbefore = 0.0;
            for (int w2 = 0; w2 < warp; ++w2) wbefore += s_warp_tot[w2];
            double tile_tot = 0.0;
            for (int w2 = 0; w2 < kThreads / 32; ++w2) tile_tot += s_warp_tot[w2];
            const double C = run + wbefore + incl;
            const bool cross = x < hi && C > target && (C - w) <= target;
            if (cross) {
                s_found = x;
                s_c_before = C - w;
                s_c_at = C;
            }
            const unsigned pos = __ballot_sync(0xffffffffu, x < hi && w > 0.0);
            if (pos) {
                const int lw = 31 - __clz(pos);
                const int cand = __shfl_sync(0xffffffffu, x, lw);
                last_pos = max(last_pos, cand);
            }
            __syncthreads();
            run += tile_tot;
            if (s_found >= 0) break;
            __syncthreads();
        }
        if (s_found >= 0) break;
    }
    __syncthreads();
    // fallback: rounding left v*Z at or past the total -> last positive-weight position
    __shared__ int s_last[kThreads / 32];
    if (lane == 0) s_last[warp] = last_pos;
    __syncthreads();
    if (tid == 0) {
        int tok = s_found;
        int near = dec.near;
        if (tok < 0) {
            for (int w2 = 0; w2 < kThreads / 32; ++w2) tok = max(tok, s_last[w2]);
            if (tok < 0) tok = 0;
            ++near;
        } else if (target - s_c_before < kNearBoundary * Z || s_c_at - target < kNearBoundary * Z) {
            ++near;
        }
        int32_t *out = p.out_tok + (int64_t)b * p.out_stride;
        for (int e = 0; e < dec.n; ++e) out[e] = __ldg(p.draft_tok + off_d + e);
        out[dec.n] = tok;
        p.n_acc[b] = dec.n;
        if (p.near_boundary) p.near_boundary[b] = near;
    }
}

}  // namespace

size_t accept_workspace_bytes(int batch, int max_gamma, int vocab, int *n_chunks_out,
                              int *n_wchunks_out) {
    const int slots_t = batch * (max_gamma + 1);
    int n_chunks = (2 * 148 + slots_t - 1) / slots_t;
    const int max_chunks = (vocab + 2047) / 2048;
    if (n_chunks > max_chunks) n_chunks = max_chunks;
    if (n_chunks < 1) n_chunks = 1;
    if (n_chunks_out) *n_chunks_out = n_chunks;
    // the drawing row of each sequence: about two CTAs per SM over the batch, at least 512
    // tokens per chunk
    int n_wchunks = (2 * 148 + batch - 1) / batch;
    const int max_wchunks = (vocab + 511) / 512;
    if (n_wchunks > max_wchunks) n_wchunks = max_wchunks;
    if (n_wchunks < 1) n_wchunks = 1;
    if (n_wchunks_out) *n_wchunks_out = n_wchunks;
    const size_t greedy = (size_t)slots_t * n_chunks * sizeof(unsigned long long);
    const size_t n_slots = (size_t)batch * (2 * max_gamma + 1);
    const size_t sample = n_slots * n_chunks * sizeof(float2) + (size_t)batch * sizeof(Decision) +
                          (size_t)batch * n_wchunks * sizeof(double);
    return greedy > sample ? greedy : sample;
}

cudaError_t launch_accept_greedy(const AcceptParams &p, cudaStream_t s) {
    dim3 g1(p.n_chunks, p.batch * (p.max_gamma + 1));
    cudaError_t e = launch_pdl(accept_argmax_kernel, g1, dim3(kThreads), 0, s, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(accept_greedy_kernel, dim3(p.batch), dim3(256),
                      (p.max_gamma + 1) * sizeof(int), s, p);
}

cudaError_t launch_accept_sample(const AcceptParams &p, cudaStream_t s) {
    dim3 g1(p.n_chunks, p.batch * (2 * p.max_gamma + 1));
    cudaError_t e = launch_pdl(accept_stats_kernel, g1, dim3(kThreads), 0, s, p);
    if (e != cudaSuccess) return e;
    if ((e = launch_pdl(accept_decide_kernel, dim3(p.batch), dim3(kDecideWarps * 32),
                        (size_t)(3 * p.max_gamma + 1) * sizeof(double), s, p)) != cudaSuccess)
        return e;
    dim3 g3(p.n_wchunks, p.batch);
    if ((e = launch_pdl(accept_wsum_kernel, g3, dim3(kThreads), 0, s, p)) != cudaSuccess)
        return e;
    return launch_pdl(accept_draw_kernel, dim3(p.batch), dim3(kThreads), 0, s, p);
}

}  // namespace sd
