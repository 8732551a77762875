// CUDA-core split-KV attention engine for the three attention kinds, plus the split merge.
//
// Serves fp32 caches and every bf16 problem with fewer than 16 query rows per KV head (the
// Sparrow and Sparse-to-Dense draft steps have one query row and G = 7 heads per KV head).
//
// Decomposition: grid (splits x row blocks, KV heads, sequences).  Every CTA owns one KV head
// g of one sequence b, a block of up to RB query rows of that head's group (rows ordered
// (query row i, head h) with h fastest), and one contiguous chunk of the sequence's
// *position stream*:
//   verify          [0, kv_len)
//   text-anchored   the non-visual positions from the lowest windowed position to kv_len
//   sparse          the compacted selected indices, then [tail_begin, kv_len)
// Per 128-position tile: each thread scores one position against all RB rows (its K row is
// streamed from HBM with 16-byte loads; the rows come from shared memory as broadcasts);
// one warp per row updates the running max / sum (online softmax, base 2); then each warp
// accumulates P.V for a quarter of the positions with lanes spread over head_dim (coalesced
// V rows).  The four warps' partial outputs are summed in a fixed order (deterministic).
// With one split the normalised output is written directly; otherwise the unnormalised
// partial and its (max, sum) go to the workspace and attn_merge_kernel combines the splits
// by their log-sum-exp.
#include "sd_internal.h"

namespace sd {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;

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

template <bool BF16, int D, int RB>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(const AttnParams p) {
    using CH = Chunk<BF16>;
    constexpr int ESZ = BF16 ? 2 : 4;
    constexpr int NCHUNK = D * ESZ / 16;  // 16-byte chunks per KV row
    constexpr int EPL = D / 32;           // head_dim elements per lane in the P.V phase
    static_assert(RB % 4 == 0 && RB * D <= RB * kTile, "tile shapes");

    extern __shared__ int s_sel[];  // sparse: compacted selected positions
    __shared__ __align__(16) float s_q[RB][D];
    __shared__ __align__(16) float s_s[RB][kTile];
    __shared__ __align__(16) float s_p[kTile][RB];
    __shared__ int64_t s_off[kTile];
    __shared__ int s_lo1[RB], s_hi1[RB], s_lo2[RB], s_hi2[RB];
    __shared__ float s_m[RB], s_l[RB], s_corr[RB];
    __shared__ int s_stream[4];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, g = blockIdx.y;
    const int split = blockIdx.x % p.n_splits, rb = blockIdx.x / p.n_splits;
    const KVView &kv = p.kv;
    const int G = p.group;
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    const int R = n_q * G;
    if (rb * RB >= R) return;
    if (n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (kv.page_size != 0 && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }

    // Visual span / window (text-anchored only).
    int vb = 0, ve = 0, W = 0;
    if (p.kind == SD_ATTN_TEXT_ANCHORED) {
        vb = __ldg(p.vis_begin + b);
        ve = __ldg(p.vis_end + b);
        W = __ldg(p.window + b);
        if (vb > ve) {
            if (tid == 0) set_dev_err(p.dev_err, SD_DEVERR_INDEX);
            vb = ve = 0;
        }
        vb = min(max(vb, 0), kv_len);
        ve = min(max(ve, 0), kv_len);
    }

    // Sparse: compact the valid, strictly ascending selected positions below the tail.
    int tail = 0;
    if (p.kind == SD_ATTN_SPARSE) {
        tail = min(max(__ldg(p.tail_begin + b), 0), kv_len);
        if (warp == 0) {
            const int32_t *sel = p.idx + ((int64_t)b * kv.h_kv + g) * p.k_sel;
            int count = 0, prev = -1;
            for (int base = 0; base < p.k_sel; base += 32) {
                const int e = base + lane;
                const int x = e < p.k_sel ? __ldg(sel + e) : -1;
                const bool in = x >= 0 && x < tail;
                int pm = in ? x : -1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, pm, o);
                    if (lane >= o) pm = max(pm, y);
                }
                int before = __shfl_up_sync(0xffffffffu, pm, 1);
                if (lane == 0) before = -1;
                before = max(before, prev);
                const bool keep = in && x > before;
                if (in && !keep) set_dev_err(p.dev_err, SD_DEVERR_INDEX);
                const unsigned m = __ballot_sync(0xffffffffu, keep);
                if (keep) s_sel[count + __popc(m & ((1u << lane) - 1u))] = x;
                count += __popc(m);
                prev = max(prev, __shfl_sync(0xffffffffu, pm, 31));
            }
            if (lane == 0) {
                s_stream[0] = 0;
                s_stream[1] = count;
                s_stream[2] = tail;
                s_stream[3] = kv_len - tail;
            }
        }
    } else if (tid == 0) {
        int s0 = 0, len0 = 0, s1 = 0, len1 = 0;
        if (p.kind == SD_ATTN_VERIFY) {
            len0 = kv_len;
        } else {
            // Lowest position any row of this sequence may see (windows slide up with rows).
            int lowest = kv_len;
            for (int i = 0; i < n_q; ++i) {
                int lo1, hi1, lo2, hi2;
                window_ranges(kv_len - n_q + i, vb, ve, W, lo1, hi1, lo2, hi2);
                if (lo2 <= hi2) lowest = min(lowest, lo2);
                if (lo1 <= hi1) lowest = min(lowest, lo1);
            }
            if (vb < ve && lowest < vb) {
                s0 = lowest;
                len0 = vb - lowest;
                s1 = ve;
            } else {
                s1 = (vb < ve && lowest >= vb) ? max(lowest, ve) : lowest;
            }
            len1 = max(0, kv_len - s1);
        }
        s_stream[0] = s0;
        s_stream[1] = len0;
        s_stream[2] = s1;
        s_stream[3] = len1;
    }

    // Per-row allowed ranges, running statistics and the pre-scaled query rows.
    if (tid < RB) {
        const int r = tid, lr = rb * RB + r;
        int lo1 = 1, hi1 = 0, lo2 = 1, hi2 = 0;
        if (lr < R) {
            const int limit = kv_len - n_q + lr / G;
            if (p.kind == SD_ATTN_TEXT_ANCHORED) {
                window_ranges(limit, vb, ve, W, lo1, hi1, lo2, hi2);
            } else {
                lo1 = 0;
                hi1 = limit;
            }
        }
        s_lo1[r] = lo1;
        s_hi1[r] = hi1;
        s_lo2[r] = lo2;
        s_hi2[r] = hi2;
        s_m[r] = -INFINITY;
        s_l[r] = 0.f;
    }
    for (int e = tid; e < RB * D; e += kThreads) {
        const int r = e / D, d = e % D, lr = rb * RB + r;
        float val = 0.f;
        if (lr < R) {
            const int64_t off = ((int64_t)(q0 + lr / G) * p.h_q + g * G + lr % G) * D + d;
            if (BF16)
                val = __uint_as_float(
                    (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.q) + off) << 16);
            else
                val = __ldg(reinterpret_cast<const float *>(p.q) + off);
        }
        s_q[r][d] = val * p.scale_log2;
    }
    __syncthreads();

    const int s0 = s_stream[0], len0 = s_stream[1], s1 = s_stream[2], len1 = s_stream[3];
    const int64_t P = (int64_t)len0 + len1;
    const int c0 = (int)(P * split / p.n_splits), c1 = (int)(P * (split + 1) / p.n_splits);
    const bool sparse = p.kind == SD_ATTN_SPARSE;

    float acc[RB][EPL];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[r][e] = 0.f;

    for (int t0 = c0; t0 < c1; t0 += kTile) {
        // ---- scores: one position per thread, all RB rows ----
        const int pl = t0 + tid;
        int j = -1;
        int64_t off = -1;
        if (pl < c1) {
            j = pl < len0 ? (sparse ? s_sel[pl] : s0 + pl) : s1 + (pl - len0);
            off = kv_row_offset(kv, b, g, j, p.dev_err);
            if (off < 0) j = -1;
        }
        s_off[tid] = j >= 0 ? off : -1;
        float2 sc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) sc[r] = make_float2(0.f, 0.f);
        if (j >= 0) {
            const char *krow = reinterpret_cast<const char *>(kv.k) + off * ESZ;
#pragma unroll
            for (int c = 0; c < NCHUNK; c += 4) {
                uint4 raw[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) raw[u] = ldg_stream16(krow + (c + u) * 16);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float f[CH::kElems];
                    CH::to_float(raw[u], f);
                    const int e0 = (c + u) * CH::kElems;
#pragma unroll
                    for (int r = 0; r < RB; ++r) {
#pragma unroll
                        for (int e = 0; e < CH::kElems; e += 4) {
                            const float4 qv = *reinterpret_cast<const float4 *>(&s_q[r][e0 + e]);
                            sc[r] = __ffma2_rn(make_float2(qv.x, qv.y), make_float2(f[e], f[e + 1]),
                                               sc[r]);
                            sc[r] = __ffma2_rn(make_float2(qv.z, qv.w),
                                               make_float2(f[e + 2], f[e + 3]), sc[r]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const bool ok = j >= 0 && ((j >= s_lo1[r] && j <= s_hi1[r]) ||
                                       (j >= s_lo2[r] && j <= s_hi2[r]));
            s_s[r][tid] = ok ? sc[r].x + sc[r].y : -INFINITY;
        }
        __syncthreads();

        // ---- online softmax: one warp per row ----
        for (int r = warp; r < RB; r += 4) {
            float v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = s_s[r][lane + 32 * c];
            const float tmax = warp_max(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])));
            const float m_old = s_m[r];
            const float m_new = fmaxf(m_old, tmax);
            float corr = 1.f, sum = 0.f;
            if (m_new != -INFINITY) {
                corr = exp2f(m_old - m_new);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    v[c] = exp2f(v[c] - m_new);
                    sum += v[c];
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) v[c] = 0.f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) s_p[lane + 32 * c][r] = v[c];
            sum = warp_sum(sum);
            if (lane == 0) {
                s_l[r] = s_l[r] * corr + sum;
                s_m[r] = m_new;
                s_corr[r] = corr;
            }
        }
        __syncthreads();

        // ---- P.V: warp w takes positions w, w+4, ...; lanes spread over head_dim ----
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const float cr = s_corr[r];
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[r][e] *= cr;
        }
        const char *vbase = reinterpret_cast<const char *>(kv.v);
        for (int t = warp; t < kTile; t += 4 * 8) {
            float vf[8][EPL];
            bool have[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int tt = t + 4 * u;
                const int64_t o = tt < kTile ? s_off[tt] : -1;
                have[u] = o >= 0;
                if (have[u]) {
                    const char *src = vbase + (o + lane * EPL) * ESZ;
                    if (BF16) {
                        if (EPL == 4) {
                            const uint2 w2 = __ldg(reinterpret_cast<const uint2 *>(src));
                            vf[u][0] = bf16_lo(w2.x);
                            vf[u][1] = bf16_hi(w2.x);
                            vf[u][2] = bf16_lo(w2.y);
                            vf[u][3] = bf16_hi(w2.y);
                        } else {
                            const uint32_t w1 = __ldg(reinterpret_cast<const uint32_t *>(src));
                            vf[u][0] = bf16_lo(w1);
                            vf[u][1] = bf16_hi(w1);
                        }
                    } else {
                        if (EPL == 4) {
                            const float4 f4 = __ldg(reinterpret_cast<const float4 *>(src));
                            vf[u][0] = f4.x;
                            vf[u][1] = f4.y;
                            vf[u][2] = f4.z;
                            vf[u][3] = f4.w;
                        } else {
                            const float2 f2 = __ldg(reinterpret_cast<const float2 *>(src));
                            vf[u][0] = f2.x;
                            vf[u][1] = f2.y;
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (!have[u]) continue;
                const int tt = t + 4 * u;
#pragma unroll
                for (int r4 = 0; r4 < RB; r4 += 4) {
                    const float4 pv = *reinterpret_cast<const float4 *>(&s_p[tt][r4]);
                    const float pr[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
#pragma unroll
                        for (int e = 0; e < EPL; e += 2) {
                            float2 a = make_float2(acc[r4 + q][e], acc[r4 + q][e + 1]);
                            a = __ffma2_rn(make_float2(pr[q], pr[q]),
                                           make_float2(vf[u][e], vf[u][e + 1]), a);
                            acc[r4 + q][e] = a.x;
                            acc[r4 + q][e + 1] = a.y;
                        }
                    }
                }
            }
        }
        __syncthreads();
    }

    // ---- sum the four warps' partial outputs in a fixed order ----
    float *s_o = &s_s[0][0];  // [RB][D]
    for (int w = 0; w < 4; ++w) {
        if (warp == w) {
#pragma unroll
            for (int r = 0; r < RB; ++r)
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    const int ix = r * D + lane * EPL + e;
                    s_o[ix] = (w == 0 ? 0.f : s_o[ix]) + acc[r][e];
                }
        }
        __syncthreads();
    }

    for (int e = tid; e < RB * D; e += kThreads) {
        const int r = e / D, d = e % D, lr = rb * RB + r;
        if (lr >= R) continue;
        const int row = q0 + lr / G, h = g * G + lr % G;
        if (p.n_splits == 1) {
            const float l = s_l[r];
            const float o = l > 0.f ? s_o[e] / l : 0.f;
            const int64_t oi = ((int64_t)row * p.h_q + h) * D + d;
            if (BF16)
                reinterpret_cast<unsigned short *>(p.out)[oi] = (unsigned short)f32_to_bf16_bits(o);
            else
                reinterpret_cast<float *>(p.out)[oi] = o;
        } else {
            const int64_t base = ((int64_t)split * p.rows_cap + row) * p.h_q + h;
            p.ws_o[base * D + d] = s_o[e];
            if (d == 0) {
                p.ws_ml[base * 2] = s_m[r];
                p.ws_ml[base * 2 + 1] = s_l[r];
            }
        }
    }
}

// Combine the splits of every (row, head): O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
template <bool BF16, int D>
__global__ void __launch_bounds__(128) attn_merge_kernel(const AttnParams p) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int row = (int)(gw / p.h_q), h = (int)(gw % p.h_q);
    const int total = __ldg(p.q_start + p.batch);
    if (row >= total || row >= p.rows_cap) return;
    float M = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s)
        M = fmaxf(M, p.ws_ml[(((int64_t)s * p.rows_cap + row) * p.h_q + h) * 2]);
    float den = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < p.n_splits; ++s) {
            const int64_t base = ((int64_t)s * p.rows_cap + row) * p.h_q + h;
            const float m = p.ws_ml[base * 2], l = p.ws_ml[base * 2 + 1];
            if (m == -INFINITY) continue;
            const float w = exp2f(m - M);
            den += w * l;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] += w * p.ws_o[base * D + lane * EPL + e];
        }
    }
    const int64_t oi = ((int64_t)row * p.h_q + h) * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        const float val = den > 0.f ? o[e] / den : 0.f;
        if (BF16)
            reinterpret_cast<unsigned short *>(p.out)[oi + e] = (unsigned short)f32_to_bf16_bits(val);
        else
            reinterpret_cast<float *>(p.out)[oi + e] = val;
    }
}

template <bool BF16, int D, int RB>
cudaError_t launch_simt_t(const AttnParams &p, const AttnPlan &plan, cudaStream_t s) {
    const size_t dyn = p.kind == SD_ATTN_SPARSE ? (size_t)p.k_sel * sizeof(int) : 0;
    auto kern = attn_simt_kernel<BF16, D, RB>;
    if (dyn > 16 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)dyn);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(p.n_splits * plan.n_rowblocks, p.kv.h_kv, p.batch);
    kern<<<grid, kThreads, dyn, s>>>(p);
    return cudaGetLastError();
}

template <bool BF16, int D>
cudaError_t launch_merge_t(const AttnParams &p, cudaStream_t s) {
    const int64_t warps = (int64_t)p.rows_cap * p.h_q;
    const int blocks = (int)((warps + 3) / 4);
    attn_merge_kernel<BF16, D><<<blocks, 128, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_simt(const AttnParams &p, const AttnPlan &plan, cudaStream_t s) {
    const bool bf = p.kv.dtype == SD_BF16;
    const int D = p.kv.head_dim;
    const int RB = plan.rows_per_block;
    if (bf && D == 128) return RB == 8 ? launch_simt_t<true, 128, 8>(p, plan, s)
                                       : launch_simt_t<true, 128, 16>(p, plan, s);
    if (bf && D == 64) return RB == 8 ? launch_simt_t<true, 64, 8>(p, plan, s)
                                      : launch_simt_t<true, 64, 16>(p, plan, s);
    if (!bf && D == 128) return RB == 8 ? launch_simt_t<false, 128, 8>(p, plan, s)
                                        : launch_simt_t<false, 128, 16>(p, plan, s);
    return RB == 8 ? launch_simt_t<false, 64, 8>(p, plan, s)
                   : launch_simt_t<false, 64, 16>(p, plan, s);
}

cudaError_t launch_attention_merge(const AttnParams &p, cudaStream_t s) {
    const bool bf = p.kv.dtype == SD_BF16;
    if (p.kv.head_dim == 128) return bf ? launch_merge_t<true, 128>(p, s) : launch_merge_t<false, 128>(p, s);
    return bf ? launch_merge_t<true, 64>(p, s) : launch_merge_t<false, 64>(p, s);
}

}  // namespace sd
