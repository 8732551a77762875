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
//   sparse          the selected indices (ascending), then [tail_begin, kv_len)
// K and V rows of 64-position tiles are copied with 16-byte cp.async into a 3-stage
// shared-memory ring (rows gathered through the position map, chunks XOR-swizzled so that
// both the row-per-thread and the lanes-over-head_dim reads are conflict-free), so the copies
// of the next two tiles overlap the arithmetic of the current one.  Per tile (256 threads,
// 64 positions): four threads per position score it against a quarter of the RB rows each
// (packed fp32 FMA, query rows broadcast from shared memory); one warp per row updates the
// running max / sum (online softmax, base 2); then each warp accumulates P.V over an eighth
// of the positions with lanes spread over head_dim.  The warps' partial outputs are summed in a fixed order (deterministic).  With
// one split the normalised output is written directly; otherwise the unnormalised partial and
// its (max, sum) go to the workspace and attn_merge_kernel combines the splits by their
// log-sum-exp.
#include "attn_stream.cuh"

namespace sd {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;    // positions per tile
constexpr int kStages = 3;  // cp.async ring depth

template <bool BF16, int D>
struct SimtCfg {
    static constexpr int ESZ = BF16 ? 2 : 4;
    static constexpr int ROWB = D * ESZ;               // bytes per KV row
    static constexpr int CH = ROWB / 16;               // 16-byte chunks per row
    static constexpr int SWZ = CH < 16 ? CH - 1 : 15;  // chunk swizzle mask
    static constexpr int TILEB = kTile * ROWB;         // one K (or V) tile
    static constexpr int DYN = kStages * 2 * TILEB;    // dynamic shared memory
};

__device__ __forceinline__ uint32_t smem_u32(const void *ptr) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool BF16, int D, int RB>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(const AttnParams p) {
    using C = SimtCfg<BF16, D>;
    using CHK = Chunk<BF16>;
    constexpr int EPL = D / 32;                  // head_dim elements per lane in the P.V phase
    constexpr int PARTS = kThreads / kTile;       // threads sharing one position's scores
    constexpr int RH = RB / PARTS;                // rows per thread in the score phase
    constexpr int NW = kThreads / 32;
    static_assert(RB % PARTS == 0 && RH % 2 == 0 && kThreads % kTile == 0, "tile shapes");

    extern __shared__ __align__(128) uint8_t s_kv[];  // [stage][K | V][kTile][ROWB]
    __shared__ __align__(16) float s_q[RB][D];         // pre-scaled rows; output buffer at the end
    __shared__ __align__(16) float s_s[RB][kTile];
    __shared__ __align__(16) float s_p[kTile][RB];
    __shared__ int64_t s_off[kStages][kTile];
    __shared__ int s_pos[kStages][kTile];
    __shared__ int s_lo1[RB], s_hi1[RB], s_lo2[RB], s_hi2[RB];
    __shared__ float s_m[RB], s_l[RB], s_corr[RB];
    __shared__ int s_stream[4 + kThreads / 32];

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

    const StreamInfo si = stream_setup<kThreads>(p, b, g, n_q, kv_len, s_stream);

    // Per-row allowed ranges, running statistics and the pre-scaled query rows.
    if (tid < RB) {
        const int r = tid;
        int lo1, hi1, lo2, hi2;
        row_ranges(p, si, rb * RB + r, R, n_q, kv_len, lo1, hi1, lo2, hi2);
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
    const int len0 = si.len0, len1 = si.len1;
    const int64_t P = (int64_t)len0 + len1;
    const int c0 = (int)(P * split / p.n_splits), c1 = (int)(P * (split + 1) / p.n_splits);
    const int n_tiles = (c1 - c0 + kTile - 1) / kTile;

    // Physical position and element offset of every slot of tile u (threads < kTile).
    auto map_tile = [&](int u) {
        const int pl = c0 + u * kTile + tid;
        int j = pl < c1 ? stream_position(p, si, pl, kv_len) : -1;
        int64_t off = -1;
        if (j >= 0) {
            off = kv_row_offset(kv, b, g, j, p.dev_err);
            if (off < 0) j = -1;
        }
        s_pos[u % kStages][tid] = j;
        s_off[u % kStages][tid] = j >= 0 ? off : -1;
    };
    // Asynchronous copies of the K and V rows of tile u.
    auto issue_tile = [&](int u) {
        const int st = u % kStages;
        const uint32_t kdst = smem_u32(s_kv) + st * 2 * C::TILEB;
        const uint32_t vdst = kdst + C::TILEB;
        const char *kbase = reinterpret_cast<const char *>(kv.k);
        const char *vbase = reinterpret_cast<const char *>(kv.v);
        for (int e = tid; e < kTile * C::CH; e += kThreads) {
            const int row = e / C::CH, ch = e % C::CH;
            const int64_t off = s_off[st][row];
            if (off < 0) continue;
            const uint32_t d = row * C::ROWB + ((ch ^ (row & C::SWZ)) << 4);
            cp_async16(kdst + d, kbase + off * C::ESZ + ch * 16);
            cp_async16(vdst + d, vbase + off * C::ESZ + ch * 16);
        }
    };

    float acc[RB][EPL];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[r][e] = 0.f;

    for (int u = 0; u < kStages - 1; ++u) {
        if (u < n_tiles && tid < kTile) map_tile(u);
        __syncthreads();
        if (u < n_tiles) issue_tile(u);
        cp_async_commit();
    }

    for (int t = 0; t < n_tiles; ++t) {
        const int u = t + kStages - 1;
        if (u < n_tiles && tid < kTile) map_tile(u);
        cp_async_wait<kStages - 2>();
        __syncthreads();
        if (u < n_tiles) issue_tile(u);
        cp_async_commit();
        const int st = t % kStages;
        const uint8_t *ktile = s_kv + st * 2 * C::TILEB;
        const uint8_t *vtile = ktile + C::TILEB;

        // ---- scores: PARTS threads per position, RH rows each ----
        {
            const int prow = tid % kTile, half = tid / kTile;  // half: which RH-row slice
            const int j = s_pos[st][prow];
            float2 sc[RH];
#pragma unroll
            for (int r = 0; r < RH; ++r) sc[r] = make_float2(0.f, 0.f);
            if (j >= 0) {
                const uint8_t *krow = ktile + prow * C::ROWB;
#pragma unroll
                for (int ch = 0; ch < C::CH; ++ch) {
                    const uint4 raw =
                        *reinterpret_cast<const uint4 *>(krow + ((ch ^ (prow & C::SWZ)) << 4));
                    float f[CHK::kElems];
                    CHK::to_float(raw, f);
                    const int e0 = ch * CHK::kElems;
#pragma unroll
                    for (int r = 0; r < RH; ++r) {
#pragma unroll
                        for (int e = 0; e < CHK::kElems; e += 4) {
                            const float4 qv =
                                *reinterpret_cast<const float4 *>(&s_q[half * RH + r][e0 + e]);
                            sc[r] = __ffma2_rn(make_float2(qv.x, qv.y),
                                               make_float2(f[e], f[e + 1]), sc[r]);
                            sc[r] = __ffma2_rn(make_float2(qv.z, qv.w),
                                               make_float2(f[e + 2], f[e + 3]), sc[r]);
                        }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RH; ++r) {
                const int rr = half * RH + r;
                const bool ok = j >= 0 && ((j >= s_lo1[rr] && j <= s_hi1[rr]) ||
                                           (j >= s_lo2[rr] && j <= s_hi2[rr]));
                s_s[rr][prow] = ok ? sc[r].x + sc[r].y : -INFINITY;
            }
        }
        __syncthreads();

        // ---- online softmax: one warp per row ----
        for (int r = warp; r < RB; r += NW) {
            float v0 = s_s[r][lane], v1 = s_s[r][lane + 32];
            const float tmax = warp_max(fmaxf(v0, v1));
            const float m_old = s_m[r];
            const float m_new = fmaxf(m_old, tmax);
            float corr = 1.f, sum = 0.f;
            if (m_new != -INFINITY) {
                corr = exp2f(m_old - m_new);
                v0 = exp2f(v0 - m_new);
                v1 = exp2f(v1 - m_new);
                sum = v0 + v1;
            } else {
                v0 = v1 = 0.f;
            }
            s_p[lane][r] = v0;
            s_p[lane + 32][r] = v1;
            sum = warp_sum(sum);
            if (lane == 0) {
                s_l[r] = s_l[r] * corr + sum;
                s_m[r] = m_new;
                s_corr[r] = corr;
            }
        }
        __syncthreads();

        // ---- P.V: warp w takes positions w, w+NW, ...; lanes spread over head_dim ----
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const float cr = s_corr[r];
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[r][e] *= cr;
        }
        {
            constexpr int LANEB = EPL * C::ESZ;  // bytes per lane in a V row
            const int lb = lane * LANEB;
#pragma unroll 2
            for (int t0 = warp; t0 < kTile; t0 += NW * 4) {
                float vf[4][EPL];
                bool have[4];
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4) {
                    const int pp = t0 + NW * u4;
                    have[u4] = s_pos[st][pp] >= 0;
                    const uint8_t *src = vtile + pp * C::ROWB +
                                         ((((lb >> 4) ^ (pp & C::SWZ)) << 4) | (lb & 15));
                    if (BF16) {
                        if (EPL == 4) {
                            const uint2 w2 = *reinterpret_cast<const uint2 *>(src);
                            vf[u4][0] = bf16_lo(w2.x);
                            vf[u4][1] = bf16_hi(w2.x);
                            vf[u4][2] = bf16_lo(w2.y);
                            vf[u4][3] = bf16_hi(w2.y);
                        } else {
                            const uint32_t w1 = *reinterpret_cast<const uint32_t *>(src);
                            vf[u4][0] = bf16_lo(w1);
                            vf[u4][1] = bf16_hi(w1);
                        }
                    } else {
                        if (EPL == 4) {
                            const float4 f4 = *reinterpret_cast<const float4 *>(src);
                            vf[u4][0] = f4.x;
                            vf[u4][1] = f4.y;
                            vf[u4][2] = f4.z;
                            vf[u4][3] = f4.w;
                        } else {
                            const float2 f2 = *reinterpret_cast<const float2 *>(src);
                            vf[u4][0] = f2.x;
                            vf[u4][1] = f2.y;
                        }
                    }
                }
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4) {
                    if (!have[u4]) continue;
                    const int pp = t0 + NW * u4;
#pragma unroll
                    for (int r4 = 0; r4 < RB; r4 += 4) {
                        const float4 pv = *reinterpret_cast<const float4 *>(&s_p[pp][r4]);
                        const float pr[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
#pragma unroll
                            for (int e = 0; e < EPL; e += 2) {
                                float2 a = make_float2(acc[r4 + q][e], acc[r4 + q][e + 1]);
                                a = __ffma2_rn(make_float2(pr[q], pr[q]),
                                               make_float2(vf[u4][e], vf[u4][e + 1]), a);
                                acc[r4 + q][e] = a.x;
                                acc[r4 + q][e + 1] = a.y;
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    // ---- sum the warps' partial outputs in a fixed order (into s_q) ----
    float *s_o = &s_q[0][0];  // [RB][D]
    __syncthreads();
    for (int w = 0; w < NW; ++w) {
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
// One warp per (sequence, row of the sequence, head), so a row's sequence is known without a
// search.  Lanes read the splits' statistics in parallel, and the first four splits' partial
// outputs are loaded in the same round trip (their weights are applied once the maximum is
// known).
template <bool BF16, int D>
__global__ void __launch_bounds__(128) attn_merge_kernel(const AttnParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    constexpr int EPL = D / 32;
    constexpr int kPre = 4;  // splits whose outputs are loaded with the statistics
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int64_t per_seq = (int64_t)p.max_q_rows * p.h_q;
    const int b = (int)(gw / per_seq);
    if (b >= p.batch) return;
    const int i = (int)((gw % per_seq) / p.h_q), h = (int)(gw % p.h_q);
    const int q0 = __ldg(p.q_start + b);
    if (i >= __ldg(p.q_start + b + 1) - q0) return;
    const int row = q0 + i;
    if (row >= p.rows_cap) return;
    const int64_t stride = (int64_t)p.rows_cap * p.h_q;  // between splits, in (row, head) units
    const int64_t rh = (int64_t)row * p.h_q + h;
    int n_splits = p.n_splits;
    if (p.persist_s) {
        // Persistent tensor-core decomposition: the CTAs whose item ranges meet the row's unit
        // wrote slots 0.. in order; a unit inside one CTA's range has its output already.
        const long long n_items = (long long)p.batch * p.kv.h_kv * p.persist_s;
        const long long base = ((long long)b * p.kv.h_kv + h / p.group) * p.persist_s;
        const int c0 = (int)(((base + 1) * p.persist_g - 1) / n_items);
        const int c1 = (int)(((base + p.persist_s) * p.persist_g - 1) / n_items);
        if (c1 == c0) return;
        n_splits = min(c1 - c0 + 1, p.n_splits);
    }
    float ov[kPre][EPL];
#pragma unroll
    for (int k = 0; k < kPre; ++k)
#pragma unroll
        for (int e = 0; e < EPL; ++e)
            ov[k][e] = k < n_splits ? p.ws_o[((int64_t)k * stride + rh) * D + lane * EPL + e] : 0.f;
    float M = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, p.ws_ml[(s * stride + rh) * 2]);
    M = warp_max(M);
    float o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
        for (int s0 = 0; s0 < n_splits; s0 += 32) {
            const int s = s0 + lane;
            float w = 0.f, l = 0.f;
            if (s < n_splits) {
                const float m = p.ws_ml[(s * stride + rh) * 2];
                l = p.ws_ml[(s * stride + rh) * 2 + 1];
                w = m == -INFINITY ? 0.f : exp2f(m - M);
            }
            den += warp_sum(w * l);
            const int n = min(32, n_splits - s0);
            int k = 0;
            if (s0 == 0) {  // the preloaded splits
#pragma unroll
                for (int q = 0; q < kPre; ++q) {
                    const float wq = __shfl_sync(0xffffffffu, w, q);
                    if (q < n)
#pragma unroll
                        for (int e = 0; e < EPL; ++e) o[e] += wq * ov[q][e];
                }
                k = min(kPre, n);
            }
            for (; k < n; ++k) {
                const float wk = __shfl_sync(0xffffffffu, w, k);
                const float *src = p.ws_o + ((s0 + k) * stride + rh) * D + lane * EPL;
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[e] += wk * src[e];
            }
        }
    }
    const int64_t oi = rh * D + lane * EPL;
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
    const size_t dyn = SimtCfg<BF16, D>::DYN;
    auto kern = attn_simt_kernel<BF16, D, RB>;
    cudaError_t e = set_max_dynamic_smem<attn_simt_kernel<BF16, D, RB>>((int)dyn);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits * plan.n_rowblocks, p.kv.h_kv, p.batch);
    kern<<<grid, kThreads, dyn, s>>>(p);
    return cudaGetLastError();
}

template <bool BF16, int D>
cudaError_t launch_merge_t(const AttnParams &p, cudaStream_t s) {
    const int64_t warps = (int64_t)p.rows_cap * p.h_q;
    const int blocks = (int)((warps + 3) / 4);
    return launch_pdl(attn_merge_kernel<BF16, D>, dim3(blocks), dim3(128), 0, s, p);
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
