// Hidden-state-reuse projection: y = W [emb ; hid] (+ bias), bf16 in/out, fp32 accumulation.
//
// A weight-streaming GEMV with n_rows <= 16 right-hand sides, balanced so that every SM
// streams the same number of weight bytes: one CTA per SM owns an even share of the output
// features [r0, r1) and splits each weight row into four quarter-rows (items); one partial per
// (feature, quarter) is stored and the four are summed in a fixed order (deterministic).  The
// input rows are copied once per CTA into shared memory as the concatenation [emb ; hid] (the
// concatenation only ever exists there).  Weights are read once per group of up to four input
// rows.
//
// Ring kernel (the weight share's items are contiguous in memory): stage u holds items
// [16u, 16u + 16), one bulk copy issued by a copy warp up to S stages ahead (full / empty
// mbarriers per stage; 56 KB per stage for d_model = 3584), so the copies stream
// continuously; warp w dots item 16u + w with the input rows and releases its share of the
// stage.
// Fallback kernel (rows too large for a ring of at least two stages): the 16 warps take the
// items round-robin, two at a time (14 coalesced 16-byte loads per lane in flight).
#include "sd_internal.h"
#include "tc_ptx.cuh"

namespace sd {
namespace {

constexpr int kWarps = 16;
constexpr int kParts = 4;  // quarter-rows per weight row

template <int NR>
__global__ void __launch_bounds__(kWarps * 32)
hsr_kernel(const uint16_t *emb, const uint16_t *hid, int n_rows, int d_model, const uint16_t *w,
           const uint16_t *bias, uint16_t *y, int max_rows_per_cta) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    extern __shared__ uint4 s_x4[];  // [NR][2*d_model] bf16 chunks, then [rows][kParts][NR] f32
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g0 = blockIdx.y * NR;
    const int nr = min(NR, n_rows - g0);
    const int cpr = 2 * d_model / 8;    // 16-byte chunks per weight row
    const int cpp = cpr / kParts;       // chunks per quarter-row
    const int r0 = (int)((int64_t)d_model * blockIdx.x / gridDim.x);
    const int r1 = (int)((int64_t)d_model * (blockIdx.x + 1) / gridDim.x);
    float *s_part = reinterpret_cast<float *>(s_x4 + NR * cpr);
    for (int e = tid; e < NR * cpr; e += kWarps * 32) {
        const int r = e / cpr, c = e % cpr;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < nr) {
            const int col = c * 8;
            const uint16_t *src = col < d_model ? emb + (int64_t)(g0 + r) * d_model + col
                                                : hid + (int64_t)(g0 + r) * d_model + (col - d_model);
            v = *reinterpret_cast<const uint4 *>(src);
        }
        s_x4[e] = v;
    }
    __syncthreads();
    const int items = (r1 - r0) * kParts;
    const uint4 *wbase = reinterpret_cast<const uint4 *>(w) + (int64_t)r0 * cpr;
    for (int it0 = warp; it0 < items; it0 += 2 * kWarps) {
        const int it1 = it0 + kWarps;  // second item of the pair (may not exist)
        float part[2][NR];
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int r = 0; r < NR; ++r) part[k][r] = 0.f;
        for (int c0 = lane; c0 < cpp; c0 += 32 * 7) {
            uint4 wv[2][7];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int it = k == 0 ? it0 : it1;
#pragma unroll
                for (int u = 0; u < 7; ++u) {
                    const int c = c0 + 32 * u;
                    wv[k][u] = (it < items && c < cpp)
                                   ? ldg_stream16(wbase + (int64_t)(it / kParts) * cpr +
                                                  (it % kParts) * cpp + c)
                                   : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int it = k == 0 ? it0 : it1;
                if (it >= items) break;
#pragma unroll
                for (int u = 0; u < 7; ++u) {
                    const int c = c0 + 32 * u;
                    if (c >= cpp) break;
                    float wf[8];
                    Chunk<true>::to_float(wv[k][u], wf);
                    const int col = (it % kParts) * cpp + c;
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        float xf[8];
                        Chunk<true>::to_float(s_x4[r * cpr + col], xf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) part[k][r] = fmaf(wf[e], xf[e], part[k][r]);
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int it = k == 0 ? it0 : it1;
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const float sum = warp_sum(part[k][r]);
                if (lane == 0 && it < items) s_part[(it * NR) + r] = sum;
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < nr * (r1 - r0); e += kWarps * 32) {
        const int r = e / (r1 - r0), i = e % (r1 - r0);
        float val = 0.f;
#pragma unroll
        for (int q = 0; q < kParts; ++q) val += s_part[((i * kParts + q) * NR) + r];
        if (bias) val += __uint_as_float((uint32_t)bias[r0 + i] << 16);
        y[(int64_t)(g0 + r) * d_model + r0 + i] = (uint16_t)f32_to_bf16_bits(val);
    }
}

constexpr int kRingWarps = 16;                     // consumer warps: one item each per stage
constexpr int kRingThreads = (kRingWarps + 1) * 32;  // + the copy warp
constexpr size_t kRingSmemMax = 227 * 1024 - 256;  // (dynamic: the barriers are static)
constexpr unsigned long long kRingWaitNs = 1000000000ull;  // bound of every pipeline wait

template <int NR, int S>
__global__ void __launch_bounds__(kRingThreads, 1)
hsr_ring_kernel(const uint16_t *emb, const uint16_t *hid, int n_rows, int d_model,
                const uint16_t *w, const uint16_t *bias, uint16_t *y) {
    using namespace tc;
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    // [NR][cpr] input chunks, then the ring [S][16][cpp] chunks, then [items][NR] f32 partials
    extern __shared__ __align__(16) uint4 s_x4[];
    __shared__ __align__(8) uint64_t s_full[S], s_empty[S];
    __shared__ int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g0 = blockIdx.y * NR;
    const int nr = min(NR, n_rows - g0);
    const int cpr = 2 * d_model / 8;  // 16-byte chunks per weight row
    const int cpp = cpr / kParts;     // chunks per item (quarter-row)
    const int r0 = (int)((int64_t)d_model * blockIdx.x / gridDim.x);
    const int r1 = (int)((int64_t)d_model * (blockIdx.x + 1) / gridDim.x);
    const int items = (r1 - r0) * kParts;
    uint4 *ring = s_x4 + NR * cpr;
    float *s_part = reinterpret_cast<float *>(ring + (size_t)S * kRingWarps * cpp);
    const uint4 *wbase = reinterpret_cast<const uint4 *>(w) + (int64_t)r0 * cpr;
    const int n_stages = (items + kRingWarps - 1) / kRingWarps;
    if (tid == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(saddr(&s_full[st]), 1);
            mbar_init(saddr(&s_empty[st]), kRingWarps);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort_flag = &s_abort;
    int n_issued = 0;
    if (warp == kRingWarps) {
        // ---- copy warp: stage u (items [16u, 16u + 16), contiguous) is one bulk copy ----
        if (lane == 0) {
            for (int u = 0; u < n_stages; ++u) {
                const int st = u % S;
                if (u >= S && !mbar_wait(saddr(&s_empty[st]), ((u / S) - 1) & 1, abort_flag,
                                         nullptr, kRingWaitNs))
                    break;
                const int i0 = u * kRingWarps;
                const uint32_t bytes = (uint32_t)(min(kRingWarps, items - i0) * cpp * 16);
                mbar_arrive_tx(saddr(&s_full[st]), bytes);
                bulk_load(saddr(ring + (size_t)st * kRingWarps * cpp), wbase + (int64_t)i0 * cpp,
                          bytes, saddr(&s_full[st]));
                n_issued = u + 1;
                if (*abort_flag) break;
            }
        }
    } else {
        for (int e = tid; e < NR * cpr; e += kRingWarps * 32) {
            const int r = e / cpr, c = e % cpr;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < nr) {
                const int col = c * 8;
                const uint16_t *src = col < d_model
                                          ? emb + (int64_t)(g0 + r) * d_model + col
                                          : hid + (int64_t)(g0 + r) * d_model + (col - d_model);
                v = *reinterpret_cast<const uint4 *>(src);
            }
            s_x4[e] = v;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kRingWarps * 32) : "memory");  // input rows in
        for (int u = 0; u < n_stages; ++u) {
            const int st = u % S;
            const bool got =
                mbar_wait(saddr(&s_full[st]), (u / S) & 1, abort_flag, nullptr, kRingWaitNs);
            if (!__all_sync(0xffffffffu, got)) break;  // (the warp leaves together)
            const int it = u * kRingWarps + warp;
            if (it < items) {
                const uint4 *wr = ring + (size_t)st * kRingWarps * cpp + (size_t)warp * cpp;
                const int col0 = (it % kParts) * cpp;
                float part[NR];
#pragma unroll
                for (int r = 0; r < NR; ++r) part[r] = 0.f;
                for (int c = lane; c < cpp; c += 32) {
                    float wf[8];
                    Chunk<true>::to_float(wr[c], wf);
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        float xf[8];
                        Chunk<true>::to_float(s_x4[r * cpr + col0 + c], xf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) part[r] = fmaf(wf[e], xf[e], part[r]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(saddr(&s_empty[st]));  // the item is read
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float sum = warp_sum(part[r]);
                    if (lane == 0) s_part[it * NR + r] = sum;
                }
            } else if (lane == 0) {
                mbar_arrive(saddr(&s_empty[st]));
            }
        }
    }
    // ---- teardown: after an abort, the copy lane waits (bounded) for its copies in flight ----
    if (warp == kRingWarps && lane == 0 && *abort_flag) {
        const unsigned long long t0 = now_ns();
        for (int u = (n_issued > S ? n_issued - S : 0); u < n_issued; ++u)
            while (!mbar_try(saddr(&s_full[u % S]), (u / S) & 1) && now_ns() - t0 < kDrainNs) {
            }
    }
    __syncthreads();
    for (int e = tid; e < nr * (r1 - r0); e += kRingThreads) {
        const int r = e / (r1 - r0), i = e % (r1 - r0);
        float val = 0.f;
#pragma unroll
        for (int q = 0; q < kParts; ++q) val += s_part[((i * kParts + q) * NR) + r];
        if (bias) val += __uint_as_float((uint32_t)bias[r0 + i] << 16);
        y[(int64_t)(g0 + r) * d_model + r0 + i] = (uint16_t)f32_to_bf16_bits(val);
    }
}

template <int NR, int S>
cudaError_t launch_ring_t(const void *emb, const void *hid, int n_rows, int d_model,
                          const void *w, const void *bias, void *y, size_t smem, int ctas,
                          cudaStream_t s) {
    auto kern = hsr_ring_kernel<NR, S>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ctas, (n_rows + NR - 1) / NR);
    return launch_pdl(kern, grid, dim3(kRingThreads), smem, s,
                      reinterpret_cast<const uint16_t *>(emb),
                      reinterpret_cast<const uint16_t *>(hid), n_rows, d_model,
                      reinterpret_cast<const uint16_t *>(w),
                      reinterpret_cast<const uint16_t *>(bias), reinterpret_cast<uint16_t *>(y));
}

template <int NR>
cudaError_t launch_hsr_t(const void *emb, const void *hid, int n_rows, int d_model, const void *w,
                         const void *bias, void *y, cudaStream_t s) {
    const int ctas = min(device_sm_count(), d_model);
    const int max_rows = (d_model + ctas - 1) / ctas;
    {
        // ring: as many stages (2..4) as fit next to the input rows and the partials
        const size_t fixed = (size_t)NR * 2 * d_model * sizeof(uint16_t) +
                             (size_t)max_rows * kParts * NR * sizeof(float);
        const size_t stage = (size_t)kRingWarps * (2 * d_model / 8 / kParts) * 16;
        const int S = fixed < kRingSmemMax ? (int)min((size_t)4, (kRingSmemMax - fixed) / stage)
                                           : 0;
        if (S >= 2) {
            const size_t smem = fixed + (size_t)S * stage;
            auto ring = S == 2 ? launch_ring_t<NR, 2>
                        : S == 3 ? launch_ring_t<NR, 3>
                                 : launch_ring_t<NR, 4>;
            return ring(emb, hid, n_rows, d_model, w, bias, y, smem, ctas, s);
        }
    }
    const size_t smem = (size_t)NR * 2 * d_model * sizeof(uint16_t) +
                        (size_t)max_rows * kParts * NR * sizeof(float);
    auto kern = hsr_kernel<NR>;
    if (smem > 48 * 1024) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(ctas, (n_rows + NR - 1) / NR);
    return launch_pdl(kern, grid, dim3(kWarps * 32), smem, s,
                      reinterpret_cast<const uint16_t *>(emb),
                      reinterpret_cast<const uint16_t *>(hid), n_rows, d_model,
                      reinterpret_cast<const uint16_t *>(w),
                      reinterpret_cast<const uint16_t *>(bias), reinterpret_cast<uint16_t *>(y),
                      max_rows);
}

}  // namespace

cudaError_t launch_hsr(const void *emb, const void *hid, int n_rows, int d_model, const void *w,
                       const void *bias, void *y, cudaStream_t s) {
    if (n_rows == 1) return launch_hsr_t<1>(emb, hid, n_rows, d_model, w, bias, y, s);
    if (n_rows == 2) return launch_hsr_t<2>(emb, hid, n_rows, d_model, w, bias, y, s);
    return launch_hsr_t<4>(emb, hid, n_rows, d_model, w, bias, y, s);
}

}  // namespace sd
