// Sparse-to-Dense's own KV selection score, computed at prefill: the mean attention weight that
// the text tokens give each candidate key, per layer (sequence) and KV head.  The text rows are
// the last n_q positions of the cache; row i (position kv_len - n_q + i) attends causally with
// its own softmax over every position it sees, and the score of key j averages its weight over
// the n_q rows and the G query heads of the KV head.  The keys of the scores then go through the
// top-K selection kernel shared with the query-key mode.
//
// Two passes, both a dense contraction of the text rows with the keys, on tcgen05 for bf16
// caches with head_dim 64 or 128:
//   1. text_lse_tc_kernel    grid (G x row tiles, KV heads, sequences).  S = Q K^T with
//      M = 128 text rows of one query head (Q in shared memory, loaded once), N = 128 positions
//      per tile streamed by TMA through a 2-stage ring; each thread owns one row (one TMEM lane)
//      and keeps its running max and sum over the positions its row sees.  Output: the row's
//      log-sum-exp in log2 units of the scaled score.
//   2. text_colsum_tc_kernel grid (key tiles, KV heads, sequences).  S^T = K Q^T with M = 128
//      candidate keys (loaded once by TMA) and N = 128 text rows per tile (the G heads' row tiles
//      in turn, copied by the same threads with cp.async, double-buffered); each thread owns
//      one key and sums 2^(s - lse_row) over the tile's columns, so no reduction crosses
//      threads.  Per tile the sum is fp32 (128 terms in [0, 1]), across tiles fp64.
// Every tile runs two MMA groups deep: the tensor core computes tile t+1 while the threads
// exponentiate tile t (double-buffered S in TMEM).  Every mbarrier wait is bounded (1 s); on
// expiry the CTA records SD_DEVERR_TIMEOUT, drains its own copies and MMAs and exits.
// Other caches (fp32, or layouts the copy engine cannot describe) use CUDA-core kernels with
// the same two passes.
#include "topk_common.cuh"
#include "tc_ptx.cuh"

namespace sd {
namespace {

using namespace tc;

constexpr int kTT = 128;             // rows (pass 1) / keys (pass 2) per tile, and MMA M and N
constexpr int kTaThreads = 192;      // warps 0-3 compute, 4 copy producer, 5 MMA issuer
constexpr int kTaProducer = 4;
constexpr int kTaMma = 5;
constexpr uint32_t kTaTmemCols = 256;  // two 128-column S buffers
constexpr uint32_t kHalf = kTT * 128;  // bytes of one 64-column half of a 128-row bf16 tile

template <int D>
struct TaCfg {
    static constexpr int kTileBytes = kTT * D * 2;
    static constexpr int kStages = 2;  // pass-1 K ring (two CTAs per SM)
    // pass 1: Q tile, K ring, barriers
    static constexpr int kSmem1 = (1 + kStages) * kTileBytes + 256 + 1024;
    // pass 2: K tile, two Q tiles, three lse rows, barriers
    static constexpr int kSmem2 = 3 * kTileBytes + 3 * kTT * 4 + 256 + 1024;
};

// Row r of a 128-row tile, 16-byte chunk c of its d elements: the 128-byte-swizzled K-major
// layout the MMA descriptors describe (64-element halves 16 KB apart, 128 bytes per row,
// chunk index XOR row % 8 within each 1024-byte atom).
__device__ __forceinline__ uint32_t swz_off(int r, int c) {
    return (uint32_t)((c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Copy producer: K tiles [p0, p0 + 128) of (b, g) into the stage at dst through TMA; paged
// caches one box per 16-position page (positions past kv_len read an out-of-range page: zeros).
template <int D, bool PAGED>
__device__ __forceinline__ void load_k_tile(const TcMaps &maps, const KVView &kv, int b, int g,
                                            int p0, int kv_len, uint32_t dst, uint32_t bar,
                                            int32_t *dev_err) {
    constexpr int H = D / 64;
    mbar_arrive_tx(bar, TaCfg<D>::kTileBytes);
    if (!PAGED) {
#pragma unroll
        for (int h = 0; h < H; ++h) tma_load_4d(dst + h * kHalf, &maps.k, bar, h * 64, p0, g, b);
    } else {
        for (int pg = 0; pg < kTT / kPageSize; ++pg) {
            const int pos = p0 + pg * kPageSize;
            int page = kv.num_pages;
            if (pos >= 0 && pos < kv_len) {
                const int e = __ldg(kv.block_table + (int64_t)b * kv.max_pages + pos / kPageSize);
                if (e >= 0 && e < kv.num_pages)
                    page = e;
                else
                    set_dev_err(dev_err, SD_DEVERR_PAGE);
            }
#pragma unroll
            for (int h = 0; h < H; ++h)
                tma_load_4d(dst + h * kHalf + pg * kPageSize * 128, &maps.k, bar, h * 64, 0, g,
                            page);
        }
    }
}

// ---------------------------------------------------------------- pass 1: row lse ----------

template <int D, bool PAGED>
__global__ void __launch_bounds__(kTaThreads, 2)
text_lse_tc_kernel(const TopkParams p, const __grid_constant__ TcMaps maps) {
    using C = TaCfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = smem + C::kTileBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (1 + S) * C::kTileBytes);
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int KF = 0, KE = S, SF = 2 * S, SE = 2 * S + 2, QF = 2 * S + 4, DR = 2 * S + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y;
    const int G = p.group;
    const int n_rt = (p.max_q_rows + kTT - 1) / kTT;
    const int hh = blockIdx.x / n_rt, rt = blockIdx.x % n_rt;
    const int h = g * G + hh;
    const KVView &kv = p.kv;
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    if (n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (PAGED && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0 && hh == 0 && rt == 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    const int row0 = rt * kTT;
    if (row0 >= n_q) return;
    const int rows = min(kTT, n_q - row0);
    // positions seen by the tile's last row: [0, hi)
    const int hi = kv_len - n_q + row0 + rows;
    const int n_tiles = (hi + kTT - 1) / kTT;

    if (warp == kTaMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kTaTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(BAR(KF + s), 1);
            mbar_init(BAR(KE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(SF + s), 1);
            mbar_init(BAR(SE + s), 128);
        }
        mbar_init(BAR(QF), 128);
        mbar_init(BAR(DR), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;

    int n_issued = 0;
    if (warp == kTaProducer) {
        if (lane == 0) {
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % S, use = t / S;
                if (t >= S && !mbar_wait(BAR(KE + s), (use - 1) & 1, abort_flag, p.dev_err, p.wait_ns))
                    break;
                load_k_tile<D, PAGED>(maps, kv, b, g, t * kTT, kv_len,
                                      saddr(sK + (size_t)s * C::kTileBytes), BAR(KF + s),
                                      p.dev_err);
                n_issued = t + 1;
                if (*abort_flag) break;
            }
        }
    } else if (warp == kTaMma) {
        const uint32_t idesc = idesc_bf16(kTT, false);
        bool issued = false;
        bool alive = true;
        if (lane == 0) alive = mbar_wait(BAR(QF), 0, abort_flag, p.dev_err, p.wait_ns);
        alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
        for (int t = 0; alive && t < n_tiles; ++t) {
            const int s = t % S, use = t / S, sb = t & 1;
            bool ok = true;
            if (lane == 0) {
                ok = mbar_wait(BAR(KF + s), use & 1, abort_flag, p.dev_err, p.wait_ns);
                if (ok && t >= 2) ok = mbar_wait(BAR(SE + sb), ((t >> 1) - 1) & 1, abort_flag,
                                                 p.dev_err, p.wait_ns);
            }
            alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!alive) break;
            tc_after();
            if (lane == 0) {
                const uint32_t qb = saddr(sQ), kb = saddr(sK + (size_t)s * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                    mma_ss(tmem + sb * kTT, desc_k_sw128(qb + off), desc_k_sw128(kb + off), idesc,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(SF + sb));
                mma_commit(BAR(KE + s));
                issued = true;
            }
            __syncwarp();
        }
        if (lane == 0 && issued) {
            mma_commit(BAR(DR));
            const unsigned long long t0 = now_ns();
            while (!mbar_try(BAR(DR), 0) && now_ns() - t0 < kDrainNs) {
            }
        }
        __syncwarp();
    } else {
        // ---- compute warps: thread r owns text row row0 + r (TMEM lane r) ----
        const int r = tid;
        const bool valid = r < rows;
        const int i = row0 + r;
        {  // the tile's query rows into shared memory (zeros past the sequence's rows)
            const uint4 *src = reinterpret_cast<const uint4 *>(
                reinterpret_cast<const unsigned short *>(p.q) +
                ((int64_t)(q0 + (valid ? i : 0)) * p.h_q + h) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 x = valid ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sQ + swz_off(r, c)) = x;
            }
            fence_async_smem();
            mbar_arrive(BAR(QF));
        }
        const int limit = kv_len - n_q + i;  // last position the row sees
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok_run = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int sb = t & 1;
            const bool got = mbar_wait(BAR(SF + sb), (t >> 1) & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(0xffffffffu, got)) {
                ok_run = false;
                break;
            }
            tc_after();
            const int p0 = t * kTT;
            const bool whole = p0 + kTT - 1 <= limit;
#pragma unroll
            for (int q = 0; q < kTT / 32; ++q) {
                float v[32];
                tmem_ld32(lane_base + sb * kTT + q * 32, v);
                float cm = -INFINITY;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const bool vis = whole || p0 + q * 32 + e <= limit;
                    v[e] = vis ? v[e] * sl2 : -INFINITY;
                    cm = fmaxf(cm, v[e]);
                }
                const float mn = fmaxf(m, cm);
                if (mn != -INFINITY) {  // (no position of the row seen yet otherwise)
                    float acc = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) acc += ex2(v[e] - mn);
                    l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + acc;
                    m = mn;
                }
            }
            tc_before();
            mbar_arrive(BAR(SE + sb));
        }
        if (ok_run && valid) {
            float lg;
            asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
            p.lse[(int64_t)(q0 + i) * p.h_q + h] = l > 0.f ? m + lg : INFINITY;
        }
    }

    // ---- teardown: the producer drains its own copies if the CTA aborted ----
    if (warp == kTaProducer && lane == 0 && *abort_flag) {
        const unsigned long long t0 = now_ns();
        for (int t = (n_issued > S ? n_issued - S : 0); t < n_issued; ++t) {
            const int s = t % S, use = t / S;
            while (!mbar_try(BAR(KF + s), use & 1) && now_ns() - t0 < kDrainNs) {
            }
        }
    }
    tc_before();
    __syncthreads();
    tc_after();
    if (warp == kTaMma)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTaTmemCols)
                     : "memory");
}

// ---------------------------------------------------------------- pass 2: column sums ------

template <int D, bool PAGED>
__global__ void __launch_bounds__(kTaThreads, 2)
text_colsum_tc_kernel(const TopkParams p, const __grid_constant__ TcMaps maps) {
    using C = TaCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem;
    uint8_t *sQ = smem + C::kTileBytes;                              // two Q tiles
    float *sL = reinterpret_cast<float *>(smem + 3 * C::kTileBytes);  // three lse rows
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 3 * C::kTileBytes + 3 * kTT * 4);
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int KF = 0, QF = 1, SF = 3, SE = 5, DR = 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y, kt = blockIdx.x;
    const int G = p.group;
    const KVView &kv = p.kv;
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    if (n_q < 1 || n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (PAGED && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0 && kt == 0 && n_q != 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    int cb, n;
    cand_range(p, b, cb, n);
    // key tiles start at the candidate range's start (its page boundary for paged caches)
    const int a = PAGED ? (cb & ~(kPageSize - 1)) : cb;
    const int k0 = a + kt * kTT;
    if (k0 >= cb + n) return;
    const int n_rt = (n_q + kTT - 1) / kTT;
    const int n_tiles = G * n_rt;  // (head, row tile) pairs, head-major

    if (warp == kTaMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kTaTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(BAR(KF), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(QF + s), 128);
            mbar_init(BAR(SF + s), 1);
            mbar_init(BAR(SE + s), 128);
        }
        mbar_init(BAR(DR), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;

    bool k_issued = false;
    if (warp == kTaProducer) {
        if (lane == 0) {
            load_k_tile<D, PAGED>(maps, kv, b, g, k0, kv_len, saddr(sK), BAR(KF), p.dev_err);
            k_issued = true;
        }
    } else if (warp == kTaMma) {
        const uint32_t idesc = idesc_bf16(kTT, false);
        bool issued = false;
        bool alive = true;
        if (lane == 0) alive = mbar_wait(BAR(KF), 0, abort_flag, p.dev_err, p.wait_ns);
        alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
        for (int u = 0; alive && u < n_tiles; ++u) {
            const int sb = u & 1;
            bool ok = true;
            if (lane == 0) {
                ok = mbar_wait(BAR(QF + sb), (u >> 1) & 1, abort_flag, p.dev_err, p.wait_ns);
                if (ok && u >= 2) ok = mbar_wait(BAR(SE + sb), ((u >> 1) - 1) & 1, abort_flag,
                                                 p.dev_err, p.wait_ns);
            }
            alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!alive) break;
            tc_after();
            if (lane == 0) {
                const uint32_t kb = saddr(sK), qb = saddr(sQ + (size_t)sb * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                    mma_ss(tmem + sb * kTT, desc_k_sw128(kb + off), desc_k_sw128(qb + off), idesc,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(SF + sb));
                issued = true;
            }
            __syncwarp();
        }
        if (lane == 0 && issued) {
            mma_commit(BAR(DR));
            const unsigned long long t0 = now_ns();
            while (!mbar_try(BAR(DR), 0) && now_ns() - t0 < kDrainNs) {
            }
        }
        __syncwarp();
    } else {
        // ---- compute warps: thread r owns key k0 + r (TMEM lane r) and copies row r of
        // every Q tile ----
        const int r = tid;
        auto load_tile = [&](int u) {  // Q rows and their lse of tile u, one cp.async group
            if (u < n_tiles) {
                const int hh = u / n_rt, rt = u % n_rt, hq = g * G + hh;
                const int i = rt * kTT + r;
                const uint32_t qd = saddr(sQ + (size_t)(u & 1) * C::kTileBytes);
                const uint32_t ld = saddr(sL + (u % 3) * kTT + r);
                if (i < n_q) {
                    const unsigned short *src = reinterpret_cast<const unsigned short *>(p.q) +
                                                ((int64_t)(q0 + i) * p.h_q + hq) * D;
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) cp_async16(qd + swz_off(r, c), src + 8 * c);
                    cp_async4(ld, p.lse + (int64_t)(q0 + i) * p.h_q + hq);
                } else {
#pragma unroll
                    for (int c = 0; c < D / 8; ++c)
                        *reinterpret_cast<uint4 *>(sQ + (size_t)(u & 1) * C::kTileBytes +
                                                   swz_off(r, c)) = make_uint4(0, 0, 0, 0);
                    sL[(u % 3) * kTT + r] = INFINITY;  // no weight from a missing row
                }
            }
            cp_async_commit();
        };
        load_tile(0);
        load_tile(1);
        const int key = k0 + r;
        const bool key_ok = key >= cb && key < cb + n;
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        double total = 0.0;
        bool ok_run = true;
        for (int u = 0; u < n_tiles; ++u) {
            const int sb = u & 1;
            cp_async_wait<1>();  // this thread's part of tile u has landed
            fence_async_smem();
            mbar_arrive(BAR(QF + sb));
            // every thread's part of tile u has landed (and every thread is done with tile
            // u - 1, whose lse buffer the copy of tile u + 2 reuses), then S^T of tile u
            const bool got = mbar_wait(BAR(QF + sb), (u >> 1) & 1, abort_flag, p.dev_err, p.wait_ns) &&
                             mbar_wait(BAR(SF + sb), (u >> 1) & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(0xffffffffu, got)) {
                ok_run = false;
                break;
            }
            tc_after();
            const int rt = u % n_rt;
            // row c of the tile sees this key iff key <= kv_len - n_q + rt*128 + c
            const int cmin = key - (kv_len - n_q) - rt * kTT;
            const float *lse = sL + (u % 3) * kTT;
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < kTT / 32; ++q) {
                float v[32];
                tmem_ld32(lane_base + sb * kTT + q * 32, v);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 lv = *reinterpret_cast<const float4 *>(lse + q * 32 + e);
                    const float w0 = ex2(fmaf(v[e], sl2, -lv.x));
                    const float w1 = ex2(fmaf(v[e + 1], sl2, -lv.y));
                    const float w2 = ex2(fmaf(v[e + 2], sl2, -lv.z));
                    const float w3 = ex2(fmaf(v[e + 3], sl2, -lv.w));
                    const int c = q * 32 + e;
                    acc += (c >= cmin ? w0 : 0.f) + (c + 1 >= cmin ? w1 : 0.f) +
                           (c + 2 >= cmin ? w2 : 0.f) + (c + 3 >= cmin ? w3 : 0.f);
                }
            }
            tc_before();
            mbar_arrive(BAR(SE + sb));
            total += (double)acc;
            load_tile(u + 2);
        }
        cp_async_wait<0>();
        if (ok_run && key_ok) {
            const double score = total / ((double)G * (double)n_q);
            const int64_t slot = ((int64_t)b * kv.h_kv + g) * p.max_cand + (key - cb);
            p.keys[slot] = score_key(score);
            if (p.scores) p.scores[slot] = score;
        }
    }

    // ---- teardown: the producer waits for its one copy if the CTA aborted ----
    if (warp == kTaProducer && lane == 0 && k_issued && *abort_flag) {
        const unsigned long long t0 = now_ns();
        while (!mbar_try(BAR(KF), 0) && now_ns() - t0 < kDrainNs) {
        }
    }
    tc_before();
    __syncthreads();
    tc_after();
    if (warp == kTaMma)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTaTmemCols)
                     : "memory");
}

// ---------------------------------------------------------------- CUDA-core passes ---------

template <bool BF16>
__device__ __forceinline__ float ld_elem(const void *base, int64_t off) {
    return BF16 ? __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(base) +
                                                  off) << 16)
                : __ldg(reinterpret_cast<const float *>(base) + off);
}

// Pass 1: one warp per (text row, query head); lanes stride over the row's positions.
template <bool BF16>
__global__ void __launch_bounds__(32) text_lse_simt_kernel(const TopkParams p) {
    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z, lane = threadIdx.x;
    const KVView &kv = p.kv;
    const int D = kv.head_dim;
    const int q0 = __ldg(p.q_start + b), n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    if (i >= n_q || n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (kv.page_size != 0 && kv_len > kv.max_pages * kPageSize))
        return;
    const int g = h / p.group;
    const int limit = kv_len - n_q + i;
    const int64_t qoff = ((int64_t)(q0 + i) * p.h_q + h) * D;
    float m = -INFINITY, l = 0.f;
    for (int j = lane; j <= limit; j += 32) {
        const int64_t kr = kv_row_offset(kv, b, g, j, p.dev_err);
        if (kr < 0) continue;
        float s = 0.f;
        for (int e = 0; e < D; ++e) s = fmaf(ld_elem<BF16>(p.q, qoff + e), ld_elem<BF16>(kv.k, kr + e), s);
        s *= p.scale_log2;
        const float mn = fmaxf(m, s);
        l = (m == -INFINITY ? 0.f : l * exp2f(m - mn)) + exp2f(s - mn);
        m = mn;
    }
    const float M = warp_max(m);
    float lw = m == -INFINITY ? 0.f : l * exp2f(m - M);
    lw = warp_sum(lw);
    if (lane == 0)
        p.lse[(int64_t)(q0 + i) * p.h_q + h] = lw > 0.f ? M + log2f(lw) : INFINITY;
}

// Pass 2: one thread per candidate key; the group's text rows in turn.
template <bool BF16>
__global__ void __launch_bounds__(128) text_colsum_simt_kernel(const TopkParams p) {
    const int g = blockIdx.y, b = blockIdx.z;
    const KVView &kv = p.kv;
    const int D = kv.head_dim;
    const int q0 = __ldg(p.q_start + b), n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    if (n_q < 1 || n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (kv.page_size != 0 && kv_len > kv.max_pages * kPageSize))
        return;
    int cb, n;
    cand_range(p, b, cb, n);
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n) return;
    const int j = cb + t;
    const int64_t kr = kv_row_offset(kv, b, g, j, p.dev_err);
    double total = 0.0;
    if (kr >= 0) {
        for (int h = g * p.group; h < (g + 1) * p.group; ++h)
            for (int i = max(0, j - (kv_len - n_q)); i < n_q; ++i) {
                const int64_t qoff = ((int64_t)(q0 + i) * p.h_q + h) * D;
                float s = 0.f;
                for (int e = 0; e < D; ++e)
                    s = fmaf(ld_elem<BF16>(p.q, qoff + e), ld_elem<BF16>(kv.k, kr + e), s);
                total += (double)exp2f(s * p.scale_log2 - p.lse[(int64_t)(q0 + i) * p.h_q + h]);
            }
    }
    const double score = total / ((double)p.group * (double)n_q);
    const int64_t slot = ((int64_t)b * kv.h_kv + g) * p.max_cand + t;
    p.keys[slot] = score_key(score);
    if (p.scores) p.scores[slot] = score;
}

// ---------------------------------------------------------------- host side ---------------

template <int D, bool PAGED>
cudaError_t launch_tc_t(const TopkParams &p, const TcMaps &maps, cudaStream_t s) {
    cudaError_t e = set_max_dynamic_smem<text_lse_tc_kernel<D, PAGED>>(TaCfg<D>::kSmem1);
    if (e != cudaSuccess) return e;
    e = set_max_dynamic_smem<text_colsum_tc_kernel<D, PAGED>>(TaCfg<D>::kSmem2);
    if (e != cudaSuccess) return e;
    const int n_rt = (p.max_q_rows + kTT - 1) / kTT;
    dim3 g1(p.group * n_rt, p.kv.h_kv, p.batch);
    text_lse_tc_kernel<D, PAGED><<<g1, kTaThreads, TaCfg<D>::kSmem1, s>>>(p, maps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int span = p.max_cand + (PAGED ? kPageSize - 1 : 0);
    dim3 g2((span + kTT - 1) / kTT, p.kv.h_kv, p.batch);
    text_colsum_tc_kernel<D, PAGED><<<g2, kTaThreads, TaCfg<D>::kSmem2, s>>>(p, maps);
    return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_simt_t(const TopkParams &p, cudaStream_t s) {
    dim3 g1(p.max_q_rows, p.h_q, p.batch);
    text_lse_simt_kernel<BF16><<<g1, 32, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2((p.max_cand + 127) / 128, p.kv.h_kv, p.batch);
    text_colsum_simt_kernel<BF16><<<g2, 128, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_text_attention_scores(const TopkParams &p, cudaStream_t s) {
    cudaError_t e = cudaErrorNotSupported;
    if (p.kv.dtype == SD_BF16 && (p.kv.head_dim == 64 || p.kv.head_dim == 128) &&
        ((reinterpret_cast<uintptr_t>(p.q) & 15) == 0)) {
        AttnParams ap{};  // the K map only needs the cache view, the batch and the capacity
        ap.kind = SD_ATTN_VERIFY;
        ap.kv = p.kv;
        ap.batch = p.batch;
        TcMaps maps;
        if (encode_kv_maps(ap, p.max_kv_len, &maps)) {
            const bool paged = p.kv.page_size != 0;
            if (p.kv.head_dim == 128)
                e = paged ? launch_tc_t<128, true>(p, maps, s) : launch_tc_t<128, false>(p, maps, s);
            else
                e = paged ? launch_tc_t<64, true>(p, maps, s) : launch_tc_t<64, false>(p, maps, s);
            if (e != cudaSuccess) return e;
        }
    }
    if (e == cudaErrorNotSupported)
        e = p.kv.dtype == SD_BF16 ? launch_simt_t<true>(p, s) : launch_simt_t<false>(p, s);
    if (e != cudaSuccess) return e;
    return launch_topk_select(p, s);
}

}  // namespace sd
