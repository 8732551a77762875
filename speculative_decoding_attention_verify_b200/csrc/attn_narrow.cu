// Tensor-core (tcgen05 + TMA) split-KV attention for ONE query row per sequence and at most 16
// query heads per KV head (R = G <= 16 rows per KV head): the draft steps of the speculative
// cycle (sparse draft attention over a staged selection, text-anchored draft attention) and
// single-row dense decoding, bf16 caches with head_dim 128.
//
// The products are taken transposed, so that the 128 positions of a tile, not the few rows,
// fill the MMA's M dimension:
//   S^T = K Q^T      M = 128 positions (A = K tile, shared memory, K-major), N = 16 rows
//                    (B = Q, shared memory, K-major; rows past R are zero), K = d
//   O^T += V^T P^T   M = d = 128 (A = V tile read MN-major), N = 16 rows (B = P^T, written to
//                    shared memory by the softmax threads), K = 128 positions
// A tile costs 16 MMAs of N = 16 instead of 16 MMAs of 128 x 128, and the softmax work is one
// TMEM lane (one position) per thread with R exponentials.
//
// One CTA per (split, KV head, sequence); 6 warps, one CTA per SM:
//   warps 0-3  softmax: thread p owns position p of each tile (TMEM lane p of S^T) and lane p
//              of O^T (head dimension p) in the epilogue
//   warp 4     TMA producer: lane 0 K tiles, lane 1 V tiles (128 positions, 128-byte swizzle),
//              3-stage ring, each half released on its own (as in the wide kernel)
//   warp 5     MMA issuer and TMEM owner (S^T double-buffered in columns [0, 32), O^T in
//              [32, 48))
// Softmax per tile: each warp reduces its 32 positions' maximum of every row with shuffles, the
// four warps exchange them through shared memory (an mbarrier of four arrivals per tile), and
// every thread then holds the same tile maximum per row.  The exponent's reference maximum of a
// row only moves when the tile maximum exceeds it by more than 2^8 ("lazy rescale"); then O^T's
// column of that row is rescaled in TMEM (each thread its own lane) after the previous P.V.
// Each thread keeps partial row sums of its own positions; they are added across the CTA once,
// in the epilogue.  Partial outputs (O, max, sum) go to the split workspace exactly as the other
// engines write them, or, with a single split, O / sum is written directly.
// Every wait on an mbarrier is bounded (the launch's wait bound); on expiry the CTA records
// SD_DEVERR_TIMEOUT, drains its own copies and MMAs (at most 1 s), frees TMEM and exits.
#include "attn_stream.cuh"
#include "tc_ptx.cuh"

namespace sd {
namespace {

using namespace tc;

constexpr int kNT = 128;                   // positions per tile (MMA M of S^T)
constexpr int kNR = 16;                    // MMA N: rows per KV head, padded
constexpr int kND = 128;                   // head_dim
constexpr int kNThreads = 6 * 32;
constexpr int kNProducer = 4;
constexpr int kNMma = 5;
constexpr int kNStages = 3;
constexpr uint32_t kNTmemCols = 64;        // S^T 0 [0,16), S^T 1 [16,32), O^T [32,48)
constexpr uint32_t kNColO = 32;
constexpr float kNRescale = 8.0f;
constexpr uint32_t kTileB = kNT * kND * 2;  // one K (or V) tile: 32 KB
constexpr uint32_t kHalfT = kNT * 128;      // one 64-column half of a 128-row tile
constexpr uint32_t kHalfR = kNR * 128;      // one 64-column half of a 16-row operand
constexpr uint32_t kOffQ = kNStages * 2 * kTileB;  // 192 KB
constexpr uint32_t kOffP = kOffQ + 2 * kHalfR;     // two P^T buffers of 2 * kHalfR
constexpr uint32_t kOffRed = kOffP + 4 * kHalfR;   // [2][4][16] float tile maxima
constexpr uint32_t kOffSum = kOffRed + 2 * 4 * kNR * 4;
constexpr uint32_t kOffBar = kOffSum + 4 * kNR * 4;
constexpr int kNSmem = kOffBar + 256 + 1024;  // barriers and slots + alignment slack

// Row r, position p of a 16-row K-major operand with 128-byte swizzle (P^T: rows are query
// rows, the K dimension is the tile's positions).
__device__ __forceinline__ uint32_t small_off(int r, int p) {
    return (uint32_t)((p >> 6) * kHalfR + r * 128 + ((((p & 63) >> 3) ^ (r & 7)) << 4) +
                      (p & 7) * 2);
}

template <bool PAGED>
__global__ void __launch_bounds__(kNThreads, 1)
attn_narrow_kernel(const AttnParams p, const __grid_constant__ TcMaps maps) {
    constexpr int S = kNStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKV = smem;  // stage s: K at s*2*tile, V at s*2*tile + tile
    uint8_t *sQ = smem + kOffQ;
    uint8_t *sP = smem + kOffP;
    float *sRed = reinterpret_cast<float *>(smem + kOffRed);
    float *sSum = reinterpret_cast<float *>(smem + kOffSum);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    // k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], p_full[2], max_x[2], o_done,
    // drain, q_full
    const int KF = 0, VF = S, KE = 2 * S, VE = 3 * S, SF = 4 * S, PF = 4 * S + 2, MX = 4 * S + 4,
              OD = 4 * S + 6, DR = 4 * S + 7, QF = 4 * S + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 9);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_stream = reinterpret_cast<int *>(tmem_slot + 2);  // stream set-up scratch (10 ints)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const KVView &kv = p.kv;
    const int G = p.group;  // == R: one query row
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    if (n_q != 1 || G > kNR || q0 + 1 > p.rows_cap || kv_len < 1 ||
        (PAGED && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0 && n_q != 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    const int R = G;
    const bool sparse = p.kind == SD_ATTN_SPARSE;
    StreamInfo si{};
    if (sparse) {
        si.s0 = 0;
        si.len0 = __ldg(p.k_eff + b * kv.h_kv + g);
        si.s1 = min(max(__ldg(p.tail_begin + b), 0), kv_len);
        si.len1 = kv_len - si.s1;
    } else {
        si = stream_setup<kNThreads>(p, b, g, 1, kv_len, s_stream);
    }
    const int a0 = (PAGED && !sparse) ? (si.s0 & ~(kPageSize - 1)) : si.s0;
    const int a1 = PAGED ? (si.s1 & ~(kPageSize - 1)) : si.s1;
    const int nt0 = si.len0 > 0 ? (si.s0 + si.len0 - a0 + kNT - 1) / kNT : 0;
    const int nt1 = si.len1 > 0 ? (si.s1 + si.len1 - a1 + kNT - 1) / kNT : 0;
    const int n_tiles = nt0 + nt1;
    auto tile_start = [&](int t) { return t < nt0 ? a0 + t * kNT : a1 + (t - nt0) * kNT; };
    const int tile_lo = (int)((int64_t)n_tiles * split / p.n_splits);
    const int tile_hi = (int)((int64_t)n_tiles * (split + 1) / p.n_splits);
    const int n_my = tile_hi - tile_lo;

    if (warp == kNMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kNTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(BAR(KF + s), 1);
            mbar_init(BAR(VF + s), 1);
            mbar_init(BAR(KE + s), 1);
            mbar_init(BAR(VE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(SF + s), 1);
            mbar_init(BAR(PF + s), 128);
            mbar_init(BAR(MX + s), 4);
        }
        mbar_init(BAR(OD), 1);
        mbar_init(BAR(DR), 1);
        mbar_init(BAR(QF), 128);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    // Q (the B operand of S^T): row r < R is query head g*G + r of the sequence's row; the
    // 16 x 128 tile is 256 16-byte chunks, two per softmax thread; rows past R are zero.
    if (warp < 4) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int c = tid + 128 * k, r = c >> 4, ch = c & 15;
            uint4 x = make_uint4(0, 0, 0, 0);
            if (r < R)
                x = __ldg(reinterpret_cast<const uint4 *>(
                          reinterpret_cast<const unsigned short *>(p.q) +
                          ((int64_t)q0 * p.h_q + g * G + r) * kND) + ch);
            *reinterpret_cast<uint4 *>(sQ + (ch >> 3) * kHalfR + r * 128 +
                                       (((ch & 7) ^ (r & 7)) << 4)) = x;
        }
        fence_async_smem();
        mbar_arrive(BAR(QF));
    }

    int n_issued = 0;
    if (warp == kNProducer) {
        // ---------------------------------------------------------- TMA producer ----------
        if (lane < 2) {
            const int half = lane;
            const int full = half == 0 ? KF : VF, empty = half == 0 ? KE : VE;
            int pages[kNT / kPageSize];
            for (int t = 0; t < n_my; ++t) {
                const int s = t % S, use = t / S;
                const int p0 = tile_start(tile_lo + t);
                const bool cmp = sparse && tile_lo + t < nt0;
                const uint32_t dst = saddr(sKV + (size_t)s * 2 * kTileB + (size_t)half * kTileB);
                if (PAGED && !cmp) {
                    for (int pg = 0; pg < kNT / kPageSize; ++pg) {
                        const int pos = p0 + pg * kPageSize;
                        int page = kv.num_pages;  // out of range: zero-filled box
                        if (pos < kv_len) {
                            const int e = __ldg(kv.block_table + (int64_t)b * kv.max_pages +
                                                pos / kPageSize);
                            if (e >= 0 && e < kv.num_pages)
                                page = e;
                            else
                                set_dev_err(p.dev_err, SD_DEVERR_PAGE);
                        }
                        pages[pg] = page;
                    }
                }
                const CUtensorMap *map = cmp ? (half == 0 ? &maps.k2 : &maps.v2)
                                             : (half == 0 ? &maps.k : &maps.v);
                if (t >= S && !mbar_wait(BAR(empty + s), (use - 1) & 1, abort_flag, p.dev_err,
                                         p.wait_ns))
                    break;
                mbar_arrive_tx(BAR(full + s), kTileB);
                if (!PAGED || cmp) {
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load_4d(dst + h * kHalfT, map, BAR(full + s), h * 64, p0, g, b);
                } else {
                    for (int pg = 0; pg < kNT / kPageSize; ++pg)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tma_load_4d(dst + h * kHalfT + pg * kPageSize * 128, map,
                                        BAR(full + s), h * 64, 0, g, pages[pg]);
                }
                n_issued = t + 1;
                if (*abort_flag) break;
            }
        }
    } else if (warp == kNMma) {
        // ---------------------------------------------------------- MMA issuer ------------
        const uint32_t idesc_s = idesc_bf16_ab(kNR, false, false);
        const uint32_t idesc_o = idesc_bf16_ab(kNR, true, false);
        const uint32_t qb = saddr(sQ);
        bool issued = false;
        auto issue_s = [&](int t) {  // S^T = K Q^T of tile t (its K stage has landed)
            const int s = t % S, sb = t & 1;
            const uint32_t kb = saddr(sKV + (size_t)s * 2 * kTileB);
            tc_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < kND / 16; ++kk)
                    mma_ss(tmem + sb * kNR, desc_k_sw128(kb + (kk >> 2) * kHalfT + (kk & 3) * 32),
                           desc_k_sw128(qb + (kk >> 2) * kHalfR + (kk & 3) * 32), idesc_s,
                           kk > 0 ? 1u : 0u);
                mma_commit(BAR(SF + sb));
                mma_commit(BAR(KE + s));
                issued = true;
            }
            __syncwarp();
        };
        auto issue_o = [&](int t) {  // O^T += V^T P^T of tile t (its P^T and V stage are ready)
            const int s = t % S, sb = t & 1;
            uint8_t *vs = sKV + (size_t)s * 2 * kTileB + kTileB;
            // V rows past the run's end may hold anything (NaN included): zero them so that
            // 0 * V cannot poison O
            const int tt = tile_lo + t;
            const int run_hi = tt < nt0 ? si.s0 + si.len0 : si.s1 + si.len1;
            const int valid = max(0, min(kNT, run_hi - tile_start(tt)));
            if (valid < kNT) {
                const int nchunk = (kNT - valid) * 8;
                for (int h = 0; h < 2; ++h)
                    for (int e = lane; e < nchunk; e += 32)
                        *reinterpret_cast<uint4 *>(vs + h * kHalfT + valid * 128 + e * 16) =
                            make_uint4(0, 0, 0, 0);
                fence_async_smem();
                __syncwarp();
            }
            tc_after();
            if (lane == 0) {
                const uint32_t vb = saddr(vs), pb = saddr(sP + (size_t)sb * 2 * kHalfR);
#pragma unroll
                for (int kk = 0; kk < kNT / 16; ++kk)
                    mma_ss(tmem + kNColO, desc_mn_sw128(vb + kk * 2048, kHalfT),
                           desc_k_sw128(pb + (kk >> 2) * kHalfR + (kk & 3) * 32), idesc_o,
                           (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(BAR(VE + s));
                mma_commit(BAR(OD));
            }
            __syncwarp();
        };
        bool alive = true;
        if (n_my > 0) {
            bool qok = true;
            if (lane == 0)
                qok = mbar_wait(BAR(QF), 0, abort_flag, p.dev_err, p.wait_ns) &&
                      mbar_wait(BAR(KF), 0, abort_flag, p.dev_err, p.wait_ns);
            alive = __shfl_sync(0xffffffffu, qok ? 1 : 0, 0) != 0;
            if (alive) issue_s(0);
        }
        for (int t = 0; alive && t < n_my; ++t) {
            // S^T of tile t+1 and P.V of tile t in whichever order their operands arrive
            // (S^T first when both are ready).  S^T of t+1 overwrites the buffer of tile t-1,
            // whose softmax ended before the P.V of t-1 (issued in the previous iteration).
            const int s = t % S, use = t / S, sb = t & 1;
            const int s1 = (t + 1) % S, use1 = (t + 1) / S;
            bool s_done = t + 1 >= n_my, o_done = false;
            const unsigned long long t0 = now_ns();
            const uint32_t hint = poll_hint(p.wait_ns);
            for (unsigned it = 1; !(s_done && o_done); ++it) {
                int flags = 0;  // bit 0: S^T can go, bit 1: P.V can go, bit 2: give up
                if (lane == 0) {
                    if (!s_done && mbar_try_for(BAR(KF + s1), use1 & 1, hint)) flags |= 1;
                    if (!o_done && mbar_try_for(BAR(PF + sb), (t >> 1) & 1, hint) &&
                        mbar_try_for(BAR(VF + s), use & 1, hint))
                        flags |= 2;
                    if (flags == 0) {
                        if (now_ns() - t0 > p.wait_ns) {
                            *abort_flag = 1;
                            set_dev_err(p.dev_err, SD_DEVERR_TIMEOUT);
                            flags = 4;
                        } else if ((it & 7u) == 0 && *abort_flag) {
                            flags = 4;
                        }
                    }
                }
                flags = __shfl_sync(0xffffffffu, flags, 0);
                if (flags & 4) {
                    alive = false;
                    break;
                }
                if (flags & 1) {
                    issue_s(t + 1);
                    s_done = true;
                }
                if (flags & 2) {
                    issue_o(t);
                    o_done = true;
                }
            }
        }
        // Drain: every MMA this warp issued has completed once the drain barrier flips.
        const bool any_issued = __any_sync(0xffffffffu, issued);
        if (lane == 0 && any_issued) {
            mma_commit(BAR(DR));
            const unsigned long long t0 = now_ns();
            while (!mbar_try(BAR(DR), 0) && now_ns() - t0 < kDrainNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax ---------------
        const unsigned FULL = 0xffffffffu;
        const int pos = tid;  // this thread's position in every tile
        const int limit = kv_len - 1;
        // The row's visible positions as two ranges (unsigned: visible(j) <=> j - lo1 <= w1 or
        // j - lo2 <= w2); verify and sparse rows see every position of their runs.
        uint32_t lo1 = 0u, w1 = (uint32_t)limit, lo2 = 0x80000000u, w2 = 0u;
        if (p.kind == SD_ATTN_TEXT_ANCHORED) {
            int x1 = 0, y1 = limit, x2 = 1, y2 = 0;
            window_ranges(limit, si.vb, si.ve, si.W, x1, y1, x2, y2);
            lo1 = 0x80000000u;
            w1 = 0u;
            if (y1 >= x1) {
                lo1 = (uint32_t)x1;
                w1 = (uint32_t)(y1 - x1);
            }
            if (y2 >= x2) {
                lo2 = (uint32_t)x2;
                w2 = (uint32_t)(y2 - x2);
            }
        }
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m_used[kNR], lsum[kNR];
#pragma unroll
        for (int r = 0; r < kNR; ++r) {
            m_used[r] = -INFINITY;
            lsum[r] = 0.f;
        }
        bool ok_run = true;
        for (int t = 0; t < n_my; ++t) {
            const int sb = t & 1;
            const int tt = tile_lo + t;
            const int j = tile_start(tt) + pos;  // stream coordinate of this thread's position
            const int seg_lo = tt < nt0 ? si.s0 : si.s1;
            const int seg_hi = tt < nt0 ? si.s0 + si.len0 : si.s1 + si.len1;
            const bool cmp = sparse && tt < nt0;  // list coordinates: all selected are visible
            const bool vis = j >= seg_lo && j < seg_hi &&
                             (cmp || ((uint32_t)j - lo1 <= w1) || ((uint32_t)j - lo2 <= w2));
            const bool got =
                mbar_wait(BAR(SF + sb), (t >> 1) & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(FULL, got)) {
                ok_run = false;
                break;
            }
            tc_after();
            float x[kNR];
            tmem_ld16(lane_base + sb * kNR, x);
            // this warp's maximum of every row over its 32 positions
#pragma unroll
            for (int r = 0; r < kNR; ++r) {
                x[r] = (vis && r < R) ? x[r] * sl2 : -INFINITY;
                if (r < R) {
                    float wm = x[r];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(FULL, wm, o));
                    if (lane == 0) sRed[(sb * 4 + warp) * kNR + r] = wm;
                }
            }
            if (lane == 0) mbar_arrive(BAR(MX + sb));
            const bool xg = mbar_wait(BAR(MX + sb), (t >> 1) & 1, abort_flag, p.dev_err,
                                      p.wait_ns);
            if (!__all_sync(FULL, xg)) {
                ok_run = false;
                break;
            }
            // the tile maximum of every row (the same in every thread) and the rescale decision
            float corr[kNR];
            bool rescale = false;
#pragma unroll
            for (int r = 0; r < kNR; ++r) {
                corr[r] = 1.f;
                if (r < R) {
                    const float tm = fmaxf(fmaxf(sRed[(sb * 4 + 0) * kNR + r],
                                                 sRed[(sb * 4 + 1) * kNR + r]),
                                           fmaxf(sRed[(sb * 4 + 2) * kNR + r],
                                                 sRed[(sb * 4 + 3) * kNR + r]));
                    if (tm > m_used[r] + kNRescale) {
                        if (m_used[r] != -INFINITY) {
                            corr[r] = ex2(m_used[r] - tm);
                            rescale = true;
                        }
                        lsum[r] *= corr[r];
                        m_used[r] = tm;
                    }
                }
            }
            if (rescale) {
                // O^T holds tiles < t: wait for the P.V of tile t-1, then rescale the changed
                // rows' columns (each thread its own lane).  S^T of t was committed after the
                // P.V of t-2 and the P.V of t needs this thread's arrival, so o_done is in
                // phase t-1 or t: its parity test is exact.
                const bool done =
                    mbar_wait(BAR(OD), (t - 1) & 1, abort_flag, p.dev_err, p.wait_ns);
                if (!__all_sync(FULL, done)) {
                    ok_run = false;
                    break;
                }
                tc_after();
                float o[kNR];
                tmem_ld16(lane_base + kNColO, o);
#pragma unroll
                for (int r = 0; r < kNR; ++r) o[r] *= corr[r];
                tmem_st16(lane_base + kNColO, o);
            }
            // P^T of this position: 2^(s - m) (0 where masked or no position seen yet)
            uint8_t *pbuf = sP + (size_t)sb * 2 * kHalfR;
#pragma unroll
            for (int r = 0; r < kNR; ++r) {
                if (r < R) {
                    const float pe = x[r] == -INFINITY ? 0.f : ex2(x[r] - m_used[r]);
                    lsum[r] += pe;
                    *reinterpret_cast<__nv_bfloat16 *>(pbuf + small_off(r, pos)) =
                        __float2bfloat16_rn(pe);
                }
            }
            fence_async_smem();
            tc_before();
            mbar_arrive(BAR(PF + sb));
        }
        // ---- epilogue ----
        bool done = ok_run;
        if (ok_run && n_my > 0)
            done = mbar_wait(BAR(DR), 0, abort_flag, p.dev_err, p.wait_ns);
        const bool read_o = __all_sync(FULL, done) && n_my > 0;
        tc_after();
        // the row sums: each warp's, then the four warps' in a fixed order
#pragma unroll
        for (int r = 0; r < kNR; ++r) {
            if (r < R) {
                float v = lsum[r];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
                if (lane == 0) sSum[warp * kNR + r] = v;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        float o[kNR];
        if (read_o) {
            tmem_ld16(lane_base + kNColO, o);
        } else {
#pragma unroll
            for (int r = 0; r < kNR; ++r) o[r] = 0.f;
        }
        const int d = pos;  // O^T lane = head dimension
#pragma unroll
        for (int r = 0; r < kNR; ++r) {
            if (r >= R) continue;
            const float l = ((sSum[r] + sSum[kNR + r]) + sSum[2 * kNR + r]) + sSum[3 * kNR + r];
            const bool have = read_o && m_used[r] != -INFINITY && l > 0.f;
            const int h = g * G + r;
            if (p.n_splits == 1) {
                const float v = have ? o[r] / l : 0.f;
                reinterpret_cast<unsigned short *>(p.out)[((int64_t)q0 * p.h_q + h) * kND + d] =
                    (unsigned short)f32_to_bf16_bits(v);
            } else {
                const int64_t base = ((int64_t)split * p.rows_cap + q0) * p.h_q + h;
                p.ws_o[base * kND + d] = have ? o[r] : 0.f;
                if (d == 0) {
                    p.ws_ml[base * 2] = have ? m_used[r] : -INFINITY;
                    p.ws_ml[base * 2 + 1] = have ? l : 0.f;
                }
            }
        }
    }

    // ---- teardown: the producer drains its own copies if the CTA aborted ----
    if (warp == kNProducer && lane < 2 && *abort_flag) {
        const unsigned long long t0 = now_ns();
        const int full = lane == 0 ? KF : VF;
        for (int t = (n_issued > S ? n_issued - S : 0); t < n_issued; ++t) {
            const int s = t % S, use = t / S;
            while (!mbar_try(BAR(full + s), use & 1) && now_ns() - t0 < kDrainNs) {
            }
        }
    }
    tc_before();
    __syncthreads();
    tc_after();
    if (warp == kNMma)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kNTmemCols)
                     : "memory");
}

template <bool PAGED>
cudaError_t launch_narrow_t(const AttnParams &p, const TcMaps &maps, cudaStream_t s) {
    cudaError_t e = set_max_dynamic_smem<attn_narrow_kernel<PAGED>>(kNSmem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, p.kv.h_kv, p.batch);
    attn_narrow_kernel<PAGED><<<grid, kNThreads, kNSmem, s>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

bool narrow_supported(int head_dim, int group, int max_q_rows) {
    return head_dim == kND && max_q_rows == 1 && group >= 1 && group <= kNR;
}

cudaError_t launch_attention_narrow(const AttnParams &p, const TcMaps &maps, cudaStream_t s) {
    return p.kv.page_size != 0 ? launch_narrow_t<true>(p, maps, s)
                               : launch_narrow_t<false>(p, maps, s);
}

}  // namespace sd
