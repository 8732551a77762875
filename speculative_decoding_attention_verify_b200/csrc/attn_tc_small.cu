// Split-KV attention for at most 8 query rows per KV head (G * max_q_rows <= 8; the draft steps
// of the 7B-like layers: one row x 7 heads), bf16 caches, head_dim 64 or 128: the scores
// S = Q K^T on the tensor core (tcgen05, TMA-fed K tiles), the weighted sum P.V on CUDA cores.
//
// With so few rows a tile's two MMA groups cost far more than their arithmetic (a tcgen05.mma
// costs about 200 SM cycles whatever its N), so the tensor core only computes S (8 MMAs per
// 128-position tile instead of 16) and the four softmax warps form P.V themselves while it
// computes the next tile's S.
//
// One CTA per (split, KV head, sequence); 10 warps, one CTA per SM:
//   warps 0-7  Q is placed four times in the 128 MMA rows (copy c in TMEM lanes [32c, 32c+32));
//              warp w reads the scores of copy w % 4 for the tile's 16 columns
//              [32 (w % 4) + 16 (w / 4), +16) (lane r = row r), keeps its own running max and
//              sum per row, writes its P (fp32) to shared memory, then every lane of the warp
//              accumulates O[r][head dims of the lane] for the rows over those 16 positions,
//              reading V straight from the TMA-staged tile.  Two such warps per SM
//              sub-partition hide each other's latencies.
//   warp 8     TMA producer: lane 0 K tiles, lane 1 V tiles (128 positions, 128-byte swizzle),
//              3-stage ring, K released when S is computed, V when the eight warps are done
//   warp 9     MMA issuer (S = Q K^T into one of two 128-column TMEM buffers) and TMEM owner
// O stays in registers (a rescale is a register multiply); the eight partial results are merged
// in shared memory at the end.  Partial outputs (O, max, sum) go to the split workspace exactly as the
// other engines write them, or, with a single split, O / sum is written directly.
// Every wait on an mbarrier is bounded (the launch's wait bound); on expiry the CTA records
// SD_DEVERR_TIMEOUT, drains its own copies and MMAs (at most 1 s), frees TMEM and exits.
#include "attn_stream.cuh"
#include "tc_ptx.cuh"

namespace sd {
namespace {

using namespace tc;

constexpr int kST = 128;             // positions per tile
constexpr int kSRows = 8;            // rows per KV head served here
constexpr int kSCompute = 8;           // compute warps
constexpr int kSCols = kST / kSCompute;  // tile columns per compute warp
constexpr int kSThreads = (kSCompute + 2) * 32;
constexpr int kSProducer = kSCompute;
constexpr int kSMma = kSCompute + 1;
constexpr int kSStages = 3;
constexpr uint32_t kSTmemCols = 512;  // S0 [0,128) S1 [128,256) Q [384, 384 + D/2)
constexpr uint32_t kSColQ = 384;
constexpr float kSRescale = 8.0f;
constexpr uint32_t kSHalf = kST * 128;  // one 64-column half of a 128-row bf16 tile

template <int D>
struct SCfg {
    static constexpr int kTileBytes = kST * D * 2;
    static constexpr int kRing = kSStages * 2 * kTileBytes;
    static constexpr int kPBytes = kSCompute * kSCols * kSRows * 4;  // [warp][position][row]
    static constexpr int kBarOffset = kRing + kPBytes;
    static constexpr int kSmem = kBarOffset + 256 + 1024;
};

template <int D, bool PAGED>
__global__ void __launch_bounds__(kSThreads, 1)
attn_tc_small_kernel(const AttnParams p, const __grid_constant__ TcMaps maps) {
    using C = SCfg<D>;
    constexpr int S = kSStages;
    constexpr int DPL = D / 32;  // head dims per lane in P.V
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKV = smem;  // stage s: K at s*2*tile, V at s*2*tile + tile
    float *sP = reinterpret_cast<float *>(smem + C::kRing);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    // k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], s_empty[2], drain, q_full
    const int KF = 0, VF = S, KE = 2 * S, VE = 3 * S, SF = 4 * S, SE = 4 * S + 2, DR = 4 * S + 4,
              QF = 4 * S + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_stream = reinterpret_cast<int *>(tmem_slot + 2);  // stream set-up scratch (14 ints)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const KVView &kv = p.kv;
    const int G = p.group;
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    const int R = n_q * G;
    if (n_q < 1 || R > kSRows || n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (PAGED && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0 && n_q != 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    const bool sparse = p.kind == SD_ATTN_SPARSE;
    StreamInfo si{};
    if (sparse) {
        si.s0 = 0;
        si.len0 = __ldg(p.k_eff + b * kv.h_kv + g);
        si.s1 = min(max(__ldg(p.tail_begin + b), 0), kv_len);
        si.len1 = kv_len - si.s1;
    } else {
        si = stream_setup<kSThreads>(p, b, g, n_q, kv_len, s_stream);
    }
    const int a0 = (PAGED && !sparse) ? (si.s0 & ~(kPageSize - 1)) : si.s0;
    const int a1 = PAGED ? (si.s1 & ~(kPageSize - 1)) : si.s1;
    const int nt0 = si.len0 > 0 ? (si.s0 + si.len0 - a0 + kST - 1) / kST : 0;
    const int nt1 = si.len1 > 0 ? (si.s1 + si.len1 - a1 + kST - 1) / kST : 0;
    const int n_tiles = nt0 + nt1;
    auto tile_start = [&](int t) { return t < nt0 ? a0 + t * kST : a1 + (t - nt0) * kST; };
    const int tile_lo = (int)((int64_t)n_tiles * split / p.n_splits);
    const int tile_hi = (int)((int64_t)n_tiles * (split + 1) / p.n_splits);
    const int n_my = tile_hi - tile_lo;

    if (warp == kSMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kSTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(BAR(KF + s), 1);
            mbar_init(BAR(VF + s), 1);
            mbar_init(BAR(KE + s), 1);
            mbar_init(BAR(VE + s), kSCompute);  // one arrival per compute warp
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(SF + s), 1);
            mbar_init(BAR(SE + s), kSCompute);
        }
        mbar_init(BAR(DR), 1);
        mbar_init(BAR(QF), 128);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    // Q rows into TMEM columns [kSColQ, kSColQ + D/2) as packed bf16 pairs: lane rr holds query
    // row rr % 32 of the group (zero past R), four copies.
    if (warp < 4) {
        const int r = lane;
        uint32_t qv[D / 2];
        if (r < R) {
            const uint4 *src = reinterpret_cast<const uint4 *>(
                reinterpret_cast<const unsigned short *>(p.q) +
                ((int64_t)(q0 + r / G) * p.h_q + g * G + r % G) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 x = __ldg(src + c);
                qv[4 * c] = x.x;
                qv[4 * c + 1] = x.y;
                qv[4 * c + 2] = x.z;
                qv[4 * c + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int c = 0; c < D / 2; ++c) qv[c] = 0u;
        }
        const uint32_t qaddr = tmem + ((uint32_t)(warp * 32) << 16) + kSColQ;
        if constexpr (D == 128) {
            tmem_st64(qaddr, qv);
        } else {
            float qf[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) qf[c] = __uint_as_float(qv[c]);
            tmem_st32(qaddr, qf);
        }
        tc_before();
        mbar_arrive(BAR(QF));
    }

    int n_issued = 0;
    if (warp == kSProducer) {
        // ---------------------------------------------------------- TMA producer ----------
        if (lane < 2) {
            const int half = lane;
            const int full = half == 0 ? KF : VF, empty = half == 0 ? KE : VE;
            int pages[kST / kPageSize];
            for (int t = 0; t < n_my; ++t) {
                const int s = t % S, use = t / S;
                const int p0 = tile_start(tile_lo + t);
                const bool cmp = sparse && tile_lo + t < nt0;
                const uint32_t dst =
                    saddr(sKV + (size_t)s * 2 * C::kTileBytes + (size_t)half * C::kTileBytes);
                if (PAGED && !cmp) {
                    for (int pg = 0; pg < kST / kPageSize; ++pg) {
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
                mbar_arrive_tx(BAR(full + s), C::kTileBytes);
                if (!PAGED || cmp) {
#pragma unroll
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_4d(dst + h * kSHalf, map, BAR(full + s), h * 64, p0, g, b);
                } else {
                    for (int pg = 0; pg < kST / kPageSize; ++pg)
#pragma unroll
                        for (int h = 0; h < D / 64; ++h)
                            tma_load_4d(dst + h * kSHalf + pg * kPageSize * 128, map,
                                        BAR(full + s), h * 64, 0, g, pages[pg]);
                }
                n_issued = t + 1;
                if (*abort_flag) break;
            }
        }
    } else if (warp == kSMma) {
        // ---------------------------------------------------------- MMA issuer ------------
        const uint32_t idesc = idesc_bf16(kST, false);
        bool issued = false, alive = true;
        if (n_my > 0 && lane == 0) alive = mbar_wait(BAR(QF), 0, abort_flag, p.dev_err, p.wait_ns);
        alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
        for (int t = 0; alive && t < n_my; ++t) {
            // S of tile t into buffer t & 1 once its K has landed and the softmax warps are
            // done with the buffer's previous tile (t - 2)
            const int s = t % S, use = t / S, sb = t & 1;
            bool ok = true;
            if (lane == 0) {
                ok = mbar_wait(BAR(KF + s), use & 1, abort_flag, p.dev_err, p.wait_ns);
                if (ok && t >= 2)
                    ok = mbar_wait(BAR(SE + sb), ((t >> 1) - 1) & 1, abort_flag, p.dev_err,
                                   p.wait_ns);
            }
            alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!alive) break;
            tc_after();
            if (lane == 0) {
                const uint32_t kb = saddr(sKV + (size_t)s * 2 * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kSHalf + (kk & 3) * 32;
                    mma_ts(tmem + sb * kST, tmem + kSColQ + kk * 8, desc_k_sw128(kb + off), idesc,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(SF + sb));
                mma_commit(BAR(KE + s));
                issued = true;
            }
            __syncwarp();
        }
        // Drain: every MMA this warp issued has completed once the drain barrier flips.
        if (lane == 0 && __any_sync(1u, issued)) {
            mma_commit(BAR(DR));
            const unsigned long long t0 = now_ns();
            while (!mbar_try(BAR(DR), 0) && now_ns() - t0 < kDrainNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax + P.V ---------
        const unsigned FULL = 0xffffffffu;
        const int cp = warp & 3;                // this warp's row copy (its TMEM lanes)
        const int c0 = cp * 32 + (warp >> 2) * kSCols;  // its first tile column
        const int r = lane;                     // this lane's row (real when r < R)
        const bool row_ok = r < R;
        const int limit = kv_len - n_q + (row_ok ? r / G : 0);
        uint32_t lo1 = 0x80000000u, w1 = 0u, lo2 = 0x80000000u, w2 = 0u;
        {
            int x1 = 0, y1 = limit, x2 = 1, y2 = 0;
            if (p.kind == SD_ATTN_TEXT_ANCHORED)
                window_ranges(limit, si.vb, si.ve, si.W, x1, y1, x2, y2);
            if (row_ok && y1 >= x1) {
                lo1 = (uint32_t)x1;
                w1 = (uint32_t)(y1 - x1);
            }
            if (row_ok && y2 >= x2) {
                lo2 = (uint32_t)x2;
                w2 = (uint32_t)(y2 - x2);
            }
        }
        // every selected position lies below the tail; when the tail starts at or below the
        // smallest row limit + 1 every row sees the whole selection
        const bool sel_all = !sparse || si.s1 <= kv_len - n_q + 1;
        const int32_t *cpos = sparse ? p.cpos + ((int64_t)b * kv.h_kv + g) * p.k_cap : nullptr;
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(cp * 32) << 16);
        float *pw = sP + warp * kSCols * kSRows;  // [position][row]
        float2 o[kSRows][DPL / 2];  // head dims (2x, 2x + 1) of this lane's DPL, every row
#pragma unroll
        for (int q = 0; q < kSRows; ++q)
#pragma unroll
            for (int e = 0; e < DPL / 2; ++e) o[q][e] = make_float2(0.f, 0.f);
        float m_used = -INFINITY, l = 0.f;
        bool ok_run = true;
        for (int t = 0; t < n_my; ++t) {
            const int sb = t & 1, s = t % S, use = t / S;
            const int tt = tile_lo + t;
            const int p0 = tile_start(tt);
            const int seg_lo = tt < nt0 ? si.s0 : si.s1;
            const int seg_hi = tt < nt0 ? si.s0 + si.len0 : si.s1 + si.len1;
            const bool cmp = sparse && tt < nt0;
            const bool got =
                mbar_wait(BAR(SF + sb), (t >> 1) & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(FULL, got)) {
                ok_run = false;
                break;
            }
            tc_after();
            float v[kSCols];
            tmem_ld16(lane_base + sb * kST + c0, v);
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(SE + sb));  // this warp is done with the S buffer
            // mask (skipped for columns inside the run and visible in full to every row of the
            // warp), then this row's max over the warp's 32 columns, in base 2
            const int q0p = p0 + c0;
            const bool in_run = q0p >= seg_lo && q0p + kSCols <= seg_hi;
            const uint32_t d1 = (uint32_t)q0p - lo1, d2 = (uint32_t)q0p - lo2;
            const bool whole = !row_ok || (cmp ? sel_all
                                               : ((w1 >= kSCols - 1 && d1 <= w1 - (kSCols - 1)) ||
                                                  (w2 >= kSCols - 1 && d2 <= w2 - (kSCols - 1))));
            if (!__all_sync(FULL, in_run && whole)) {
                const uint32_t seg_w = (uint32_t)(seg_hi - seg_lo);
#pragma unroll
                for (int e = 0; e < kSCols; ++e) {
                    bool vis;
                    if (!cmp) {
                        const uint32_t j = (uint32_t)(q0p + e);
                        vis = (j - (uint32_t)seg_lo < seg_w) && ((j - lo1 <= w1) || (j - lo2 <= w2));
                    } else {
                        const bool in = (uint32_t)(q0p + e) < seg_w;
                        vis = in && row_ok &&
                              (sel_all || (uint32_t)__ldg(cpos + q0p + e) - lo1 <= w1);
                    }
                    v[e] = vis ? v[e] : -INFINITY;
                }
            }
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < kSCols; e += 2) mx = max3(mx, v[e], v[e + 1]);
            mx = mx == -INFINITY ? -INFINITY : mx * sl2;
            // lazy rescale: the reference max moves only when the row's max grows by > 2^8
            const bool grow = mx > m_used + kSRescale;
            float corr = 1.f;
            if (grow) {
                corr = m_used == -INFINITY ? 1.f : ex2(m_used - mx);
                m_used = mx;
                l *= corr;
            }
            // P = 2^(s * scale - m) in fp32 (masked entries: 2^-inf = 0)
            const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
            const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
            float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < kSCols; e += 2) {
                const float2 x = __ffma2_rn(make_float2(v[e], v[e + 1]), sc2, nm2);
                const float2 pe = make_float2(ex2(x.x), ex2(x.y));
                acc2 = __fadd2_rn(acc2, pe);
                if (r < kSRows) {
                    pw[e * kSRows + r] = pe.x;
                    pw[(e + 1) * kSRows + r] = pe.y;
                }
            }
            l += acc2.x + acc2.y;
            // rescale the accumulators of the rows whose reference max moved
            if (__any_sync(FULL, grow && corr != 1.f)) {
#pragma unroll
                for (int q = 0; q < kSRows; ++q) {
                    const float cq = __shfl_sync(FULL, corr, q);
#pragma unroll
                    for (int e = 0; e < DPL / 2; ++e) o[q][e] = __fmul2_rn(o[q][e], make_float2(cq, cq));
                }
            }
            __syncwarp();
            // P.V over this copy's 32 positions: lane holds head dims [lane*DPL, +DPL) of every row
            const bool vok = mbar_wait(BAR(VF + s), use & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(FULL, vok)) {
                ok_run = false;
                break;
            }
            const int n_cols = max(0, min(kSCols, seg_hi - q0p));  // V rows past the run: skipped
            const int dl = lane * DPL;                          // first head dim of this lane
            // this lane's bytes of V row c0 + e sit at vrow + e * 128 + voff[e & 7] (128-byte
            // swizzle: 16-byte chunk c of row r is stored in slot c ^ (r & 7))
            const uint8_t *vrow = sKV + (size_t)s * 2 * C::kTileBytes + C::kTileBytes +
                                  (size_t)(dl >> 6) * kSHalf + (size_t)c0 * 128;
            uint32_t voff[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                voff[j] = ((((uint32_t)(dl & 63) >> 3) ^ (uint32_t)j) << 4) | (uint32_t)(dl & 7) * 2;
            auto pv = [&](int e, uint32_t off) {  // off: voff[e & 7]
                const uint8_t *src = vrow + e * 128 + off;
                float2 vf[DPL / 2];
                if constexpr (DPL == 4) {
                    const uint2 w2v = *reinterpret_cast<const uint2 *>(src);
                    vf[0] = make_float2(bf16_lo(w2v.x), bf16_hi(w2v.x));
                    vf[1] = make_float2(bf16_lo(w2v.y), bf16_hi(w2v.y));
                } else {
                    const uint32_t w1v = *reinterpret_cast<const uint32_t *>(src);
                    vf[0] = make_float2(bf16_lo(w1v), bf16_hi(w1v));
                }
                const float4 pa = *reinterpret_cast<const float4 *>(pw + e * kSRows);
                const float4 pb = *reinterpret_cast<const float4 *>(pw + e * kSRows + 4);
                const float pr[kSRows] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
                for (int q = 0; q < kSRows; ++q)
#pragma unroll
                    for (int x = 0; x < DPL / 2; ++x)
                        o[q][x] = __ffma2_rn(make_float2(pr[q], pr[q]), vf[x], o[q][x]);
            };
            if (n_cols == kSCols) {
#pragma unroll 1
                for (int e0 = 0; e0 < kSCols; e0 += 8)
#pragma unroll
                    for (int j = 0; j < 8; ++j) pv(e0 + j, voff[j]);
            } else {
#pragma unroll 1
                for (int e = 0; e < n_cols; ++e)
                    pv(e, ((((uint32_t)(dl & 63) >> 3) ^ (uint32_t)(e & 7)) << 4) |
                              (uint32_t)(dl & 7) * 2);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(VE + s));  // this warp is done with the V stage
        }
        // ---- epilogue: merge the eight partials through shared memory ----
        // Once every compute warp is past its last tile (the barrier) and the MMAs have drained,
        // no copy or MMA touches the ring any more.
        bool done = ok_run;
        if (ok_run && n_my > 0)
            done = mbar_wait(BAR(DR), 0, abort_flag, p.dev_err, p.wait_ns);
        const bool have_any = __all_sync(FULL, done) && n_my > 0;
        asm volatile("bar.sync 1, %0;" ::"n"(kSCompute * 32) : "memory");
        float *s_m = reinterpret_cast<float *>(sKV);       // [warp][row]
        float *s_l = s_m + kSCompute * kSRows;             // [warp][row]
        float *s_o = s_l + kSCompute * kSRows;             // [warp][row][D]
        if (r < kSRows) {
            s_m[warp * kSRows + r] = (have_any && row_ok && l > 0.f) ? m_used : -INFINITY;
            s_l[warp * kSRows + r] = (have_any && row_ok) ? l : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kSRows; ++q)
#pragma unroll
            for (int x = 0; x < DPL / 2; ++x)
                *reinterpret_cast<float2 *>(s_o + (warp * kSRows + q) * D + lane * DPL + 2 * x) =
                    have_any ? o[q][x] : make_float2(0.f, 0.f);
        asm volatile("bar.sync 1, %0;" ::"n"(kSCompute * 32) : "memory");
        // thread tid: head dim tid % D of rows tid / D, tid / D + 256 / D, ...
        for (int idx = tid; idx < R * D; idx += kSCompute * 32) {
            const int rr = idx / D, d = idx % D;
            float M = -INFINITY;
#pragma unroll
            for (int c = 0; c < kSCompute; ++c) M = fmaxf(M, s_m[c * kSRows + rr]);
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int c = 0; c < kSCompute; ++c) {
                const float mc = s_m[c * kSRows + rr];
                const float f = mc == -INFINITY ? 0.f : ex2(mc - M);
                L += f * s_l[c * kSRows + rr];
                O += f * s_o[(c * kSRows + rr) * D + d];
            }
            const int row = q0 + rr / G, h = g * G + rr % G;
            if (p.n_splits == 1) {
                const float val = L > 0.f ? O / L : 0.f;
                reinterpret_cast<unsigned short *>(p.out)[((int64_t)row * p.h_q + h) * D + d] =
                    (unsigned short)f32_to_bf16_bits(val);
            } else {
                const int64_t base = ((int64_t)split * p.rows_cap + row) * p.h_q + h;
                p.ws_o[base * D + d] = L > 0.f ? O : 0.f;
                if (d == 0) {
                    p.ws_ml[base * 2] = L > 0.f ? M : -INFINITY;
                    p.ws_ml[base * 2 + 1] = L;
                }
            }
        }
    }

    // ---- teardown: the producer drains its own copies if the CTA aborted ----
    if (warp == kSProducer && lane < 2 && *abort_flag) {
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
    if (warp == kSMma)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kSTmemCols)
                     : "memory");
}

template <int D, bool PAGED>
cudaError_t launch_small_t(const AttnParams &p, const TcMaps &maps, cudaStream_t s) {
    cudaError_t e = set_max_dynamic_smem<attn_tc_small_kernel<D, PAGED>>(SCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, p.kv.h_kv, p.batch);
    attn_tc_small_kernel<D, PAGED><<<grid, kSThreads, SCfg<D>::kSmem, s>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

bool tc_small_supported(int head_dim, int rows) {
    return (head_dim == 64 || head_dim == 128) && rows >= 1 && rows <= kSRows;
}

cudaError_t launch_attention_tc_small(const AttnParams &p, const TcMaps &maps, cudaStream_t s) {
    const bool paged = p.kv.page_size != 0;
    if (p.kv.head_dim == 128)
        return paged ? launch_small_t<128, true>(p, maps, s) : launch_small_t<128, false>(p, maps, s);
    return paged ? launch_small_t<64, true>(p, maps, s) : launch_small_t<64, false>(p, maps, s);
}

}  // namespace sd
