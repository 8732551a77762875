// Tensor-core (tcgen05 + TMA) split-KV attention for bf16 caches: dense verification,
// text-anchored draft attention and sparse draft attention (over a staged selection).
//
// Serves every bf16 attention call with d = 64 or 128 and R = G * max_q_rows <= 128 rows per
// KV head (7B-like layers: R = 7 for a draft step, 42..63 for verification of 6..9 rows).
//
// One CTA per (split, KV head g, sequence b); 7 warps, one CTA per SM:
//   warps 0-3  softmax: TMEM lane r holds MMA row r; with NCP row copies the R rows are
//              placed NCP times (copy c in lanes [c * 128/NCP, ...)) and each warp handles
//              the 128/NCP tile columns of its copy (rows past R are padding, never read back)
//   warp 4     TMA producer: lane 0 streams K tiles, lane 1 V tiles (128 positions,
//              128-byte swizzle) into a 3-4 stage shared-memory ring, each through its own
//              half of every stage (a stage's K is released once S is computed, its V once
//              P.V is); contiguous caches: one 4-D box per half of head_dim; paged caches: one
//              box per 16-position page
//   warp 5     S = Q K^T issuer (one thread) and TMEM owner
//   warp 6     O += P V issuer (one thread)
// Per tile t (three S buffers in TMEM):
//   S_t = Q K_t^T        tcgen05.mma kind::f16, M=128, N=128, A = Q (a shared-memory tile in
//                        the K tile's layout, written once by the softmax warps), B = K tile
//                        (smem, K-major), fp32 accumulators
//   softmax              each thread reads its row's columns of S_t from TMEM, applies the
//                        run bounds and the row's visible ranges, updates its running max
//                        (base 2) and writes P_t = 2^(s - m) as bf16 over S_t in TMEM.  The
//                        running max used for the exponent only moves when the true max grows
//                        by more than 2^8 ("lazy rescale"), so O is rarely touched.
//   O += P_t V_t         tcgen05.mma with A = P_t from TMEM, B = V tile (smem, MN-major)
// One thread issues a tcgen05.mma no faster than every ~150 SM cycles whatever its shape, and
// a tile takes 16 of them (8 for S over d = 128, 8 for P.V over the tile's 128 positions), so
// the two products have an issuing warp each and S runs up to three tiles ahead: S of tile t
// goes into buffer t % 3 once the P.V of tile t-3, which reads P from that buffer, has
// completed.  (Q sits in shared memory to leave TMEM room for the third buffer.)
// The row copies' partial (m, l, O) are merged in shared memory at the end.  Partial outputs
// (O, max, sum) go to the split workspace exactly like the CUDA-core engine, or, with a single
// split, O / sum is written directly.
//
// Two decompositions of the same per-tile pipeline:
//   attn_tc_kernel          one CTA per (split, KV head, sequence): right for few tiles per
//                           unit (the draft calls), where every CTA starts together
//   attn_tc_persist_kernel  one CTA per SM, each taking an equal contiguous share of all units'
//                           tiles and running its units back to back (long streams: verify,
//                           plain decoding), so no partial last wave idles SMs; partials of
//                           units shared by two CTAs are merged by attn_merge_kernel.  Its
//                           streams are bound by HBM and its merge scratch leaves no shared
//                           memory for Q: Q stays in TMEM, S is double-buffered and one
//                           thread issues both products, S of tile t+1 and P.V of tile t in
//                           whichever order their operands arrive (6 warps)
// The host plans one or the other from a time model.  They are separate kernels because the
// per-unit bookkeeping costs the short draft calls registers and time per tile.
// Every wait on an mbarrier is bounded (the launch's wait bound, 1 s by default); on expiry the
// CTA records SD_DEVERR_TIMEOUT, drains its own copies and MMAs (bounded), frees TMEM and exits.
#include <type_traits>

#include "attn_stream.cuh"
#include "tc_ptx.cuh"

namespace sd {
namespace {

using namespace tc;

constexpr int kTile = 128;            // positions per tile
constexpr int kRows = 128;            // MMA M
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;           // S = Q K^T issuer (persistent: both products), TMEM owner
constexpr int kPvWarp = 6;            // per-unit kernel: O += P V issuer
constexpr int kThreads = 6 * 32;      // persistent kernel
constexpr int kThreadsUnit = 7 * 32;  // per-unit kernel
constexpr uint32_t kTmemCols = 512;
// persistent kernel: S0 [0,128) S1 [128,256) O [256,256+D) Q [384,384+D/2)
constexpr uint32_t kColO = 256;
constexpr uint32_t kColQ = 384;       // Q as packed bf16 pairs: the A operand of S = Q K^T
// per-unit kernel: S0 S1 S2 [0,384) O [384,384+D)
constexpr int kSBufs = 3;
constexpr uint32_t kColOUnit = 384;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kHalfBytes = kTile * 128;  // one 64-column half of a 128-row tile
constexpr int kMaxSegs = 8;      // segments (units) one CTA may touch
constexpr int kSegBytes = 768;   // their table in shared memory

template <int D>
struct Cfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr int kStages = D == 128 ? 3 : 4;
    static constexpr int kBarOffset = kStages * 2 * kTileBytes;
    static constexpr int kSegOffset = kBarOffset + 256;  // the CTA's segment table
    static constexpr int kMergeOffset = kSegOffset + kSegBytes;  // persistent: merge scratch
    static constexpr int kSmem = kMergeOffset + 1024;  // (+ slack to align the base to 1 KB)
    // per-unit kernel: the Q tile (the K tile's layout, 1 KB aligned) where the persistent
    // kernel keeps its merge scratch
    static constexpr int kQOffset = kMergeOffset;
    static constexpr int kSmemUnit = kQOffset + kTileBytes + 1024;
};

// ---------------------------------------------------------------- the kernel --------------

// One (sequence b, KV head g) unit's share of a CTA: tiles [t_lo, t_hi) of the unit's position
// stream, and where the result goes.  Every thread that needs it computes it on its own.
struct TcSeg {
    int b, g;
    int q0, n_q, kv_len;
    bool valid;  // the shape checks passed
    StreamInfo si;
    int a0, a1, nt0, nt1;  // runs tiled from a0 / a1: nt0 + nt1 tiles
    int t_lo, t_hi;
    int slot;  // split-workspace slot of the partial result, or -1: the normalised output
    __device__ __forceinline__ int tile_start(int t) const {
        return t < nt0 ? a0 + t * kTile : a1 + (t - nt0) * kTile;
    }
    __device__ __forceinline__ bool active() const { return valid && t_hi > t_lo; }
};

// The unit (b, g): its rows and its position stream as at most two runs [s0, s0+len0) and
// [s1, s1+len1) (verify: [0, kv_len); text-anchored: the non-visual positions from the lowest
// windowed one; sparse: run 0 is the compacted selection [0, k_eff) in its own buffer, run 1
// the tail).  Each run is tiled from its start, or from the page boundary below it for paged
// caches.
template <bool PAGED>
__device__ __forceinline__ TcSeg make_seg(const AttnParams &p, int b, int g, int rpc) {
    TcSeg sg{};
    sg.b = b;
    sg.g = g;
    sg.q0 = __ldg(p.q_start + b);
    sg.n_q = __ldg(p.q_start + b + 1) - sg.q0;
    sg.kv_len = __ldg(p.kv.kv_len + b);
    const int R = sg.n_q * p.group;
    sg.valid = !(sg.n_q < 1 || R > rpc || sg.n_q > p.max_q_rows || sg.q0 + sg.n_q > p.rows_cap ||
                 sg.kv_len < sg.n_q || (PAGED && sg.kv_len > p.kv.max_pages * kPageSize));
    if (!sg.valid) return sg;
    const bool sparse = p.kind == SD_ATTN_SPARSE;
    if (sparse) {
        sg.si.s0 = 0;
        sg.si.len0 = __ldg(p.k_eff + b * p.kv.h_kv + g);
        sg.si.s1 = min(max(__ldg(p.tail_begin + b), 0), sg.kv_len);
        sg.si.len1 = sg.kv_len - sg.si.s1;
    } else {
        sg.si = stream_info_single(p, b, sg.n_q, sg.kv_len);
    }
    sg.a0 = (PAGED && !sparse) ? (sg.si.s0 & ~(kPageSize - 1)) : sg.si.s0;
    sg.a1 = PAGED ? (sg.si.s1 & ~(kPageSize - 1)) : sg.si.s1;
    sg.nt0 = sg.si.len0 > 0 ? (sg.si.s0 + sg.si.len0 - sg.a0 + kTile - 1) / kTile : 0;
    sg.nt1 = sg.si.len1 > 0 ? (sg.si.s1 + sg.si.len1 - sg.a1 + kTile - 1) / kTile : 0;
    return sg;
}

// The CTA's item range in the persistent decomposition (see AttnParams::persist_s).
struct TcWork {
    long long lo, hi, n_items;
    int u0, nseg;
};

__device__ __forceinline__ TcWork cta_work(const AttnParams &p) {
    TcWork w{};
    w.n_items = (long long)p.batch * p.kv.h_kv * p.persist_s;
    w.lo = w.n_items * blockIdx.x / p.persist_g;
    w.hi = w.n_items * (blockIdx.x + 1) / p.persist_g;
    if (w.hi <= w.lo) return w;
    w.u0 = (int)(w.lo / p.persist_s);
    w.nseg = (int)((w.hi - 1) / p.persist_s) - w.u0 + 1;
    return w;
}

// The CTA (of persist_g) whose item range holds item x.
__device__ __forceinline__ int persist_cta_of(long long x, long long n_items, int ctas) {
    return (int)(((x + 1) * ctas - 1) / n_items);
}

// Segment j of the CTA: the j-th unit its item range touches, with the unit-local tiles of
// those items.  Computed once per segment into the CTA's shared-memory table (a single call
// site, so inlining it does not swell the kernel past the instruction cache).
template <bool PAGED>
__device__ __forceinline__ TcSeg cta_seg(const AttnParams &p, const TcWork &w, int j, int rpc) {
    const int u = w.u0 + j;
    TcSeg sg = make_seg<PAGED>(p, u / p.kv.h_kv, u % p.kv.h_kv, rpc);
    const long long s = p.persist_s, base = (long long)u * s;
    int n_tiles = sg.valid ? sg.nt0 + sg.nt1 : 0;
    if (n_tiles > s) {  // longer than the host's bound: a hint was violated
        set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        n_tiles = (int)s;
    }
    sg.t_lo = min((int)max(w.lo - base, 0LL), n_tiles);
    sg.t_hi = min((int)min(w.hi - base, s), n_tiles);
    const int c0 = persist_cta_of(base, w.n_items, p.persist_g);
    const int c1 = persist_cta_of(base + s - 1, w.n_items, p.persist_g);
    sg.slot = c1 == c0 ? -1 : (int)blockIdx.x - c0;
    if (sg.slot >= p.n_splits) {  // cannot happen with the host's slot count; never written
        set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        sg.valid = false;
    }
    return sg;
}

// What the producer and the MMA issuer need of an active segment.
struct TcRuns {
    int b, g, kv_len;
    int a0, a1, nt0;  // tile starts (TcSeg::tile_start)
    int hi0, hi1;     // ends of the two runs
    int t_lo, t_hi;
    __device__ __forceinline__ int tile_start(int t) const {
        return t < nt0 ? a0 + t * kTile : a1 + (t - nt0) * kTile;
    }
    __device__ __forceinline__ int run_end(int t) const { return t < nt0 ? hi0 : hi1; }
};

static_assert(sizeof(TcSeg) * kMaxSegs <= kSegBytes, "segment table");

// Walks the tiles of the CTA's active segments in order (global tile index t), from the
// CTA's segment table in shared memory.
struct TileCursor {
    TcRuns sg;
    int j, lt, a;  // segment, unit-local tile, ordinal of the active segment
    bool done;
    __device__ __forceinline__ void seek(const TcSeg *segs, int nseg, int from) {
        for (j = from; j < nseg; ++j) {
            const TcSeg f = segs[j];
            if (f.active()) {
                sg.b = f.b;
                sg.g = f.g;
                sg.kv_len = f.kv_len;
                sg.a0 = f.a0;
                sg.a1 = f.a1;
                sg.nt0 = f.nt0;
                sg.hi0 = f.si.s0 + f.si.len0;
                sg.hi1 = f.si.s1 + f.si.len1;
                sg.t_lo = f.t_lo;
                sg.t_hi = f.t_hi;
                lt = f.t_lo;
                done = false;
                return;
            }
        }
        done = true;
    }
    __device__ __forceinline__ void start(const TcSeg *segs, int nseg) {
        a = 0;
        seek(segs, nseg, 0);
    }
    __device__ __forceinline__ bool first() const { return lt == sg.t_lo; }
    __device__ __forceinline__ bool last() const { return lt + 1 == sg.t_hi; }
    __device__ __forceinline__ void next(const TcSeg *segs, int nseg) {
        if (++lt < sg.t_hi) return;
        ++a;
        seek(segs, nseg, j + 1);
    }
};

// Drain of one issuing warp: once `bar` (committed here) flips, every MMA its lane 0 issued
// has completed.  Bounded (kDrainNs): an aborted CTA must still free its TMEM.
__device__ __forceinline__ void mma_drain(uint32_t bar, bool issued, int lane) {
    const bool any_issued = __any_sync(0xffffffffu, issued);
    if (lane == 0 && any_issued) {
        mma_commit(bar);
        const unsigned long long t0 = now_ns();
        while (!mbar_try(bar, 0) && now_ns() - t0 < kDrainNs) {
        }
    }
    __syncwarp();
}

// NCP row copies: with R <= 128 / NCP rows per KV head, the rows are placed NCP times in the
// 128 MMA rows (copy c in rows [c * 128/NCP, (c+1) * 128/NCP)) and softmax warp w, of copy
// c = w / (4 / NCP), handles the columns [c * 128/NCP, (c+1) * 128/NCP) of every tile: the
// exponentials of a tile are spread over four warps (and their SM sub-partitions) instead of
// one or two.  Each copy keeps its own running max, sum and output rows; the copies are
// merged in shared memory at the end.
template <int D, bool PAGED, int NCP>
__global__ void __launch_bounds__(kThreadsUnit, 1)
attn_tc_kernel(const AttnParams p, const __grid_constant__ TcMaps maps) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    constexpr int RPC = kRows / NCP;  // rows per copy
    constexpr int NC = kTile / NCP;   // columns per softmax warp
    using C = Cfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKV = smem;  // stage s: K at s*2*tile, V at s*2*tile + tile
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint8_t *sQ = smem + C::kQOffset;  // Q rows: the A operand of S = Q K^T
    // barrier slots: k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[3], p_full[3],
    // pv_done[3] (per S buffer), drain (P.V issuer), s_drain (S issuer), q_full.  A stage's K
    // half is released as soon as S = Q K^T is computed, its V half once P.V is, so the next
    // K copy starts a softmax earlier.
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int KF = 0, VF = S, KE = 2 * S, VE = 3 * S, SF = 4 * S, PF = SF + kSBufs,
              PD = PF + kSBufs, DR = PD + kSBufs, DS = DR + 1, QF = DS + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + QF + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // stream set-up scratch: 4 ints (sparse streams are set up without it, so stream_setup's
    // per-warp counts are never written here)
    int *s_stream = reinterpret_cast<int *>(tmem_slot + 2);
    static_assert((4 * S + 3 * kSBufs + 3) * 8 + 8 + 16 <= C::kSegOffset - C::kBarOffset,
                  "barrier region");

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const KVView &kv = p.kv;
    const int G = p.group;
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    const int R = n_q * G;
    if (n_q < 1 || R > RPC || n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (PAGED && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0 && n_q != 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    // The unit's position stream as at most two runs [s0, s0+len0) and [s1, s1+len1) (verify:
    // [0, kv_len); text-anchored: the non-visual positions from the lowest windowed one).  Each
    // run is tiled from a0 (a1): its start, or the page boundary below it for paged caches.
    // Sparse: run 0 is the compacted selection [0, k_eff) in its own buffer, run 1 the tail.
    const bool sparse = p.kind == SD_ATTN_SPARSE;
    StreamInfo si{};
    if (sparse) {
        si.s0 = 0;
        si.len0 = __ldg(p.k_eff + b * kv.h_kv + g);
        si.s1 = min(max(__ldg(p.tail_begin + b), 0), kv_len);
        si.len1 = kv_len - si.s1;
    } else {
        si = stream_setup<kThreadsUnit>(p, b, g, n_q, kv_len, s_stream);
    }
    const int a0 = (PAGED && !sparse) ? (si.s0 & ~(kPageSize - 1)) : si.s0;
    const int a1 = PAGED ? (si.s1 & ~(kPageSize - 1)) : si.s1;
    const int nt0 = si.len0 > 0 ? (si.s0 + si.len0 - a0 + kTile - 1) / kTile : 0;
    const int nt1 = si.len1 > 0 ? (si.s1 + si.len1 - a1 + kTile - 1) / kTile : 0;
    const int n_tiles = nt0 + nt1;
    // first position of tile t of the unit
    auto tile_start = [&](int t) { return t < nt0 ? a0 + t * kTile : a1 + (t - nt0) * kTile; };
    const int tile_lo = (int)((int64_t)n_tiles * split / p.n_splits);
    const int tile_hi = (int)((int64_t)n_tiles * (split + 1) / p.n_splits);
    const int n_my = tile_hi - tile_lo;
    const int n_active = NCP > 1 ? 4 : (R + 31) / 32;  // softmax warps holding real rows

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kTmemCols)
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
        for (int s = 0; s < kSBufs; ++s) {
            mbar_init(BAR(SF + s), 1);
            mbar_init(BAR(PF + s), 32 * n_active);
            mbar_init(BAR(PD + s), 1);
        }
        mbar_init(BAR(DR), 1);
        mbar_init(BAR(DS), 1);
        mbar_init(BAR(QF), 128);  // Q in shared memory (warps 0-3)
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    // Q rows into shared memory in the K tile's layout (64-element halves of 128-byte rows,
    // 16-byte chunk c of row rr in slot c ^ (rr & 7): the 128-byte swizzle), the A operand of
    // S = Q K^T: row rr holds query row rr % RPC of the group (zero past R).  Each of warps
    // 0-3 writes its own 32 rows, after the producer has started its first copies; the S
    // issuer waits for all of them.
    if (warp < 4) {
        const int rr = warp * 32 + lane, r = rr % RPC;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const unsigned short *>(p.q) +
            ((int64_t)(q0 + (r < R ? r / G : 0)) * p.h_q + g * G + (r < R ? r % G : 0)) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 x = r < R ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sQ + (c >> 3) * kHalfBytes + rr * 128 +
                                       (((c & 7) ^ (rr & 7)) << 4)) = x;
        }
        fence_async_smem();
        mbar_arrive(BAR(QF));
    }

    int n_issued = 0;  // producer lanes: tiles whose copy this lane has issued
    if (warp == kProducerWarp) {
        // ---------------------------------------------------------- TMA producer ----------
        // Lane 0 streams K, lane 1 streams V, each through its own half of the stage ring, so
        // a K copy never waits behind the release of a V stage (which needs the P.V).
        if (lane < 2) {
            const int half = lane;
            const int full = half == 0 ? KF : VF, empty = half == 0 ? KE : VE;
            int pages[kTile / kPageSize];
            for (int t = 0; t < n_my; ++t) {
                const int s = t % S, use = t / S;
                const int p0 = tile_start(tile_lo + t);
                // compacted sparse selection: its own contiguous buffer
                const bool cmp = sparse && tile_lo + t < nt0;
                const uint32_t dst =
                    saddr(sKV + (size_t)s * 2 * C::kTileBytes + (size_t)half * C::kTileBytes);
                if (PAGED && !cmp) {
                    for (int pg = 0; pg < kTile / kPageSize; ++pg) {
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
                    for (int h = 0; h < C::kHalves; ++h)
                        tma_load_4d(dst + h * kHalfBytes, map, BAR(full + s), h * 64, p0, g, b);
                } else {
                    for (int pg = 0; pg < kTile / kPageSize; ++pg)
#pragma unroll
                        for (int h = 0; h < C::kHalves; ++h)
                            tma_load_4d(dst + h * kHalfBytes + pg * kPageSize * 128, map,
                                        BAR(full + s), h * 64, 0, g, pages[pg]);
                }
                n_issued = t + 1;
                if (*abort_flag) break;
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------- S = Q K^T issuer ---------
        // Lane 0 waits and issues; the decision is broadcast so the warp stays converged.
        // S of tile t waits for its K stage, for Q (first tile) and for the completion of the
        // P.V of tile t-3, which reads P from the S buffer this S overwrites.
        const uint32_t idesc_qk = idesc_bf16(kTile, false);
        const uint32_t qb = saddr(sQ);
        bool issued = false;
        for (int t = 0; t < n_my; ++t) {
            const int s = t % S, use = t / S, sb = t % kSBufs;
            bool ok = true;
            if (lane == 0)
                ok = (t > 0 || mbar_wait(BAR(QF), 0, abort_flag, p.dev_err, p.wait_ns)) &&
                     mbar_wait(BAR(KF + s), use & 1, abort_flag, p.dev_err, p.wait_ns) &&
                     (t < kSBufs || mbar_wait(BAR(PD + sb), ((t - kSBufs) / kSBufs) & 1,
                                              abort_flag, p.dev_err, p.wait_ns));
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
            tc_after();
            if (lane == 0) {
                const uint32_t kb = saddr(sKV + (size_t)s * 2 * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + sb * kTile, desc_k_sw128(qb + off), desc_k_sw128(kb + off),
                           idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(SF + sb));
                mma_commit(BAR(KE + s));
                issued = true;
            }
            __syncwarp();
        }
        mma_drain(BAR(DS), issued, lane);
    } else if (warp == kPvWarp) {
        // ------------------------------------------------------- O += P V issuer ----------
        // P.V of tile t waits for P_t (the softmax warps) and its V stage; its completion
        // releases the V stage and frees S buffer t % 3 for S of tile t+3.
        const uint32_t idesc_pv = idesc_bf16(D, true);
        bool issued = false;
        for (int t = 0; t < n_my; ++t) {
            const int s = t % S, use = t / S, sb = t % kSBufs;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(BAR(PF + sb), (t / kSBufs) & 1, abort_flag, p.dev_err,
                               p.wait_ns) &&
                     mbar_wait(BAR(VF + s), use & 1, abort_flag, p.dev_err, p.wait_ns);
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
            // V rows past the end of the sequence may hold anything (NaN included): zero
            // them so that 0 * V cannot poison O.
            uint8_t *vs = sKV + (size_t)s * 2 * C::kTileBytes + C::kTileBytes;
            // (rows past the run's end in its tensor: the sequence end, or the compacted count)
            const int tt = tile_lo + t;
            const int run_hi = tt < nt0 ? si.s0 + si.len0 : si.s1 + si.len1;
            const int valid = max(0, min(kTile, run_hi - tile_start(tt)));
            if (valid < kTile) {
                const int nchunk = (kTile - valid) * 8;  // 16-byte chunks per half
                for (int h = 0; h < C::kHalves; ++h)
                    for (int e = lane; e < nchunk; e += 32)
                        *reinterpret_cast<uint4 *>(vs + h * kHalfBytes + valid * 128 + e * 16) =
                            make_uint4(0, 0, 0, 0);
                fence_async_smem();
                __syncwarp();
            }
            tc_after();
            if (lane == 0) {
                const uint32_t vb = saddr(vs);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_ts(tmem + kColOUnit, tmem + sb * kTile + kk * 8,
                           desc_mn_sw128(vb + kk * 2048, kHalfBytes), idesc_pv,
                           (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(BAR(VE + s));
                mma_commit(BAR(PD + sb));
                issued = true;
            }
            __syncwarp();
        }
        // (the softmax warps' epilogue waits on the same drain barrier: O is complete)
        mma_drain(BAR(DR), issued, lane);
    } else if (warp < n_active) {
        // ---------------------------------------------------------- softmax ---------------
        // tcgen05.ld / st are warp-collective: every lane executes them, row validity only
        // selects values, and decisions that gate them are made warp-uniform by votes.
        const unsigned FULL = 0xffffffffu;
        const int cp = NCP > 1 ? warp / (4 / NCP) : 0;  // this warp's row copy
        const int c0 = cp * NC;                         // its first tile column
        const int r = warp * 32 + lane - cp * RPC;      // its row
        const bool row_ok = r < R;
        const int limit = kv_len - n_q + (row_ok ? r / G : 0);
        // The row's visible positions as two ranges: visible(j) <=> j - lo1 <= w1 or
        // j - lo2 <= w2 (unsigned; an empty range is lo = 2^31, w = 0).  Verify: [0, limit];
        // text-anchored: the row's window.
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
        // Sparse: every selected position is below the tail; when the tail starts at or below
        // the smallest row limit + 1, every row sees the whole selection, else the compacted
        // positions are tested one by one.
        const bool sel_all = !sparse || si.s1 <= kv_len - n_q + 1;
        const uint32_t row_ok_u = row_ok ? 1u : 0u;
        const int32_t *cpos = sparse ? p.cpos + ((int64_t)b * kv.h_kv + g) * p.k_cap : nullptr;
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m_used = -INFINITY, l = 0.f;
        bool ok_run = true;
        for (int t = 0; t < n_my; ++t) {
            const int sb = t % kSBufs;
            const int tt = tile_lo + t;
            const int p0 = tile_start(tt);
            // the run this tile belongs to: positions [seg_lo, seg_hi)
            const int seg_lo = tt < nt0 ? si.s0 : si.s1;
            const int seg_hi = tt < nt0 ? si.s0 + si.len0 : si.s1 + si.len1;
            const bool got =
                mbar_wait(BAR(SF + sb), (t / kSBufs) & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(FULL, got)) {
                ok_run = false;
                break;
            }
            tc_after();
            const uint32_t s_addr = lane_base + sb * kTile;
            float v[NC];
            tmem_ld_cols<NC>(s_addr + c0, v);
            const int q0p = p0 + c0;  // stream coordinate of this warp's first column
            // Interior tiles (inside the run and visible in full to every row of this warp)
            // skip masking.
            // (tiles of the compacted selection are in list coordinates: the positions are
            // cpos[...], all below the tail)
            const bool cmp = sparse && tt < nt0;
            const bool in_run = q0p >= seg_lo && q0p + NC <= seg_hi;
            const uint32_t d1 = (uint32_t)q0p - lo1, d2 = (uint32_t)q0p - lo2;
            const bool whole = !row_ok || (cmp ? sel_all
                                               : ((w1 >= NC - 1 && d1 <= w1 - (NC - 1)) ||
                                                  (w2 >= NC - 1 && d2 <= w2 - (NC - 1))));
            const bool interior = __all_sync(FULL, in_run && whole);
            float mx = -INFINITY;
            if (!interior) {
                const uint32_t seg_w = (uint32_t)(seg_hi - seg_lo);
                if (!cmp) {
#pragma unroll
                    for (int e = 0; e < NC; ++e) {
                        const uint32_t j = (uint32_t)(q0p + e);
                        const uint32_t vis = (j - (uint32_t)seg_lo < seg_w) &
                                             ((j - lo1 <= w1) | (j - lo2 <= w2));
                        v[e] = vis ? v[e] : -INFINITY;
                    }
                } else if (sel_all) {
#pragma unroll
                    for (int e = 0; e < NC; ++e) {
                        const uint32_t vis = ((uint32_t)(q0p + e) < seg_w) & row_ok_u;
                        v[e] = vis ? v[e] : -INFINITY;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < NC; ++e) {
                        const bool in = q0p + e < (int)seg_w;
                        const uint32_t j = in ? (uint32_t)__ldg(cpos + q0p + e) : 0u;
                        const uint32_t vis = (uint32_t)in & (j - lo1 <= w1);
                        v[e] = vis ? v[e] : -INFINITY;
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < NC; e += 2) mx = max3(mx, v[e], v[e + 1]);
            mx = mx == -INFINITY ? -INFINITY : mx * sl2;
            const bool grow = mx > m_used + kRescaleLog2;
            const bool rescale_o = grow && m_used != -INFINITY;
            if (__any_sync(FULL, rescale_o)) {
                // O holds tiles < t: wait for the P.V of tile t-1, then rescale O in TMEM.
                // (pv_done of buffer (t-1) % 3: S_{t-1} was issued once the P.V of tile t-4,
                // that buffer's previous use, had completed, and its next use, tile t+2, needs
                // this warp's later arrivals, so the parity test is exact.)
                const int pb = (t - 1) % kSBufs;
                const bool done = mbar_wait(BAR(PD + pb), ((t - 1) / kSBufs) & 1, abort_flag,
                                            p.dev_err, p.wait_ns);
                if (!__all_sync(FULL, done)) {
                    ok_run = false;
                    break;
                }
                tc_after();
                const float corr = rescale_o ? ex2(m_used - mx) : 1.f;
                float o[32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    tmem_ld32(lane_base + kColOUnit + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= corr;
                    tmem_st32(lane_base + kColOUnit + c * 32, o);
                }
                l *= corr;
            }
            if (grow) m_used = mx;
            // P = 2^(s*scale - m).  Masked entries are -inf and give exactly 0; while no
            // position of the row has been visible (m = -inf) every entry is masked.
            const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
            const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
            float2 acc2 = make_float2(0.f, 0.f);
            uint32_t pk[NC / 2];
#pragma unroll
            for (int e = 0; e < NC; e += 2) {
                const float2 x = __ffma2_rn(make_float2(v[e], v[e + 1]), sc2, nm2);
                const float2 pe = make_float2(ex2(x.x), ex2(x.y));
                acc2 = __fadd2_rn(acc2, pe);
                pk[e >> 1] = pack_bf16(pe.x, pe.y);
            }
            // P over S: the warp's NC columns are packed into NC/2 TMEM columns at c0/2; the
            // other copies' columns of these rows are zero
            uint32_t prow[kTile / 2];
#pragma unroll
            for (int i = 0; i < kTile / 2; ++i) prow[i] = 0u;
#pragma unroll
            for (int q = 0; q < NCP; ++q)
                if (q == cp)
#pragma unroll
                    for (int i = 0; i < NC / 2; ++i) prow[q * (NC / 2) + i] = pk[i];
            tmem_st64(s_addr, prow);
            const float sum = acc2.x + acc2.y;
            l += sum;
            tc_before();
            mbar_arrive(BAR(PF + sb));
        }
        // ---- epilogue ----
        // Wait on the one-shot drain barrier (committed after the last P.V), not on the
        // per-tile o_done barrier: here only the P.V of tiles < n_my - 2 is known to be
        // complete, so o_done could be two phases behind and its parity test would pass early.
        bool done = ok_run;
        if (ok_run && n_my > 0)
            done = mbar_wait(BAR(DR), 0, abort_flag, p.dev_err, p.wait_ns);
        const bool read_o = __all_sync(FULL, done) && n_my > 0;
        tc_after();
        const bool have = read_o && m_used != -INFINITY;
        const int i = row_ok ? r / G : 0, h = g * G + (row_ok ? r % G : 0);
        const int row = q0 + i;
        float m_out = have ? m_used : -INFINITY, l_out = have ? l : 0.f;
        // merged copies: [copy][RPC][D/4] float4 of unscaled outputs (stage memory); 16-byte
        // chunk j of row r sits in slot j ^ (r & 7), so the eight rows of a quarter-warp
        // access hit distinct banks
        float4 *s_o = nullptr;
        float fq[NCP];  // copy 0: the factor 2^(m_c - M) of every copy
        if constexpr (NCP > 1) {
            // Merge the copies through shared memory (the K/V ring is idle now): every copy
            // writes its (m, l) and its O, read from TMEM in one load; copy 0 then forms
            // M = max over copies, the factors 2^(m_c - M), L = sum of scaled sums and the
            // sum of scaled outputs, in a fixed order.
            float *s_m = reinterpret_cast<float *>(sKV);
            float *s_l = s_m + kRows;
            s_o = reinterpret_cast<float4 *>(s_l + kRows);
            s_m[cp * RPC + r] = m_out;
            s_l[cp * RPC + r] = l_out;
            {
                float o[D];
                if (read_o) tmem_ld_cols<D>(lane_base + kColOUnit, o);
                float4 *dst = s_o + (cp * RPC + r) * (D / 4);
#pragma unroll
                for (int k = 0; k < D / 4; ++k)
                    dst[k ^ (r & 7)] = have ? make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2],
                                                          o[4 * k + 3])
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (cp == 0) {
                float M = -INFINITY;
#pragma unroll
                for (int q = 0; q < NCP; ++q) M = fmaxf(M, s_m[q * RPC + r]);
                float L = 0.f;
#pragma unroll
                for (int q = 0; q < NCP; ++q) {
                    const float mq = s_m[q * RPC + r];
                    fq[q] = mq == -INFINITY ? 0.f : ex2(mq - M);
                    L += fq[q] * s_l[q * RPC + r];
                }
                m_out = M;
                l_out = L;
            }
        }
        const float inv = l_out > 0.f ? 1.f / l_out : 0.f;
        const bool writer = row_ok && cp == 0;  // copy 0 holds the merged row
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            float o[32];
            if constexpr (NCP > 1) {
                if (!writer) continue;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int q = 0; q < NCP; ++q) {
                        const float4 x = s_o[(q * RPC + r) * (D / 4) + ((c * 8 + k) ^ (r & 7))];
                        acc.x = fmaf(fq[q], x.x, acc.x);
                        acc.y = fmaf(fq[q], x.y, acc.y);
                        acc.z = fmaf(fq[q], x.z, acc.z);
                        acc.w = fmaf(fq[q], x.w, acc.w);
                    }
                    o[4 * k] = acc.x;
                    o[4 * k + 1] = acc.y;
                    o[4 * k + 2] = acc.z;
                    o[4 * k + 3] = acc.w;
                }
            } else {
                if (read_o) tmem_ld32(lane_base + kColOUnit + c * 32, o);
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (!have) o[e] = 0.f;
            }
            if (!writer) continue;
            if (p.n_splits == 1) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) pk[e >> 1] = pack_bf16(o[e] * inv, o[e + 1] * inv);
                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<unsigned short *>(p.out) +
                                                       ((int64_t)row * p.h_q + h) * D + c * 32);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            } else {
                const int64_t base = ((int64_t)split * p.rows_cap + row) * p.h_q + h;
                float4 *dst = reinterpret_cast<float4 *>(p.ws_o + base * D + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                if (c == 0) {
                    p.ws_ml[base * 2] = l_out > 0.f ? m_out : -INFINITY;
                    p.ws_ml[base * 2 + 1] = l_out;
                }
            }
        }
    }

    // ---- teardown: the producer drains its own copies if the CTA aborted ----
    if (warp == kProducerWarp && lane < 2 && *abort_flag) {
        // only the last S copies this lane issued can still be in flight
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
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

// NCP row copies: with R <= 128 / NCP rows per KV head, the rows are placed NCP times in the
// 128 MMA rows (copy c in rows [c * 128/NCP, (c+1) * 128/NCP)) and softmax warp w, of copy
// c = w / (4 / NCP), handles the columns [c * 128/NCP, (c+1) * 128/NCP) of every tile: the
// exponentials of a tile are spread over four warps (and their SM sub-partitions) instead of
// one or two.  Each copy keeps its own running max, sum and output rows; the copies are
// merged in shared memory at the end of every segment.
//
// Persistent decomposition: the CTA runs its segments back to back through one pipeline (the
// global tile index t drives the ring stages and barrier phases).  At the end of a segment the
// softmax warps write the next segment's Q into TMEM (the issuer waits for it before that
// segment's first S = Q K^T), then read O once the segment-done barrier (committed after its
// last P.V) flips; the next segment's first P.V, which starts O afresh, needs their P of its
// first tile and so comes after that read.
template <int D, bool PAGED, int NCP>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_persist_kernel(const AttnParams p, const __grid_constant__ TcMaps maps) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    constexpr int RPC = kRows / NCP;  // rows per copy
    constexpr int NC = kTile / NCP;   // columns per softmax warp
    using C = Cfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKV = smem;  // stage s: K at s*2*tile, V at s*2*tile + tile
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    // barrier slots: k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], p_full[2],
    // o_done, seg_done, drain, q_full.  A stage's K half is released as soon as S = Q K^T is
    // computed, its V half once P.V is, so the next K copy starts a softmax earlier.
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int KF = 0, VF = S, KE = 2 * S, VE = 3 * S, SF = 4 * S, PF = 4 * S + 2, OD = 4 * S + 4,
              SD = 4 * S + 5, DR = 4 * S + 6, QF = 4 * S + 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // copies' merge scratch: its own region after the segment table (the ring is busy with
    // the next segment's tiles)
    float *s_merge = reinterpret_cast<float *>(smem + C::kMergeOffset);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const KVView &kv = p.kv;
    const int G = p.group;
    const bool sparse = p.kind == SD_ATTN_SPARSE;
    const int rows_max = G * p.max_q_rows;  // rows per KV head the launch was planned for
    const TcWork work = cta_work(p);
    if (work.nseg == 0) return;  // (more CTAs than items)
    // The CTA's segments, computed once, in parallel (producer lane j: segment j), while the
    // TMEM is allocated and the barriers initialised; every role then reads them from shared
    // memory.
    TcSeg *s_segs = reinterpret_cast<TcSeg *>(smem + C::kSegOffset);
    const int nseg = work.nseg <= kMaxSegs ? work.nseg : 0;
    if (warp == kProducerWarp && lane < nseg) s_segs[lane] = cta_seg<PAGED>(p, work, lane, RPC);
    if (tid == 0 && nseg == 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);  // (not planned)
    const int n_active = NCP > 1 ? 4 : min(4, (rows_max + 31) / 32);  // softmax warps with rows

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kTmemCols)
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
            mbar_init(BAR(PF + s), 32 * n_active);
        }
        mbar_init(BAR(OD), 1);
        mbar_init(BAR(SD), 1);
        mbar_init(BAR(DR), 1);
        mbar_init(BAR(QF), 32 * n_active);  // Q in TMEM (the softmax warps)
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    // Q rows of segment sg into TMEM columns [kColQ, kColQ + D/2) as packed bf16 pairs, the A
    // operand of S = Q K^T (read by the tensor core from TMEM, not re-read from shared memory
    // every tile): lane rr holds query row rr % RPC of the group (zero past R).  Each softmax
    // warp writes its own 32 lanes; the MMA issuer waits for all of them.
    auto write_q = [&](const TcSeg &sg) {
        const int rr = warp * 32 + lane, r = rr % RPC;
        const bool has = r < sg.n_q * G;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const unsigned short *>(p.q) +
            ((int64_t)(sg.q0 + (has ? r / G : 0)) * p.h_q + sg.g * G + (has ? r % G : 0)) * D);
        const uint32_t qaddr = tmem + ((uint32_t)(warp * 32) << 16) + kColQ;
        // 32 packed columns (64 elements) at a time
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
            float qf[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 x = has ? __ldg(src + hh * 8 + c) : make_uint4(0, 0, 0, 0);
                qf[4 * c] = __uint_as_float(x.x);
                qf[4 * c + 1] = __uint_as_float(x.y);
                qf[4 * c + 2] = __uint_as_float(x.z);
                qf[4 * c + 3] = __uint_as_float(x.w);
            }
            tmem_st32(qaddr + hh * 32, qf);
        }
        tc_before();
        mbar_arrive(BAR(QF));
    };

    int n_issued = 0;  // producer lanes: tiles whose copy this lane has issued
    if (warp == kProducerWarp) {
        // ---------------------------------------------------------- TMA producer ----------
        // Lane 0 streams K, lane 1 streams V, each through its own half of the stage ring, so
        // a K copy never waits behind the release of a V stage (which needs the P.V).
        if (lane < 2) {
            const int half = lane;
            const int full = half == 0 ? KF : VF, empty = half == 0 ? KE : VE;
            int pages[kTile / kPageSize];
            TileCursor cur;
            cur.start(s_segs, nseg);
            for (int t = 0; !cur.done; ++t, cur.next(s_segs, nseg)) {
                const TcRuns &sg = cur.sg;
                const int s = t % S, use = t / S;
                const int p0 = sg.tile_start(cur.lt);
                // compacted sparse selection: its own contiguous buffer
                const bool cmp = sparse && cur.lt < sg.nt0;
                const uint32_t dst =
                    saddr(sKV + (size_t)s * 2 * C::kTileBytes + (size_t)half * C::kTileBytes);
                if (PAGED && !cmp) {
                    for (int pg = 0; pg < kTile / kPageSize; ++pg) {
                        const int pos = p0 + pg * kPageSize;
                        int page = kv.num_pages;  // out of range: zero-filled box
                        if (pos < sg.kv_len) {
                            const int e = __ldg(kv.block_table + (int64_t)sg.b * kv.max_pages +
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
                    for (int h = 0; h < C::kHalves; ++h)
                        tma_load_4d(dst + h * kHalfBytes, map, BAR(full + s), h * 64, p0, sg.g,
                                    sg.b);
                } else {
                    for (int pg = 0; pg < kTile / kPageSize; ++pg)
#pragma unroll
                        for (int h = 0; h < C::kHalves; ++h)
                            tma_load_4d(dst + h * kHalfBytes + pg * kPageSize * 128, map,
                                        BAR(full + s), h * 64, 0, sg.g, pages[pg]);
                }
                n_issued = t + 1;
                if (*abort_flag) break;
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer ------------
        // Lane 0 waits and issues; the decision is broadcast so the warp stays converged.
        // S = Q K^T of tile t+1 is issued before waiting for the softmax of tile t, so the
        // tensor core computes it while the softmax warps work.  The first S of a segment also
        // waits for that segment's Q; the first P.V of a segment starts O afresh; the last one
        // is followed by a commit to the segment-done barrier.
        const uint32_t idesc_qk = idesc_bf16(kTile, false);
        const uint32_t idesc_pv = idesc_bf16(D, true);
        bool issued = false;
        auto issue_qk = [&](int t) {  // S = Q K^T of tile t (its K stage has landed)
            const int s = t % S, sb = t & 1;
            const uint32_t kb = saddr(sKV + (size_t)s * 2 * C::kTileBytes);
            tc_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    mma_ts(tmem + sb * kTile, tmem + kColQ + kk * 8, desc_k_sw128(kb + off),
                           idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(SF + sb));
                mma_commit(BAR(KE + s));
                issued = true;
            }
            __syncwarp();
        };
        auto issue_pv = [&](int t, const TileCursor &c) {  // O += P V of tile t
            const int s = t % S, sb = t & 1;
            // V rows past the end of the run may hold anything (NaN included): zero them so
            // that 0 * V cannot poison O.  (The run's end: the sequence end, or the compacted
            // count.)
            uint8_t *vs = sKV + (size_t)s * 2 * C::kTileBytes + C::kTileBytes;
            const int valid = max(0, min(kTile, c.sg.run_end(c.lt) - c.sg.tile_start(c.lt)));
            if (valid < kTile) {
                const int nchunk = (kTile - valid) * 8;  // 16-byte chunks per half
                for (int h = 0; h < C::kHalves; ++h)
                    for (int e = lane; e < nchunk; e += 32)
                        *reinterpret_cast<uint4 *>(vs + h * kHalfBytes + valid * 128 + e * 16) =
                            make_uint4(0, 0, 0, 0);
                fence_async_smem();
                __syncwarp();
            }
            tc_after();
            if (lane == 0) {
                const uint32_t vb = saddr(vs);
                const bool fresh = c.first();
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_ts(tmem + kColO, tmem + sb * kTile + kk * 8,
                           desc_mn_sw128(vb + kk * 2048, kHalfBytes), idesc_pv,
                           (!fresh || kk > 0) ? 1u : 0u);
                mma_commit(BAR(VE + s));
                mma_commit(BAR(OD));
                if (c.last()) mma_commit(BAR(SD));
            }
            __syncwarp();
        };
        TileCursor cq, cv;  // next S to issue, next P.V to issue
        cq.start(s_segs, nseg);
        cv = cq;
        bool alive = !cq.done;
        if (alive) {
            bool qok = true;
            if (lane == 0)
                qok = mbar_wait(BAR(QF), 0, abort_flag, p.dev_err, p.wait_ns) &&
                      mbar_wait(BAR(KF), 0, abort_flag, p.dev_err, p.wait_ns);
            alive = __shfl_sync(0xffffffffu, qok ? 1 : 0, 0) != 0;
            if (alive) {
                issue_qk(0);
                cq.next(s_segs, nseg);
            }
        }
        for (int t = 0; alive && !cv.done; ++t) {
            // S of tile t+1 and P.V of tile t, in whichever order their operands arrive (S
            // first when both are ready, so the softmax warps get their next tile early).  S of
            // t+1 overwrites the buffer of tile t-1, whose P.V was issued in the previous
            // iteration, so either order is safe.
            const int s = t % S, use = t / S, sb = t & 1;
            const int s1 = (t + 1) % S, use1 = (t + 1) / S;
            const bool need_q = !cq.done && cq.first();  // S of a new segment needs its Q
            bool qk_done = cq.done, pv_done = false;
            const unsigned long long t0 = now_ns();
            const uint32_t hint = poll_hint(p.wait_ns);
            for (unsigned it = 1; !(qk_done && pv_done); ++it) {
                int flags = 0;  // bit 0: S can go, bit 1: P.V can go, bit 2: give up
                if (lane == 0) {
                    if (!qk_done && mbar_try_for(BAR(KF + s1), use1 & 1, hint) &&
                        (!need_q || mbar_try_for(BAR(QF), cq.a & 1, hint)))
                        flags |= 1;
                    if (!pv_done && mbar_try_for(BAR(PF + sb), (t >> 1) & 1, hint) &&
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
                    issue_qk(t + 1);
                    cq.next(s_segs, nseg);
                    qk_done = true;
                }
                if (flags & 2) {
                    issue_pv(t, cv);
                    cv.next(s_segs, nseg);
                    pv_done = true;
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
    } else if (warp < n_active) {
        // ---------------------------------------------------------- softmax ---------------
        // tcgen05.ld / st are warp-collective: every lane executes them, row validity only
        // selects values, and decisions that gate them are made warp-uniform by votes.
        const unsigned FULL = 0xffffffffu;
        const int cp = NCP > 1 ? warp / (4 / NCP) : 0;  // this warp's row copy
        const int c0 = cp * NC;                         // its first tile column
        const int r = warp * 32 + lane - cp * RPC;      // its row
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float *s_m = s_merge;             // [copy][RPC]
        float *s_l = s_merge + kRows;     // [copy][RPC]
        float4 *s_o = reinterpret_cast<float4 *>(s_merge + 2 * kRows);  // [copy-1][rows_max][D/4]
        bool ok_run = true;
        int t = 0;  // global tile index
        int a = 0;  // ordinal of the active segment
        // the first active segment's Q
        for (int jj = 0; jj < nseg; ++jj) {
            const TcSeg f = s_segs[jj];
            if (f.active()) {
                write_q(f);
                break;
            }
        }
        for (int j = 0; j < nseg; ++j) {
            // (segment descriptions are re-read from the table where needed rather than kept
            // live across the tile loop, whose registers are tight)
            const TcSeg sg = s_segs[j];
            if (!sg.valid) {
                if (warp == 0 && lane == 0 && sg.n_q != 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
                continue;
            }
            const int R = sg.n_q * G;
            const bool row_ok = r < R;
            const int kv_len = sg.kv_len, n_q = sg.n_q;
            const int limit = kv_len - n_q + (row_ok ? r / G : 0);
            // The row's visible positions as two ranges: visible(j) <=> j - lo1 <= w1 or
            // j - lo2 <= w2 (unsigned; an empty range is lo = 2^31, w = 0).  Verify: [0, limit];
            // text-anchored: the row's window.
            uint32_t lo1 = 0x80000000u, w1 = 0u, lo2 = 0x80000000u, w2 = 0u;
            {
                int x1 = 0, y1 = limit, x2 = 1, y2 = 0;
                if (p.kind == SD_ATTN_TEXT_ANCHORED)
                    window_ranges(limit, sg.si.vb, sg.si.ve, sg.si.W, x1, y1, x2, y2);
                if (row_ok && y1 >= x1) {
                    lo1 = (uint32_t)x1;
                    w1 = (uint32_t)(y1 - x1);
                }
                if (row_ok && y2 >= x2) {
                    lo2 = (uint32_t)x2;
                    w2 = (uint32_t)(y2 - x2);
                }
            }
            // Sparse: every selected position is below the tail; when the tail starts at or
            // below the smallest row limit + 1, every row sees the whole selection, else the
            // compacted positions are tested one by one.
            const bool sel_all = !sparse || sg.si.s1 <= kv_len - n_q + 1;
            const uint32_t row_ok_u = row_ok ? 1u : 0u;
            const int32_t *cpos =
                sparse ? p.cpos + ((int64_t)sg.b * kv.h_kv + sg.g) * p.k_cap : nullptr;
            float m_used = -INFINITY, l = 0.f;
            const int n_seg = sg.t_hi - sg.t_lo;
            for (int lt = sg.t_lo; ok_run && lt < sg.t_hi; ++lt, ++t) {
                const int sb = t & 1;
                const int p0 = sg.tile_start(lt);
                // the run this tile belongs to: positions [seg_lo, seg_hi)
                const int seg_lo = lt < sg.nt0 ? sg.si.s0 : sg.si.s1;
                const int seg_hi = lt < sg.nt0 ? sg.si.s0 + sg.si.len0 : sg.si.s1 + sg.si.len1;
                const bool got =
                    mbar_wait(BAR(SF + sb), (t >> 1) & 1, abort_flag, p.dev_err, p.wait_ns);
                if (!__all_sync(FULL, got)) {
                    ok_run = false;
                    break;
                }
                tc_after();
                const uint32_t s_addr = lane_base + sb * kTile;
                float v[NC];
                tmem_ld_cols<NC>(s_addr + c0, v);
                const int q0p = p0 + c0;  // stream coordinate of this warp's first column
                // Interior tiles (inside the run and visible in full to every row of this warp)
                // skip masking.  (Tiles of the compacted selection are in list coordinates: the
                // positions are cpos[...], all below the tail.)
                const bool cmp = sparse && lt < sg.nt0;
                const bool in_run = q0p >= seg_lo && q0p + NC <= seg_hi;
                const uint32_t d1 = (uint32_t)q0p - lo1, d2 = (uint32_t)q0p - lo2;
                const bool whole = !row_ok || (cmp ? sel_all
                                                   : ((w1 >= NC - 1 && d1 <= w1 - (NC - 1)) ||
                                                      (w2 >= NC - 1 && d2 <= w2 - (NC - 1))));
                const bool interior = __all_sync(FULL, in_run && whole);
                float mx = -INFINITY;
                if (!interior) {
                    const uint32_t seg_w = (uint32_t)(seg_hi - seg_lo);
                    if (!cmp) {
#pragma unroll
                        for (int e = 0; e < NC; ++e) {
                            const uint32_t jp = (uint32_t)(q0p + e);
                            const uint32_t vis = (jp - (uint32_t)seg_lo < seg_w) &
                                                 ((jp - lo1 <= w1) | (jp - lo2 <= w2));
                            v[e] = vis ? v[e] : -INFINITY;
                        }
                    } else if (sel_all) {
#pragma unroll
                        for (int e = 0; e < NC; ++e) {
                            const uint32_t vis = ((uint32_t)(q0p + e) < seg_w) & row_ok_u;
                            v[e] = vis ? v[e] : -INFINITY;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < NC; ++e) {
                            const bool in = q0p + e < (int)seg_w;
                            const uint32_t jp = in ? (uint32_t)__ldg(cpos + q0p + e) : 0u;
                            const uint32_t vis = (uint32_t)in & (jp - lo1 <= w1);
                            v[e] = vis ? v[e] : -INFINITY;
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < NC; e += 2) mx = max3(mx, v[e], v[e + 1]);
                mx = mx == -INFINITY ? -INFINITY : mx * sl2;
                const bool grow = mx > m_used + kRescaleLog2;
                const bool rescale_o = grow && m_used != -INFINITY;
                if (__any_sync(FULL, rescale_o)) {
                    // O holds this segment's tiles < t: wait for the P.V of tile t-1, then
                    // rescale O in TMEM.  S_t was committed after the P.V of tile t-2 and the
                    // P.V of tile t needs this warp's arrival, so o_done is in phase t-1 or t:
                    // its parity test is exact.
                    const bool done =
                        mbar_wait(BAR(OD), (t - 1) & 1, abort_flag, p.dev_err, p.wait_ns);
                    if (!__all_sync(FULL, done)) {
                        ok_run = false;
                        break;
                    }
                    tc_after();
                    const float corr = rescale_o ? ex2(m_used - mx) : 1.f;
                    float o[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        tmem_ld32(lane_base + kColO + c * 32, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= corr;
                        tmem_st32(lane_base + kColO + c * 32, o);
                    }
                    l *= corr;
                }
                if (grow) m_used = mx;
                // P = 2^(s*scale - m).  Masked entries are -inf and give exactly 0; while no
                // position of the row has been visible (m = -inf) every entry is masked.
                const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
                const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
                float2 acc2 = make_float2(0.f, 0.f);
                uint32_t pk[NC / 2];
#pragma unroll
                for (int e = 0; e < NC; e += 2) {
                    const float2 x = __ffma2_rn(make_float2(v[e], v[e + 1]), sc2, nm2);
                    const float2 pe = make_float2(ex2(x.x), ex2(x.y));
                    acc2 = __fadd2_rn(acc2, pe);
                    pk[e >> 1] = pack_bf16(pe.x, pe.y);
                }
                // P over S: the warp's NC columns are packed into NC/2 TMEM columns at c0/2;
                // the other copies' columns of these rows are zero (written first)
                if constexpr (NCP == 1) {
                    tmem_st64(s_addr, pk);
                } else {
                    // one store, specialised per copy so that the zeros are compile-time
                    // constants (no registers of their own)
                    auto st_copy = [&](auto cq) {
                        constexpr int CQ = decltype(cq)::value;
                        uint32_t prow[kTile / 2];
#pragma unroll
                        for (int i = 0; i < kTile / 2; ++i)
                            prow[i] = (i / (NC / 2) == CQ) ? pk[i % (NC / 2)] : 0u;
                        tmem_st64(s_addr, prow);
                    };
                    if (cp == 0)
                        st_copy(std::integral_constant<int, 0>{});
                    else if (cp == 1)
                        st_copy(std::integral_constant<int, 1>{});
                    else if (cp == 2)
                        st_copy(std::integral_constant<int, (NCP > 2 ? 2 : 0)>{});
                    else
                        st_copy(std::integral_constant<int, (NCP > 3 ? 3 : 0)>{});
                }
                const float sum = acc2.x + acc2.y;
                l += sum;
                tc_before();
                mbar_arrive(BAR(PF + sb));
            }
            // ---- end of the segment: the next active segment's Q, then this one's output ----
            // (after a failed wait every warp still passes each segment's barriers, with no
            // further waits)
            // (every S of this segment has completed: the last was waited for above)
            if (n_seg > 0 && ok_run) {
                for (int jj = j + 1; jj < nseg; ++jj) {
                    const TcSeg f = s_segs[jj];
                    if (f.active()) {
                        write_q(f);
                        break;
                    }
                }
            }
            // Wait on the segment-done barrier (committed after the segment's last P.V), not
            // on the per-tile o_done barrier, which could be two phases behind here.
            bool done = ok_run;
            if (n_seg > 0 && ok_run)
                done = mbar_wait(BAR(SD), a & 1, abort_flag, p.dev_err, p.wait_ns);
            const bool read_o = __all_sync(FULL, done) && n_seg > 0;
            if (!read_o && n_seg > 0) ok_run = false;
            tc_after();
            const TcSeg eg = s_segs[j];
            const bool have = read_o && m_used != -INFINITY;
            const int i = row_ok ? r / G : 0, h = eg.g * G + (row_ok ? r % G : 0);
            const int row = eg.q0 + i;
            float m_out = have ? m_used : -INFINITY, l_out = have ? l : 0.f;
            float fq[NCP];  // copy 0: the factor 2^(m_c - M) of every copy
            if constexpr (NCP > 1) {
                // Merge the copies through shared memory: every copy writes its (m, l), copies
                // 1.. their O rows (16-byte chunk k of row r in slot k ^ (r & 7), so the eight
                // rows of a quarter-warp access hit distinct banks); copy 0 then forms
                // M = max over copies, the factors 2^(m_c - M), L = sum of scaled sums and the
                // sum of scaled outputs (its own O straight from TMEM), in a fixed order.
                asm volatile("bar.sync 1, 128;" ::: "memory");  // the last segment's merge done
                s_m[cp * RPC + r] = m_out;
                s_l[cp * RPC + r] = l_out;
                if (cp > 0) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        float o[32];
                        if (read_o) tmem_ld32(lane_base + kColO + c * 32, o);  // warp-collective
                        if (r < rows_max) {
                            float4 *dst = s_o + ((cp - 1) * rows_max + r) * (D / 4);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                dst[(c * 8 + k) ^ (r & 7)] =
                                    have ? make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2],
                                                       o[4 * k + 3])
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (cp == 0) {
                    float M = -INFINITY;
#pragma unroll
                    for (int q = 0; q < NCP; ++q) M = fmaxf(M, s_m[q * RPC + r]);
                    float L = 0.f;
#pragma unroll
                    for (int q = 0; q < NCP; ++q) {
                        const float mq = s_m[q * RPC + r];
                        fq[q] = mq == -INFINITY ? 0.f : ex2(mq - M);
                        L += fq[q] * s_l[q * RPC + r];
                    }
                    m_out = M;
                    l_out = L;
                }
            }
            const float inv = l_out > 0.f ? 1.f / l_out : 0.f;
            const bool writer = row_ok && cp == 0;  // copy 0 holds the merged row
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                if (cp == 0) {
                    if (read_o) tmem_ld32(lane_base + kColO + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = have ? o[e] : 0.f;
                }
                if (!writer) continue;
                if constexpr (NCP > 1) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= fq[0];
                    if (r < rows_max) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            float4 acc = make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2],
                                                     o[4 * k + 3]);
#pragma unroll
                            for (int q = 1; q < NCP; ++q) {
                                const float4 x =
                                    s_o[((q - 1) * rows_max + r) * (D / 4) + ((c * 8 + k) ^ (r & 7))];
                                acc.x = fmaf(fq[q], x.x, acc.x);
                                acc.y = fmaf(fq[q], x.y, acc.y);
                                acc.z = fmaf(fq[q], x.z, acc.z);
                                acc.w = fmaf(fq[q], x.w, acc.w);
                            }
                            o[4 * k] = acc.x;
                            o[4 * k + 1] = acc.y;
                            o[4 * k + 2] = acc.z;
                            o[4 * k + 3] = acc.w;
                        }
                    }
                }
                if (eg.slot < 0) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        pk[e >> 1] = pack_bf16(o[e] * inv, o[e + 1] * inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        reinterpret_cast<unsigned short *>(p.out) + ((int64_t)row * p.h_q + h) * D +
                        c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                } else {
                    const int64_t base = ((int64_t)eg.slot * p.rows_cap + row) * p.h_q + h;
                    float4 *dst = reinterpret_cast<float4 *>(p.ws_o + base * D + c * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                    if (c == 0) {
                        p.ws_ml[base * 2] = l_out > 0.f ? m_out : -INFINITY;
                        p.ws_ml[base * 2 + 1] = l_out;
                    }
                }
            }
            if (n_seg > 0) ++a;
        }
    }

    // ---- teardown: the producer drains its own copies if the CTA aborted ----
    if (warp == kProducerWarp && lane < 2 && *abort_flag) {
        // only the last S copies this lane issued can still be in flight
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
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

// ---------------------------------------------------------------- host side ---------------

constexpr int kNcp2Rows = 64;  // largest row count per KV head served with two copies
constexpr int kMaxDynSmem = 227 * 1024;  // per CTA on sm_100

// Row copies for `rows` rows per KV head: four when they fit in 32 (the draft steps), two when
// they fit in 64 (verification of up to 9 rows x 7 heads).
int row_copies(int rows) { return rows <= 32 ? 4 : rows <= kNcp2Rows ? 2 : 1; }

// Shared memory of a launch: the ring and barriers, plus, for a persistent launch with row
// copies, the merge scratch ((m, l) of every MMA row and the O rows of copies 1..).
int tc_smem_bytes(int head_dim, int rows, bool persistent) {
    if (!persistent) return head_dim == 128 ? Cfg<128>::kSmemUnit : Cfg<64>::kSmemUnit;
    const int base = head_dim == 128 ? Cfg<128>::kSmem : Cfg<64>::kSmem;
    const int ncp = row_copies(rows);
    if (ncp == 1) return base;
    return base + (2 * kRows + (ncp - 1) * rows * head_dim) * 4;
}

template <int D, bool PAGED, int NCP>
cudaError_t launch_t(const AttnParams &p, const TcMaps &maps, cudaStream_t s) {
    if (p.persist_s == 0) {
        cudaError_t e = set_max_dynamic_smem<attn_tc_kernel<D, PAGED, NCP>>(Cfg<D>::kSmemUnit);
        if (e != cudaSuccess) return e;
        return launch_pdl(attn_tc_kernel<D, PAGED, NCP>, dim3(p.n_splits, p.kv.h_kv, p.batch),
                          dim3(kThreadsUnit), Cfg<D>::kSmemUnit, s, p, maps);
    }
    const int smem = tc_smem_bytes(D, p.group * p.max_q_rows, true);
    // (the opt-in is the largest any launch may ask for: the merge scratch varies)
    cudaError_t e = set_max_dynamic_smem<attn_tc_persist_kernel<D, PAGED, NCP>>(kMaxDynSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_tc_persist_kernel<D, PAGED, NCP>, dim3(p.persist_g), dim3(kThreads),
                      smem, s, p, maps);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
        else
            cudaGetLastError();
    }
    return fn;
}

bool encode_kv_maps(const AttnParams &p, int max_kv_len, TcMaps *maps) {
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    const KVView &kv = p.kv;
    const cuuint64_t d = (cuuint64_t)kv.head_dim;
    cuuint64_t dims[4], strides[3];
    cuuint32_t box[4] = {64, 0, 1, 1}, elem[4] = {1, 1, 1, 1};
    if (kv.page_size == 0) {
        cuuint64_t lcap;
        if (kv.h_kv > 1)
            lcap = (cuuint64_t)kv.stride_h / d;
        else if (p.batch > 1)
            lcap = (cuuint64_t)kv.stride_b / d;
        else
            lcap = (cuuint64_t)max_kv_len;
        if (lcap < (cuuint64_t)max_kv_len || lcap < 1) return false;
        dims[0] = d;
        dims[1] = lcap;
        dims[2] = (cuuint64_t)kv.h_kv;
        dims[3] = (cuuint64_t)p.batch;
        strides[0] = d * 2;
        strides[1] = (cuuint64_t)kv.stride_h * 2;
        strides[2] = (cuuint64_t)kv.stride_b * 2;
        if (kv.h_kv == 1) strides[1] = lcap * d * 2;
        if (p.batch == 1) strides[2] = strides[1] * (cuuint64_t)kv.h_kv;
        box[1] = kTile;
    } else {
        dims[0] = d;
        dims[1] = kPageSize;
        dims[2] = (cuuint64_t)kv.h_kv;
        dims[3] = (cuuint64_t)kv.num_pages;
        strides[0] = d * 2;
        strides[1] = (cuuint64_t)kPageSize * d * 2;
        strides[2] = (cuuint64_t)kv.h_kv * kPageSize * d * 2;
        box[1] = kPageSize;
    }
    for (int i = 0; i < 3; ++i)
        if (strides[i] % 16 != 0) return false;
    CUresult rk = enc(&maps->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(kv.k), dims,
                      strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CUresult rv = enc(&maps->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(kv.v), dims,
                      strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (rk != CUDA_SUCCESS || rv != CUDA_SUCCESS) return false;
    if (p.kind != SD_ATTN_SPARSE) return true;
    // compacted selection [batch][h_kv][k_cap][d]
    const cuuint64_t kc = (cuuint64_t)(p.k_cap > 0 ? p.k_cap : 1);
    const cuuint64_t cdims[4] = {d, kc, (cuuint64_t)kv.h_kv, (cuuint64_t)p.batch};
    const cuuint64_t cstr[3] = {d * 2, kc * d * 2, (cuuint64_t)kv.h_kv * kc * d * 2};
    const cuuint32_t cbox[4] = {64, kTile, 1, 1};
    CUresult ck = enc(&maps->k2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.ck, cdims, cstr, cbox, elem,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CUresult cv = enc(&maps->v2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.cv, cdims, cstr, cbox, elem,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return ck == CUDA_SUCCESS && cv == CUDA_SUCCESS;
}

bool tc_persistent_fits(int head_dim, int rows) {
    return tc_smem_bytes(head_dim, rows, true) <= kMaxDynSmem;
}

int tc_persistent_max_segments() { return kMaxSegs; }

bool tc_supported(int kind, int dtype, int head_dim, int rows) {
    return dtype == SD_BF16 && (head_dim == 64 || head_dim == 128) && rows >= 1 &&
           rows <= kRows;  // every kind (sparse through the compacted selection)
}

cudaError_t launch_attention_tc(const AttnParams &p, const AttnPlan &plan, cudaStream_t s) {
    TcMaps maps;
    if (!encode_kv_maps(p, p.max_kv_len, &maps)) return cudaErrorNotSupported;
    (void)plan;
    const bool paged = p.kv.page_size != 0;
    const int ncp = row_copies(p.group * p.max_q_rows);
#define SD_TC_LAUNCH(DD, PG)                                                                   \
    (ncp == 4   ? launch_t<DD, PG, 4>(p, maps, s)                                              \
     : ncp == 2 ? launch_t<DD, PG, 2>(p, maps, s)                                              \
                : launch_t<DD, PG, 1>(p, maps, s))
    if (p.kv.head_dim == 128) return paged ? SD_TC_LAUNCH(128, true) : SD_TC_LAUNCH(128, false);
    return paged ? SD_TC_LAUNCH(64, true) : SD_TC_LAUNCH(64, false);
#undef SD_TC_LAUNCH
}

}  // namespace sd
