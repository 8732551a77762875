// Top-K KV selection per (sequence, KV head).
//
// 1. topk_score_kernel: grid (splits, KV heads, sequences).  The group's last query rows are
//    summed once in fp64 (qbar).  Candidate key rows are staged through a 4-stage cp.async
//    ring in 64-row tiles with coalesced 16-byte copies (two CTAs per SM); four threads share
//    a row, each holding its quarter of qbar in registers, and accumulate in fp64 (four
//    independent chains per thread; bf16 x bf16 products are exact in fp64, and the sum of the
//    group's dot products equals qbar . k up to fp64 rounding).  The score is stored as an
//    order-preserving 64-bit key (larger score -> larger key; -0 == +0; NaN lowest).  A
//    non-finite score (the row holds an infinite or NaN element) is recomputed head by head,
//    since the sum over heads and qbar . k can differ there.
// 2. topk_select_kernel: one CTA per (sequence, KV head).  An MSB-first radix select (eight
//    8-bit digits, shared-memory histograms) finds the k-th largest key T exactly; then one
//    pass in position order keeps every key > T and the first (k - #greater) keys == T, so
//    equal scores go to the lower position, and block-wide prefix sums write the kept
//    positions in ascending order.  When the keys fit in shared memory (up to 26,624) they are
//    loaded once and the select touches shared memory only.
// These two serve every call that asks for the scores themselves, and the mean text attention
// mode's selection.  A last-query selection without a scores output takes the fp32 pair below
// (topk_score_fast_kernel, topk_select_fast_kernel): the scores only decide the kept set, and
// fp64 is spent only where it can change it.
#include "tc_ptx.cuh"
#include "topk_common.cuh"

namespace sd {
namespace {

constexpr int kRowThreads = 4;    // threads per candidate (each holds a quarter of qbar)
constexpr int kScoreTile = 64;    // candidates per staged tile
constexpr int kScoreThreads = kRowThreads * kScoreTile;
constexpr int kScoreCtasPerSm = 2;
constexpr int kSelectThreads = 1024;

// cp.async ring depth: 4 stages of 64 rows (bf16, d = 128: two CTAs x 48 KB ahead per SM),
// 3 for fp32 rows
constexpr int score_stages(int row_bytes) { return row_bytes >= 512 ? 3 : 4; }

// Shared-memory chunk slot of chunk ch of tile row `row`.  A quarter-warp (the unit of a
// 16-byte shared load) covers two rows x four threads; thread j of a row reads chunks
// j, j + 4, ...; flipping bit 2 of the slot on odd rows puts the two rows on disjoint bank
// quads, and the copy side's eight consecutive chunks of one row stay distinct.
__device__ __forceinline__ int score_swizzle(int ch, int row) { return ch ^ ((row & 1) << 2); }

// Element e of query head h in row `row`.
template <bool BF16, int D>
__device__ __forceinline__ float query_elem(const void *q, int h_q, int row, int h, int e) {
    const int64_t off = ((int64_t)row * h_q + h) * D + e;
    return BF16 ? __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(q) +
                                                  off) << 16)
                : __ldg(reinterpret_cast<const float *>(q) + off);
}

// Part score (one thread's chunks) of a key row whose qbar score is not finite: the row holds
// an infinite or NaN element (or the query does).  The score is then +inf, -inf or NaN, and
// which one follows the group's own dot products (the sum over heads of q_h . k): qbar . k can
// differ there (+inf against heads of both signs is NaN).  Rare, so it is recomputed head by
// head, outside the scoring loop.
template <bool BF16, int D>
__device__ __noinline__ double nonfinite_part_score(const void *q, int h_q, int row, int h0,
                                                    int h1, const uint8_t *rp, int c,
                                                    int part) {
    using CH = Chunk<BF16>;
    constexpr int NCHUNK = D * (BF16 ? 2 : 4) / 16;
    constexpr int QCH = NCHUNK / kRowThreads;
    double t = 0.0;
    for (int k = 0; k < QCH; ++k) {
        const int ch = part + kRowThreads * k;
        const uint4 raw = *reinterpret_cast<const uint4 *>(rp + (score_swizzle(ch, c) << 4));
        float f[CH::kElems];
        CH::to_float(raw, f);
#pragma unroll
        for (int e = 0; e < CH::kElems; ++e)
            for (int h = h0; h < h1; ++h)
                t = fma((double)query_elem<BF16, D>(q, h_q, row, h, ch * CH::kElems + e),
                        (double)f[e], t);
    }
    return t;
}

template <bool BF16, int D>
__global__ void __launch_bounds__(kScoreThreads, kScoreCtasPerSm) topk_score_kernel(const TopkParams p) {
    using CH = Chunk<BF16>;
    constexpr int ESZ = BF16 ? 2 : 4;
    constexpr int ROWB = D * ESZ;
    constexpr int NCHUNK = ROWB / 16;
    constexpr int QCH = NCHUNK / kRowThreads;  // chunks per thread
    constexpr int QE = D / kRowThreads;        // elements per thread
    constexpr int kScoreStages = score_stages(ROWB);
    static_assert(kScoreThreads == kRowThreads * kScoreTile, "four threads per candidate");
    extern __shared__ __align__(128) uint8_t s_ring[];  // [stage][kScoreTile][ROWB]
    __shared__ double s_qbar[D];
    __shared__ int64_t s_off[kScoreStages][kScoreTile];
    const int tid = threadIdx.x;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const int last = __ldg(p.q_start + b + 1) - 1;
    if (last < __ldg(p.q_start + b)) {
        if (tid == 0 && split == 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    int cb, n;
    cand_range(p, b, cb, n);
    for (int e = tid; e < D; e += kScoreThreads) {
        double acc = 0.0;
        for (int h = g * p.group; h < (g + 1) * p.group; ++h)
            acc += (double)query_elem<BF16, D>(p.q, p.h_q, last, h, e);
        s_qbar[e] = acc;
    }
    __syncthreads();
    // thread quad (4c .. 4c+3) scores candidate c of a tile; thread 4c+j takes chunks
    // j, j+4, ... of the row and holds their qbar elements in registers
    const int c = tid / kRowThreads, quarter = tid % kRowThreads;
    double qr[QE];
#pragma unroll
    for (int k = 0; k < QCH; ++k)
#pragma unroll
        for (int e = 0; e < CH::kElems; ++e)
            qr[k * CH::kElems + e] = s_qbar[(quarter + kRowThreads * k) * CH::kElems + e];

    unsigned long long *keys = p.keys + ((int64_t)b * p.kv.h_kv + g) * p.max_cand;
    const int t_begin = (int)((int64_t)n * split / p.n_splits);
    const int t_end = (int)((int64_t)n * (split + 1) / p.n_splits);
    const int n_tiles = (t_end - t_begin + kScoreTile - 1) / kScoreTile;
    const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(s_ring));
    const char *kbase = reinterpret_cast<const char *>(p.kv.k);

    auto map_tile = [&](int u) {
        if (tid < kScoreTile) {
            const int t = t_begin + u * kScoreTile + tid;
            s_off[u % kScoreStages][tid] =
                t < t_end ? kv_row_offset(p.kv, b, g, cb + t, p.dev_err) : -1;
        }
    };
    auto issue_tile = [&](int u) {  // coalesced: consecutive threads take consecutive chunks
        const int st = u % kScoreStages;
#pragma unroll
        for (int i = 0; i < kScoreTile * NCHUNK / kScoreThreads; ++i) {
            const int e = tid + i * kScoreThreads;
            const int row = e / NCHUNK, ch = e % NCHUNK;
            const int64_t off = s_off[st][row];
            if (off < 0) continue;
            cp_async16(ring + (st * kScoreTile + row) * ROWB + (score_swizzle(ch, row) << 4),
                       kbase + off * ESZ + ch * 16);
        }
    };
    for (int u = 0; u < kScoreStages - 1; ++u) {
        if (u < n_tiles) map_tile(u);
        __syncthreads();
        if (u < n_tiles) issue_tile(u);
        cp_async_commit();
    }
    for (int t = 0; t < n_tiles; ++t) {
        const int u = t + kScoreStages - 1;
        if (u < n_tiles) map_tile(u);
        cp_async_wait<kScoreStages - 2>();
        __syncthreads();
        if (u < n_tiles) issue_tile(u);
        cp_async_commit();
        const int st = t % kScoreStages;
        const int cand = t_begin + t * kScoreTile + c;
        const bool live = cand < t_end && s_off[st][c] >= 0;
        const uint8_t *rp = s_ring + (st * kScoreTile + c) * ROWB;
        double a[4] = {0.0, 0.0, 0.0, 0.0};  // independent chains
        if (live) {
#pragma unroll
            for (int k = 0; k < QCH; ++k) {
                const int ch = quarter + kRowThreads * k;
                const uint4 raw = *reinterpret_cast<const uint4 *>(rp + (score_swizzle(ch, c) << 4));
                float f[CH::kElems];
                CH::to_float(raw, f);
#pragma unroll
                for (int e = 0; e < CH::kElems; ++e)
                    a[e & 3] = fma((double)f[e], qr[k * CH::kElems + e], a[e & 3]);
            }
        }
        double part = (a[0] + a[1]) + (a[2] + a[3]);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);  // the same sum in all four threads
        // converted elements carry infinities and NaNs into the score
        const bool redo = live && !isfinite(part);
        if (__any_sync(0xffffffffu, redo)) {
            double r = redo ? nonfinite_part_score<BF16, D>(p.q, p.h_q, last, g * p.group,
                                                            (g + 1) * p.group, rp, c, quarter)
                            : 0.0;
            r += __shfl_xor_sync(0xffffffffu, r, 1);
            r += __shfl_xor_sync(0xffffffffu, r, 2);
            if (redo) part = r;
        }
        if (quarter == 0 && cand < t_end) {
            keys[cand] = live ? score_key(part) : 0ull;
            if (p.scores)
                p.scores[((int64_t)b * p.kv.h_kv + g) * p.max_cand + cand] = live ? part : NAN;
        }
        __syncthreads();
    }
    cp_async_wait<0>();
}

// Inclusive block-wide prefix sum of one int per thread (kSelectThreads threads).
__device__ __forceinline__ int block_inclusive_scan(int x, int *s_warp, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int before = warp > 0 ? s_warp[warp - 1] : 0;
    total = s_warp[31];
    __syncthreads();
    return x + before;
}

// Selection over n > k 64-bit keys in global memory (one CTA of kSelectThreads): the radix
// select of the k-th largest key T, then one pass in position order that keeps every key > T
// and the first keys == T.
__device__ void select_keys64(const TopkParams &p, int32_t *out, int cb, int n,
                              const unsigned long long *keys, int *s_hist, int *s_warp,
                              unsigned long long &s_prefix, int &s_remaining) {
    const int tid = threadIdx.x;
    // ---- radix select of the k-th largest key ----
    unsigned long long prefix = 0ull, mask = 0ull;
    int remaining = p.k;
    for (int digit = 7; digit >= 0; --digit) {
        const int shift = digit * 8;
        if (tid < 256) s_hist[tid] = 0;
        __syncthreads();
        for (int t = tid; t < n; t += kSelectThreads) {
            const unsigned long long key = keys[t];
            if ((key & mask) == prefix) atomicAdd(&s_hist[(int)((key >> shift) & 255ull)], 1);
        }
        __syncthreads();
        // Cumulative counts from the largest bucket down; 256 threads, descending order.
        int c = tid < 256 ? s_hist[255 - tid] : 0;
        int total;
        const int incl = block_inclusive_scan(c, s_warp, total);
        if (tid < 256 && incl >= remaining && incl - c < remaining) {
            s_prefix = prefix | ((unsigned long long)(255 - tid) << shift);
            s_remaining = remaining - (incl - c);
        }
        __syncthreads();
        prefix = s_prefix;
        remaining = s_remaining;
        mask |= 255ull << shift;
        __syncthreads();
    }
    // prefix == T exactly; `remaining` keys equal to T are taken, lowest positions first.
    const unsigned long long T = prefix;
    int eq_carry = 0, out_carry = 0;
    for (int base = 0; base < n; base += kSelectThreads) {
        const int t = base + tid;
        const unsigned long long key = t < n ? keys[t] : 0ull;
        const bool gt = t < n && key > T;
        const bool eq = t < n && key == T;
        int eq_total;
        const int eq_incl = block_inclusive_scan(eq ? 1 : 0, s_warp, eq_total);
        const bool keep = gt || (eq && eq_carry + eq_incl <= remaining);
        int keep_total;
        const int keep_incl = block_inclusive_scan(keep ? 1 : 0, s_warp, keep_total);
        if (keep) out[out_carry + keep_incl - 1] = cb + t;
        eq_carry += eq_total;
        out_carry += keep_total;
    }
}

__global__ void __launch_bounds__(kSelectThreads) topk_select_kernel(const TopkParams p) {
    __shared__ int s_hist[256];
    __shared__ int s_warp[32];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_remaining;
    const int b = blockIdx.y, g = blockIdx.x, tid = threadIdx.x;
    int32_t *out = p.idx_out + ((int64_t)b * p.kv.h_kv + g) * p.k;
    const int last = __ldg(p.q_start + b + 1) - 1;
    if (last < __ldg(p.q_start + b)) {
        for (int e = tid; e < p.k; e += kSelectThreads) out[e] = -1;
        return;
    }
    int cb, n;
    cand_range(p, b, cb, n);
    const unsigned long long *keys = p.keys + ((int64_t)b * p.kv.h_kv + g) * p.max_cand;
    if (n <= p.k) {  // everything is selected
        for (int e = tid; e < p.k; e += kSelectThreads) out[e] = e < n ? cb + e : -1;
        return;
    }
    select_keys64(p, out, cb, n, keys, s_hist, s_warp, s_prefix, s_remaining);
}

// Selection with every key in shared memory (up to kSmemKeys): the keys are loaded once,
// coalesced; thread t then owns the contiguous candidates [t*kpt, t*kpt + kpt).  The eight
// radix passes touch shared memory only, and the compaction needs a single block-wide scan
// because each thread's candidates are contiguous.
constexpr int kSmemKeys = 26624;  // 208 KB of keys

__global__ void __launch_bounds__(kSelectThreads) topk_select_smem_kernel(const TopkParams p) {
    extern __shared__ unsigned long long s_keys[];
    __shared__ int s_hist[256];
    __shared__ int s_warp[32];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_remaining;
    const int b = blockIdx.y, g = blockIdx.x, tid = threadIdx.x;
    int32_t *out = p.idx_out + ((int64_t)b * p.kv.h_kv + g) * p.k;
    const int last = __ldg(p.q_start + b + 1) - 1;
    if (last < __ldg(p.q_start + b)) {
        for (int e = tid; e < p.k; e += kSelectThreads) out[e] = -1;
        return;
    }
    int cb, n;
    cand_range(p, b, cb, n);
    const unsigned long long *keys = p.keys + ((int64_t)b * p.kv.h_kv + g) * p.max_cand;
    if (n <= p.k) {
        for (int e = tid; e < p.k; e += kSelectThreads) out[e] = e < n ? cb + e : -1;
        return;
    }
    for (int e = tid; e < n; e += kSelectThreads) s_keys[e] = keys[e];
    const int kpt = (n + kSelectThreads - 1) / kSelectThreads;
    const int first = tid * kpt;
    const int mine = max(0, min(kpt, n - first));  // keys owned by this thread
    const unsigned long long *my = s_keys + first;
    unsigned long long prefix = 0ull, mask = 0ull;
    int remaining = p.k;
    for (int digit = 7; digit >= 0; --digit) {
        const int shift = digit * 8;
        if (tid < 256) s_hist[tid] = 0;
        __syncthreads();
        for (int i = 0; i < mine; ++i) {
            const unsigned long long kk = my[i];
            if ((kk & mask) == prefix) atomicAdd(&s_hist[(int)((kk >> shift) & 255ull)], 1);
        }
        __syncthreads();
        const int c = tid < 256 ? s_hist[255 - tid] : 0;
        int total;
        const int incl = block_inclusive_scan(c, s_warp, total);
        if (tid < 256 && incl >= remaining && incl - c < remaining) {
            s_prefix = prefix | ((unsigned long long)(255 - tid) << shift);
            s_remaining = remaining - (incl - c);
        }
        __syncthreads();
        prefix = s_prefix;
        remaining = s_remaining;
        mask |= 255ull << shift;
    }
    const unsigned long long T = prefix;
    // keys > T are all kept; the first `remaining` keys == T in position order are kept
    int eq = 0, gt = 0;
    for (int i = 0; i < mine; ++i) {
        eq += my[i] == T ? 1 : 0;
        gt += my[i] > T ? 1 : 0;
    }
    int eq_total;
    const int eq_before = block_inclusive_scan(eq, s_warp, eq_total) - eq;
    int eq_left = max(0, min(eq, remaining - eq_before));  // equal keys this thread keeps
    const int keep_n = gt + eq_left;
    int keep_total;
    int pos = block_inclusive_scan(keep_n, s_warp, keep_total) - keep_n;
    for (int i = 0; i < mine; ++i) {
        const unsigned long long kk = my[i];
        bool keep = kk > T;
        if (kk == T && eq_left > 0) {
            keep = true;
            --eq_left;
        }
        if (keep) out[pos++] = cb + first + i;
    }
}

// ---------------------------------------------------------------- fp32 scoring -------------
// A last-query selection without a scores output.  With y_j the fp32 score of candidate j and
// x_j its fp64 score, |y_j - x_j| <= E for every candidate of the unit, so the k-th largest y
// (tau) lies within E of the k-th largest x (T): a candidate with y_j > tau + 2E has x_j > T
// and is kept; one with y_j < tau - 2E has x_j < T and is not.  The band between is rescored
// in fp64 and ranked (score, then position) for the places left, so the kept set is the fp64
// selection's.  A unit with a score or a bound that is not finite (infinite or NaN elements,
// fp32 overflow), a row without a valid page, or a band too wide to rank in shared memory is
// scored in fp64 from scratch by the select kernel.
//
// The bound.  The fp32 query q_i rounds the group's sum qbar_i (fp64); with Q_i the sum over
// the group of |q_h,i| (fp64), |q_i - exact qbar_i| <= 2^-24 Q_i (1 + 2^-39) + 2^-150 (the fp64
// sum errs by ~G 2^-53 Q_i; 2^-150 for an fp32 subnormal), which is at most 2^-23 Qu_i with
// Qu_i = (fp32 round-up of Q_i) + 2^-126.  A sum of products accumulated in fp32 with FMAs
// along a tree of height h <= D errs by at most gamma_h = h 2^-24 / (1 - h 2^-24) times the
// sum of |q_i k_i|, plus h 2^-150 for gradual underflow; |q_i| <= (1 + 2^-23) Qu_i.  With
// S = sum Qu_i |k_i| and B its fp32 value (B >= S (1 - gamma_D) - D 2^-150):
//     |y - x| <= (gamma_D (1 + 2^-23) + 2^-23) S + D 2^-150 + (fp64 rounding of x, ~2^-46 S)
//            <= 2^-15 B + 2^-140                    for D <= 128
// (the coefficient is below 2^-16 for D = 128: a factor of two to spare).  E = 2^-15 max_j B_j
// + 2^-140 over the unit's candidates.

// Order-preserving 32-bit key of a finite fp32 score (-0 == +0); 0 (NaN) and 0xffffffff are
// never the key of a finite score and serve as the select kernel's marks.
__device__ __forceinline__ uint32_t score_key32(float x) {
    if (x != x) return 0u;
    x += 0.0f;
    const uint32_t u = __float_as_uint(x);
    return (u >> 31) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key32_value(uint32_t k) {
    return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k);
}

constexpr uint32_t kKeyKept = 0xffffffffu;   // band candidate ranked in
constexpr uint32_t kKeyDropped = 0u;         // band candidate ranked out
constexpr float kErrScale = 0x1p-15f;        // E = kErrScale * max B + kErrFloor
constexpr double kErrFloor = 0x1p-140;

constexpr int kGroupRowsCap = 2048;  // group x d query elements staged in shared memory

// The group's query elements of row `last` into s_qh [G][D] (floats: exact for both dtypes),
// by `nthreads` threads numbered t, four independent loads in flight per thread (a loop over
// the heads would wait for each load in turn).  Requires G * D <= kGroupRowsCap.
template <bool BF16, int D>
__device__ __forceinline__ void stage_group_rows(const TopkParams &p, int last, int g, float *s_qh,
                                                 int t, int nthreads) {
    const int total = p.group * D;
    for (int base = 0; base < total; base += 4 * nthreads) {
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = base + t + j * nthreads;
            v[j] = i < total ? query_elem<BF16, D>(p.q, p.h_q, last, g * p.group + i / D, i % D)
                             : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = base + t + j * nthreads;
            if (i < total) s_qh[i] = v[j];
        }
    }
}

// The fp32 scoring streams each CTA's candidate rows through a ring of 64-row stages filled by
// plain bulk copies (one per run of rows contiguous in the cache: the whole tile, or a page's
// rows) issued by a copy warp; eight warps score (four threads per candidate, as the fp64
// kernel).  Rows sit linearly in shared memory; thread j of a candidate reads chunks
// j + 4k on even rows and j + 4(k ^ 1) on odd ones, so the two rows of a quarter-warp load
// from disjoint banks, and holds its query elements in that order.
constexpr int kFastTile = 64;                                 // candidates per stage
constexpr int kFastWarps = kFastTile * kRowThreads / 32;      // scoring warps
constexpr int kFastThreads = (kFastWarps + 1) * 32;           // + the copy warp
// ring depth: about 96 KB of rows per CTA (two CTAs per SM)
constexpr int fast_stages(int tile_bytes) { return tile_bytes <= 16384 ? 6 : 3; }

// Parts of the fp32 scoring.  Every part holds `chunk` candidates of one (sequence, KV head)
// unit, the same count for every unit, so a batch of ragged sequences gives its long sequences
// more parts instead of longer ones: chunk = the batch's candidates over units * n_splits parts
// (the host's split count for this batch size), at least four 128-candidate spans and at least
// max_cand / part_stride (no unit needs more parts than its part slots).  A unit of n
// candidates takes max(1, ceil(n / chunk)) parts; their sum is at most units * (n_splits + 1),
// the launch's CTA count.  Warp-collective: every lane returns chunk.
constexpr long long kMinPart = 4 * 128;
__device__ long long fast_part_chunk(const TopkParams &p, int lane) {
    long long tot = 0;
    for (int bb = lane; bb < p.batch; bb += 32) {
        int c0, nn;
        cand_range(p, bb, c0, nn, false);
        tot += nn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    const long long units = (long long)p.batch * p.kv.h_kv;
    const long long parts = units * p.n_splits;
    long long chunk = (tot * p.kv.h_kv + parts - 1) / parts;
    chunk = max(chunk, kMinPart);
    chunk = max(chunk, ((long long)p.max_cand + p.part_stride - 1) / p.part_stride);
    return chunk;
}

__device__ __forceinline__ int fast_parts_of(long long n, long long chunk) {
    return (int)max(1LL, (n + chunk - 1) / chunk);
}

// The part CTA x scores: m[0] = sequence (-1: x is past the batch's parts), m[1] = KV head,
// m[2] = part, m[3] = chunk.  Units in (sequence, KV head) order, each unit's parts together.
// Warp-collective; lane 0 writes m.
__device__ void fast_part_of_cta(const TopkParams &p, long long x, int lane, long long *m) {
    const long long chunk = fast_part_chunk(p, lane);
    long long base = 0;
    int fb = -1, fg = 0, fs = 0;
    for (int b0 = 0; b0 < p.batch; b0 += 32) {
        const int bb = b0 + lane;
        int parts = 0;
        if (bb < p.batch) {
            int c0, nn;
            cand_range(p, bb, c0, nn, false);
            parts = fast_parts_of(nn, chunk);
        }
        const long long cnt = (long long)parts * p.kv.h_kv;  // CTAs of sequence bb
        long long inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        const long long lo = base + inc - cnt;
        const unsigned hit = __ballot_sync(0xffffffffu, bb < p.batch && x >= lo && x < lo + cnt);
        if (hit) {
            const int src = __ffs(hit) - 1;
            const long long r = x - __shfl_sync(0xffffffffu, lo, src);
            const int np = __shfl_sync(0xffffffffu, parts, src);
            fb = b0 + src;
            fg = (int)(r / np);
            fs = (int)(r % np);
            break;
        }
        base += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
        m[0] = fb;
        m[1] = fg;
        m[2] = fs;
        m[3] = chunk;
    }
}

template <bool BF16, int D>
__global__ void __launch_bounds__(kFastThreads, kScoreCtasPerSm)
topk_score_fast_kernel(const TopkParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    using CH = Chunk<BF16>;
    using namespace tc;
    constexpr int ESZ = BF16 ? 2 : 4;
    constexpr int ROWB = D * ESZ;
    constexpr int NCHUNK = ROWB / 16;
    constexpr int QCH = NCHUNK / kRowThreads;  // chunks per thread
    constexpr int QE = D / kRowThreads;        // elements per thread
    constexpr int TILEB = kFastTile * ROWB;
    constexpr int S = fast_stages(TILEB);
    static_assert(QCH % 2 == 0 && CH::kElems % 2 == 0 && D <= 128, "chunk pairs; the bound's D");
    extern __shared__ __align__(128) uint8_t s_ring[];  // [S][kFastTile][ROWB]
    __shared__ __align__(8) uint64_t s_full[S], s_empty[S];
    __shared__ unsigned long long s_live[S];  // bit r: row r of the stage holds a cache row
    __shared__ float s_q[D], s_qu[D];
    __shared__ float s_qh[kGroupRowsCap];  // the group's query elements [G][D]
    __shared__ float s_bmax[kFastWarps];
    __shared__ int s_bad[kFastWarps];
    __shared__ int s_abort;
    __shared__ long long s_part[4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (warp == 0) fast_part_of_cta(p, blockIdx.x, lane, s_part);
    __syncthreads();
    if (s_part[0] < 0) return;  // (past the batch's parts)
    const int b = (int)s_part[0], g = (int)s_part[1], split = (int)s_part[2];
    const long long chunk = s_part[3];
    const int last = __ldg(p.q_start + b + 1) - 1;
    if (last < __ldg(p.q_start + b)) {  // (the select kernel writes -1 without reading more)
        if (tid == 0 && split == 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    int cb, n;
    cand_range(p, b, cb, n, tid == 0 && split == 0);
    if (tid == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(saddr(&s_full[st]), 1);
            mbar_init(saddr(&s_empty[st]), kFastWarps);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort_flag = &s_abort;
    const int unit = b * p.kv.h_kv + g;
    const int t_begin = (int)min((long long)n, split * chunk);
    const int t_end = (int)min((long long)n, (split + 1) * chunk);
    const int n_tiles = (t_end - t_begin + kFastTile - 1) / kFastTile;
    float bmax = 0.f;
    bool bad = false;
    int n_issued = 0;
    if (warp == kFastWarps) {
        // ---- copy warp: lane 0 fills the ring ----
        if (lane == 0) {
            const char *kbase = reinterpret_cast<const char *>(p.kv.k);
            constexpr int kMaxRuns = kFastTile / kPageSize + 1;
            const bool paged = p.kv.page_size != 0;
            // Paged caches: the block-table entries of the pages tile u touches (-1 past its
            // rows), loaded together and one tile ahead, so that their latency passes while
            // the lane waits for a free stage instead of once per page on the issue path.
            const int32_t *btab = paged ? p.kv.block_table + (int64_t)b * p.kv.max_pages : nullptr;
            auto tile_pages = [&](int u, int *ent) {
                const int pos0 = cb + t_begin + u * kFastTile;
                const int end = u < n_tiles ? cb + min(t_begin + (u + 1) * kFastTile, t_end) : 0;
#pragma unroll
                for (int i = 0; i < kMaxRuns; ++i) {
                    const int pg = (pos0 >> 4) + i;
                    ent[i] = pg * kPageSize < end ? __ldg(btab + pg) : -1;
                }
            };
            int ent[kMaxRuns];
            if (paged) tile_pages(0, ent);
            for (int u = 0; u < n_tiles; ++u) {
                const int st = u % S;
                if (u >= S && !mbar_wait(saddr(&s_empty[st]), ((u / S) - 1) & 1, abort_flag,
                                         p.dev_err, p.wait_ns))
                    break;
                const int t0 = t_begin + u * kFastTile;
                const int rows = min(kFastTile, t_end - t0);
                int64_t roff[kMaxRuns];
                int rbeg[kMaxRuns], rlen[kMaxRuns];
                int nruns = 0;
                unsigned long long live = 0ull;
                if (!paged) {  // every row of the tile, one run
                    roff[0] = kv_row_offset(p.kv, b, g, cb + t0, p.dev_err);
                    rbeg[0] = 0;
                    rlen[0] = rows;
                    nruns = 1;
                    live = rows == 64 ? ~0ull : ((1ull << rows) - 1ull);
                } else {  // a run per page (pages without a valid entry: no copy, not live)
                    const int pos0 = cb + t0;
#pragma unroll
                    for (int i = 0; i < kMaxRuns; ++i) {
                        const int pg = (pos0 >> 4) + i;
                        const int r = max(pg * kPageSize - pos0, 0);  // the page's first row
                        if (r >= rows) continue;
                        const int len = min(rows - r, kPageSize - ((pos0 + r) & (kPageSize - 1)));
                        const int e = ent[i];
                        if (e >= 0 && e < p.kv.num_pages) {
                            roff[nruns] = (((int64_t)e * p.kv.h_kv + g) * kPageSize +
                                           ((pos0 + r) & (kPageSize - 1))) * p.kv.head_dim;
                            rbeg[nruns] = r;
                            rlen[nruns] = len;
                            ++nruns;
                            live |= ((len == 64 ? ~0ull : ((1ull << len) - 1ull)) << r);
                        } else {
                            set_dev_err(p.dev_err, SD_DEVERR_PAGE);
                        }
                    }
                    tile_pages(u + 1, ent);  // (the next tile's entries, while this one copies)
                }
                uint32_t bytes = 0;
                for (int i = 0; i < nruns; ++i) bytes += (uint32_t)(rlen[i] * ROWB);
                s_live[st] = live;
                const uint32_t dst = saddr(s_ring + (size_t)st * TILEB);
                mbar_arrive_tx(saddr(&s_full[st]), bytes);
                for (int i = 0; i < nruns; ++i)
                    bulk_load(dst + rbeg[i] * ROWB, kbase + roff[i] * ESZ,
                              (uint32_t)(rlen[i] * ROWB), saddr(&s_full[st]));
                n_issued = u + 1;
                if (*abort_flag) break;
            }
        }
    } else {
        // ---- scoring warps: thread quad (4c .. 4c+3) takes candidate c of each stage ----
        // (the query sums are formed while the first copies are in flight; the group's
        // elements are summed in head order, in fp64)
        const bool staged = p.group * D <= kGroupRowsCap;
        if (staged) {
            stage_group_rows<BF16, D>(p, last, g, s_qh, tid, kFastWarps * 32);
            asm volatile("bar.sync 1, %0;" ::"n"(kFastWarps * 32) : "memory");
        }
        for (int e = tid; e < D; e += kFastWarps * 32) {
            double acc = 0.0, mag = 0.0;
            for (int h = 0; h < p.group; ++h) {
                const double x = staged ? (double)s_qh[h * D + e]
                                        : (double)query_elem<BF16, D>(p.q, p.h_q, last,
                                                                      g * p.group + h, e);
                acc += x;
                mag += fabs(x);
            }
            s_q[e] = __double2float_rn(acc);
            s_qu[e] = __fadd_ru(__double2float_ru(mag), 0x1p-126f);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kFastWarps * 32) : "memory");  // scoring warps
        const int c = tid / kRowThreads, quarter = tid % kRowThreads;
        const int par = c & 1;
        float qr[QE], qu[QE];
        int choff[QCH];  // byte offsets of this thread's chunks, in its reading order
#pragma unroll
        for (int k = 0; k < QCH; ++k) {
            const int ch = quarter + kRowThreads * (k ^ par);
            choff[k] = ch * 16;
#pragma unroll
            for (int e = 0; e < CH::kElems; ++e) {
                qr[k * CH::kElems + e] = s_q[ch * CH::kElems + e];
                qu[k * CH::kElems + e] = s_qu[ch * CH::kElems + e];
            }
        }
        uint32_t *keys = reinterpret_cast<uint32_t *>(p.keys + (int64_t)unit * p.max_cand);
        for (int u = 0; u < n_tiles; ++u) {
            const int st = u % S;
            const bool got =
                mbar_wait(saddr(&s_full[st]), (u / S) & 1, abort_flag, p.dev_err, p.wait_ns);
            if (!__all_sync(0xffffffffu, got)) break;  // (the warp leaves together)
            const int cand = t_begin + u * kFastTile + c;
            const bool in_range = cand < t_end;
            const bool live = in_range && ((s_live[st] >> c) & 1ull);
            const uint8_t *rp = s_ring + (size_t)st * TILEB + c * ROWB;
            float2 y2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // four chains
            float2 b2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            if (live) {
#pragma unroll
                for (int k = 0; k < QCH; ++k) {
                    const uint4 raw = *reinterpret_cast<const uint4 *>(rp + choff[k]);
                    float f[CH::kElems];
                    CH::to_float(raw, f);
#pragma unroll
                    for (int e = 0; e < CH::kElems; e += 2) {
                        const int i = k * CH::kElems + e, a = (e >> 1) & 1;
                        y2[a] = __ffma2_rn(make_float2(f[e], f[e + 1]),
                                           make_float2(qr[i], qr[i + 1]), y2[a]);
                        b2[a] = __ffma2_rn(make_float2(fabsf(f[e]), fabsf(f[e + 1])),
                                           make_float2(qu[i], qu[i + 1]), b2[a]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(saddr(&s_empty[st]));  // the stage's rows are read
            float y = (y2[0].x + y2[1].x) + (y2[0].y + y2[1].y);
            float bb = (b2[0].x + b2[1].x) + (b2[0].y + b2[1].y);
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            y += __shfl_xor_sync(0xffffffffu, y, 2);  // the same sum in all four threads
            bb += __shfl_xor_sync(0xffffffffu, bb, 1);
            bb += __shfl_xor_sync(0xffffffffu, bb, 2);
            if (in_range) {
                if (live) {
                    bad |= !(isfinite(y) && isfinite(bb));
                    bmax = fmaxf(bmax, bb);
                } else {
                    bad = true;  // a row without a valid page: the fp64 path decides
                }
                if (quarter == 0) keys[cand] = live ? score_key32(y) : 0u;
            }
        }
        if (*abort_flag) bad = true;  // (an expired wait: the scores are incomplete)
    }
    // ---- teardown: after an abort, the copy lane waits (bounded) for its copies in flight ----
    if (warp == kFastWarps && lane == 0 && *abort_flag) {
        const unsigned long long t0 = now_ns();
        for (int u = (n_issued > S ? n_issued - S : 0); u < n_issued; ++u)
            while (!mbar_try(saddr(&s_full[u % S]), (u / S) & 1) && now_ns() - t0 < kDrainNs) {
            }
    }
    // the CTA's partial: its largest B and whether anything was not finite
    if (warp < kFastWarps) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
        const bool any_bad = __any_sync(0xffffffffu, bad);
        if (lane == 0) {
            s_bmax[warp] = bmax;
            s_bad[warp] = any_bad ? 1 : 0;
        }
    }
    __syncthreads();
    if (tid == 0) {
        float m = 0.f;
        int f = 0;
        for (int w = 0; w < kFastWarps; ++w) {
            m = fmaxf(m, s_bmax[w]);
            f |= s_bad[w];
        }
        p.parts[(int64_t)unit * p.part_stride + split] = make_uint2(__float_as_uint(m), (uint32_t)f);
    }
}

// D / 32 elements of a key row per lane (lane l: elements [l * D/32, (l+1) * D/32)).
template <bool BF16, int D>
__device__ __forceinline__ void lane_elems(const char *row, int lane, float (&f)[D / 32]) {
    constexpr int EPL = D / 32;
    static_assert(EPL == 2 || EPL == 4, "d = 64 or 128");
    if constexpr (BF16) {
        if constexpr (EPL == 4) {
            const uint2 v = *reinterpret_cast<const uint2 *>(row + lane * 8);
            f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        } else {
            const uint32_t v = *reinterpret_cast<const uint32_t *>(row + lane * 4);
            f[0] = bf16_lo(v); f[1] = bf16_hi(v);
        }
    } else {
        if constexpr (EPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(row + lane * 16);
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2 *>(row + lane * 8);
            f[0] = v.x; f[1] = v.y;
        }
    }
}

// fp64 score of the key row at element offset `off` (warp-collective; the same value in every
// lane): qbar . k, or, when that is not finite, the sum over the group's heads of q_h . k (the
// two differ there: +inf against heads of both signs is NaN).
template <bool BF16, int D>
__device__ double exact_score(const TopkParams &p, const double *s_qbar, int last, int g,
                              int64_t off, int lane) {
    constexpr int EPL = D / 32;
    const char *row = reinterpret_cast<const char *>(p.kv.k) + off * (BF16 ? 2 : 4);
    float f[EPL];
    lane_elems<BF16, D>(row, lane, f);
    double x = 0.0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) x = fma(s_qbar[lane * EPL + e], (double)f[e], x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (!isfinite(x)) {
        x = 0.0;
        for (int h = g * p.group; h < (g + 1) * p.group; ++h)
#pragma unroll
            for (int e = 0; e < EPL; ++e)
                x = fma((double)query_elem<BF16, D>(p.q, p.h_q, last, h, lane * EPL + e),
                        (double)f[e], x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    }
    return x;
}

constexpr int kSmemKeys32 = 49152;  // 192 KB of 32-bit keys
constexpr int kRadixBins = 2048;    // 11-bit digits
constexpr int kKeyGroups = 8;       // 32-key groups a warp reads per step (loads in flight)
constexpr int kGroupKeys = 32 * kKeyGroups;
constexpr int kBandCap = 1024;      // band candidates ranked in shared memory

// One CTA per (sequence, KV head): the radix select of the k-th largest fp32 key (tau), the
// band [tau - 2E, tau + 2E] rescored in fp64 and ranked, then the kept positions written in
// ascending order.  Falls back to fp64 scores of every candidate (select_keys64) when the
// scoring flagged the unit or the band does not fit.
template <bool BF16, int D>
__global__ void __launch_bounds__(kSelectThreads) topk_select_fast_kernel(const TopkParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    extern __shared__ uint32_t s_k32[];  // the unit's keys when max_cand <= kSmemKeys32
    __shared__ int s_hist[kRadixBins];
    __shared__ int s_warp[32];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_remaining;
    __shared__ double s_qbar[D];
    __shared__ float s_qh[kGroupRowsCap];             // the group's query elements [G][D]
    __shared__ int s_band[kBandCap];                  // band: local candidate index
    __shared__ unsigned long long s_bkey[kBandCap];   // and its fp64 score key
    __shared__ float s_bmax;
    __shared__ int s_flag;
    const int b = blockIdx.y, g = blockIdx.x, tid = threadIdx.x, lane = tid & 31,
              warp = tid >> 5;
    const int unit = b * p.kv.h_kv + g;
    int32_t *out = p.idx_out + (int64_t)unit * p.k;
    const int last = __ldg(p.q_start + b + 1) - 1;
    if (last < __ldg(p.q_start + b)) {
        for (int e = tid; e < p.k; e += kSelectThreads) out[e] = -1;
        return;
    }
    int cb, n;
    cand_range(p, b, cb, n);
    if (n <= p.k) {  // everything is selected
        for (int e = tid; e < p.k; e += kSelectThreads) out[e] = e < n ? cb + e : -1;
        return;
    }
    const bool staged = p.group * D <= kGroupRowsCap;
    if (staged) {
        stage_group_rows<BF16, D>(p, last, g, s_qh, tid, kSelectThreads);
        __syncthreads();
    }
    for (int e = tid; e < D; e += kSelectThreads) {  // (head order, fp64)
        double acc = 0.0;
        for (int h = 0; h < p.group; ++h)
            acc += staged ? (double)s_qh[h * D + e]
                          : (double)query_elem<BF16, D>(p.q, p.h_q, last, g * p.group + h, e);
        s_qbar[e] = acc;
    }
    if (warp == 0) {
        float m = 0.f;
        uint32_t f = 0u;
        const int n_parts = fast_parts_of(n, fast_part_chunk(p, lane));  // (the scoring's)
        for (int i = lane; i < n_parts; i += 32) {
            const uint2 v = p.parts[(int64_t)unit * p.part_stride + i];
            m = fmaxf(m, __uint_as_float(v.x));
            f |= v.y;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        f = __any_sync(0xffffffffu, f != 0u) ? 1u : 0u;
        if (lane == 0) {
            s_bmax = m;
            s_flag = (int)f;
        }
    }
    uint32_t *gkeys = reinterpret_cast<uint32_t *>(p.keys + (int64_t)unit * p.max_cand);
    const bool in_smem = p.max_cand <= kSmemKeys32;
    if (in_smem) {  // (the unit's key slots start 8-byte aligned: two keys per load, four
                    // loads in flight per thread)
        const uint2 *src = reinterpret_cast<const uint2 *>(gkeys);
        uint2 *dst = reinterpret_cast<uint2 *>(s_k32);
        const int n2 = n / 2;
        for (int base = 0; base < n2; base += 4 * kSelectThreads) {
            uint2 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = base + tid + j * kSelectThreads;
                v[j] = e < n2 ? src[e] : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = base + tid + j * kSelectThreads;
                if (e < n2) dst[e] = v[j];
            }
        }
        if ((n & 1) && tid == 0) s_k32[n - 1] = gkeys[n - 1];
    }
    __syncthreads();
    bool exact = s_flag != 0;
    if (!exact) {
        uint32_t *keys = in_smem ? s_k32 : gkeys;
        // warp w owns the keys [w * seg, w * seg + seg) (seg a multiple of kGroupKeys), which its
        // lanes read 32 consecutive keys at a time (coalesced in global memory, conflict-free in
        // shared memory), kKeyGroups groups in flight; keys past the segment or n read 0
        const int seg = ((n + 32 * kGroupKeys - 1) / (32 * kGroupKeys)) * kGroupKeys;
        const int wbeg = warp * seg;
        const int wend = min(n, wbeg + seg);
        auto load_groups = [&](int i, uint32_t (&kg)[kKeyGroups]) {  // (i: offset in the segment)
#pragma unroll
            for (int j = 0; j < kKeyGroups; ++j) {
                const int idx = wbeg + i + 32 * j + lane;
                kg[j] = idx < wend ? keys[idx] : 0u;
            }
        };
        // ---- radix select of the k-th largest key (digits of 11, 11 and 10 bits) ----
        // (a real key is never 0: that is the key of NaN, which flags the unit)
        uint32_t prefix = 0u, mask = 0u;
        int remaining = p.k;
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const uint32_t dmask = pass == 2 ? 1023u : 2047u;
            for (int i = tid; i < kRadixBins; i += kSelectThreads) s_hist[i] = 0;
            __syncthreads();
            for (int i = 0; wbeg + i < wend; i += kGroupKeys) {
                uint32_t kg[kKeyGroups];
                load_groups(i, kg);
#pragma unroll
                for (int j = 0; j < kKeyGroups; ++j)
                    if (kg[j] != 0u && (kg[j] & mask) == prefix)
                        atomicAdd(&s_hist[(kg[j] >> shift) & dmask], 1);
            }
            __syncthreads();
            // cumulative counts from the largest bucket down: thread t takes buckets
            // dmask - 2t and dmask - 2t - 1
            const int b0 = (int)dmask - 2 * tid, b1 = b0 - 1;
            const int c0 = b0 >= 0 ? s_hist[b0] : 0, c1 = b1 >= 0 ? s_hist[b1] : 0;
            int total;
            const int incl = block_inclusive_scan(c0 + c1, s_warp, total);
            const int before = incl - c0 - c1;
            if (before < remaining && incl >= remaining) {
                const bool in0 = before + c0 >= remaining;
                s_prefix = prefix | ((uint32_t)(in0 ? b0 : b1) << shift);
                s_remaining = remaining - before - (in0 ? 0 : c0);
            }
            __syncthreads();
            prefix = (uint32_t)s_prefix;
            remaining = s_remaining;
            mask |= dmask << shift;
        }
        // ---- the band around tau ----
        // For an fp32 y: y > hi <=> y > (hi rounded down to fp32), and y >= lo <=> y >= (lo
        // rounded up), so the band is a range of keys: [key_lo, key_hi].
        const double tau = (double)key32_value(prefix);
        const double E = (double)kErrScale * (double)s_bmax + kErrFloor;
        const uint32_t key_hi = score_key32(__double2float_rd(tau + 2.0 * E));
        const uint32_t key_lo = score_key32(__double2float_ru(tau - 2.0 * E));
        int n_in = 0, n_band = 0;
        for (int i = 0; wbeg + i < wend; i += kGroupKeys) {
            uint32_t kg[kKeyGroups];
            load_groups(i, kg);
#pragma unroll
            for (int j = 0; j < kKeyGroups; ++j) {  // (0, past the range, is below key_lo)
                n_in += kg[j] > key_hi ? 1 : 0;
                n_band += (kg[j] >= key_lo && kg[j] <= key_hi) ? 1 : 0;
            }
        }
        int in_total, band_total;
        block_inclusive_scan(n_in, s_warp, in_total);
        int pos = block_inclusive_scan(n_band, s_warp, band_total) - n_band;
        // (every candidate with x > T is kept or in the band, and those with x >= T number at
        // least k; a violation would mean a broken bound: the fp64 path decides then)
        exact = band_total > kBandCap || in_total >= p.k || in_total + band_total < p.k;
        if (!exact) {
            for (int i = 0; wbeg + i < wend; i += kGroupKeys) {
                uint32_t kg[kKeyGroups];
                load_groups(i, kg);
#pragma unroll
                for (int j = 0; j < kKeyGroups; ++j)
                    if (kg[j] >= key_lo && kg[j] <= key_hi) s_band[pos++] = wbeg + i + 32 * j + lane;
            }
            __syncthreads();
            for (int m = warp; m < band_total; m += kSelectThreads / 32) {
                const int64_t off = kv_row_offset(p.kv, b, g, cb + s_band[m], p.dev_err);
                // (rows without a valid page were flagged by the scoring: off >= 0 here)
                const double x = exact_score<BF16, D>(p, s_qbar, last, g, off, lane);
                if (lane == 0) s_bkey[m] = score_key(x);
            }
            __syncthreads();
            // rank within the band by (score descending, position ascending); the first
            // k - in_total are kept
            const int need = p.k - in_total;
            for (int m = tid; m < band_total; m += kSelectThreads) {
                const unsigned long long km = s_bkey[m];
                const int pm = s_band[m];
                int rank = 0;
                for (int o = 0; o < band_total; ++o) {
                    const unsigned long long ko = s_bkey[o];
                    rank += (ko > km || (ko == km && s_band[o] < pm)) ? 1 : 0;
                }
                keys[pm] = rank < need ? kKeyKept : kKeyDropped;
            }
            __syncthreads();
            // ---- output: kept positions, ascending ----
            // (kKeyKept is above every key, kKeyDropped below: the kept keys are those above
            // key_hi.)  Each warp counts its segment's, one scan over the warps gives its first
            // slot, and the warp writes its kept positions in order, 32 keys at a time.
            int keep_n = 0;
            for (int i = 0; wbeg + i < wend; i += kGroupKeys) {
                uint32_t kg[kKeyGroups];
                load_groups(i, kg);
#pragma unroll
                for (int j = 0; j < kKeyGroups; ++j) keep_n += kg[j] > key_hi ? 1 : 0;
            }
            keep_n = __reduce_add_sync(0xffffffffu, keep_n);
            if (lane == 0) s_warp[warp] = keep_n;
            __syncthreads();
            if (warp == 0) {
                const int c = s_warp[lane];
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                s_warp[lane] = incl - c;
            }
            __syncthreads();
            int w = s_warp[warp];
            for (int i = 0; wbeg + i < wend; i += kGroupKeys) {
                uint32_t kg[kKeyGroups];
                load_groups(i, kg);
#pragma unroll
                for (int j = 0; j < kKeyGroups; ++j) {
                    const bool keep = kg[j] > key_hi;
                    const unsigned bal = __ballot_sync(0xffffffffu, keep);
                    if (keep)
                        out[w + __popc(bal & ((1u << lane) - 1u))] = cb + wbeg + i + 32 * j + lane;
                    w += __popc(bal);
                }
            }
        }
    }
    if (exact) {  // (uniform: from the flag or from block-wide totals)
        // fp64 scores of every candidate, one warp per candidate, as 64-bit keys over the
        // unit's key slots (its 32-bit keys are no longer needed)
        unsigned long long *k64 = p.keys + (int64_t)unit * p.max_cand;
        __syncthreads();
        for (int t = warp; t < n; t += kSelectThreads / 32) {
            const int64_t off = kv_row_offset(p.kv, b, g, cb + t, p.dev_err);
            double x = 0.0;
            if (off >= 0) x = exact_score<BF16, D>(p, s_qbar, last, g, off, lane);
            if (lane == 0) k64[t] = off >= 0 ? score_key(x) : 0ull;
        }
        __syncthreads();
        select_keys64(p, out, cb, n, k64, s_hist, s_warp, s_prefix, s_remaining);
    }
}

template <bool BF16, int D>
cudaError_t launch_score_t(const TopkParams &p, cudaStream_t s) {
    const int dyn = score_stages(D * (BF16 ? 2 : 4)) * kScoreTile * D * (BF16 ? 2 : 4);
    auto kern = topk_score_kernel<BF16, D>;
    cudaError_t e = set_max_dynamic_smem<topk_score_kernel<BF16, D>>(dyn);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, p.kv.h_kv, p.batch);
    kern<<<grid, kScoreThreads, dyn, s>>>(p);
    return cudaGetLastError();
}

template <bool BF16, int D>
cudaError_t launch_fast_t(const TopkParams &p, cudaStream_t s) {
    const int tile = kFastTile * D * (BF16 ? 2 : 4);
    const int dyn = fast_stages(tile) * tile;
    cudaError_t e = set_max_dynamic_smem<topk_score_fast_kernel<BF16, D>>(dyn);
    if (e != cudaSuccess) return e;
    // one CTA per part, enough for every partition of the batch (fast_part_chunk)
    const long long ctas = (long long)p.batch * p.kv.h_kv * (p.n_splits + 1);
    if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    e = launch_pdl(topk_score_fast_kernel<BF16, D>, dim3((unsigned)ctas), dim3(kFastThreads), dyn,
                   s, p);
    if (e != cudaSuccess) return e;
    const size_t sdyn = p.max_cand <= kSmemKeys32 ? (size_t)p.max_cand * sizeof(uint32_t) : 0;
    e = set_max_dynamic_smem<topk_select_fast_kernel<BF16, D>>(
        (int)(kSmemKeys32 * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_select_fast_kernel<BF16, D>, dim3(p.kv.h_kv, p.batch),
                      dim3(kSelectThreads), sdyn, s, p);
}

}  // namespace

int topk_score_ctas_per_sm() { return kScoreCtasPerSm; }

int topk_part_stride(int max_cand) {
    const long long tiles = ((long long)max_cand + 127) / 128;
    return (int)std::max(1LL, std::min(1024LL, tiles / 4));
}

size_t topk_workspace_bytes(int batch, int h_kv, int max_cand) {
    if (max_cand < 1) return 0;
    const size_t units = (size_t)batch * h_kv;
    return units * (size_t)max_cand * sizeof(unsigned long long) +
           units * (size_t)topk_part_stride(max_cand) * sizeof(uint2);
}

cudaError_t launch_topk(const TopkParams &p, cudaStream_t s) {
    const bool bf = p.kv.dtype == SD_BF16;
    if (!p.scores && p.parts && p.max_cand > 0 && p.n_splits <= p.part_stride) {
        if (p.kv.head_dim == 128)
            return bf ? launch_fast_t<true, 128>(p, s) : launch_fast_t<false, 128>(p, s);
        return bf ? launch_fast_t<true, 64>(p, s) : launch_fast_t<false, 64>(p, s);
    }
    cudaError_t e;
    if (p.kv.head_dim == 128)
        e = bf ? launch_score_t<true, 128>(p, s) : launch_score_t<false, 128>(p, s);
    else
        e = bf ? launch_score_t<true, 64>(p, s) : launch_score_t<false, 64>(p, s);
    if (e != cudaSuccess) return e;
    return launch_topk_select(p, s);
}

cudaError_t launch_topk_select(const TopkParams &p, cudaStream_t s) {
    cudaError_t e;
    dim3 grid(p.kv.h_kv, p.batch);
    if (p.max_cand <= kSmemKeys) {
        const size_t dyn = (size_t)p.max_cand * sizeof(unsigned long long);
        e = set_max_dynamic_smem<topk_select_smem_kernel>(
            (int)(kSmemKeys * sizeof(unsigned long long)));
        if (e != cudaSuccess) return e;
        topk_select_smem_kernel<<<grid, kSelectThreads, dyn, s>>>(p);
    } else {
        topk_select_kernel<<<grid, kSelectThreads, 0, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace sd
