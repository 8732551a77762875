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

}  // namespace

int topk_score_ctas_per_sm() { return kScoreCtasPerSm; }

size_t topk_workspace_bytes(int batch, int h_kv, int max_cand) {
    return (size_t)batch * h_kv * (size_t)max_cand * sizeof(unsigned long long);
}

cudaError_t launch_topk(const TopkParams &p, cudaStream_t s) {
    const bool bf = p.kv.dtype == SD_BF16;
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
