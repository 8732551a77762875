// Compaction of the sparse draft's selected KV rows, so that the tensor-core attention kernel
// can stream them with TMA as one run of positions.
//
// For every (sequence b, KV head g) the ascending list idx[b][g][0..k) names cache positions;
// an entry is kept when 0 <= x < tail_begin[b] and it differs from the entry before it (the
// selected set; entries at or past the tail are covered by the dense tail, negative ones are
// padding).  Kept entry number c goes to row c of the compact K and V buffers
// [batch][h_kv][k_cap][d], its position to cpos, and the count to k_eff[b][g].  A list that is
// not ascending sets SD_DEVERR_INDEX (the result is then unspecified, as for every engine).
//
// Grid (parts, h_kv, batch): part r copies the kept entries among list entries
// [k*r/parts, k*(r+1)/parts); each CTA first counts the kept entries before its range (about
// eight CTAs per SM, all resident at once).  Warps copy two rows (d = 128) or four (d = 64) per
// 16-byte-per-lane instruction, four such row groups loaded before any is stored.
#include "attn_stream.cuh"

namespace sd {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ bool kept(const int32_t *sel, int e, int tail) {
    const int x = __ldg(sel + e);
    return x >= 0 && x < tail && (e == 0 || __ldg(sel + e - 1) != x);
}

template <int D>
__global__ void __launch_bounds__(kThreads) sparse_compact_kernel(const AttnParams p) {
    pdl_trigger();  // (see launch_pdl)
    pdl_wait();
    constexpr int CPR = D * 2 / 16;  // 16-byte chunks per row (bf16)
    constexpr int RPI = 32 / CPR;    // rows per warp instruction
    __shared__ int s_warp[kThreads / 32];
    __shared__ int s_base;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, g = blockIdx.y, part = blockIdx.x, parts = gridDim.x;
    const int unit = b * p.kv.h_kv + g;
    const int kv_len = __ldg(p.kv.kv_len + b);
    const int tail = min(max(__ldg(p.tail_begin + b), 0), kv_len);
    const int32_t *sel = p.idx + (int64_t)unit * p.k_sel;
    const int e_lo = (int)((int64_t)p.k_sel * part / parts);
    const int e_hi = (int)((int64_t)p.k_sel * (part + 1) / parts);

    // kept entries before e_lo (and, from part 0, the order check of the whole list)
    int cnt = 0;
    for (int e = tid; e < e_lo; e += kThreads) cnt += kept(sel, e, tail) ? 1 : 0;
    if (part == 0)
        for (int e = 1 + tid; e < p.k_sel; e += kThreads) {
            const int x = __ldg(sel + e), prev = __ldg(sel + e - 1);
            if (x >= 0 && x < tail && (prev > x || prev < 0)) set_dev_err(p.dev_err, SD_DEVERR_INDEX);
        }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) s_warp[warp] = cnt;
    __syncthreads();
    if (tid == 0) {
        int base = 0;
        for (int w = 0; w < kThreads / 32; ++w) base += s_warp[w];
        s_base = base;
    }
    __syncthreads();
    int base = s_base;

    const int64_t row0 = (int64_t)unit * p.k_cap;  // first compact row of this unit
    const uint4 *kb = reinterpret_cast<const uint4 *>(p.kv.k);
    const uint4 *vb = reinterpret_cast<const uint4 *>(p.kv.v);
    uint4 *ck = reinterpret_cast<uint4 *>(p.ck);
    uint4 *cv = reinterpret_cast<uint4 *>(p.cv);
    // walk the range in chunks of kThreads entries: flag, block scan, copy
    for (int c0 = e_lo; c0 < e_hi; c0 += kThreads) {
        const int e = c0 + tid;
        const bool keep = e < e_hi && kept(sel, e, tail);
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) s_warp[warp] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            const int n = s_warp[w];
            before += w < warp ? n : 0;
            total += n;
        }
        const int slot = base + before + __popc(bal & ((1u << lane) - 1u));
        int64_t off = -1;
        if (keep) {
            const int x = __ldg(sel + e);
            p.cpos[row0 + slot] = x;
            off = kv_row_offset(p.kv, b, g, x, p.dev_err);  // element offset, or -1 (bad page)
        }
        // copy the chunk's kept rows: each warp takes its own 32 entries, loading kBatch
        // row groups before storing them so that several loads per lane are in flight
        constexpr int kBatch = 4;
        for (int r0 = 0; r0 < 32; r0 += RPI * kBatch) {
            uint4 kx[kBatch], vx[kBatch];
            int64_t dst[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int r = r0 + u * RPI + lane / CPR, ch = lane % CPR;
                const int64_t o = __shfl_sync(0xffffffffu, off, r);
                const bool kr = r < 32 && ((bal >> r) & 1u);
                dst[u] = -1;
                kx[u] = make_uint4(0, 0, 0, 0);
                vx[u] = make_uint4(0, 0, 0, 0);
                if (kr) {
                    dst[u] = (row0 + base + before + __popc(bal & ((1u << r) - 1u))) * CPR + ch;
                    if (o >= 0) {
                        kx[u] = ldg_stream16(kb + o / 8 + ch);
                        vx[u] = ldg_stream16(vb + o / 8 + ch);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                if (dst[u] >= 0) {
                    ck[dst[u]] = kx[u];
                    cv[dst[u]] = vx[u];
                }
        }
        base += total;
        __syncthreads();  // s_warp is reused by the next chunk
    }
    if (part == parts - 1 && tid == 0) p.k_eff[unit] = base;
}

}  // namespace

cudaError_t launch_sparse_compact(const AttnParams &p, cudaStream_t s) {
    const int units = p.batch * p.kv.h_kv;
    const int want = (8 * device_sm_count() + units - 1) / units;  // about eight CTAs per SM
    const int by_len = (p.k_sel + 127) / 128;
    const int parts = max(1, min(want, by_len));
    dim3 grid(parts, p.kv.h_kv, p.batch);
    if (p.kv.head_dim == 128)
        return launch_pdl(sparse_compact_kernel<128>, grid, dim3(kThreads), 0, s, p);
    else
        return launch_pdl(sparse_compact_kernel<64>, grid, dim3(kThreads), 0, s, p);
    return cudaGetLastError();
}

}  // namespace sd
