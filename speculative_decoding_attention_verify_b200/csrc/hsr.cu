// Hidden-state-reuse projection: y = W [emb ; hid] (+ bias), bf16 in/out, fp32 accumulation.
//
// A weight-streaming GEMV with n_rows <= 16 right-hand sides: every weight row (2*d_model
// bf16) is read from HBM exactly once per group of up to 4 input rows, with 16-byte loads,
// one warp per output feature.  The input rows are copied once per CTA into shared memory as
// the concatenation [emb ; hid] (the concatenation only ever exists in shared memory).
#include "sd_internal.h"

namespace sd {
namespace {

constexpr int kWarps = 8;

template <int NR>
__global__ void __launch_bounds__(kWarps * 32)
hsr_kernel(const uint16_t *emb, const uint16_t *hid, int n_rows, int d_model, const uint16_t *w,
           const uint16_t *bias, uint16_t *y) {
    extern __shared__ uint4 s_x4[];  // [NR][2*d_model] bf16, as 16-byte chunks
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r0 = blockIdx.y * NR;
    const int nr = min(NR, n_rows - r0);
    const int in_dim = 2 * d_model;
    const int chunks = in_dim / 8;  // 16-byte chunks per concatenated row
    for (int e = tid; e < NR * chunks; e += kWarps * 32) {
        const int r = e / chunks, c = e % chunks;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < nr) {
            const int col = c * 8;
            const uint16_t *src = col < d_model ? emb + (int64_t)(r0 + r) * d_model + col
                                                : hid + (int64_t)(r0 + r) * d_model + (col - d_model);
            v = *reinterpret_cast<const uint4 *>(src);
        }
        s_x4[e] = v;
    }
    __syncthreads();
    const int o = blockIdx.x * kWarps + warp;
    if (o >= d_model) return;
    const uint16_t *wrow = w + (int64_t)o * in_dim;
    float acc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = 0.f;
    constexpr int U = 14;  // 14 x 16 bytes per lane in flight
    for (int c0 = lane; c0 < chunks; c0 += 32 * U) {
        uint4 wv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + 32 * u;
            wv[u] = c < chunks ? ldg_stream16(wrow + c * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + 32 * u;
            if (c >= chunks) break;
            float wf[8];
            Chunk<true>::to_float(wv[u], wf);
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                float xf[8];
                Chunk<true>::to_float(s_x4[r * chunks + c], xf);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[r] = fmaf(wf[e], xf[e], acc[r]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        const float s = warp_sum(acc[r]);
        if (lane == 0 && r < nr) {
            float val = s;
            if (bias) val += __uint_as_float((uint32_t)bias[o] << 16);
            y[(int64_t)(r0 + r) * d_model + o] = (uint16_t)f32_to_bf16_bits(val);
        }
    }
}

template <int NR>
cudaError_t launch_hsr_t(const void *emb, const void *hid, int n_rows, int d_model, const void *w,
                         const void *bias, void *y, cudaStream_t s) {
    const size_t smem = (size_t)NR * 2 * d_model * sizeof(uint16_t);
    auto kern = hsr_kernel<NR>;
    if (smem > 48 * 1024) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((d_model + kWarps - 1) / kWarps, (n_rows + NR - 1) / NR);
    kern<<<grid, kWarps * 32, smem, s>>>(
        reinterpret_cast<const uint16_t *>(emb), reinterpret_cast<const uint16_t *>(hid), n_rows,
        d_model, reinterpret_cast<const uint16_t *>(w), reinterpret_cast<const uint16_t *>(bias),
        reinterpret_cast<uint16_t *>(y));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hsr(const void *emb, const void *hid, int n_rows, int d_model, const void *w,
                       const void *bias, void *y, cudaStream_t s) {
    if (n_rows == 1) return launch_hsr_t<1>(emb, hid, n_rows, d_model, w, bias, y, s);
    if (n_rows == 2) return launch_hsr_t<2>(emb, hid, n_rows, d_model, w, bias, y, s);
    return launch_hsr_t<4>(emb, hid, n_rows, d_model, w, bias, y, s);
}

}  // namespace sd
