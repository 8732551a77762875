// Sparrow's draft layer for a few draft rows: hidden-state reuse, RMSNorm, QKV with RoPE and the
// cache append, text-anchored attention over the draft's own cache, output projection, RMSNorm
// and the gated SiLU MLP.  Every projection is a weight-streaming GEMV (bf16 weights, fp32
// accumulation, at most kMaxRows rows) whose input vector is built in shared memory by a fused
// prologue and whose result is finished by a fused epilogue:
//   prologue  concat    [e ; h]                               (the HSR FC)
//             norm      RMSNorm(x) * gamma of an fp32 vector  (before QKV and before the MLP)
//             swiglu    silu(gate) * up of an fp32 vector      (before the down projection)
//             plain     a bf16 vector                          (the attention output)
//   epilogue  f32       fp32 out (+ bias) (+ fp32 residual)
//             bf16res   bf16 out = acc + fp32 residual         (the layer's output)
//             qkv       + bias; RoPE on the query and key heads (pairs (i, i + d/2), one unit
//                       of work), queries to a bf16 buffer, keys and values written into the
//                       cache at the rows' positions
// One 16-warp CTA per SM owns an even share of the output rows (of row pairs for qkv) and cuts
// each row into P parts (items), P chosen so that every warp gets several items of at least a
// few KB (the down projection's 18,944-weight rows spread over all warps instead of one warp per
// row).  Each warp streams two items at a time (seven 16-byte loads per lane per item in
// flight) and stores one partial per (item, input row); the parts of a row are then summed in a
// fixed order (deterministic) and finished by the epilogue.  The input vector is rebuilt by
// every CTA (it is tiny beside the weights).  The attention step is the library's own
// text-anchored attention call on the draft's text-only cache.
#include "sd_internal.h"

namespace sd {
namespace {

constexpr int kDlThreads = 512;  // 16 warps
constexpr int kDlWarps = kDlThreads / 32;
constexpr int kDlMaxRows = 4;
constexpr int kDlSmemMax = 200 * 1024;  // the input vectors of every row, bf16
constexpr int kDlSmemOptIn = 226 * 1024;  // dynamic shared memory a launch may use

enum { IN_CONCAT = 0, IN_NORM = 1, IN_SWIGLU = 2, IN_PLAIN = 3 };
enum { OUT_F32 = 0, OUT_BF16_RES = 1, OUT_QKV = 2 };

struct GemvArgs {
    const uint16_t *w;     // [m][k] bf16
    const uint16_t *bias;  // [m] or null
    int m, k, n;           // outputs, inputs, rows
    // prologue inputs
    const uint16_t *in_a;  // concat: e [n][k/2]; plain: [n][k]
    const uint16_t *in_b;  // concat: h [n][k/2]
    const float *in_f;     // norm: x [n][k]; swiglu: gate/up [n][2k]
    const uint16_t *gamma; // norm weight [k]
    float eps;
    // epilogue outputs
    float *out_f;          // f32: [n][m]
    uint16_t *out_b;       // bf16res: [n][m]; qkv: queries [n][h_q * d]
    const float *res;      // residual [n][m] or null
    // qkv
    int h_q, h_kv, d;
    double theta;
    KVView kv;             // the draft cache (batch 1): keys and values are written into it
    int32_t *params;       // qkv: [q_start0, q_start1, vis_b, vis_e, window] for the attention
    int window;
    int32_t *dev_err;
    int parts;             // items per weight row (chosen by the host)
};

__device__ __forceinline__ float silu(float t) { return t / (1.f + __expf(-t)); }

// The bf16 input vectors of every row into shared memory (s_x: [n][k]).
template <int IN>
__device__ __forceinline__ void build_input(const GemvArgs &a, uint16_t *s_x, float *s_red) {
    const int tid = threadIdx.x;
    const int k = a.k;
    if constexpr (IN == IN_CONCAT || IN == IN_PLAIN) {
        const int half = IN == IN_CONCAT ? k / 2 : k;
        for (int e = tid; e < a.n * (k / 8); e += kDlThreads) {
            const int r = e / (k / 8), c = (e % (k / 8)) * 8;
            const uint16_t *src = (IN == IN_PLAIN || c < half)
                                      ? a.in_a + (int64_t)r * half + c
                                      : a.in_b + (int64_t)r * half + (c - half);
            *reinterpret_cast<uint4 *>(s_x + (int64_t)r * k + c) =
                *reinterpret_cast<const uint4 *>(src);
        }
    } else if constexpr (IN == IN_NORM) {
        // 1 / sqrt(mean(x^2) + eps) per row: a block reduction in a fixed order.  The fp32
        // inputs are read as float4, four per thread in flight (the loads, not the arithmetic,
        // set the time of this prologue).
        const int k4 = k / 4;
        for (int r = 0; r < a.n; ++r) {
            const float4 *x4 = reinterpret_cast<const float4 *>(a.in_f + (int64_t)r * k);
            float ss = 0.f;
            for (int e0 = tid; e0 < k4; e0 += 4 * kDlThreads) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + u * kDlThreads;
                    v[u] = e < k4 ? x4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    ss = fmaf(v[u].x, v[u].x, ss);
                    ss = fmaf(v[u].y, v[u].y, ss);
                    ss = fmaf(v[u].z, v[u].z, ss);
                    ss = fmaf(v[u].w, v[u].w, ss);
                }
            }
            ss = warp_sum(ss);
            if ((tid & 31) == 0) s_red[tid >> 5] = ss;
            __syncthreads();
            if (tid == 0) {
                float t = 0.f;
                for (int w = 0; w < kDlWarps; ++w) t += s_red[w];
                s_red[kDlWarps + r] = rsqrtf(t / (float)k + a.eps);
            }
            __syncthreads();
        }
        for (int e0 = tid; e0 < a.n * k4; e0 += 4 * kDlThreads) {
            float4 v[4];
            uint2 gm[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * kDlThreads;
                const bool in = e < a.n * k4;
                v[u] = in ? reinterpret_cast<const float4 *>(a.in_f)[e]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
                gm[u] = in ? reinterpret_cast<const uint2 *>(a.gamma)[e % k4] : make_uint2(0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * kDlThreads;
                if (e >= a.n * k4) break;
                const float sc = s_red[kDlWarps + e / k4];
                const uint32_t lo = f32_to_bf16_bits(v[u].x * sc * bf16_lo(gm[u].x)) |
                                    (f32_to_bf16_bits(v[u].y * sc * bf16_hi(gm[u].x)) << 16);
                const uint32_t hi = f32_to_bf16_bits(v[u].z * sc * bf16_lo(gm[u].y)) |
                                    (f32_to_bf16_bits(v[u].w * sc * bf16_hi(gm[u].y)) << 16);
                reinterpret_cast<uint2 *>(s_x)[e] = make_uint2(lo, hi);
            }
        }
    } else {  // swiglu: gate/up [n][2k], read as float4, four per thread in flight
        const int k4 = k / 4;
        for (int e0 = tid; e0 < a.n * k4; e0 += 4 * kDlThreads) {
            float4 gt[4], up[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * kDlThreads;
                const bool in = e < a.n * k4;
                const int r = in ? e / k4 : 0, i = in ? e % k4 : 0;
                const float4 *row = reinterpret_cast<const float4 *>(a.in_f + (int64_t)r * 2 * k);
                gt[u] = in ? row[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                up[u] = in ? row[k4 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * kDlThreads;
                if (e >= a.n * k4) break;
                const uint32_t lo = f32_to_bf16_bits(silu(gt[u].x) * up[u].x) |
                                    (f32_to_bf16_bits(silu(gt[u].y) * up[u].y) << 16);
                const uint32_t hi = f32_to_bf16_bits(silu(gt[u].z) * up[u].z) |
                                    (f32_to_bf16_bits(silu(gt[u].w) * up[u].w) << 16);
                reinterpret_cast<uint2 *>(s_x)[e] = make_uint2(lo, hi);
            }
        }
    }
    __syncthreads();
}

constexpr int kItemLoads = 7;  // 16-byte loads per lane per item in flight

// Finishes a QKV row pair (h, i) / (h, i + d/2) of input row r from its two dot products: bias,
// RoPE for query and key heads (angle in double: positions reach 1e5 radians), then the query
// buffer or the cache.
__device__ __forceinline__ void finish_qkv(const GemvArgs &a, int h, int i, int kv_len, int r,
                                           float v1, float v2) {
    const int half = a.d / 2;
    const int o1 = h * a.d + i, o2 = o1 + half;
    if (a.bias) {
        v1 += __uint_as_float((uint32_t)a.bias[o1] << 16);
        v2 += __uint_as_float((uint32_t)a.bias[o2] << 16);
    }
    const int pos = kv_len - a.n + r;
    if (h < a.h_q + a.h_kv) {
        const double ang = (double)pos * pow(a.theta, -2.0 * (double)i / (double)a.d);
        double sn, cs;
        sincos(ang, &sn, &cs);
        const float c = (float)cs, s = (float)sn;
        const float r1 = v1 * c - v2 * s, r2 = v2 * c + v1 * s;
        v1 = r1;
        v2 = r2;
    }
    if (h < a.h_q) {
        uint16_t *q = a.out_b + ((int64_t)r * a.h_q + h) * a.d;
        q[i] = (uint16_t)f32_to_bf16_bits(v1);
        q[i + half] = (uint16_t)f32_to_bf16_bits(v2);
    } else {
        const bool is_k = h < a.h_q + a.h_kv;
        const int g = is_k ? h - a.h_q : h - a.h_q - a.h_kv;
        const int64_t row = kv_row_offset(a.kv, 0, g, pos, a.dev_err);
        if (row >= 0) {
            uint16_t *dst =
                reinterpret_cast<uint16_t *>(const_cast<void *>(is_k ? a.kv.k : a.kv.v)) + row;
            dst[i] = (uint16_t)f32_to_bf16_bits(v1);
            dst[i + half] = (uint16_t)f32_to_bf16_bits(v2);
        }
    }
}

// Finishes output o of input row r: bias, residual, fp32 or bf16 store.
template <int OUT>
__device__ __forceinline__ void finish_row(const GemvArgs &a, int o, int r, float v) {
    if (a.bias) v += __uint_as_float((uint32_t)a.bias[o] << 16);
    if (a.res) v += a.res[(int64_t)r * a.m + o];
    if (OUT == OUT_F32)
        a.out_f[(int64_t)r * a.m + o] = v;
    else
        a.out_b[(int64_t)r * a.m + o] = (uint16_t)f32_to_bf16_bits(v);
}

// Units of a GEMV: output rows, or (for qkv) row pairs (h, i) / (h, i + d/2).
template <int OUT>
__host__ __device__ __forceinline__ int gemv_units(const GemvArgs &a) {
    return OUT == OUT_QKV ? (a.h_q + 2 * a.h_kv) * (a.d / 2) : a.m;
}

template <int IN, int OUT>
__global__ void __launch_bounds__(kDlThreads, 1) draft_gemv_kernel(const GemvArgs a) {
    constexpr int RU = OUT == OUT_QKV ? 2 : 1;  // weight rows per unit
    constexpr int NR = kDlMaxRows;
    extern __shared__ __align__(16) uint16_t s_x[];  // [n][k] bf16, then [items][NR] f32
    __shared__ float s_red[kDlWarps + kDlMaxRows];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (OUT == OUT_QKV && blockIdx.x == 0 && tid == 0) {
        a.params[0] = 0;
        a.params[1] = a.n;
        a.params[2] = 0;
        a.params[3] = 0;
        a.params[4] = a.window;
    }
    const int U = gemv_units<OUT>(a);
    const int u0 = (int)((int64_t)U * blockIdx.x / gridDim.x);
    const int u1 = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
    const int P = a.parts;
    const int items = (u1 - u0) * RU * P;
    const int cpr = a.k / 8;  // 16-byte chunks per weight row
    float *s_part = reinterpret_cast<float *>(s_x + (size_t)a.n * a.k);
    build_input<IN>(a, s_x, s_red);  // (ends with a block barrier)
    // weight row of local item it, and its chunk range [c_lo, c_hi)
    auto item_row = [&](int it, int &c_lo, int &c_hi) -> const uint4 * {
        const int u = u0 + it / (RU * P), rr = (it / P) % RU, part = it % P;
        int row;
        if constexpr (OUT == OUT_QKV) {
            const int half = a.d / 2;
            row = (u / half) * a.d + u % half + rr * half;
        } else {
            row = u;
        }
        c_lo = (int)((int64_t)cpr * part / P);
        c_hi = (int)((int64_t)cpr * (part + 1) / P);
        return reinterpret_cast<const uint4 *>(a.w + (int64_t)row * a.k);
    };
    for (int it0 = warp; it0 < items; it0 += 2 * kDlWarps) {
        const int its[2] = {it0, it0 + kDlWarps};
        const uint4 *wr[2];
        int lo[2], hi[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            lo[k] = hi[k] = 0;
            wr[k] = its[k] < items ? item_row(its[k], lo[k], hi[k]) : nullptr;
        }
        float part[2][NR];
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int r = 0; r < NR; ++r) part[k][r] = 0.f;
        const int span = max(hi[0] - lo[0], hi[1] - lo[1]);
        for (int c0 = lane; c0 < span; c0 += 32 * kItemLoads) {
            uint4 wv[2][kItemLoads];
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
                for (int u = 0; u < kItemLoads; ++u) {
                    const int c = lo[k] + c0 + 32 * u;
                    wv[k][u] = c < hi[k] ? ldg_stream16(wr[k] + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
                for (int u = 0; u < kItemLoads; ++u) {
                    const int c = lo[k] + c0 + 32 * u;
                    if (c >= hi[k]) break;
                    float wf[8];
                    Chunk<true>::to_float(wv[k][u], wf);
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        if (r >= a.n) break;
                        float xf[8];
                        Chunk<true>::to_float(
                            *reinterpret_cast<const uint4 *>(s_x + (int64_t)r * a.k + c * 8), xf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) part[k][r] = fmaf(wf[e], xf[e], part[k][r]);
                    }
                }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const float sum = warp_sum(part[k][r]);
                if (lane == 0 && its[k] < items) s_part[its[k] * NR + r] = sum;
            }
    }
    __syncthreads();
    // epilogue: thread per (unit, input row); the unit's parts summed in a fixed order
    const int kv_len = OUT == OUT_QKV ? __ldg(a.kv.kv_len) : 0;
    for (int e = tid; e < (u1 - u0) * a.n; e += kDlThreads) {
        const int lu = e / a.n, r = e % a.n, u = u0 + lu;
        float v[RU];
#pragma unroll
        for (int rr = 0; rr < RU; ++rr) {
            float acc = 0.f;
            for (int q = 0; q < P; ++q) acc += s_part[((lu * RU + rr) * P + q) * NR + r];
            v[rr] = acc;
        }
        if constexpr (OUT == OUT_QKV)
            finish_qkv(a, u / (a.d / 2), u % (a.d / 2), kv_len, r, v[0], v[RU - 1]);
        else
            finish_row<OUT>(a, u, r, v[0]);
    }
}

// Parts per weight row: doubled (up to 8) while a CTA would hold fewer than six items per warp
// and each part keeps at least 64 chunks per half (so two loads per lane stay in flight).
template <int OUT>
int gemv_parts(const GemvArgs &a, int ctas) {
    const int ru = OUT == OUT_QKV ? 2 : 1;
    const int units_max = (gemv_units<OUT>(a) + ctas - 1) / ctas;
    const int cpr = a.k / 8;
    int p = 1;
    while (p < 8 && units_max * ru * p < 6 * kDlWarps && cpr / (2 * p * 2) >= 64) p *= 2;
    return p;
}

// Dynamic shared memory of a launch: the input vectors and the partials.
template <int OUT>
size_t gemv_smem(const GemvArgs &a, int ctas) {
    const int ru = OUT == OUT_QKV ? 2 : 1;
    const int units_max = (gemv_units<OUT>(a) + ctas - 1) / ctas;
    return (size_t)a.n * a.k * 2 + (size_t)units_max * ru * a.parts * kDlMaxRows * 4;
}

template <int IN, int OUT>
cudaError_t launch_gemv(GemvArgs a, cudaStream_t s) {
    // (the opt-in leaves room for the kernel's static shared memory within the 227 KB)
    cudaError_t e = set_max_dynamic_smem<draft_gemv_kernel<IN, OUT>>(kDlSmemOptIn);
    if (e != cudaSuccess) return e;
    const int ctas = device_sm_count();
    a.parts = gemv_parts<OUT>(a, ctas);
    const size_t smem = gemv_smem<OUT>(a, ctas);
    if (smem > (size_t)kDlSmemOptIn) return cudaErrorInvalidValue;
    draft_gemv_kernel<IN, OUT><<<ctas, kDlThreads, smem, s>>>(a);
    return cudaGetLastError();
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace regions of a draft-layer call.
struct DlLayout {
    size_t x, q, params, o, x2, gu, attn, end;
};

DlLayout dl_layout(const sd_draft_layer_desc *w, int n, size_t attn_ws) {
    DlLayout l{};
    const size_t D = w->d_model, HD = (size_t)w->h_q * w->head_dim, F = w->d_ff;
    l.x = 0;
    l.q = l.x + up256(n * D * 4);
    l.params = l.q + up256(n * HD * 2);
    l.o = l.params + 256;
    l.x2 = l.o + up256(n * HD * 2);
    l.gu = l.x2 + up256(n * D * 4);
    l.attn = l.gu + up256(n * 2 * F * 4);
    l.end = l.attn + up256(attn_ws);
    return l;
}

// The query and cache descriptors of the layer's attention (rows = the last n positions).
void attn_descs(const sd_draft_layer_desc *w, int n, const sd_kv_desc *cache, int max_kv_len,
                const int32_t *q_start, sd_q_desc *q) {
    (void)cache;
    q->h_q = w->h_q;
    q->max_q_rows = n;
    q->max_kv_len = max_kv_len;
    q->softmax_scale = 0.f;
    q->q_start = q_start;
}

bool layer_desc_ok(const sd_draft_layer_desc *w, int n) {
    if (!w || n < 1 || n > kDlMaxRows) return false;
    if (w->d_model < 16 || w->d_model % 16 || w->h_q < 1 || w->h_kv < 1 || w->h_q % w->h_kv ||
        (w->head_dim != 64 && w->head_dim != 128) || w->d_ff < 8 || w->d_ff % 8 ||
        !(w->rms_eps > 0.f) || !(w->rope_theta > 0.f))
        return false;
    if (!w->w_hsr || !w->ln1 || !w->w_qkv || !w->w_o || !w->ln2 || !w->w_gate_up || !w->w_down)
        return false;
    const uintptr_t al = reinterpret_cast<uintptr_t>(w->w_hsr) |
                         reinterpret_cast<uintptr_t>(w->ln1) | reinterpret_cast<uintptr_t>(w->ln2) |
                         reinterpret_cast<uintptr_t>(w->w_qkv) |
                         reinterpret_cast<uintptr_t>(w->w_o) |
                         reinterpret_cast<uintptr_t>(w->w_gate_up) |
                         reinterpret_cast<uintptr_t>(w->w_down);
    if (al & 15) return false;
    // every input vector fits the GEMV's shared memory
    const size_t kmax = (size_t)n * 2 *
                        ((size_t)2 * w->d_model > (size_t)w->d_ff
                             ? ((size_t)2 * w->d_model > (size_t)w->h_q * w->head_dim
                                    ? (size_t)2 * w->d_model
                                    : (size_t)w->h_q * w->head_dim)
                             : ((size_t)w->d_ff > (size_t)w->h_q * w->head_dim
                                    ? (size_t)w->d_ff
                                    : (size_t)w->h_q * w->head_dim));
    return kmax <= (size_t)kDlSmemMax;
}

}  // namespace

}  // namespace sd

using namespace sd;

extern "C" {

sd_status sd_draft_layer_workspace_size(const sd_draft_layer_desc *w, int32_t n_rows,
                                        const sd_kv_desc *cache, int32_t max_kv_len,
                                        int32_t window, size_t *bytes) {
    if (!bytes || !cache || !layer_desc_ok(w, n_rows) || max_kv_len < n_rows || window < 1)
        return SD_ERR_INVALID_ARG;
    sd_q_desc q;
    attn_descs(w, n_rows, cache, max_kv_len, nullptr, &q);
    q.q_start = reinterpret_cast<const int32_t *>(16);  // not read by the size query
    size_t attn = 0;
    const sd_status st = sd_attention_workspace_size(SD_ATTN_TEXT_ANCHORED, &q, cache, 1, &attn);
    if (st != SD_OK) return st;
    *bytes = dl_layout(w, n_rows, attn).end;
    return SD_OK;
}

sd_status sd_draft_layer(const sd_draft_layer_desc *w, const void *emb, const void *hid,
                         int32_t n_rows, const sd_kv_desc *cache, int32_t max_kv_len,
                         int32_t window, void *y, void *workspace, size_t workspace_bytes,
                         int32_t *dev_err, void *stream) {
    SD_RANGE("sd_draft_layer");
    if (!emb || !hid || !y || !cache || !layer_desc_ok(w, n_rows) || max_kv_len < n_rows ||
        window < 1)
        return SD_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(emb) | reinterpret_cast<uintptr_t>(hid)) & 15) ||
        cache->dtype != SD_BF16 || cache->h_kv != w->h_kv || cache->head_dim != w->head_dim ||
        !cache->k || !cache->v || !cache->kv_len)
        return SD_ERR_INVALID_ARG;
    size_t need = 0;
    sd_status st = sd_draft_layer_workspace_size(w, n_rows, cache, max_kv_len, window, &need);
    if (st != SD_OK) return st;
    if (!workspace || need > workspace_bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return SD_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    const DlLayout l = dl_layout(w, n_rows, need - dl_layout(w, n_rows, 0).end);
    float *x = reinterpret_cast<float *>(ws + l.x);
    uint16_t *qb = reinterpret_cast<uint16_t *>(ws + l.q);
    int32_t *params = reinterpret_cast<int32_t *>(ws + l.params);
    uint16_t *ob = reinterpret_cast<uint16_t *>(ws + l.o);
    float *x2 = reinterpret_cast<float *>(ws + l.x2);
    float *gu = reinterpret_cast<float *>(ws + l.gu);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = w->d_model, HD = w->h_q * w->head_dim, F = w->d_ff;
    KVView kv{};
    kv.dtype = cache->dtype;
    kv.h_kv = cache->h_kv;
    kv.head_dim = cache->head_dim;
    kv.page_size = cache->page_size;
    kv.k = cache->k;
    kv.v = cache->v;
    kv.stride_b = cache->stride_b;
    kv.stride_h = cache->stride_h;
    kv.stride_pos = cache->stride_pos;
    kv.block_table = cache->block_table;
    kv.max_pages = cache->max_pages_per_seq;
    kv.num_pages = cache->num_pages;
    kv.kv_len = cache->kv_len;
    GemvArgs a{};
    a.n = n_rows;
    a.eps = w->rms_eps;
    a.dev_err = dev_err;
    // x = W_hsr [e ; h]
    a.w = static_cast<const uint16_t *>(w->w_hsr);
    a.m = D;
    a.k = 2 * D;
    a.in_a = static_cast<const uint16_t *>(emb);
    a.in_b = static_cast<const uint16_t *>(hid);
    a.out_f = x;
    if (launch_gemv<IN_CONCAT, OUT_F32>(a, s) != cudaSuccess) return SD_ERR_CUDA;
    // q, k, v = W_qkv RMSNorm(x) + b; RoPE; k, v into the cache
    a = GemvArgs{};
    a.n = n_rows;
    a.eps = w->rms_eps;
    a.dev_err = dev_err;
    a.w = static_cast<const uint16_t *>(w->w_qkv);
    a.bias = static_cast<const uint16_t *>(w->b_qkv);
    a.m = (w->h_q + 2 * w->h_kv) * w->head_dim;
    a.k = D;
    a.in_f = x;
    a.gamma = static_cast<const uint16_t *>(w->ln1);
    a.out_b = qb;
    a.h_q = w->h_q;
    a.h_kv = w->h_kv;
    a.d = w->head_dim;
    a.theta = w->rope_theta;
    a.kv = kv;
    a.params = params;
    a.window = window;
    if (launch_gemv<IN_NORM, OUT_QKV>(a, s) != cudaSuccess) return SD_ERR_CUDA;
    // o = text-anchored attention of the rows over the draft cache (no visual span)
    sd_q_desc q;
    attn_descs(w, n_rows, cache, max_kv_len, params, &q);
    st = sd_text_anchored_attention(&q, qb, cache, 1, params + 2, params + 3, params + 4, window,
                                    ob, ws + l.attn, need - l.attn, dev_err, stream);
    if (st != SD_OK) return st;
    // x2 = x + W_o o
    a = GemvArgs{};
    a.n = n_rows;
    a.dev_err = dev_err;
    a.w = static_cast<const uint16_t *>(w->w_o);
    a.m = D;
    a.k = HD;
    a.in_a = ob;
    a.res = x;
    a.out_f = x2;
    if (launch_gemv<IN_PLAIN, OUT_F32>(a, s) != cudaSuccess) return SD_ERR_CUDA;
    // [gate ; up] = W_gate_up RMSNorm(x2)
    a = GemvArgs{};
    a.n = n_rows;
    a.eps = w->rms_eps;
    a.dev_err = dev_err;
    a.w = static_cast<const uint16_t *>(w->w_gate_up);
    a.m = 2 * F;
    a.k = D;
    a.in_f = x2;
    a.gamma = static_cast<const uint16_t *>(w->ln2);
    a.out_f = gu;
    if (launch_gemv<IN_NORM, OUT_F32>(a, s) != cudaSuccess) return SD_ERR_CUDA;
    // y = x2 + W_down (silu(gate) * up)
    a = GemvArgs{};
    a.n = n_rows;
    a.dev_err = dev_err;
    a.w = static_cast<const uint16_t *>(w->w_down);
    a.m = D;
    a.k = F;
    a.in_f = gu;
    a.res = x2;
    a.out_b = static_cast<uint16_t *>(y);
    if (launch_gemv<IN_SWIGLU, OUT_BF16_RES>(a, s) != cudaSuccess) return SD_ERR_CUDA;
    return SD_OK;
}

}  // extern "C"
