// Device-side helpers shared by the kernels of libsdattn (sm_100a).
#pragma once

#include <atomic>

#include <cuda_runtime.h>
#include <stdint.h>

#include "sd_attn.h"

namespace sd {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPageSize = 16;

// KV cache view passed by value to kernels (mirrors sd_kv_desc).
struct KVView {
    int dtype;
    int h_kv;
    int head_dim;
    int page_size;
    const void *k;
    const void *v;
    int64_t stride_b, stride_h, stride_pos;
    const int32_t *block_table;
    int max_pages;
    int num_pages;
    const int32_t *kv_len;
};

// Programmatic dependent launch.  A kernel launched by launch_pdl may be scheduled while the
// previous kernel on its stream is still running (once that kernel's CTAs have all started,
// each of them calling pdl_trigger first); every such kernel calls pdl_wait before its first
// global memory access, which returns once the previous kernel has completed and its writes
// are visible.  The next call's launch and CTA scheduling thus overlap this call's tail.  Only
// launches made one by one take it: on a stream being captured into a CUDA graph the launch
// is plain (a replayed graph has its launches prepared already, and there the waiting CTAs
// only held SMs early: a speculative-decoding cycle replayed 1.6% slower with it, while the
// same cycle launched call by call ran 6% faster).  Without the attribute pdl_wait returns at
// once.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const bool eager = cudaStreamIsCapturing(s, &cs) == cudaSuccess &&
                       cs == cudaStreamCaptureStatusNone;
    cfg.attrs = attr;
    cfg.numAttrs = eager ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Opt kernel Kern in to `bytes` of dynamic shared memory, once per device (the attribute is
// per device, and a process may drive several).  `bytes` must be the same on every call.
template <auto Kern>
cudaError_t set_max_dynamic_smem(int bytes) {
    static std::atomic<unsigned long long> done{0};  // bit d: set on device d
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// 16-byte global -> shared copy through L2 only (cp.async), with its group commit and wait.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void set_dev_err(int32_t *flag, unsigned bits) {
    if (flag) atomicOr(reinterpret_cast<unsigned *>(flag), bits);
}

// Element offset of row (b, h, j) in the cache, or -1 when a paged cache has no valid page.
__device__ __forceinline__ int64_t kv_row_offset(const KVView &kv, int b, int h, int j,
                                                 int32_t *dev_err) {
    if (kv.page_size == 0)
        return (int64_t)b * kv.stride_b + (int64_t)h * kv.stride_h + (int64_t)j * kv.stride_pos;
    const int page = __ldg(kv.block_table + (int64_t)b * kv.max_pages + (j >> 4));
    if (page < 0 || page >= kv.num_pages) {
        set_dev_err(dev_err, SD_DEVERR_PAGE);
        return -1;
    }
    return (((int64_t)page * kv.h_kv + h) * kPageSize + (j & 15)) * kv.head_dim;
}

// bf16 bit pattern -> float (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// float -> bf16 bits, round to nearest even (finite inputs; NaN stays NaN).
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float x) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7fc0u;
    u += 0x7fffu + ((u >> 16) & 1u);
    return u >> 16;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Read-only 16-byte global load that bypasses L1 allocation (streamed KV data).
__device__ __forceinline__ uint4 ldg_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Convert a 16-byte chunk of the KV dtype to floats: 8 values for bf16, 4 for fp32.
template <bool BF16>
struct Chunk;

template <>
struct Chunk<true> {
    static constexpr int kElems = 8;
    __device__ __forceinline__ static void to_float(const uint4 &c, float *f) {
        f[0] = bf16_lo(c.x); f[1] = bf16_hi(c.x);
        f[2] = bf16_lo(c.y); f[3] = bf16_hi(c.y);
        f[4] = bf16_lo(c.z); f[5] = bf16_hi(c.z);
        f[6] = bf16_lo(c.w); f[7] = bf16_hi(c.w);
    }
};

template <>
struct Chunk<false> {
    static constexpr int kElems = 4;
    __device__ __forceinline__ static void to_float(const uint4 &c, float *f) {
        f[0] = __uint_as_float(c.x); f[1] = __uint_as_float(c.y);
        f[2] = __uint_as_float(c.z); f[3] = __uint_as_float(c.w);
    }
};

}  // namespace sd
