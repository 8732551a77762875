// Verify attention that allocates nothing: the split-KV partials live in a fixed scratch
// array of this library instead of a caller workspace.
//
// Who needs it: a caller that cannot allocate device memory at the moment of the call, e.g.
// a serving engine that hands all free HBM to its paged KV pool at start-up (a later
// cudaMalloc would fail, or would shrink the pool), or a host program that only holds device
// pointers given to it by another runtime and has no allocator of its own.  cudaMalloc may also
// synchronise the device, which such callers cannot afford in a decode loop.
//
// The scratch is a file-scope device array of kScratchBytes (64 MiB: enough for a 28-layer
// batch of 9 verify rows x 28 heads at d=128 and 26k cached positions, whose plan needs 38.5 MiB
// on 148 SMs, sized for either attention engine).  A call whose plan needs more is rejected
// with SD_ERR_WORKSPACE before anything is launched.  Nothing in the scratch has to start at
// zero: every split writes the partial output and (max, sum) of every row before the merge
// kernel reads them.
//
// The scratch is shared by every call on a device: two calls that may overlap on the device
// (different streams, or host threads, without ordering between them) race on it and give
// wrong results.  Calls on one stream are ordered and safe.
//
// The first call on each device looks up the scratch's device address with
// cudaGetSymbolAddress (which may load this module onto the device); make that first call
// before any stream capture.  The address is kept per device for later calls.
#include <atomic>
#include <mutex>

#include "sd_internal.h"

namespace {

constexpr size_t kScratchBytes = SD_VERIFY_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_verify_scratch[kScratchBytes];

std::atomic<void *> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch on the current device (looked up once per device).
sd_status scratch_on_current_device(void **ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SD_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SD_ERR_UNSUPPORTED;
    void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || !p) {
                cudaGetLastError();
                return SD_ERR_CUDA;
            }
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *ptr = p;
    return SD_OK;
}

}  // namespace

extern "C" {

sd_status sd_verify_attention_noalloc(const sd_q_desc *q, const void *q_data,
                                      const sd_kv_desc *kv, int32_t batch, void *out,
                                      int32_t *dev_err, void *stream) {
    SD_RANGE("sd_verify_attention_noalloc");
    sd::AttnPlan plan;
    sd_status st = sd::verify_plan(q, q_data, kv, batch, out, &plan);
    if (st != SD_OK) return st;
    if (plan.ws_bytes > kScratchBytes) return SD_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = scratch_on_current_device(&scratch);
    if (st != SD_OK) return st;
    return sd::verify_run(q, q_data, kv, batch, out, plan, scratch, dev_err, stream);
}

}  // extern "C"
