// route_noalloc.cu -- beam_moe_route_noalloc: the routing call for callers
// that cannot allocate device memory, with its scratch in a fixed device
// array that this file owns.
//
// Who cannot allocate: plugins embedded in a host runtime whose memory pool
// owns all of the device's memory and gives its extensions none of their own
// (a serving engine that reserves the GPU up front, for example), and callers
// working inside a fixed memory budget where any allocation may fail or
// fragment the pool.  Such callers still own their inputs and outputs; only
// the library's scratch (the router's split-K partial logits and the
// error/counter header) moves into the array below.
#include <cuda_runtime.h>

#include <mutex>

#include "beam_internal.h"
#include "beam_moe.h"

namespace {

constexpr size_t kScratchBytes = BEAM_MOE_ROUTE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per GPU that loads the library, held until the process exits.
// Host code sees only a host-side stand-in under this name; the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_route_scratch on the current device, looked up once per
// device with that device current.
beam_status scratch_for_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BEAM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return BEAM_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return BEAM_OK;
}

}  // namespace

extern "C" beam_status beam_moe_route_noalloc(const beam_moe_desc *desc, const void *x,
                                              const void *W_gate, const void *W_mask,
                                              int32_t *topk_idx, float *topk_w,
                                              int32_t *expert_counts, int32_t *kept_hist,
                                              float *logits, void *stream) {
    const size_t need = beam::route_scratch_bytes(desc);
    if (need == 0) {
        beam_moe_plan_info P;
        return beam_moe_plan(desc, &P);  // the descriptor's own error
    }
    if (need > kScratchBytes) return BEAM_ERR_WORKSPACE;  // batch too large for the array
    void *scratch = nullptr;
    beam_status s = scratch_for_current_device(&scratch);
    if (s != BEAM_OK) return s;
    return beam::route_into_scratch(desc, x, W_gate, W_mask, topk_idx, topk_w, expert_counts,
                                    kept_hist, logits, scratch, kScratchBytes,
                                    static_cast<cudaStream_t>(stream));
}

extern "C" beam_status beam_moe_route_noalloc_check(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BEAM_ERR_CUDA;
    void *scratch = nullptr;
    beam_status s = scratch_for_current_device(&scratch);
    if (s != BEAM_OK) return s;
    int err = 0;  // the header's error word (offset 0 of the scratch)
    if (cudaMemcpy(&err, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return BEAM_ERR_CUDA;
    if (err == beam::DEV_ERR_TIMEOUT) return BEAM_ERR_TIMEOUT;
    if (err != beam::DEV_OK) return BEAM_ERR_INTERNAL;
    return BEAM_OK;
}
