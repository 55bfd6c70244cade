// attn_bwd_noalloc: the backward pass with its scratch memory taken from a fixed, library-owned
// device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where they run the
// backward pass — for example code embedded in a host framework that owns every device
// allocation and gives plug-ins no allocator, or a latency-critical loop that must not call
// cudaMalloc (which can synchronise the device). attn_bwd needs a workspace from the caller;
// this entry point needs none, and it calls no cudaMalloc, cudaFree or any other allocating
// routine.
//
// Cost and limits:
//   - kNoAllocScratchBytes (32 MiB) of device memory are reserved on every GPU on which this
//     library's device code is loaded, for the lifetime of the process.
//   - Sizes whose workspace (attn_bwd_workspace_bytes) exceeds that are rejected with
//     ATTN_ERR_WORKSPACE before anything is launched.
//   - The array is shared by all calls on a device and keeps the previous call's contents. The
//     backward pass itself rewrites or zeroes every part it reads (D, LSE·log2e, the dQ
//     accumulator and the semaphores are produced by its first kernel), so no clearing is needed
//     between calls; but two calls whose kernels overlap on the GPU (different streams without an
//     ordering between them, or several host threads) race on the array and give wrong results.
//   - The device address of the array is looked up with cudaGetSymbolAddress by the first call
//     on each device (with that device current); make that first call before any stream capture.
#include <mutex>

#include "../../include/attn.h"
#include "kernels.h"

namespace attn {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

// In host code this name is only a host-side stand-in for the device array: its device address
// must come from cudaGetSymbolAddress (see scratch_for_current_device).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
cudaError_t scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace attn

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                int B, int H, int n, int d, float scale, int causal, int dtype,
                                int deterministic, void* stream) {
    void* scratch = nullptr;
    if (attn::scratch_for_current_device(&scratch) != cudaSuccess) return ATTN_ERR_CUDA;
    // Same validation, kernels and error codes as attn_bwd; the workspace is the fixed array.
    return attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, n, d, scale, causal, dtype,
                    deterministic, scratch, attn::kNoAllocScratchBytes, stream);
}
