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
//   - Outside stream capture every call looks up the array's device address on the current
//     device (cudaGetSymbolAddress, cheap), so a context that was reset and re-created is seen
//     at once. While the stream is being captured into a graph no runtime lookup is made: the
//     address that the latest uncaptured call on that device found is used, so make one call on
//     each device (outside capture) before capturing; a captured call without one fails with
//     ATTN_ERR_CUDA.
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

// Device address of the scratch array on the current device: looked up afresh outside capture,
// taken from the last lookup on this device while `stream` is capturing.
cudaError_t scratch_for_current_device(cudaStream_t stream, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    bool capturing = false;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        (void)cudaGetLastError();   // e.g. the legacy stream while another stream captures
        capturing = true;
    } else {
        capturing = cap != cudaStreamCaptureStatusNone;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (capturing) {
        if (!g_noalloc_ptr[dev]) return cudaErrorStreamCaptureUnsupported;
        *out = g_noalloc_ptr[dev];
        return cudaSuccess;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace attn

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                int B, int H, int n, int d, float scale, int causal, int dtype,
                                int deterministic, void* stream) {
    // The arguments and the size limit are checked before the device is touched, so an invalid
    // call returns its own error even where no device is usable.
    int rc = attn::validate_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, H, n, n, d, scale, dtype);
    if (rc != ATTN_OK) return rc;
    if (attn_bwd_workspace_bytes(B, H, n, d, deterministic) > attn::kNoAllocScratchBytes)
        return ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (attn::scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch) !=
        cudaSuccess)
        return ATTN_ERR_CUDA;
    // Same validation, kernels and error codes as attn_bwd; the workspace is the fixed array.
    return attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, n, d, scale, causal, dtype,
                    deterministic, scratch, attn::kNoAllocScratchBytes, stream);
}
