// Launch interface of the ring-attention helper kernels (ring.cu) for the C-ABI layer.
#pragma once

#include <cuda_runtime.h>

namespace attn {

cudaError_t launch_ring_merge(float* o_acc, float* lse_acc, const void* o_part,
                              const float* lse_part, long long rows, int d, int part_bf16,
                              int first, void* o_out, int out_bf16, cudaStream_t stream);
cudaError_t launch_ring_accumulate(float* acc, const void* part, long long count, int part_bf16,
                                   int first, void* out, int out_bf16, cudaStream_t stream);

}  // namespace attn
