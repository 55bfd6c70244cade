// Ring attention helpers: merging partial attention results over key shards, and accumulating
// gradient partials ("Attention Mechanism: Revolusi Representasi Sequence", §16 "Long Context
// Training", Ring Attention; §6 "Kompleksitas", long-context techniques table: the sequence is split
// across GPUs, each holds one chunk, and attention over all chunks is computed by passing K/V
// chunks around a ring).
//
// A query row attended over two disjoint key sets A and B has, with the softmax over their union,
//     LSE = log(exp(LSE_A) + exp(LSE_B)),   O = exp(LSE_A - LSE) * O_A + exp(LSE_B - LSE) * O_B,
// since each partial O is normalised by its own sum exp(LSE_X). A set that holds no visible key
// has LSE = -inf and weight 0. Both kernels are elementwise and HBM-bound: one warp per row for
// the merge (d/32 consecutive elements per lane), 8 elements per thread for the accumulation.
#include <cuda_bf16.h>

#include "ring.h"

namespace attn {

namespace {

template <int D>
__global__ void __launch_bounds__(256) ring_merge_kernel(float* __restrict__ o_acc,
                                                         float* __restrict__ lse_acc,
                                                         const void* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         long long rows, int part_bf16, int first,
                                                         void* __restrict__ o_out, int out_bf16) {
    constexpr int E = D / 32;   // elements per lane
    const int lane = threadIdx.x & 31;
    const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long row = w0; row < rows; row += nw) {
        const float la = first ? -INFINITY : lse_acc[row];
        const float lb = lse_part[row];
        const float mx = fmaxf(la, lb);
        float L, wa, wb;
        if (mx == -INFINITY) {
            L = -INFINITY;
            wa = 0.f;
            wb = 0.f;
        } else {
            const float ea = expf(la - mx), eb = expf(lb - mx);   // exp(-inf) = 0
            L = mx + logf(ea + eb);
            wa = ea / (ea + eb);
            wb = eb / (ea + eb);
        }
        const size_t base = static_cast<size_t>(row) * D + lane * E;
        float pv[E];
        if (part_bf16) {
            const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(o_part) + base;
#pragma unroll
            for (int x = 0; x < E; ++x) pv[x] = __bfloat162float(p[x]);
        } else {
            const float* p = static_cast<const float*>(o_part) + base;
#pragma unroll
            for (int x = 0; x < E; ++x) pv[x] = p[x];
        }
        float ov[E];
#pragma unroll
        for (int x = 0; x < E; ++x) {
            const float a = first ? 0.f : o_acc[base + x];
            ov[x] = (wa == 0.f ? 0.f : wa * a) + (wb == 0.f ? 0.f : wb * pv[x]);
            o_acc[base + x] = ov[x];
        }
        if (lane == 0) lse_acc[row] = L;
        if (o_out) {
            if (out_bf16) {
                __nv_bfloat16* q = static_cast<__nv_bfloat16*>(o_out) + base;
#pragma unroll
                for (int x = 0; x < E; ++x) q[x] = __float2bfloat16_rn(ov[x]);
            } else {
                float* q = static_cast<float*>(o_out) + base;
#pragma unroll
                for (int x = 0; x < E; ++x) q[x] = ov[x];
            }
        }
    }
}

__global__ void __launch_bounds__(256) ring_accumulate_kernel(float* __restrict__ acc,
                                                              const void* __restrict__ part,
                                                              long long count8, int part_bf16,
                                                              int first, void* __restrict__ out,
                                                              int out_bf16) {
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < count8;
         t += static_cast<long long>(gridDim.x) * blockDim.x) {
        float v[8];
        float4* a4 = reinterpret_cast<float4*>(acc + t * 8);
        if (first) {
#pragma unroll
            for (int x = 0; x < 8; ++x) v[x] = 0.f;
        } else {
            const float4 a = a4[0], b = a4[1];
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        if (part) {
            if (part_bf16) {
                const uint4 u = reinterpret_cast<const uint4*>(part)[t];
                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float2 f = __bfloat1622float2(h[x]);
                    v[2 * x] += f.x;
                    v[2 * x + 1] += f.y;
                }
            } else {
                const float4* p4 = reinterpret_cast<const float4*>(part) + 2 * t;
                const float4 a = p4[0], b = p4[1];
                v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
                v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
            }
        }
        a4[0] = make_float4(v[0], v[1], v[2], v[3]);
        a4[1] = make_float4(v[4], v[5], v[6], v[7]);
        if (out) {
            if (out_bf16) {
                uint4 u;
                __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                for (int x = 0; x < 4; ++x) h[x] = __floats2bfloat162_rn(v[2 * x], v[2 * x + 1]);
                reinterpret_cast<uint4*>(out)[t] = u;
            } else {
                float4* o4 = reinterpret_cast<float4*>(out) + 2 * t;
                o4[0] = make_float4(v[0], v[1], v[2], v[3]);
                o4[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
    }
}

unsigned grid_for(long long units, int per_block) {
    long long b = (units + per_block - 1) / per_block;
    if (b > 148LL * 16) b = 148LL * 16;
    return static_cast<unsigned>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_ring_merge(float* o_acc, float* lse_acc, const void* o_part,
                              const float* lse_part, long long rows, int d, int part_bf16,
                              int first, void* o_out, int out_bf16, cudaStream_t stream) {
    const unsigned grid = grid_for(rows, 8);   // 8 warps (rows) per block
    switch (d) {
        case 32:
            ring_merge_kernel<32><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, rows,
                                                            part_bf16, first, o_out, out_bf16);
            break;
        case 64:
            ring_merge_kernel<64><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, rows,
                                                            part_bf16, first, o_out, out_bf16);
            break;
        case 128:
            ring_merge_kernel<128><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part,
                                                             rows, part_bf16, first, o_out,
                                                             out_bf16);
            break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_ring_accumulate(float* acc, const void* part, long long count, int part_bf16,
                                   int first, void* out, int out_bf16, cudaStream_t stream) {
    const long long count8 = count / 8;
    ring_accumulate_kernel<<<grid_for(count8, 256), 256, 0, stream>>>(acc, part, count8, part_bf16,
                                                                      first, out, out_bf16);
    return cudaGetLastError();
}

}  // namespace attn
