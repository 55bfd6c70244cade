// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace attn {

struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    int B, H, n, d;
    int Hkv;          // K/V heads; query head h reads K/V head h / (H / Hkv)
    float scale;
    int causal;
    uint64_t timeout_ns;
};

struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* o;
    const void* dO;
    const float* lse;
    void* dq;
    void* dk;
    void* dv;
    int B, H, n, d;
    int Hkv;          // K/V heads (dk, dv have Hkv heads)
    float scale;
    int causal;
    int deterministic;
    float* Dvec;      // workspace: B*H*n_pad, D_i = rowsum(dO∘O) (0 on padding rows)
    float* L2vec;     // workspace: B*H*n_pad, LSE_i·log2(e) (+inf on padding rows)
    float* dq_acc;    // workspace: B*H*n_pad*d
    int* sems;        // workspace: B*H*(n_pad/64), deterministic mode only
    uint64_t timeout_ns;
    const cudaEvent_t* phase_events;   // 4 events or nullptr (measurement hook)
};

// Encodes a 3-D bf16 tensor map over a (B*H, n, d) tensor with a box of (chunk, box_rows, 1) and
// the swizzle that matches `chunk` (64 elements: 128-byte, 32 elements: 64-byte).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int BH, int n, int d,
                           int box_rows = 128);

cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint64_t timeout_ns, cudaStream_t stream);

}  // namespace attn
