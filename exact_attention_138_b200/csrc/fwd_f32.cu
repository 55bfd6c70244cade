// Forward pass in plain fp32 on the FMA pipes, for the float32 examples of "Efficient Attention"
// (efficient_attention.py: (2,3,128,32) and the (4096,64) row-tiling case), whose results are
// compared at an absolute tolerance of 1e-5. TF32 tensor-core products cannot meet that, so
// every product here is an fp32 FFMA and exponentials use the accurate expf.
//
// Same method as the bf16 kernel (tiles of Q/K/V in on-chip memory, online softmax with running
// max m and sum l, output rescaled by exp(m_old - m_new); "Attention Mechanism: Revolusi
// Representasi Sequence", §13), laid out for SIMT: one CTA per 64-row query tile of one (b,h);
// 256 threads as a 16 x 16 grid, each thread owning 4 query rows x 4 key columns of the score
// tile and 4 rows x D/16 columns of the output accumulator.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;

template <int D>
constexpr int f32_smem_bytes() {
    return (kBM * (D + 1) + kBN * (D + 1) + kBN * D + kBM * (kBN + 1)) * 4;
}

template <int D>
__global__ void __launch_bounds__(256) fwd_f32_kernel(const float* __restrict__ Q,
                                                      const float* __restrict__ K,
                                                      const float* __restrict__ V,
                                                      float* __restrict__ O,
                                                      float* __restrict__ lse, MaskSpec mk,
                                                      int n_qtiles, float scale, int kv_group) {
    constexpr int DP = D + 1;
    constexpr int PP = kBN + 1;
    constexpr int OC = D / 16;
    extern __shared__ float fsm[];
    float* Qs = fsm;
    float* Ks = Qs + kBM * DP;
    float* Vs = Ks + kBN * DP;
    float* Ps = Vs + kBN * D;

    const int qt = n_qtiles - 1 - static_cast<int>(blockIdx.x);   // longest causal rows first
    const int bh = blockIdx.y;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int nq = mk.nq, nk = mk.nk;
    const size_t base = static_cast<size_t>(bh) * nq * D;
    const size_t kvbase = static_cast<size_t>(bh / kv_group) * nk * D;   // grouped-query K/V head
    const int q0 = qt * kBM;

    for (int idx = tid; idx < kBM * D; idx += 256) {
        const int r = idx / D, c = idx % D;
        Qs[r * DP + c] = (q0 + r < nq) ? Q[base + static_cast<size_t>(q0 + r) * D + c] : 0.f;
    }
    // visible keys [klo[i], khi[i]] of this thread's 4 rows
    int klo[4], khi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        long long lo, hi;
        visible_keys(mk, q0 + ty * 4 + i, q0 + ty * 4 + i, lo, hi);
        klo[i] = clamp_int(lo);
        khi[i] = clamp_int(hi);
    }

    float m[4], l[4], acc[4][OC];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int c = 0; c < OC; ++c) acc[i][c] = 0.f;
    }

    // key tiles that hold a key some row of this tile sees
    long long tlo, thi;
    visible_keys(mk, q0, min(q0 + kBM, nq) - 1, tlo, thi);
    const int kv_begin = tlo <= thi ? static_cast<int>(tlo / kBN) : 0;
    const int kv_end = tlo <= thi ? static_cast<int>(thi / kBN) + 1 : 0;
    for (int kt = kv_begin; kt < kv_end; ++kt) {
        const int k0 = kt * kBN;
        __syncthreads();
        for (int idx = tid; idx < kBN * D; idx += 256) {
            const int r = idx / D, c = idx % D;
            const bool in = k0 + r < nk;
            const size_t g = kvbase + static_cast<size_t>(k0 + r) * D + c;
            Ks[r * DP + c] = in ? K[g] : 0.f;
            Vs[r * D + c] = in ? V[g] : 0.f;
        }
        __syncthreads();

        float s[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[i][c] = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < D; ++kk) {
            float qv[4], kv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) qv[i] = Qs[(ty * 4 + i) * DP + kk];
#pragma unroll
            for (int c = 0; c < 4; ++c) kv[c] = Ks[(tx + 16 * c) * DP + kk];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[i][c] = fmaf(qv[i], kv[c], s[i][c]);
        }

#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int kidx = k0 + tx + 16 * c;
                s[i][c] = (kidx < klo[i] || kidx > khi[i]) ? -INFINITY : s[i][c] * scale;
                mx = fmaxf(mx, s[i][c]);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off, 16));
            const float m_new = fmaxf(m[i], mx);
            float alpha, rs = 0.f;
            if (m_new == -INFINITY) {
                alpha = 1.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) s[i][c] = 0.f;
            } else {
                alpha = (m[i] == -INFINITY) ? 0.f : expf(m[i] - m_new);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    s[i][c] = (s[i][c] == -INFINITY) ? 0.f : expf(s[i][c] - m_new);
                    rs += s[i][c];
                }
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off, 16);
            l[i] = l[i] * alpha + rs;
            m[i] = m_new;
#pragma unroll
            for (int c = 0; c < OC; ++c) acc[i][c] *= alpha;
#pragma unroll
            for (int c = 0; c < 4; ++c) Ps[(ty * 4 + i) * PP + tx + 16 * c] = s[i][c];
        }
        __syncthreads();

#pragma unroll 4
        for (int j = 0; j < kBN; ++j) {
            float pv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) pv[i] = Ps[(ty * 4 + i) * PP + j];
#pragma unroll
            for (int c = 0; c < OC; ++c) {
                const float vv = Vs[j * D + tx + 16 * c];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i][c] = fmaf(pv[i], vv, acc[i][c]);
            }
        }
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int qidx = q0 + ty * 4 + i;
        if (qidx >= nq) continue;
        // a row that sees no key: l = 0, accumulator 0 -> O = 0, LSE = -inf
        const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
#pragma unroll
        for (int c = 0; c < OC; ++c)
            O[base + static_cast<size_t>(qidx) * D + tx + 16 * c] = acc[i][c] * inv;
        if (tx == 0)
            lse[static_cast<size_t>(bh) * nq + qidx] = l[i] > 0.f ? m[i] + logf(l[i]) : -INFINITY;
    }
}

template <int D>
cudaError_t launch_fwd_f32_d(const FwdArgs& a, cudaStream_t stream) {
    constexpr int smem = f32_smem_bytes<D>();
    cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int nqt = (a.nq + kBM - 1) / kBM;
    const long long bh = static_cast<long long>(a.B) * a.H;
    if (bh > 65535) return cudaErrorInvalidConfiguration;
    dim3 grid(nqt, static_cast<unsigned>(bh));
    fwd_f32_kernel<D><<<grid, 256, smem, stream>>>(
        static_cast<const float*>(a.q), static_cast<const float*>(a.k),
        static_cast<const float*>(a.v), static_cast<float*>(a.o), a.lse,
        MaskSpec{a.nq, a.nk, a.wl, a.wr, static_cast<long long>(a.nk) - a.nq}, nqt, a.scale,
        a.H / a.Hkv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t stream) {
    switch (a.d) {
        case 32: return launch_fwd_f32_d<32>(a, stream);
        case 64: return launch_fwd_f32_d<64>(a, stream);
        case 128: return launch_fwd_f32_d<128>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
