// Forward pass in plain fp32 on the FMA pipes, for the float32 examples of "Efficient Attention"
// (efficient_attention.py: (2,3,128,32) and the (4096,64) row-tiling case), whose results are
// compared at an absolute tolerance of 1e-5. TF32 tensor-core products cannot meet that, so
// every product here is an fp32 FFMA and exponentials use the accurate expf.
//
// Same method as the bf16 kernel (tiles of Q/K/V in on-chip memory, online softmax with running
// max m and sum l, output rescaled by exp(m_old - m_new); "Attention Mechanism: Revolusi
// Representasi Sequence", §13), laid out for SIMT. One CTA works on a 64-row query tile of one
// (b,h) with 256 threads as a 16 x 16 grid; each thread owns 4 query rows x 4 key columns of the
// 64 x 64 score tile and 4 rows x d/16 columns of the output accumulator. Every shared-memory
// operand is read 16 bytes at a time (rows padded so that the reads are conflict-free or
// broadcast), and the next K/V tile is copied in with cp.async while the current one is used.
//
// Small grids (the pages' examples have 12 and 64 query tiles for 148 SMs) split each query
// tile's key range over a thread-block cluster of up to 8 CTAs. Each CTA keeps its own (m, l, O)
// for its share of the keys; the cluster then merges them through distributed shared memory with
// the same rule that joins two softmax blocks (weights exp(m_s - M), M the largest m_s), each CTA
// finishing a slice of the rows. No global scratch and no second launch are needed.
#include <cooperative_groups.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

namespace cg = cooperative_groups;

constexpr int kBM = 64;          // query rows per CTA
constexpr int kBN = 64;          // keys per tile
constexpr int kPP = kBN + 4;     // row stride of the P tile (floats)
constexpr int kMaxSplit = 8;     // portable cluster size

template <int D>
struct F32Cfg {
    static constexpr int QP = D + 4;                   // row stride of Q and K tiles (floats)
    static constexpr int CW = D >= 64 ? 4 : 2;          // contiguous output columns per thread
    static constexpr int NG = D / (16 * CW);           // groups of CW columns per thread
    static constexpr int OC = NG * CW;                 // = D / 16
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + kBM * QP;     // two K buffers of kBN x QP
    static constexpr int V_OFF = K_OFF + 2 * kBN * QP; // two V buffers of kBN x D
    static constexpr int P_OFF = V_OFF + 2 * kBN * D;  // kBM x kPP
    static constexpr int ML_OFF = P_OFF + kBM * kPP;   // kBM x (m, l)
    static constexpr int FLOATS = ML_OFF + 2 * kBM;
    static constexpr int SMEM = FLOATS * 4;
    static constexpr int MIN_BLOCKS = D <= 64 ? 2 : 1;
    static_assert(kBM * D <= 2 * kBN * QP, "merge buffer must fit in the K buffers");
};

__device__ __forceinline__ void cp_async16(float* dst, const float* src, bool valid) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    const int n = valid ? 16 : 0;     // 0 source bytes: the 16 destination bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// rows [0, rows) x D floats from global `src` (row stride D) into shared `dst` (row stride ld);
// rows at or past `valid_rows` are zero-filled and read nothing.
template <int D>
__device__ __forceinline__ void load_rows(float* dst, int ld, const float* src, int rows,
                                          int valid_rows, int tid) {
    constexpr int C4 = D / 4;
    for (int idx = tid; idx < rows * C4; idx += 256) {
        const int r = idx / C4, c4 = idx % C4;
        const bool ok = r < valid_rows;
        cp_async16(dst + r * ld + c4 * 4, ok ? src + static_cast<size_t>(r) * D + c4 * 4 : src,
                   ok);
    }
}

template <int D>
__global__ void __launch_bounds__(256, F32Cfg<D>::MIN_BLOCKS)
    fwd_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                   const float* __restrict__ V, float* __restrict__ O, float* __restrict__ lse,
                   MaskSpec mk, int n_qtiles, int split, float scale, int kv_group) {
    using C = F32Cfg<D>;
    constexpr int QP = C::QP, CW = C::CW, NG = C::NG, OC = C::OC;
    extern __shared__ __align__(16) float fsm[];
    float* Qs = fsm + C::Q_OFF;
    float* Ps = fsm + C::P_OFF;
    float* ML = fsm + C::ML_OFF;

    const int rank = static_cast<int>(blockIdx.x) % split;             // key share in the cluster
    const int qt = n_qtiles - 1 - static_cast<int>(blockIdx.x) / split; // longest causal rows first
    const int bh = blockIdx.y;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int nq = mk.nq, nk = mk.nk;
    const size_t base = static_cast<size_t>(bh) * nq * D;
    const size_t kvbase = static_cast<size_t>(bh / kv_group) * nk * D;   // grouped-query K/V head
    const int q0 = qt * kBM;

    // visible keys [klo[i], khi[i]] of this thread's 4 rows
    int klo[4], khi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        long long lo, hi;
        visible_keys(mk, q0 + ty * 4 + i, q0 + ty * 4 + i, lo, hi);
        klo[i] = clamp_int(lo);
        khi[i] = clamp_int(hi);
    }

    // key tiles that hold a key some row of this tile sees; this CTA takes share `rank` of them
    long long tlo, thi;
    visible_keys(mk, q0, min(q0 + kBM, nq) - 1, tlo, thi);
    const int t_begin = tlo <= thi ? static_cast<int>(tlo / kBN) : 0;
    const int t_count = tlo <= thi ? static_cast<int>(thi / kBN) + 1 - t_begin : 0;
    const int kt0 = t_begin + static_cast<int>(static_cast<long long>(t_count) * rank / split);
    const int kt1 = t_begin + static_cast<int>(static_cast<long long>(t_count) * (rank + 1) / split);

    auto load_kv = [&](int kt, int buf) {
        const int k0 = kt * kBN;
        const size_t g = kvbase + static_cast<size_t>(k0) * D;
        load_rows<D>(fsm + C::K_OFF + buf * kBN * QP, QP, K + g, kBN, nk - k0, tid);
        load_rows<D>(fsm + C::V_OFF + buf * kBN * D, D, V + g, kBN, nk - k0, tid);
    };

    load_rows<D>(Qs, QP, Q + base + static_cast<size_t>(q0) * D, kBM, nq - q0, tid);
    if (kt0 < kt1) load_kv(kt0, 0);
    cp_async_commit();

    float m[4], l[4], acc[4][OC];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int c = 0; c < OC; ++c) acc[i][c] = 0.f;
    }

    for (int kt = kt0; kt < kt1; ++kt) {
        const int buf = (kt - kt0) & 1;
        if (kt + 1 < kt1) {
            load_kv(kt + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const float* Ks = fsm + C::K_OFF + buf * kBN * QP;
        const float* Vs = fsm + C::V_OFF + buf * kBN * D;
        const int k0 = kt * kBN;

        // S = Q K^T for rows ty*4+i, keys tx+16*jj
        float s[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) s[i][jj] = 0.f;
#pragma unroll 4
        for (int c = 0; c < D; c += 4) {
            float4 qv[4], kv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                qv[i] = *reinterpret_cast<const float4*>(Qs + (ty * 4 + i) * QP + c);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                kv[jj] = *reinterpret_cast<const float4*>(Ks + (tx + 16 * jj) * QP + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    s[i][jj] = fmaf(qv[i].x, kv[jj].x, s[i][jj]);
                    s[i][jj] = fmaf(qv[i].y, kv[jj].y, s[i][jj]);
                    s[i][jj] = fmaf(qv[i].z, kv[jj].z, s[i][jj]);
                    s[i][jj] = fmaf(qv[i].w, kv[jj].w, s[i][jj]);
                }
        }

        // online softmax over the 64 keys of each row (16 threads share a row)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float mx = -INFINITY;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int kidx = k0 + tx + 16 * jj;
                s[i][jj] = (kidx < klo[i] || kidx > khi[i]) ? -INFINITY : s[i][jj] * scale;
                mx = fmaxf(mx, s[i][jj]);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off, 16));
            const float m_new = fmaxf(m[i], mx);
            float alpha, rs = 0.f;
            if (m_new == -INFINITY) {
                alpha = 1.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) s[i][jj] = 0.f;
            } else {
                alpha = (m[i] == -INFINITY) ? 0.f : expf(m[i] - m_new);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    s[i][jj] = (s[i][jj] == -INFINITY) ? 0.f : expf(s[i][jj] - m_new);
                    rs += s[i][jj];
                }
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off, 16);
            l[i] = l[i] * alpha + rs;
            m[i] = m_new;
#pragma unroll
            for (int c = 0; c < OC; ++c) acc[i][c] *= alpha;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) Ps[(ty * 4 + i) * kPP + tx + 16 * jj] = s[i][jj];
        }
        __syncthreads();

        // O += P V for rows ty*4+i, columns g*16*CW + tx*CW + e
#pragma unroll 2
        for (int j = 0; j < kBN; j += 4) {
            float4 pv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pv[i] = *reinterpret_cast<const float4*>(Ps + (ty * 4 + i) * kPP + j);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    float vv[CW];
                    const float* vp = Vs + (j + jj) * D + g * 16 * CW + tx * CW;
                    if constexpr (CW == 4) {
                        const float4 t = *reinterpret_cast<const float4*>(vp);
                        vv[0] = t.x; vv[1] = t.y; vv[2] = t.z; vv[3] = t.w;
                    } else {
                        const float2 t = *reinterpret_cast<const float2*>(vp);
                        vv[0] = t.x; vv[1] = t.y;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float p = jj == 0 ? pv[i].x : jj == 1 ? pv[i].y
                                      : jj == 2 ? pv[i].z : pv[i].w;
#pragma unroll
                        for (int e = 0; e < CW; ++e)
                            acc[i][g * CW + e] = fmaf(p, vv[e], acc[i][g * CW + e]);
                    }
                }
            }
        }
        __syncthreads();   // the buffers read here are refilled by the next iteration's copy
    }
    cp_async_wait<0>();    // nothing is in flight when the range was empty
    __syncthreads();

    // This CTA's unnormalised output (rows of the tile x D, in the K buffers) and its (m, l).
    float* Ob = fsm + C::K_OFF;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int e = 0; e < CW; ++e)
                Ob[r * D + g * 16 * CW + tx * CW + e] = acc[i][g * CW + e];
        if (tx == 0) {
            ML[2 * r] = m[i];
            ML[2 * r + 1] = l[i];
        }
    }
    cg::cluster_group cluster = cg::this_cluster();
    if (split > 1) cluster.sync(); else __syncthreads();

    // Merge: this CTA finishes rows [rank*R, rank*R + R) of the tile from all CTAs of the
    // cluster. A row that sees no key has l = 0 everywhere: O = 0, LSE = -inf.
    const int R = kBM / split;
    auto peer = [&](float* p, int s2) -> const float* {
        return split > 1 ? cluster.map_shared_rank(p, s2) : p;
    };
    constexpr int C4 = D / 4;
    for (int idx = tid; idx < R * C4; idx += 256) {
        const int r = rank * R + idx / C4, c4 = idx % C4;
        const int qidx = q0 + r;
        if (qidx >= nq) continue;
        float M = -INFINITY;
        for (int s2 = 0; s2 < split; ++s2) M = fmaxf(M, peer(ML, s2)[2 * r]);
        float L = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s2 = 0; s2 < split; ++s2) {
            const float* mls = peer(ML, s2);
            const float ms = mls[2 * r];
            const float w = ms == -INFINITY ? 0.f : (split > 1 ? expf(ms - M) : 1.f);
            L = fmaf(w, mls[2 * r + 1], L);
            const float4 t = *reinterpret_cast<const float4*>(peer(Ob, s2) + r * D + c4 * 4);
            o.x = fmaf(w, t.x, o.x);
            o.y = fmaf(w, t.y, o.y);
            o.z = fmaf(w, t.z, o.z);
            o.w = fmaf(w, t.w, o.w);
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
        *reinterpret_cast<float4*>(O + base + static_cast<size_t>(qidx) * D + c4 * 4) = o;
        if (c4 == 0)
            lse[static_cast<size_t>(bh) * nq + qidx] = L > 0.f ? M + logf(L) : -INFINITY;
    }
    if (split > 1) cluster.sync();   // peers may still be reading this CTA's shared memory
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return 148;
    return n;
}

// Key shares per query tile: 1 when the query tiles alone fill the GPU, else the smallest power
// of two (at most 8, and at most the largest number of key tiles a query tile sees) that brings
// the grid to about the number of CTAs the SMs hold at once.
int choose_split(const MaskSpec& mk, int n_qtiles, long long bh, int resident_per_sm) {
    const long long target = static_cast<long long>(sm_count()) * resident_per_sm;
    const long long base = bh * n_qtiles;
    if (base * 2 > target) return 1;
    int max_tiles = 0;
    for (int t = 0; t < n_qtiles; ++t) {
        long long lo, hi;
        const long long a = static_cast<long long>(t) * kBM;
        const long long b = a + kBM - 1 < mk.nq - 1 ? a + kBM - 1 : mk.nq - 1;
        visible_keys(mk, a, b, lo, hi);
        if (lo <= hi) {
            const int c = static_cast<int>(hi / kBN - lo / kBN + 1);
            if (c > max_tiles) max_tiles = c;
        }
    }
    int s = 1;
    while (s < kMaxSplit && base * s * 2 <= target && s * 2 <= max_tiles) s *= 2;
    return s;
}

template <int D>
cudaError_t launch_fwd_f32_d(const FwdArgs& a, cudaStream_t stream) {
    using C = F32Cfg<D>;
    cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int nqt = (a.nq + kBM - 1) / kBM;
    const long long bh = static_cast<long long>(a.B) * a.H;
    if (bh > 65535) return cudaErrorInvalidConfiguration;
    const MaskSpec mk{a.nq, a.nk, a.wl, a.wr, static_cast<long long>(a.nk) - a.nq};
    const int split = choose_split(mk, nqt, bh, C::MIN_BLOCKS);
    if (static_cast<long long>(nqt) * split > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nqt * split), static_cast<unsigned>(bh));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = split > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, fwd_f32_kernel<D>, static_cast<const float*>(a.q),
                              static_cast<const float*>(a.k), static_cast<const float*>(a.v),
                              static_cast<float*>(a.o), a.lse, mk, nqt, split, a.scale,
                              a.H / a.Hkv);
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
