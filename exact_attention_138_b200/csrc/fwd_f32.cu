// Forward pass in plain fp32 on the FMA pipes, for the float32 examples of "Efficient Attention"
// (efficient_attention.py: (2,3,128,32) and the (4096,64) row-tiling case), whose results are
// compared at an absolute tolerance of 1e-5. TF32 tensor-core products cannot meet that, so every
// product here is an fp32 fused multiply-add (packed two to an instruction); each exponential is
// one FMA (score · scale·log2 e minus the running maximum, rounded once) and the MUFU's 2^x,
// whose relative error of a few 1e-7 stays far inside that tolerance.
//
// Same method as the bf16 kernel (tiles of Q/K/V in on-chip memory, online softmax with running
// max m and sum l, output rescaled by the exponential of the change of m; "Attention Mechanism:
// Revolusi Representasi Sequence", §13), laid out for SIMT. One CTA works on a tile of BM query
// rows (BM = 64, or a smaller multiple of 4 down to 32 when that balances a small grid over the
// SMs) of one (b,h) with 2·BM threads as a (BM/4) x 8 grid (ty, tx). Thread (ty, tx) owns rows
// ty + i·BM/4 (i < 4) and keys tx + 8·jj (jj < 8) of the BM x 64 score tile, and the same rows x
// columns tx·4 + 32·g + e (e < 4) of the output accumulator. A warp thus covers 16 rows x 64 keys
// (or 16 rows x all d columns): per 4-wide step of the reduction it reads 4 Q rows and 8 K rows
// (or 4 P rows and 4·d/32 V words) as conflict-free 16-byte words (rows are padded so that
// consecutive rows start 4 or 8 banks apart), against 128 (or 64·d/32) products, which packed
// fp32x2 FMAs do two at a time (a 16-byte word is two fp32 pairs), so that instruction issue
// leaves room for the FMA pipes. The next K/V tile is copied in with cp.async while the current
// one is used. Scores are kept in the base-2 domain (scale·log2 e folded into one FMA before
// ex2), and key tiles that every row of the CTA sees skip the mask.
//
// Small grids (the pages' examples have 12 and 64 query tiles for 148 SMs) split each query
// tile's key range over a thread-block cluster of up to 8 CTAs. Each CTA keeps its own (m, l, O)
// for its share of the keys; the cluster then merges them through distributed shared memory with
// the same rule that joins two softmax blocks (weights 2^(m_s - M), M the largest m_s), each CTA
// finishing a slice of the rows. No global scratch and no second launch are needed.
#include <cooperative_groups.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

namespace cg = cooperative_groups;

constexpr int kBMMax = 64;       // query rows per CTA at most
constexpr int kBN = 64;          // keys per tile
constexpr int kPP = kBN + 8;     // row stride of the P tile (floats): 4 rows x 8 keys, 32 banks
constexpr int kMaxSplit = 8;     // portable cluster size
constexpr float kF32Log2e = 1.4426950408889634f;   // log2(e)
constexpr float kF32Ln2 = 0.6931471805599453f;     // ln(2)

template <int D>
struct F32Cfg {
    static constexpr int QP = D + 4;                   // row stride of Q and K tiles (floats)
    static constexpr int NG = D / 32;                  // 4-column groups per thread in O
    static constexpr int OC2 = NG * 2;                 // output column pairs per thread
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + kBMMax * QP;  // two K buffers of kBN x QP
    static constexpr int V_OFF = K_OFF + 2 * kBN * QP; // two V buffers of kBN x D
    static constexpr int P_OFF = V_OFF + 2 * kBN * D;  // kBMMax x kPP
    static constexpr int ML_OFF = P_OFF + kBMMax * kPP;// kBMMax x (m, l)
    static constexpr int FLOATS = ML_OFF + 2 * kBMMax;
    static constexpr int SMEM = FLOATS * 4;
    // CTAs per SM that the shared memory allows (228 KB per SM); registers are bounded to match
    static constexpr int MIN_BLOCKS = D == 32 ? 3 : (D == 64 ? 2 : 1);
    static_assert(kBMMax * D <= 2 * kBN * QP, "merge buffer must fit in the K buffers");
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

// rows [0, rows) x D floats from global `src` (row stride D) into shared `dst` (row stride ld) by
// `nthr` threads; rows at or past `valid_rows` are zero-filled and read nothing.
template <int D>
__device__ __forceinline__ void load_rows(float* dst, int ld, const float* src, int rows,
                                          int valid_rows, int tid, int nthr) {
    constexpr int C4 = D / 4;
    for (int idx = tid; idx < rows * C4; idx += nthr) {
        const int r = idx / C4, c4 = idx % C4;
        const bool ok = r < valid_rows;
        cp_async16(dst + r * ld + c4 * 4, ok ? src + static_cast<size_t>(r) * D + c4 * 4 : src,
                   ok);
    }
}

// Online-softmax step of one thread for one key tile: s (raw scores of rows ty + i·BM/4, keys
// tx + 8·jj) becomes P = 2^(s·sl2 - m) with m the rows' new running maxima (base 2); l and the
// output accumulator (column pairs) are rescaled. MASK: keys outside a row's [klo, khi] are
// dropped.
template <bool MASK, int OC2>
__device__ __forceinline__ void softmax_tile(float (&s)[4][8], float (&m)[4], float (&l)[4],
                                             uint64_t (&acc)[4][OC2], const int (&klo)[4],
                                             const int (&khi)[4], int kbase, float sl2,
                                             unsigned wmask) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float mx = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            if constexpr (MASK) {
                const int kidx = kbase + 8 * jj;
                if (kidx < klo[i] || kidx > khi[i]) s[i][jj] = -INFINITY;
            }
            mx = fmaxf(mx, s[i][jj]);
        }
#pragma unroll
        for (int off = 4; off > 0; off >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(wmask, mx, off, 8));
        // scale > 0, so the largest raw score gives the largest scaled one
        const float m_new = fmaxf(m[i], mx * sl2);
        float alpha = 1.f, rs = 0.f;
        if (!MASK || m_new != -INFINITY) {
            alpha = ex2_approx(m[i] - m_new);          // 0 while m was -inf
            const float nm = -m_new;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                s[i][jj] = ex2_approx(fmaf(s[i][jj], sl2, nm));   // dropped keys: 2^-inf = 0
                rs += s[i][jj];
            }
        } else {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) s[i][jj] = 0.f;
        }
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) rs += __shfl_xor_sync(wmask, rs, off, 8);
        l[i] = fmaf(l[i], alpha, rs);
        m[i] = m_new;
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int c = 0; c < OC2; ++c) acc[i][c] = f2_fma(acc[i][c], a2, 0ull);
    }
}

template <int D>
__global__ void __launch_bounds__(128, F32Cfg<D>::MIN_BLOCKS)
    fwd_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                   const float* __restrict__ V, float* __restrict__ O, float* __restrict__ lse,
                   MaskSpec mk, int n_qtiles, int split, float scale, int kv_group) {
    using C = F32Cfg<D>;
    constexpr int QP = C::QP, NG = C::NG, OC2 = C::OC2;
    extern __shared__ __align__(16) float fsm[];
    float* Qs = fsm + C::Q_OFF;
    float* Ps = fsm + C::P_OFF;
    float* ML = fsm + C::ML_OFF;

    const int nthr = static_cast<int>(blockDim.x);       // 2·BM
    const int R4 = nthr >> 3;                             // BM / 4: rows between a thread's rows
    const int BM = R4 * 4;
    const int rank = static_cast<int>(blockIdx.x) % split;             // key share in the cluster
    const int qt = n_qtiles - 1 - static_cast<int>(blockIdx.x) / split; // longest causal rows first
    const int bh = blockIdx.y;
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    // lanes of this warp that exist (the last warp of a CTA of 2·BM threads may be partial)
    const int wfirst = tid & ~31;
    const unsigned wmask = nthr - wfirst >= 32 ? 0xffffffffu : (1u << (nthr - wfirst)) - 1u;
    const int nq = mk.nq, nk = mk.nk;
    const size_t base = static_cast<size_t>(bh) * nq * D;
    const size_t kvbase = static_cast<size_t>(bh / kv_group) * nk * D;   // grouped-query K/V head
    const int q0 = qt * BM;
    const int qlast = min(q0 + BM, nq) - 1;
    const float sl2 = scale * kF32Log2e;

    // visible keys [klo[i], khi[i]] of this thread's 4 rows
    int klo[4], khi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        long long lo, hi;
        const int row = q0 + ty + R4 * i;
        visible_keys(mk, row, row, lo, hi);
        klo[i] = clamp_int(lo);
        khi[i] = clamp_int(hi);
    }
    // keys that every row of the tile sees: [all_lo, all_hi]
    long long all_lo, all_hi;
    visible_keys(mk, qlast, q0, all_lo, all_hi);

    // key tiles that hold a key some row of this tile sees; this CTA takes share `rank` of them
    long long tlo, thi;
    visible_keys(mk, q0, qlast, tlo, thi);
    const int t_begin = tlo <= thi ? static_cast<int>(tlo / kBN) : 0;
    const int t_count = tlo <= thi ? static_cast<int>(thi / kBN) + 1 - t_begin : 0;
    const int kt0 = t_begin + static_cast<int>(static_cast<long long>(t_count) * rank / split);
    const int kt1 = t_begin + static_cast<int>(static_cast<long long>(t_count) * (rank + 1) / split);

    auto load_kv = [&](int kt, int buf) {
        const int k0 = kt * kBN;
        const size_t g = kvbase + static_cast<size_t>(k0) * D;
        load_rows<D>(fsm + C::K_OFF + buf * kBN * QP, QP, K + g, kBN, nk - k0, tid, nthr);
        load_rows<D>(fsm + C::V_OFF + buf * kBN * D, D, V + g, kBN, nk - k0, tid, nthr);
    };

    load_rows<D>(Qs, QP, Q + base + static_cast<size_t>(q0) * D, BM, nq - q0, tid, nthr);
    if (kt0 < kt1) load_kv(kt0, 0);
    cp_async_commit();

    // output accumulator as column pairs (acc[i][2g + h]: columns tx·4 + 32·g + 2h, +1), each
    // updated by one packed fp32x2 FMA
    float m[4], l[4];
    uint64_t acc[4][OC2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int c = 0; c < OC2; ++c) acc[i][c] = 0ull;   // (+0, +0)
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

        // S = Q K^T for rows ty + R4·i, keys tx + 8·jj: each 16-byte read of Q and of K is two
        // fp32 pairs, so one packed FMA does two products and each score carries two partial
        // sums (even and odd head-dim columns) that are added at the end
        float s[4][8];
        {
            uint64_t s2[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) s2[i][jj] = 0ull;
#pragma unroll 2
            for (int c = 0; c < D; c += 4) {
                ulonglong2 qv[4], kv[8];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    qv[i] = *reinterpret_cast<const ulonglong2*>(Qs + (ty + R4 * i) * QP + c);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    kv[jj] = *reinterpret_cast<const ulonglong2*>(Ks + (tx + 8 * jj) * QP + c);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        s2[i][jj] = f2_fma(qv[i].x, kv[jj].x, s2[i][jj]);
                        s2[i][jj] = f2_fma(qv[i].y, kv[jj].y, s2[i][jj]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    float a, b;
                    f2_unpack(s2[i][jj], a, b);
                    s[i][jj] = a + b;
                }
        }

        // online softmax (8 threads share a row); the mask only where some row misses a key
        if (all_lo <= k0 && k0 + kBN - 1 <= all_hi)
            softmax_tile<false, OC2>(s, m, l, acc, klo, khi, k0 + tx, sl2, wmask);
        else
            softmax_tile<true, OC2>(s, m, l, acc, klo, khi, k0 + tx, sl2, wmask);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) Ps[(ty + R4 * i) * kPP + tx + 8 * jj] = s[i][jj];
        __syncthreads();

        // O += P V for rows ty + R4·i, columns tx·4 + 32·g + e
#pragma unroll 2
        for (int j = 0; j < kBN; j += 4) {
            float4 pv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pv[i] = *reinterpret_cast<const float4*>(Ps + (ty + R4 * i) * kPP + j);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                ulonglong2 t[NG];    // V row j + jj, this thread's columns as fp32 pairs
#pragma unroll
                for (int g = 0; g < NG; ++g)
                    t[g] = *reinterpret_cast<const ulonglong2*>(Vs + (j + jj) * D + g * 32 +
                                                                tx * 4);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float p = jj == 0 ? pv[i].x : jj == 1 ? pv[i].y
                                  : jj == 2 ? pv[i].z : pv[i].w;
                    const uint64_t pp = f2_pack(p, p);
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        acc[i][2 * g] = f2_fma(pp, t[g].x, acc[i][2 * g]);
                        acc[i][2 * g + 1] = f2_fma(pp, t[g].y, acc[i][2 * g + 1]);
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
        const int r = ty + R4 * i;
#pragma unroll
        for (int g = 0; g < NG; ++g)
            *reinterpret_cast<ulonglong2*>(Ob + r * D + g * 32 + tx * 4) =
                make_ulonglong2(acc[i][2 * g], acc[i][2 * g + 1]);
        if (tx == 0) {
            ML[2 * r] = m[i];
            ML[2 * r + 1] = l[i];
        }
    }
    cg::cluster_group cluster = cg::this_cluster();
    if (split > 1) cluster.sync(); else __syncthreads();

    // Merge: this CTA finishes rows [rank*R, rank*R + R) of the tile from all CTAs of the
    // cluster. A row that sees no key has l = 0 everywhere: O = 0, LSE = -inf.
    const int R = BM / split;
    auto peer = [&](float* p, int s2) -> const float* {
        return split > 1 ? cluster.map_shared_rank(p, s2) : p;
    };
    constexpr int C4 = D / 4;
    for (int idx = tid; idx < R * C4; idx += nthr) {
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
            const float w = ms == -INFINITY ? 0.f : (split > 1 ? ex2_approx(ms - M) : 1.f);
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
        // LSE = ln(2^M · L) = M·ln 2 + ln L (M, the base-2 maximum, is what the weights used)
        if (c4 == 0)
            lse[static_cast<size_t>(bh) * nq + qidx] =
                L > 0.f ? fmaf(M, kF32Ln2, logf(L)) : -INFINITY;
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

// CTAs of the fp32 kernel that one SM holds: its shared memory (sized for 64-row tiles whatever
// BM is) against the SM's, at most the count the register bound was compiled for.
template <int D>
int f32_ctas_per_sm() {
    int dev = 0, smem = 0, reserved = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
            cudaSuccess) {
        (void)cudaGetLastError();
        return 1;
    }
    const int n = smem / (F32Cfg<D>::SMEM + reserved);
    return n < 1 ? 1 : (n > F32Cfg<D>::MIN_BLOCKS ? F32Cfg<D>::MIN_BLOCKS : n);
}

// Clusters of `split` CTAs of `2·bm` threads that the GPU holds at once (a cluster must fit in
// one GPC, so this can be below SMs x CTAs per SM / split); queried once per (device, d, bm,
// split) into a per-device table of atomics. While `stream` is being captured into a graph the
// query is not made and 95% of the per-SM bound is assumed.
constexpr int kF32CacheDevices = 64;

template <int D>
long long f32_max_active_clusters(int bm, int split, int sms, int per_sm, cudaStream_t stream) {
    const long long fallback = static_cast<long long>(sms) * per_sm * 95 / 100 / split;
    static std::atomic<int> cache[kF32CacheDevices][9][4];
    const int bslot = (kBMMax - bm) / 4;
    const int sslot = split == 1 ? 0 : split == 2 ? 1 : split == 4 ? 2 : 3;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return fallback;
    }
    std::atomic<int>* entry = (dev >= 0 && dev < kF32CacheDevices && bslot >= 0 && bslot < 9)
                                  ? &cache[dev][bslot][sslot] : nullptr;
    if (entry) {
        const int known = entry->load(std::memory_order_relaxed);
        if (known > 0) return known;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        (void)cudaGetLastError();
        return fallback;
    }
    if (cap != cudaStreamCaptureStatusNone) return fallback;
    if (cudaFuncSetAttribute(fwd_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             F32Cfg<D>::SMEM) != cudaSuccess) {
        (void)cudaGetLastError();
        return fallback;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(split * 64));
    cfg.blockDim = dim3(static_cast<unsigned>(2 * bm));
    cfg.dynamicSmemBytes = F32Cfg<D>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fwd_f32_kernel<D>, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        return fallback;
    }
    if (entry) entry->store(n, std::memory_order_relaxed);
    return n;
}

struct F32Plan {
    int bm, split;
};

// Tile height BM and key shares per query tile. Large grids take 64-row tiles and no split. A
// small grid is costed for each BM in {64, 60, ..., 32} and split in {1, 2, 4, 8} (BM a
// multiple of the split, at most one share per key tile): per wave of resident CTAs (the SMs'
// CTA slots, or for a split the clusters the GPU holds at once), the busiest SM's CTAs x rows x
// (key tiles per share + 1 for loading Q and the merge), divided by how well that many warps
// keep the SM's pipes busy (8 or more warps: fully; 4 to 7: 0.7; fewer: 0.5). Ties keep the
// larger tile and the smaller split.
template <int D>
F32Plan plan_f32(const MaskSpec& mk, long long bh, int per_sm, cudaStream_t stream) {
    const int sms = sm_count();
    const long long tiles64 = bh * ((mk.nq + kBMMax - 1) / kBMMax);
    if (tiles64 >= 4LL * sms * per_sm) return F32Plan{kBMMax, 1};
    F32Plan best{kBMMax, 1};
    double best_cost = 0;
    bool have = false;
    for (int bm = kBMMax; bm >= 32; bm -= 4) {
        const int nqt = (mk.nq + bm - 1) / bm;
        int max_tiles = 0;
        for (int t = 0; t < nqt; ++t) {
            long long lo, hi;
            const long long a = static_cast<long long>(t) * bm;
            const long long b = a + bm - 1 < mk.nq - 1 ? a + bm - 1 : mk.nq - 1;
            visible_keys(mk, a, b, lo, hi);
            if (lo <= hi) {
                const int c = static_cast<int>(hi / kBN - lo / kBN + 1);
                if (c > max_tiles) max_tiles = c;
            }
        }
        for (int split = 1; split <= kMaxSplit; split *= 2) {
            if (bm % split != 0 || (split > 1 && split > max_tiles)) continue;
            const long long ctas = bh * nqt * split;
            long long slots = static_cast<long long>(sms) * per_sm;
            if (split > 1) {
                const long long cl = f32_max_active_clusters<D>(bm, split, sms, per_sm, stream);
                if (cl * split < slots) slots = cl * split;
            }
            if (slots < 1) continue;
            const long long waves = (ctas + slots - 1) / slots;
            const long long in_wave = ctas < slots ? ctas : slots;
            const long long on_sm = (in_wave + sms - 1) / sms;              // busiest SM
            const long long warps = on_sm * ((2 * bm + 31) / 32);
            const double eff = warps >= 8 ? 1.0 : (warps >= 4 ? 0.7 : 0.5);
            const double cost = static_cast<double>(waves) * on_sm * bm *
                                ((max_tiles + split - 1) / split + 1) / eff;
            if (!have || cost < best_cost) {
                best = F32Plan{bm, split};
                best_cost = cost;
                have = true;
            }
        }
    }
    return best;
}

template <int D>
cudaError_t launch_fwd_f32_d(const FwdArgs& a, cudaStream_t stream) {
    using C = F32Cfg<D>;
    cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const long long bh = static_cast<long long>(a.B) * a.H;
    if (bh > 65535) return cudaErrorInvalidConfiguration;
    const MaskSpec mk{a.nq, a.nk, a.wl, a.wr, static_cast<long long>(a.nk) - a.nq};
    const F32Plan plan = plan_f32<D>(mk, bh, f32_ctas_per_sm<D>(), stream);
    const int nqt = (a.nq + plan.bm - 1) / plan.bm;
    const int split = plan.split;
    if (static_cast<long long>(nqt) * split > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nqt * split), static_cast<unsigned>(bh));
    cfg.blockDim = dim3(static_cast<unsigned>(2 * plan.bm));
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
