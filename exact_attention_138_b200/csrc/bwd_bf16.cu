// Backward pass, bf16 in / bf16 out, fp32 accumulation, on the sm_100a tensor cores.
//
// The backward pass rebuilds the softmax blocks on chip from the saved row statistics instead of
// reading a stored n x n matrix ("Apa itu FlashAttention", "Cara kerja teknik Tiling dan
// Recomputation", item 2; "Flash Attention Nedir?", section "Recomputation (Yeniden
// Hesaplama)"). With LSE from the forward pass, for a key tile j and a query tile i:
//     P^T  = exp(scale·K_j·Q_i^T - LSE_i)          dV_j += P^T·dO_i
//     dP^T = V_j·dO_i^T                            dS^T  = P^T ∘ (dP^T - D_i)
//     dK_j += dS^T·Q_i                             dQ_i += dS·K_j
// with D_i = rowsum(dO_i ∘ O_i); dK and dQ are multiplied by `scale` at the end. These are the
// exact derivative of O = softmax(scale·Q·K^T + M)·V.
//
// Kernels:
//   bwd_preprocess  D = rowsum(dO∘O) per query row; zeroes the fp32 dQ accumulator (and the
//                   ordering semaphores of the deterministic mode).           HBM-bound
//   bwd_main        one CTA per (key tile j, head): K_j and V_j stay in shared memory, Q_i and
//                   dO_i stream through a 2-deep TMA ring. One thread issues the five tcgen05
//                   MMAs per query tile; 4 compute warps (one thread per key row = TMEM lane) form
//                   P^T and dS^T and add the dQ partial tile into the accumulator.
//                   TMEM (512 columns): dV | dK | S^T (P^T as bf16) | dP^T, and the dQ tile reuses
//                   the dP^T columns once dS^T is formed.
//   bwd_dq_convert  dQ = scale·acc -> bf16.                                    HBM-bound
// Causal: key tile j only meets query tiles i >= j.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

constexpr int kBwdThreads = 192;
constexpr float kBwdLog2e = 1.44269504088896340736f;

template <int D>
struct BwdCfg {
    static constexpr int CW = D >= 64 ? 64 : D;
    static constexpr int NCH = D / CW;
    static constexpr int SWB = CW * 2;
    static constexpr uint32_t SWZ = SWB == 128 ? 2u : 4u;
    static constexpr int CHUNK = 128 * SWB;
    static constexpr int TILE = NCH * CHUNK;              // 128 x D bf16
    static constexpr int DS_BYTES = 128 * 128 * 2;         // dS^T tile, 2 x [128 x 64] SW128
    static constexpr int STAT_BYTES = 2 * 2 * 128 * 4;     // LSE·log2e and D, double-buffered
    static constexpr int SMEM = 6 * TILE + DS_BYTES + STAT_BYTES + 256;
};

struct BwdBars {
    uint64_t kv_full;
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full, dp_full, p_full, ds_full, dq_full, dq_drained, ds_free, dkv_done, teardown;
    uint32_t tmem_base;
    int abort;
};

struct BwdKParams {
    const float* lse;
    const float* Dvec;
    float* dq_acc;
    int* sems;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    int n, n_pad, BH, nq, causal, deterministic;
    float scale, scale_log2;
    uint64_t timeout_ns;
};

__device__ __forceinline__ void drain_wait_bwd(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) {
            report_error(4);
            return;
        }
}

__device__ __forceinline__ void compute_bar() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// ------------------------------------------------------------------------------------------
// Preprocess: D_i = sum_c dO_ic·O_ic (fp32), zero the dQ accumulator rows (padded per head to a
// multiple of 128) and the semaphores.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ O,
                                                             const __nv_bfloat16* __restrict__ dO,
                                                             float* __restrict__ Dvec,
                                                             float* __restrict__ dq_acc,
                                                             int* __restrict__ sems, int n,
                                                             int n_pad, long long rows,
                                                             int n_sems) {
    constexpr int LPR = D / 8;            // lanes per row, 8 elements per lane
    constexpr int RPW = 32 / LPR;         // rows per warp
    const int lane = threadIdx.x & 31;
    const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int sub = lane / LPR, part = lane % LPR;
    for (long long w = warp_global; w * RPW < rows; w += nwarps) {
        const long long row = w * RPW + sub;              // in padded (bh, q) space
        float acc = 0.f;
        bool valid = false;
        long long src = 0;
        if (row < rows) {
            const long long bh = row / n_pad;
            const int q = static_cast<int>(row % n_pad);
            valid = q < n;
            src = (bh * n + q) * D + part * 8;
            float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (valid) {
            const uint4 a = *reinterpret_cast<const uint4*>(O + src);
            const uint4 b = *reinterpret_cast<const uint4*>(dO + src);
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float2 fa = __bfloat1622float2(pa[x]);
                const float2 fb = __bfloat1622float2(pb[x]);
                acc = fmaf(fa.x, fb.x, acc);
                acc = fmaf(fa.y, fb.y, acc);
            }
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
            acc += __shfl_xor_sync(0xffffffffu, acc, off, LPR);
        if (row < rows && part == 0) Dvec[row] = valid ? acc : 0.f;
    }
    if (sems) {
        for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < n_sems;
             t += static_cast<long long>(gridDim.x) * blockDim.x)
            sems[t] = 0;
    }
}

// ------------------------------------------------------------------------------------------
// dQ = scale · acc, rounded to bf16.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float* __restrict__ dq_acc,
                                                             __nv_bfloat16* __restrict__ dq, int n,
                                                             int n_pad, long long total8,
                                                             float scale) {
    constexpr int G = D / 8;   // groups of 8 elements per row
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total8;
         t += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long row = t / G;           // (bh, q) in unpadded space
        const int part = static_cast<int>(t % G);
        const long long bh = row / n;
        const int q = static_cast<int>(row % n);
        const float4* src = reinterpret_cast<const float4*>(dq_acc + (bh * n_pad + q) * D + part * 8);
        const float4 a = src[0], b = src[1];
        uint4 o;
        o.x = pack_bf16x2(a.x * scale, a.y * scale);
        o.y = pack_bf16x2(a.z * scale, a.w * scale);
        o.z = pack_bf16x2(b.x * scale, b.y * scale);
        o.w = pack_bf16x2(b.z * scale, b.w * scale);
        *reinterpret_cast<uint4*>(dq + row * D + part * 8) = o;
    }
}

// ------------------------------------------------------------------------------------------
// Main backward kernel.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdKParams p) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::TILE;
    uint8_t* sQ = sV + C::TILE;                   // 2 stages
    uint8_t* sdO = sQ + 2 * C::TILE;              // 2 stages
    uint8_t* sdS = sdO + 2 * C::TILE;             // 32 KB, 1024-aligned
    float* sStat = reinterpret_cast<float*>(sdS + C::DS_BYTES);   // [2][2][128]
    BwdBars* bars = reinterpret_cast<BwdBars*>(sdS + C::DS_BYTES + C::STAT_BYTES);

    constexpr uint32_t COL_DV = 0, COL_DK = 128, COL_S = 256, COL_DP = 384;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int L = blockIdx.x;
    const int j = L / p.BH;                        // key tile: small j (most work) first
    const int bh = L % p.BH;
    const int n = p.n;
    const int i_begin = p.causal ? j : 0;
    const int NT = p.nq - i_begin;

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->ds_full, 128);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_drained, 128);
        mbar_init(&bars->ds_free, 1);
        mbar_init(&bars->dkv_done, 1);
        mbar_init(&bars->teardown, 1);
        bars->abort = ((smem_addr(smem) & 1023u) != 0) ? 1 : 0;
        if (bars->abort) report_error(3);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 5) tmem_alloc(&bars->tmem_base, 512);
    if (warp == 4 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    const uint64_t lim = p.timeout_ns;

    if (warp == 4) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && !*abort) {
            mbar_arrive_expect_tx(&bars->kv_full, 2 * C::TILE);
            for (int ch = 0; ch < C::NCH; ++ch) {
                tma_load_3d(sK + ch * C::CHUNK, &tmK, &bars->kv_full, ch * C::CW, j * 128, bh);
                tma_load_3d(sV + ch * C::CHUNK, &tmV, &bars->kv_full, ch * C::CW, j * 128, bh);
            }
            int issued = 0;
            for (int it = 0; it < NT; ++it) {
                const int st = it & 1, f = it >> 1;
                if (f > 0 && !bounded_wait(&bars->q_empty[st], (f - 1) & 1, abort, lim)) break;
                const int i = i_begin + it;
                mbar_arrive_expect_tx(&bars->q_full[st], 2 * C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch) {
                    tma_load_3d(sQ + st * C::TILE + ch * C::CHUNK, &tmQ, &bars->q_full[st],
                                ch * C::CW, i * 128, bh);
                    tma_load_3d(sdO + st * C::TILE + ch * C::CHUNK, &tmdO, &bars->q_full[st],
                                ch * C::CW, i * 128, bh);
                }
                issued = it + 1;
            }
            if (*abort) {
                drain_wait_bwd(&bars->kv_full, 0, 100000000ull);
                for (int it = 0; it < issued; ++it)
                    drain_wait_bwd(&bars->q_full[it & 1], (it >> 1) & 1, 100000000ull);
            }
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);     // K-major x K-major
            constexpr uint32_t idKN = idesc_bf16_f32(128, D, 0, 1);      // A K-major, B MN-major
            constexpr uint32_t idQ = idesc_bf16_f32(128, D, 1, 1);       // A MN-major, B MN-major
            const uint32_t aK = smem_addr(sK), aV = smem_addr(sV), aQ = smem_addr(sQ),
                           adO = smem_addr(sdO), adS = smem_addr(sdS);
            bool ok = bounded_wait(&bars->kv_full, 0, abort, lim);
            tc_fence_after();
            for (int it = 0; ok && it < NT; ++it) {
                const int st = it & 1;
                if (!(ok = bounded_wait(&bars->q_full[st], (it >> 1) & 1, abort, lim))) break;
                tc_fence_after();
                const uint32_t q_a = aQ + st * C::TILE, do_a = adO + st * C::TILE;
                // S^T = K_j · Q_i^T   (M = keys, N = queries, K = d)
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = ((ks * 16) / C::CW) * C::CHUNK + ((ks * 16) % C::CW) * 2;
                    mma_ss(tmem + COL_S, smem_desc(aK + off, 16, 8 * C::SWB, C::SWZ),
                           smem_desc(q_a + off, 16, 8 * C::SWB, C::SWZ), idS, ks > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full);
                if (it > 0) {
                    if (!(ok = bounded_wait(&bars->dq_drained, (it - 1) & 1, abort, lim))) break;
                    tc_fence_after();
                }
                // dP^T = V_j · dO_i^T
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = ((ks * 16) / C::CW) * C::CHUNK + ((ks * 16) % C::CW) * 2;
                    mma_ss(tmem + COL_DP, smem_desc(aV + off, 16, 8 * C::SWB, C::SWZ),
                           smem_desc(do_a + off, 16, 8 * C::SWB, C::SWZ), idS, ks > 0 ? 1u : 0u);
                }
                mma_commit(&bars->dp_full);
                if (!(ok = bounded_wait(&bars->p_full, it & 1, abort, lim))) break;
                tc_fence_after();
                // dV_j += P^T · dO_i   (A = P^T from TMEM, B = dO_i MN-major; K = queries)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(tmem + COL_DV, tmem + COL_S + ks * 8,
                           smem_desc(do_a + ks * 16 * C::SWB, C::CHUNK, 8 * C::SWB, C::SWZ), idKN,
                           (it > 0 || ks > 0) ? 1u : 0u);
                if (!(ok = bounded_wait(&bars->ds_full, it & 1, abort, lim))) break;
                tc_fence_after();
                // dK_j += dS^T · Q_i   (A = dS^T K-major SW128, B = Q_i MN-major)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(tmem + COL_DK,
                           smem_desc(adS + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2u),
                           smem_desc(q_a + ks * 16 * C::SWB, C::CHUNK, 8 * C::SWB, C::SWZ), idKN,
                           (it > 0 || ks > 0) ? 1u : 0u);
                // dQ_i = dS · K_j   (A = dS MN-major view of the same buffer, B = K_j MN-major)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss(tmem + COL_DP, smem_desc(adS + ks * 2048, 16384, 1024, 2u),
                           smem_desc(aK + ks * 16 * C::SWB, C::CHUNK, 8 * C::SWB, C::SWZ), idQ,
                           ks > 0 ? 1u : 0u);
                mma_commit(&bars->dq_full);
                mma_commit(&bars->ds_free);
                mma_commit(&bars->q_empty[st]);
            }
            if (ok) mma_commit(&bars->dkv_done);
            mma_commit(&bars->teardown);
            drain_wait_bwd(&bars->teardown, 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- compute warps 0-3
        const int r = warp * 32 + lane;                    // key row within tile = TMEM lane
        const int kidx = j * 128 + r;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tS = tmem + lane_base + COL_S;
        const uint32_t tDP = tmem + lane_base + COL_DP;
        const float sl2 = p.scale_log2;
        bool ok = true;
        for (int it = 0; it < NT; ++it) {
            const int i = i_begin + it;
            const int buf = it & 1;
            float* sL = sStat + buf * 256;
            float* sD = sL + 128;
            {
                const int q = i * 128 + r;
                sL[r] = (q < n) ? p.lse[static_cast<size_t>(bh) * n + q] * kBwdLog2e : INFINITY;
                sD[r] = (q < n) ? p.Dvec[static_cast<size_t>(bh) * p.n_pad + q] : 0.f;
            }
            compute_bar();
            ok = __all_sync(0xffffffffu, bounded_wait(&bars->s_full, it & 1, abort, lim));
            if (!ok) break;
            tc_fence_after();
            float pr[128];
            {
                uint32_t u[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(tS + c * 32, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) pr[c * 32 + x] = __uint_as_float(u[x]);
                }
            }
            const bool edge = (p.causal && i == j) || (kidx >= n);
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                float v = ex2_approx(fmaf(pr[c], sl2, -sL[c]));
                if (edge && (kidx >= n || (p.causal && i * 128 + c < kidx))) v = 0.f;
                pr[c] = v;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t u[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) u[x] = pack_bf16x2(pr[h * 64 + 2 * x], pr[h * 64 + 2 * x + 1]);
                tmem_st32(tS + h * 32, u);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars->p_full);

            ok = __all_sync(0xffffffffu, bounded_wait(&bars->dp_full, it & 1, abort, lim));
            if (ok && it > 0) ok = __all_sync(0xffffffffu, bounded_wait(&bars->ds_free, (it - 1) & 1, abort, lim));
            if (!ok) break;
            tc_fence_after();
            uint8_t* ds_row = sdS + r * 128;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t u[32];
                tmem_ld32(tDP + cc * 32, u);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int c0 = cc * 32 + 2 * x;
                    const float d0 = pr[c0] * (__uint_as_float(u[2 * x]) - sD[c0]);
                    const float d1 = pr[c0 + 1] * (__uint_as_float(u[2 * x + 1]) - sD[c0 + 1]);
                    w[x] = pack_bf16x2(d0, d1);
                }
                // queries cc*32 .. cc*32+31: chunk cc/2, 16-byte units (cc&1)*4 .. +3, swizzled
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int unit = (cc & 1) * 4 + t;
                    uint4* dst = reinterpret_cast<uint4*>(ds_row + (cc >> 1) * 16384 +
                                                          ((unit ^ (r & 7)) << 4));
                    *dst = make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_full);

            ok = __all_sync(0xffffffffu, bounded_wait(&bars->dq_full, it & 1, abort, lim));
            if (!ok) break;
            tc_fence_after();
            int* sem = p.deterministic ? p.sems + static_cast<size_t>(bh) * p.nq + i : nullptr;
            if (sem) {
                // add this CTA's partial only after every lower key tile has added its own
                bool got = true;
                if (r == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (atomicAdd(sem, 0) != j) {
                        if (*abort || globaltimer_ns() - t0 > lim) {
                            *abort = 1;
                            report_error(4);
                            got = false;
                            break;
                        }
                        __nanosleep(64);
                    }
                    __threadfence();
                }
                compute_bar();
                if (*abort) got = false;
                ok = __all_sync(0xffffffffu, got);
                if (!ok) {
                    // release dQ's TMEM columns so the MMA warp does not wait for them
                    tc_fence_before();
                    mbar_arrive(&bars->dq_drained);
                    break;
                }
            }
            float* acc_row = p.dq_acc + (static_cast<size_t>(bh) * p.n_pad + i * 128 + r) * D;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t u[32];
                tmem_ld32(tDP + cc * 32, u);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 8; ++x)
                    atomicAdd(reinterpret_cast<float4*>(acc_row + cc * 32 + 4 * x),
                              make_float4(__uint_as_float(u[4 * x]), __uint_as_float(u[4 * x + 1]),
                                          __uint_as_float(u[4 * x + 2]), __uint_as_float(u[4 * x + 3])));
            }
            tc_fence_before();
            mbar_arrive(&bars->dq_drained);
            if (sem) {
                __threadfence();
                compute_bar();
                if (r == 0) atomicAdd(sem, 1);
            }
        }
        if (ok) ok = __all_sync(0xffffffffu, bounded_wait(&bars->dkv_done, 0, abort, lim));
        if (ok) {
            tc_fence_after();
            const size_t orow = (static_cast<size_t>(bh) * n + kidx) * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t tacc = tmem + lane_base + (which == 0 ? COL_DV : COL_DK);
                const float mul = which == 0 ? 1.f : p.scale;
                __nv_bfloat16* dst = which == 0 ? p.dv : p.dk;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t u[32];
                    tmem_ld32(tacc + cc * 32, u);
                    tmem_ld_wait();
                    uint32_t w[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        w[x] = pack_bf16x2(__uint_as_float(u[2 * x]) * mul,
                                           __uint_as_float(u[2 * x + 1]) * mul);
                    if (kidx < n) {
                        uint4* o = reinterpret_cast<uint4*>(dst + orow + cc * 32);
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            o[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t stream) {
    using C = BwdCfg<D>;
    const int BH = a.B * a.H;
    const int nq = (a.n + 127) / 128;
    const int n_pad = nq * 128;
    cudaError_t e;
    const cudaEvent_t* ev = a.phase_events;
    if (ev && (e = cudaEventRecord(ev[0], stream)) != cudaSuccess) return e;
    // 1. preprocess
    {
        const long long rows = static_cast<long long>(BH) * n_pad;
        const int rpw = 32 / (D / 8);
        long long blocks = (rows + (8 * rpw) - 1) / (8 * rpw);
        if (blocks > 148 * 16) blocks = 148 * 16;
        const int n_sems = a.deterministic ? BH * nq : 0;
        bwd_preprocess_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dO),
            a.Dvec, a.dq_acc, a.deterministic ? a.sems : nullptr, a.n, n_pad, rows, n_sems);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 2. main
    {
        CUtensorMap mq, mk, mv, mdo;
        if ((e = make_tmap_bf16(&mq, a.q, BH, a.n, D)) != cudaSuccess) return e;
        if ((e = make_tmap_bf16(&mk, a.k, BH, a.n, D)) != cudaSuccess) return e;
        if ((e = make_tmap_bf16(&mv, a.v, BH, a.n, D)) != cudaSuccess) return e;
        if ((e = make_tmap_bf16(&mdo, a.dO, BH, a.n, D)) != cudaSuccess) return e;
        e = cudaFuncSetAttribute(bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM);
        if (e != cudaSuccess) return e;
        BwdKParams kp;
        kp.lse = a.lse;
        kp.Dvec = a.Dvec;
        kp.dq_acc = a.dq_acc;
        kp.sems = a.sems;
        kp.dk = static_cast<__nv_bfloat16*>(a.dk);
        kp.dv = static_cast<__nv_bfloat16*>(a.dv);
        kp.n = a.n;
        kp.n_pad = n_pad;
        kp.BH = BH;
        kp.nq = nq;
        kp.causal = a.causal;
        kp.deterministic = a.deterministic;
        kp.scale = a.scale;
        kp.scale_log2 = a.scale * kBwdLog2e;
        kp.timeout_ns = a.timeout_ns;
        const long long grid = static_cast<long long>(nq) * BH;
        if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        if (ev && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess) return e;
        bwd_main_kernel<D><<<static_cast<unsigned>(grid), kBwdThreads, C::SMEM, stream>>>(
            mq, mk, mv, mdo, kp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (ev && (e = cudaEventRecord(ev[2], stream)) != cudaSuccess) return e;
    }
    // 3. dQ convert
    {
        const long long total8 = static_cast<long long>(BH) * a.n * (D / 8);
        long long blocks = (total8 + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        bwd_dq_convert_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            a.dq_acc, static_cast<__nv_bfloat16*>(a.dq), a.n, n_pad, total8, a.scale);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (ev && (e = cudaEventRecord(ev[3], stream)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream) {
    switch (a.d) {
        case 32: return launch_bwd_d<32>(a, stream);
        case 64: return launch_bwd_d<64>(a, stream);
        case 128: return launch_bwd_d<128>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
