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
//   bwd_main        (d = 32, 64) one CTA per (key tile j, K/V head): K_j and V_j stay in shared
//                   memory, Q_i and dO_i stream through a 2-deep TMA ring. One warp issues the five
//                   tcgen05 MMAs per query tile; 8 compute warps (one thread per key row = TMEM
//                   lane, half the query columns each) form P^T and dS^T and add the dQ partial
//                   tile into the accumulator. TMEM (512 columns): dV | dK | dQ x2 | S^T (P^T as
//                   bf16) | dP^T, dQ double-buffered so the next tile's MMAs never wait for it.
//   bwd_main_q64    (d = 128) see below.
//   bwd_dq_convert  dQ = scale·acc -> bf16.                                    HBM-bound
// Masks (causal, sliding window, query/key lengths that differ; see MaskSpec): key tile j only
// meets the query tiles that hold a query which sees one of its keys; a key tile that no query
// sees gets dK = dV = 0.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

constexpr int kBwdThreads = 320;
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
    static constexpr int STAT_BYTES = 2 * 2 * 128 * 4;     // [warpgroup][buffer][LSE2 | D] x 64
    static constexpr int SMEM = 6 * TILE + DS_BYTES + STAT_BYTES + 256;
};

struct BwdBars {
    uint64_t kv_full;
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full, dp_full, p_full, ds_full, ds_free, dkv_done, teardown;
    uint64_t dq_full[2], dq_drained[2];   // dQ double-buffered in its own TMEM columns
    uint32_t tmem_base;
    int abort;
};

struct BwdKParams {
    const float* lse;
    const float* Dvec;
    const float* L2vec;
    float* dq_acc;
    int* sems;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    int n_pad;        // query rows per head in the workspace arrays (multiple of 128)
    int BH;           // K/V heads (one CTA row per K/V head)
    int nkt;          // key tiles of 128 per head
    int deterministic, group;
    int kv_group;     // query heads per K/V head
    MaskSpec mask;
    float scale, scale_log2;
    uint64_t timeout_ns;
};

// Accumulating launches (the backward in parts) add dK and dV in fp32 into these arrays
// (B, Hkv, nk, d) instead of storing them; a kernel parameter of its own, used only by the
// accumulating instantiation of each main kernel.
struct AccOut {
    float* dk;
    float* dv;
    long long rows;   // rows between consecutive K/V heads of dk, dv
};

// dst[0 .. N) += mul · (TMEM words u as fp32); dst 16-byte aligned. Vector reductions performed
// in L2: nothing waits for them, and each element of dst gets one addition per launch (one CTA
// owns each key row), so the sum does not depend on timing.
template <int N>
__device__ __forceinline__ void add_row_f32(float* dst, const uint32_t* u, float mul) {
#pragma unroll
    for (int c = 0; c < N / 4; ++c)
        red_add_v4_f32(dst + 4 * c, __uint_as_float(u[4 * c]) * mul,
                       __uint_as_float(u[4 * c + 1]) * mul, __uint_as_float(u[4 * c + 2]) * mul,
                       __uint_as_float(u[4 * c + 3]) * mul);
}

__device__ __forceinline__ void drain_wait_bwd(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) {
            report_error(4);
            return;
        }
}

// ------------------------------------------------------------------------------------------
// Preprocess: D_i = sum_c dO_ic·O_ic (fp32) and LSE_i·log2(e), both padded per head to a multiple
// of 128 rows (0 and +inf on the padding), zero the dQ accumulator rows and the semaphores.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ O,
                                                             const __nv_bfloat16* __restrict__ dO,
                                                             const float* __restrict__ lse,
                                                             float* __restrict__ L2vec,
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
        if (row < rows && part == 0) {
            Dvec[row] = valid ? acc : 0.f;
            // LSE in log2 units; +inf on padding rows and on rows that see no key (LSE = -inf)
            // makes their P exactly 0 downstream
            const float l = valid ? lse[src / D] : INFINITY;
            L2vec[row] = l == -INFINITY ? INFINITY : l * 1.44269504088896340736f;
        }
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
//
// Roles (320 threads): warps 0-3 = compute warpgroup 0 (query columns 0-63 of each tile),
// warps 4-7 = compute warpgroup 1 (query columns 64-127), warp 8 = TMA producer, warp 9 = MMA
// issuer. Every compute thread owns one key row (= TMEM lane) and half of the tile's columns.
// Per query tile i the MMA warp issues, in this order,
//     dV += P^T(i)·dO(i) [after P^T(i) is in TMEM],   S^T(i+1) = K·Q(i+1)^T,
//     dK += dS^T(i)·Q(i), dQ(i) = dS·K into buffer i mod 2 [after dS^T(i) is in shared memory
//     and dQ(i-2) has been drained], then dP^T(i+1) = V·dO(i+1)^T,
// while the compute warps run P(i) -> drain dQ(i-1) -> dS(i): the dQ drain of one tile and the
// softmax of the next overlap the dK/dQ MMAs. dQ has TMEM lane = query, and each thread adds
// 16-byte pieces of its row to the fp32 accumulator with red.global.
// ------------------------------------------------------------------------------------------
template <int D, bool ACC>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdKParams p, const AccOut acc) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::TILE;
    uint8_t* sQ = sV + C::TILE;                   // 2 stages
    uint8_t* sdO = sQ + 2 * C::TILE;              // 2 stages
    uint8_t* sdS = sdO + 2 * C::TILE;             // dS^T, 2 chunks [128 keys][64 queries], SW128
    float* sStat = reinterpret_cast<float*>(sdS + C::DS_BYTES);   // [wg][buf][LSE2 64 | D 64]
    BwdBars* bars = reinterpret_cast<BwdBars*>(sdS + C::DS_BYTES + C::STAT_BYTES);

    // TMEM: dV [0,64) | dK [64,128) | dQ x2 [128,192),[192,256) | S^T [256,384) | dP^T [384,512)
    static_assert(D <= 64, "d = 128 runs bwd_main_q64_kernel");
    constexpr uint32_t COL_DV = 0, COL_DK = 64, COL_DQ = 128, COL_S = 256, COL_DP = 384;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Heads in groups of p.group (a group's Q, dO, K, V and dQ rows stay in L2); within a group,
    // key tiles go from small j (most causal work) to large j across the group's heads.
    const int L = blockIdx.x;
    const int gbase = (L / (p.group * p.nkt)) * p.group;
    const int gsize = min(p.group, p.BH - gbase);
    const int r_in = L - gbase * p.nkt;
    // deterministic mode adds dQ partials in decreasing key-tile order, so CTAs of high key tiles
    // are launched first (a CTA only ever waits for CTAs launched before it)
    const int j = p.deterministic ? p.nkt - 1 - r_in / gsize : r_in / gsize;
    const int kvbh = gbase + r_in % gsize;        // K/V head of this CTA
    const MaskSpec& mk = p.mask;
    const int nk = mk.nk;
    const int qt128 = p.n_pad / 128;              // semaphore stride per query head
    int i_begin, i_end;                           // query tiles that meet this key tile
    visible_query_tiles(mk, j * 128LL, min(j * 128LL + 127, nk - 1LL), 128, i_begin, i_end);
    const int NT = i_end - i_begin;               // query tiles per query head
    const int NTT = NT * p.kv_group;              // over all query heads sharing this K/V head

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->ds_full, 256);
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(&bars->dq_full[b2], 1);
            mbar_init(&bars->dq_drained[b2], 256);
        }
        mbar_init(&bars->ds_free, 1);
        mbar_init(&bars->dkv_done, 1);
        mbar_init(&bars->teardown, 1);
        bars->abort = ((smem_addr(smem) & 1023u) != 0) ? 1 : 0;
        if (bars->abort) report_error(3);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, 512);
    if (warp == 8 && lane == 0) {
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

    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && !*abort && NTT > 0) {
            mbar_arrive_expect_tx(&bars->kv_full, 2 * C::TILE);
            for (int ch = 0; ch < C::NCH; ++ch) {
                tma_load_3d(sK + ch * C::CHUNK, &tmK, &bars->kv_full, ch * C::CW, j * 128, kvbh);
                tma_load_3d(sV + ch * C::CHUNK, &tmV, &bars->kv_full, ch * C::CW, j * 128, kvbh);
            }
            int issued = 0;
            for (int it = 0; it < NTT; ++it) {
                const int st = it & 1, f = it >> 1;
                if (f > 0 && !bounded_wait(&bars->q_empty[st], (f - 1) & 1, abort, lim)) break;
                const int i = i_begin + it % NT;
                const int qbh = kvbh * p.kv_group + it / NT;
                mbar_arrive_expect_tx(&bars->q_full[st], 2 * C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch) {
                    tma_load_3d(sQ + st * C::TILE + ch * C::CHUNK, &tmQ, &bars->q_full[st],
                                ch * C::CW, i * 128, qbh);
                    tma_load_3d(sdO + st * C::TILE + ch * C::CHUNK, &tmdO, &bars->q_full[st],
                                ch * C::CW, i * 128, qbh);
                }
                issued = it + 1;
            }
            if (*abort) {
                drain_wait_bwd(&bars->kv_full, 0, 100000000ull);
                for (int it = 0; it < issued; ++it)
                    drain_wait_bwd(&bars->q_full[it & 1], (it >> 1) & 1, 100000000ull);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        // The whole warp runs this loop (warp-uniform state) and waits together; one elected lane
        // issues each batch of MMAs with its commits (a warp vote per tcgen05.mma would cost the
        // issuing warp ~100 cycles per instruction).
        {
            auto vss = [](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
                mma_ss(d, a, b, id, acc);
            };
            auto vts = [](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
                mma_ts(d, a, b, id, acc);
            };
            auto vcommit = [](uint64_t* bar) { mma_commit(bar); };
            constexpr uint32_t idSS = idesc_bf16_f32(128, 128, 0, 0);    // K-major x K-major
            constexpr uint32_t idKN = idesc_bf16_f32(128, D, 0, 1);      // A K-major, B MN-major
            constexpr uint32_t idDQ = idesc_bf16_f32(128, D, 1, 1);      // dQ = dS · K    // dQ
            const uint32_t aK = smem_addr(sK), aV = smem_addr(sV), aQ = smem_addr(sQ),
                           adO = smem_addr(sdO), adS = smem_addr(sdS);
            // Descriptor words of every operand view, built once (the issuing lane shares its SM
            // sub-partition with busy compute warps: keep the per-MMA instruction count minimal).
            const SDesc K_k = sdesc(aK, 16, 8 * C::SWB, C::SWZ);          // K_j, K-major
            const SDesc V_k = sdesc(aV, 16, 8 * C::SWB, C::SWZ);          // V_j, K-major
            const SDesc K_mn = sdesc(aK, C::CHUNK, 8 * C::SWB, C::SWZ);   // K_j, MN-major
            const SDesc dS_k = sdesc(adS, 16, 1024, 2u);                  // dS^T, K-major
            const SDesc dS_mn = sdesc(adS, 16384, 1024, 2u);              // dS^T, MN-major
            // stage 1 sits TILE bytes after stage 0: its start field is (TILE >> 4) larger
            const SDesc Q_k = sdesc(aQ, 16, 8 * C::SWB, C::SWZ);
            const SDesc Q_mn = sdesc(aQ, C::CHUNK, 8 * C::SWB, C::SWZ);
            const SDesc dO_k = sdesc(adO, 16, 8 * C::SWB, C::SWZ);
            const SDesc dO_mn = sdesc(adO, C::CHUNK, 8 * C::SWB, C::SWZ);
            auto stage = [](SDesc d, int st) { return SDesc{d.lo + st * (C::TILE >> 4), d.hi}; };
            // k-step offsets (16-byte units): K-major over d, MN-major over 16 rows
            auto koff = [](int ks) -> uint32_t {
                return static_cast<uint32_t>((((ks * 16) / C::CW) * C::CHUNK + ((ks * 16) % C::CW) * 2) >> 4);
            };
            auto roff = [](int ks) -> uint32_t { return static_cast<uint32_t>((ks * 16 * C::SWB) >> 4); };
            auto issue_s = [&](int it) {                // S^T = K_j · Q_i^T
                const SDesc bq = stage(Q_k, it & 1);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    vss(tmem + COL_S, sdesc_at(K_k, koff(ks)), sdesc_at(bq, koff(ks)), idSS,
                           ks > 0 ? 1u : 0u);
            };
            auto issue_dp = [&](int it) {               // dP^T = V_j · dO_i^T
                const SDesc bo = stage(dO_k, it & 1);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    vss(tmem + COL_DP, sdesc_at(V_k, koff(ks)), sdesc_at(bo, koff(ks)), idSS,
                           ks > 0 ? 1u : 0u);
            };
            bool ok = NTT > 0 && bounded_wait_warp(&bars->kv_full, 0, abort, lim);
            if (ok) ok = bounded_wait_warp(&bars->q_full[0], 0, abort, lim);
            tc_fence_after();
            if (ok) {
                if (elect_one()) {
                    issue_s(0);
                    vcommit(&bars->s_full);
                    issue_dp(0);
                    vcommit(&bars->dp_full);
                }
                __syncwarp();
            }
            for (int it = 0; ok && it < NTT; ++it) {
                const int st = it & 1;
                if (!(ok = bounded_wait_warp(&bars->p_full, it & 1, abort, lim))) break;
                tc_fence_after();
                if (elect_one()) {   // dV_j += P^T · dO_i   (P^T in TMEM: queries 0-63 at S+0.., 64-127 at S+64..)
                    const SDesc bo = stage(dO_mn, st);
                    vts(tmem + COL_DV, tmem + COL_S, sdesc_at(bo, 0), idKN, it > 0 ? 1u : 0u);
#pragma unroll
                    for (int ks = 1; ks < 8; ++ks)
                        vts(tmem + COL_DV, tmem + COL_S + (ks >> 2) * 64 + (ks & 3) * 8,
                               sdesc_at(bo, roff(ks)), idKN, 1u);
                }
                __syncwarp();
                if (it + 1 < NTT) {
                    if (!(ok = bounded_wait_warp(&bars->q_full[(it + 1) & 1], ((it + 1) >> 1) & 1,
                                            abort, lim)))
                        break;
                    tc_fence_after();
                    if (elect_one()) {
                        issue_s(it + 1);
                        vcommit(&bars->s_full);
                    }
                    __syncwarp();
                }
                if (!(ok = bounded_wait_warp(&bars->ds_full, it & 1, abort, lim))) break;
                tc_fence_after();
                if (elect_one()) {   // dK_j += dS^T · Q_i   (A = dS^T K-major, B = Q_i MN-major)
                    const SDesc bq = stage(Q_mn, st);
                    vss(tmem + COL_DK, sdesc_at(dS_k, 0), sdesc_at(bq, 0), idKN, it > 0 ? 1u : 0u);
#pragma unroll
                    for (int ks = 1; ks < 8; ++ks)
                        vss(tmem + COL_DK,
                               sdesc_at(dS_k, static_cast<uint32_t>(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4)),
                               sdesc_at(bq, roff(ks)), idKN, 1u);
                }
                __syncwarp();
                // dQ_i = dS · K_j into buffer it mod 2, once the partial of tile it-2 is drained
                const int b2 = it & 1;
                if (it >= 2) {
                    if (!(ok = bounded_wait_warp(&bars->dq_drained[b2], ((it - 2) >> 1) & 1, abort, lim))) break;
                    tc_fence_after();
                }
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint64_t kd = sdesc_at(K_mn, roff(ks));
                        const uint64_t sd = sdesc_at(dS_mn, static_cast<uint32_t>((ks * 2048) >> 4));
                        vss(tmem + COL_DQ + b2 * 64, sd, kd, idDQ, ks > 0 ? 1u : 0u);
                    }
                    vcommit(&bars->dq_full[b2]);
                    vcommit(&bars->ds_free);
                    vcommit(&bars->q_empty[st]);
                    // dP^T(i+1): its columns were last read for dS^T(i) (ds_full(i)), and dO(i+1)
                    // arrived before S^T(i+1)
                    if (it + 1 < NTT) {
                        issue_dp(it + 1);
                        vcommit(&bars->dp_full);
                    }
                }
                __syncwarp();
            }
            if (elect_one()) {
                if (ok) vcommit(&bars->dkv_done);
                vcommit(&bars->teardown);
            }
            __syncwarp();
            drain_wait_bwd(&bars->teardown, 0, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- compute warpgroups
        const int g = warp >> 2;                           // warpgroup: query columns 64g..64g+63
        const int t = threadIdx.x & 127;
        const int r = (warp & 3) * 32 + lane;              // key row within the tile = TMEM lane
        const int kidx = j * 128 + r;
        const int cb = g * 64;
        // queries that see key kidx: [qmin, qmax] (empty for a key past the end)
        int qmin = 1, qmax = 0;
        if (kidx < nk) {
            qmin = mk.wr < 0 ? -0x7fffffff : clamp_int(kidx - mk.off - mk.wr);
            qmax = mk.wl < 0 ? 0x7fffffff : clamp_int(kidx - mk.off + mk.wl);
        }
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + COL_S;
        const uint32_t tDP = tmem + lane_base + COL_DP;
        const float sl2 = p.scale_log2;
        auto wg_bar = [&]() {
            if (g == 0)
                asm volatile("bar.sync 1, 128;" ::: "memory");
            else
                asm volatile("bar.sync 2, 128;" ::: "memory");
        };
        auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
            return __all_sync(0xffffffffu, bounded_wait(bar, par, abort, lim));
        };
        float pr[64];
        bool ok = true;

        // dQ partial of tile `it` out of TMEM into the fp32 accumulator
        auto drain = [&](int it) -> bool {
            const int i = i_begin + it % NT;
            const int qbh = kvbh * p.kv_group + it / NT;
            const int b2 = it & 1;
            if (!wait_all(&bars->dq_full[b2], (it >> 1) & 1)) return false;
            tc_fence_after();
            if (p.deterministic) {
                // add this tile's partial only after every higher key tile that meets the query
                // tile has added its own (each CTA contributes two halves, one per warpgroup)
                volatile int* sem = p.sems + static_cast<size_t>(qbh) * qt128 + i;
                const int need = 2 * (last_key_tile(mk, i * 128LL, 128, 128) - j);
                bool got = true;
                if (t == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (*sem < need) {
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
                wg_bar();
                if (*abort) got = false;
                if (!__all_sync(0xffffffffu, got)) {
                    tc_fence_before();
                    mbar_arrive(&bars->dq_drained[b2]);
                    return false;
                }
            }
            float* acc_tile = p.dq_acc + (static_cast<size_t>(qbh) * p.n_pad + i * 128) * D;
            {
                // lane r = query row; columns = head-dim g*D/2 .. (g+1)*D/2-1; rows past the
                // launch's last query add nothing (they may lie outside its workspace rows)
                const uint32_t tDQ = tmem + lane_base + COL_DQ + b2 * 64 + g * (D / 2);
                const bool live = i * 128 + r < mk.nq;
                float* row = acc_tile + r * D + g * (D / 2);
                if constexpr (D / 2 == 32) {
                    uint32_t u[32];
                    tmem_ld32(tDQ, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        if (live) red_add_v4_f32(row + 4 * x, __uint_as_float(u[4 * x]), __uint_as_float(u[4 * x + 1]),
                                       __uint_as_float(u[4 * x + 2]), __uint_as_float(u[4 * x + 3]));
                } else {
                    uint32_t u[16];
                    tmem_ld16(tDQ, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        if (live) red_add_v4_f32(row + 4 * x, __uint_as_float(u[4 * x]), __uint_as_float(u[4 * x + 1]),
                                       __uint_as_float(u[4 * x + 2]), __uint_as_float(u[4 * x + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->dq_drained[b2]);
            if (p.deterministic) {
                __threadfence();
                wg_bar();
                if (t == 0) atomicAdd(p.sems + static_cast<size_t>(qbh) * qt128 + i, 1);
            }
            return true;
        };

        for (int it = 0; it < NTT; ++it) {
            const int i = i_begin + it % NT;
            const int qbh = kvbh * p.kv_group + it / NT;
            float* sL = sStat + (g * 2 + (it & 1)) * 128;
            float* sD = sL + 64;
            {
                // rows past the launch's last query (a 128-row tile that starts 64 rows into a
                // workspace block runs into the next head's rows) read as padding: P = dS = 0
                const int qr = i * 128 + cb + (t & 63);
                const size_t qq = static_cast<size_t>(qbh) * p.n_pad + qr;
                if (t < 64)
                    sL[t] = qr < mk.nq ? p.L2vec[qq] : INFINITY;
                else
                    sD[t - 64] = qr < mk.nq ? p.Dvec[qq] : 0.f;
            }
            wg_bar();
            // ---- P^T = exp2(S^T·scale·log2e - LSE·log2e), masked; bf16 copy into TMEM
            if (!(ok = wait_all(&bars->s_full, it & 1))) break;
            tc_fence_after();
            bool edge;
            {   // every key of the tile visible to every query of the tile: no mask needed
                long long flo, fhi;
                visible_keys(mk, i * 128LL + 127, i * 128LL, flo, fhi);
                edge = !(flo <= j * 128LL && j * 128LL + 127 <= fhi);
            }
            const int q0 = i * 128 + cb;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
                tmem_ld32(tS + cb + c * 32, u);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const int col = c * 32 + x;
                    float v = ex2_approx(fmaf(__uint_as_float(u[x]), sl2, -sL[col]));
                    if (edge && (q0 + col < qmin || q0 + col > qmax)) v = 0.f;
                    pr[col] = v;
                }
            }
            {
                uint32_t w[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) w[x] = pack_bf16x2(pr[2 * x], pr[2 * x + 1]);
                tmem_st32(tS + g * 64, w);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars->p_full);
            // ---- drain the previous tile's dQ while the MMAs of this tile run
            if (it > 0 && !(ok = drain(it - 1))) break;
            // ---- dS^T = P^T ∘ (dP^T - D) -> bf16 into shared memory (chunk g, swizzled)
            if (!(ok = wait_all(&bars->dp_full, it & 1))) break;
            if (it > 0 && !(ok = wait_all(&bars->ds_free, (it - 1) & 1))) break;
            tc_fence_after();
            uint8_t* ds_row = sdS + g * 16384 + r * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
                tmem_ld32(tDP + cb + c * 32, u);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int c0 = c * 32 + 2 * x;
                    const float d0 = pr[c0] * (__uint_as_float(u[2 * x]) - sD[c0]);
                    const float d1 = pr[c0 + 1] * (__uint_as_float(u[2 * x + 1]) - sD[c0 + 1]);
                    w[x] = pack_bf16x2(d0, d1);
                }
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const int unit = c * 4 + tt;
                    *reinterpret_cast<uint4*>(ds_row + ((unit ^ (r & 7)) << 4)) =
                        make_uint4(w[4 * tt], w[4 * tt + 1], w[4 * tt + 2], w[4 * tt + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_full);
        }
        if (ok && NTT > 0) ok = drain(NTT - 1);
        if (ok && NTT == 0) {
            // no query sees these keys: dK = dV = 0
            if (kidx < nk && !ACC) {     // (accumulating: nothing to add)
                const size_t orow = (static_cast<size_t>(kvbh) * nk + kidx) * D + g * (D / 2);
#pragma unroll
                for (int x = 0; x < D / 16; ++x) {
                    reinterpret_cast<uint4*>(p.dk + orow)[x] = make_uint4(0u, 0u, 0u, 0u);
                    reinterpret_cast<uint4*>(p.dv + orow)[x] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            ok = false;
        }
        if (ok) ok = wait_all(&bars->dkv_done, 0);
        if (ok) {
            tc_fence_after();
            const size_t orow = (static_cast<size_t>(kvbh) * nk + kidx) * D + g * (D / 2);
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t tacc = tmem + lane_base + (which == 0 ? COL_DV : COL_DK) + g * (D / 2);
                const float mul = which == 0 ? 1.f : p.scale;
                __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + orow;
#pragma unroll 1
                for (int cc = 0; cc < D / 2; cc += 16) {
                    uint32_t u[16];
                    tmem_ld16(tacc + cc, u);
                    tmem_ld_wait();
                    if constexpr (ACC) {
                        if (kidx < nk)
                            add_row_f32<16>((which == 0 ? acc.dv : acc.dk) +
                                                (static_cast<size_t>(kvbh) * acc.rows + kidx) * D +
                                                g * (D / 2) + cc,
                                            u, mul);
                    } else {
                        uint32_t w[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x)
                            w[x] = pack_bf16x2(__uint_as_float(u[2 * x]) * mul,
                                               __uint_as_float(u[2 * x + 1]) * mul);
                        if (kidx < nk) {
                            uint4* o = reinterpret_cast<uint4*>(dst + cc);
                            o[0] = make_uint4(w[0], w[1], w[2], w[3]);
                            o[1] = make_uint4(w[4], w[5], w[6], w[7]);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------
// Main backward kernel for d = 128: 64-row query tiles, two of them in flight.
//
// A CTA owns one 128-key tile j (K_j and V_j stay in shared memory, dK and dV accumulate in
// TMEM) and walks the 64-row query tiles that meet it. Per query tile i the work is a chain whose
// links alternate between the tensor cores and the SIMT warps:
//     S^T = K·Q^T -> P^T = exp2(S^T·c - LSE·log2e) -> dV += P^T·dO
//     dP^T = V·dO^T -> dS^T = P^T∘(dP^T - D) -> dK += dS^T·Q,  dQ^T = K^T·dS^T -> drain
// With one tile in flight the tensor cores idle whenever the warps form P^T or dS^T. Here two
// compute warpgroups each take every other query tile, so while one works on tile i the tensor
// cores run the products of its neighbour. TMEM (512 columns):
//     dV [0,128) | dK [128,256) | S^T, then P^T, of even tiles [256,320), of odd tiles
//     [320,384) | dP^T, then dQ^T, of even tiles [384,448), of odd tiles [448,512)
// dQ^T(i) is written over dP^T(i) once dS^T(i) has been formed from it; tile i+2 reuses both
// column ranges, its dP^T after the drain has read dQ^T(i) out.
// Roles (512 threads; warp 11 idle):
//   warps 0-3, 4-7  compute warpgroups 0 and 1: even and odd query tiles, all 64 query columns;
//                   one thread per key row (TMEM lane).
//   warp 8          TMA producer: K_j, V_j once; Q_i, dO_i (64 rows) and the matching 64 values of
//                   LSE·log2e and D through a 3-deep ring.
//   warps 9, 10     MMA issuers (one elected lane issues each batch of MMAs with its commits;
//                   a tcgen05.mma costs its issuing warp tens of cycles, so two warps on two SM
//                   sub-partitions feed the tensor pipe):
//                   warp 9:  S^T, dP^T of tile i [dQ^T(i-2) read out, Q/dO(i) loaded];
//                   warp 10: dV(i) [P^T(i) ready], then dK(i), dQ^T(i) [dS^T(i) ready].
//                   The commits of warp 10 cover warp 9's products of the same tile: P^T(i)
//                   and dS^T(i) exist only once S^T(i) and dP^T(i) are complete.
//   warps 12-15     dQ drain, each warp on its own: 32 head-dim columns of dQ(i) out of TMEM
//                   (one column per lane), staged per half tile as a [32 queries][32 columns]
//                   fp32 box and added to the fp32 accumulator by a TMA tensor reduction. The
//                   deterministic mode orders the additions to each (query tile, column block)
//                   by key tile, from the last key tile that meets the query tile down, with one
//                   semaphore per query tile and drain warp (acquire load before the first
//                   box, release add one tile later, once the tile's reductions are complete).
// ------------------------------------------------------------------------------------------
namespace q64 {
constexpr int kThreads = 512;              // warp 11 idle: the drain warps must be warps
                                           // 12-15 to cover TMEM lane quarters 0-3
constexpr int BQ = 64;                     // query rows per tile
constexpr int KTILE = 128 * 128 * 2;       // K_j or V_j: 2 chunks [128 rows][64 d], SW128
constexpr int QTILE = 64 * 128 * 2;        // Q_i or dO_i: 2 chunks [64 rows][64 d]
constexpr int QCHUNK = 64 * 128;           // bytes of one [64 rows][64 d] chunk
constexpr int STAGES = 3;                  // two tiles in flight plus one loading
constexpr int DS_BYTES = 128 * 64 * 2;     // dS^T [128 keys][64 queries], one SW128 chunk
constexpr int BOX = 32 * 32 * 4;           // drain box: [32 queries][32 columns] fp32
constexpr int BOXES = 2;                   // boxes per drain warp (one reduction may be reading)
constexpr int STG_BYTES = 4 * BOXES * BOX;
constexpr int OFF_K = 0, OFF_V = KTILE, OFF_Q = 2 * KTILE, OFF_DO = OFF_Q + STAGES * QTILE;
constexpr int OFF_DS = OFF_DO + STAGES * QTILE;            // two buffers, by tile parity
constexpr int OFF_STG = OFF_DS + 2 * DS_BYTES;
constexpr int OFF_L2 = OFF_STG + STG_BYTES, OFF_DV = OFF_L2 + STAGES * 256;
constexpr int OFF_BARS = OFF_DV + STAGES * 256;
constexpr int SMEM = OFF_BARS + 256;
static_assert(SMEM <= 232448, "dynamic shared memory per block");
static_assert(OFF_DS % 1024 == 0 && OFF_STG % 128 == 0, "operand and box alignment");
// registers: launched at 128 per thread; the producer/MMA warpgroup gives up 64, the drain
// warpgroup 32, and the compute warpgroups take 48 each: 128·64 + 128·96 + 256·176 <= 512·128
constexpr int kRegsIdle = 64, kRegsDrain = 96, kRegsCompute = 176;
static_assert(128 * kRegsIdle + 128 * kRegsDrain + 256 * kRegsCompute <= kThreads * 128,
              "register split");

struct Bars {
    uint64_t kv_full;
    uint64_t q_full[STAGES], q_empty[STAGES];
    // per tile parity (even / odd query tiles)
    uint64_t s_full[2], dp_full[2], p_full[2], ds_full[2], ds_free[2], dq_full[2], dq_drained[2];
    uint64_t dkv_done, teardown;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");
}  // namespace q64

template <bool ACC>
__global__ void __launch_bounds__(q64::kThreads, 1)
    bwd_main_q64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmAcc, const BwdKParams p,
                        const AccOut acc) {
    using namespace q64;
    constexpr int D = 128;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sK = smem + OFF_K;
    uint8_t* sV = smem + OFF_V;
    uint8_t* sQ = smem + OFF_Q;
    uint8_t* sdO = smem + OFF_DO;
    uint8_t* sdS = smem + OFF_DS;
    float* sStg = reinterpret_cast<float*>(smem + OFF_STG);
    float* sL2 = reinterpret_cast<float*>(smem + OFF_L2);     // [STAGES][64]
    float* sDv = reinterpret_cast<float*>(smem + OFF_DV);     // [STAGES][64]
    Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BARS);

    // S^T/P^T and dP^T/dQ^T columns of a tile: base + 64 * (tile parity)
    constexpr uint32_t COL_DV = 0, COL_DK = 128, COL_S = 256, COL_DP = 384;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Heads in groups of p.group (see bwd_main_kernel); key tiles of 128 keys, small j first.
    const int L = blockIdx.x;
    const int gbase = (L / (p.group * p.nkt)) * p.group;
    const int gsize = min(p.group, p.BH - gbase);
    const int r_in = L - gbase * p.nkt;
    // deterministic mode: high key tiles first (see bwd_main_kernel)
    const int j = p.deterministic ? p.nkt - 1 - r_in / gsize : r_in / gsize;
    const int kvbh = gbase + r_in % gsize;         // K/V head of this CTA
    const MaskSpec& mk = p.mask;
    const int nk = mk.nk;
    const int qt64 = p.n_pad / BQ;                 // 64-row query tiles per query head
    int i_begin, i_end;                            // 64-row query tiles that meet this key tile
    visible_query_tiles(mk, j * 128LL, min(j * 128LL + 127, nk - 1LL), BQ, i_begin, i_end);
    const int NT = i_end - i_begin;                // query tiles per query head
    const int NTT = NT * p.kv_group;               // over all query heads sharing this K/V head

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->dp_full[x], 1);
            mbar_init(&bars->p_full[x], 128);
            mbar_init(&bars->ds_full[x], 128);
            mbar_init(&bars->ds_free[x], 1);
            mbar_init(&bars->dq_full[x], 1);
            mbar_init(&bars->dq_drained[x], 128);
        }
        mbar_init(&bars->dkv_done, 1);
        mbar_init(&bars->teardown, 2);                 // one commit per MMA issuer
        bars->abort = ((smem_addr(smem) & 1023u) != 0) ? 1 : 0;
        if (bars->abort) report_error(3);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, 512);
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmAcc);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    const uint64_t lim = p.timeout_ns;

    if (warp >= 8 && warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIdle));
    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && !*abort && NTT > 0) {
            mbar_arrive_expect_tx(&bars->kv_full, 2 * KTILE);
            for (int ch = 0; ch < 2; ++ch) {
                tma_load_3d(sK + ch * 16384, &tmK, &bars->kv_full, ch * 64, j * 128, kvbh);
                tma_load_3d(sV + ch * 16384, &tmV, &bars->kv_full, ch * 64, j * 128, kvbh);
            }
            int issued = 0;
            for (int it = 0; it < NTT; ++it) {
                const int st = it % STAGES, f = it / STAGES;
                if (f > 0 && !bounded_wait(&bars->q_empty[st], (f - 1) & 1, abort, lim)) break;
                const int i = i_begin + it % NT;
                const int bh = kvbh * p.kv_group + it / NT;   // query head
                mbar_arrive_expect_tx(&bars->q_full[st], 2 * QTILE + 2 * 256);
                for (int ch = 0; ch < 2; ++ch) {
                    tma_load_3d(sQ + st * QTILE + ch * QCHUNK, &tmQ, &bars->q_full[st], ch * 64,
                                i * BQ, bh);
                    tma_load_3d(sdO + st * QTILE + ch * QCHUNK, &tmdO, &bars->q_full[st], ch * 64,
                                i * BQ, bh);
                }
                const size_t row0 = static_cast<size_t>(bh) * p.n_pad + i * BQ;
                bulk_load(sL2 + st * 64, p.L2vec + row0, 256, &bars->q_full[st]);
                bulk_load(sDv + st * 64, p.Dvec + row0, 256, &bars->q_full[st]);
                issued = it + 1;
            }
            if (*abort) {
                drain_wait_bwd(&bars->kv_full, 0, 100000000ull);
                for (int it = (issued > STAGES ? issued - STAGES : 0); it < issued; ++it)
                    drain_wait_bwd(&bars->q_full[it % STAGES], (it / STAGES) & 1, 100000000ull);
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ---------------------------------------------------------------- MMA issuers
        // The whole warp waits; one elected lane issues a batch of MMAs and its commits.
        constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);      // S^T, dP^T
        constexpr uint32_t idKV = idesc_bf16_f32(128, 128, 0, 1);    // dV, dK
        constexpr uint32_t idQ = idesc_bf16_f32(128, 64, 1, 1);      // dQ^T
        const uint32_t aK = smem_addr(sK), aV = smem_addr(sV), aQ = smem_addr(sQ),
                       adO = smem_addr(sdO), adS = smem_addr(sdS);
        const SDesc K_k = sdesc(aK, 16, 1024, 2u), V_k = sdesc(aV, 16, 1024, 2u);
        const SDesc K_mn = sdesc(aK, 16384, 1024, 2u);
        const SDesc dS_k = sdesc(adS, 16, 1024, 2u), dS_mn = sdesc(adS, 16384, 1024, 2u);
        const SDesc Q_k = sdesc(aQ, 16, 1024, 2u), Q_mn = sdesc(aQ, QCHUNK, 1024, 2u);
        const SDesc dO_k = sdesc(adO, 16, 1024, 2u), dO_mn = sdesc(adO, QCHUNK, 1024, 2u);
        auto shift = [](SDesc d, int bytes) { return SDesc{d.lo + static_cast<uint32_t>(bytes >> 4), d.hi}; };
        // k-step offsets over d: operand with 128 rows (16 KB chunks) / 64 rows (8 KB chunks)
        auto k128 = [](int ks) -> uint32_t { return static_cast<uint32_t>(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4); };
        auto k64 = [](int ks) -> uint32_t { return static_cast<uint32_t>(((ks >> 2) * QCHUNK + (ks & 3) * 32) >> 4); };
        // S^T(it) and dP^T(it) into the columns of the tile's parity
        auto issue_sdp = [&](int it) {
            const uint32_t x = static_cast<uint32_t>(it & 1);
            const int st = it % STAGES;
            const SDesc bq = shift(Q_k, st * QTILE), bo = shift(dO_k, st * QTILE);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(tmem + COL_S + 64 * x, sdesc_at(K_k, k128(ks)), sdesc_at(bq, k64(ks)), idS,
                       ks > 0 ? 1u : 0u);
            mma_commit(&bars->s_full[x]);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(tmem + COL_DP + 64 * x, sdesc_at(V_k, k128(ks)), sdesc_at(bo, k64(ks)), idS,
                       ks > 0 ? 1u : 0u);
            mma_commit(&bars->dp_full[x]);
        };
        // dV += P^T(it) · dO(it): P^T of query q at column q/2 of the tile's S^T range
        auto issue_dv = [&](int it) {
            const uint32_t x = static_cast<uint32_t>(it & 1);
            const SDesc bo = shift(dO_mn, (it % STAGES) * QTILE);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ts(tmem + COL_DV, tmem + COL_S + 64 * x + ks * 8,
                       sdesc_at(bo, static_cast<uint32_t>((ks * 2048) >> 4)), idKV,
                       (it > 0 || ks > 0) ? 1u : 0u);
        };
        // dK += dS^T(it) · Q(it); dQ^T(it) = K^T · dS^T(it) over dP^T(it)
        auto issue_dkdq = [&](int it) {
            const int x = it & 1, st = it % STAGES;
            const SDesc bq = shift(Q_mn, st * QTILE);
            const SDesc a_ds = shift(dS_k, x * DS_BYTES), b_ds = shift(dS_mn, x * DS_BYTES);
            // dQ^T first: the drain, and through it the next S^T of this parity, waits for it
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(tmem + COL_DP + 64 * x, sdesc_at(K_mn, static_cast<uint32_t>((ks * 2048) >> 4)),
                       sdesc_at(b_ds, static_cast<uint32_t>((ks * 2048) >> 4)), idQ, ks > 0 ? 1u : 0u);
            mma_commit(&bars->dq_full[x]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_ss(tmem + COL_DK, sdesc_at(a_ds, static_cast<uint32_t>((ks * 32) >> 4)),
                       sdesc_at(bq, static_cast<uint32_t>((ks * 2048) >> 4)), idKV,
                       (it > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&bars->ds_free[x]);
            mma_commit(&bars->q_empty[st]);
        };
        bool ok = NTT > 0;
        if (warp == 9) {
            // S^T(i), dP^T(i): tile i takes the columns of tile i-2, free once the drain has read
            // dQ^T(i-2) (which also means dV(i-2), the last reader of P^T(i-2), is complete)
            if (ok) ok = bounded_wait_warp(&bars->kv_full, 0, abort, lim);
            for (int it = 0; ok && it < NTT; ++it) {
                const int x = it & 1;
                if (it >= 2 && !(ok = bounded_wait_warp(&bars->dq_drained[x], ((it >> 1) - 1) & 1, abort, lim)))
                    break;
                if (!(ok = bounded_wait_warp(&bars->q_full[it % STAGES], (it / STAGES) & 1, abort, lim)))
                    break;
                tc_fence_after();
                if (elect_one()) issue_sdp(it);
                __syncwarp();
            }
        } else {
            for (int it = 0; ok && it < NTT; ++it) {
                const int x = it & 1;
                const uint32_t ph = static_cast<uint32_t>((it >> 1) & 1);   // tile it's phase
                if (!(ok = bounded_wait_warp(&bars->p_full[x], ph, abort, lim))) break;
                tc_fence_after();
                if (elect_one()) issue_dv(it);
                __syncwarp();
                if (!(ok = bounded_wait_warp(&bars->ds_full[x], ph, abort, lim))) break;
                tc_fence_after();
                if (elect_one()) issue_dkdq(it);
                __syncwarp();
            }
            if (ok && elect_one()) mma_commit(&bars->dkv_done);
            __syncwarp();
        }
        if (elect_one()) mma_commit(&bars->teardown);
        __syncwarp();
        drain_wait_bwd(&bars->teardown, 0, 100000000ull);
    }
    } else if (warp >= 12) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsDrain));
        // ---------------------------------------------------------------- dQ drain warps
        const int w = warp & 3;                            // head-dim columns 32w .. 32w+31
        const uint32_t lane_base = static_cast<uint32_t>(w * 32) << 16;
        float* boxes = sStg + w * (BOXES * BOX / 4);
        int nbox = 0;                                      // boxes this warp has issued
        bool run = true;
        volatile int* pending = nullptr;                   // semaphore still to be released
        for (int it = 0; run && it < NTT; ++it) {
            const int x = it & 1;
            if (!bounded_wait_warp(&bars->dq_full[x], (it >> 1) & 1, abort, lim)) break;
            tc_fence_after();
            uint32_t u[64];                                // lane = column 32w + lane, 64 queries
            tmem_ld32(tmem + lane_base + COL_DP + 64 * x, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            tmem_ld32(tmem + lane_base + COL_DP + 64 * x + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            tmem_ld_wait();
            reg_fence<64>(u);
            tc_fence_before();
            mbar_arrive(&bars->dq_drained[x]);
            const int i = i_begin + it % NT;
            const int qbh = kvbh * p.kv_group + it / NT;
            const int row0 = qbh * p.n_pad + i * BQ;       // accumulator row of the tile's query 0
            volatile int* sem = p.deterministic
                                    ? p.sems + (static_cast<size_t>(qbh) * qt64 + i) * 4 + w
                                    : nullptr;
#pragma unroll
            for (int h = 0; h < 2; ++h, ++nbox) {
                float* box = boxes + (nbox % BOXES) * (BOX / 4);
                // the reduction issued from this box BOXES boxes ago has finished reading it
                if (lane == 0) bulk_wait_read_le1();
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 32; ++q) box[q * 32 + lane] = __uint_as_float(u[h * 32 + q]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    bool got = true;
                    if (h == 0 && sem) {
                        // the key tiles above this one that meet query tile i add first
                        const int need = last_key_tile(mk, static_cast<long long>(i) * BQ, BQ, 128) - j;
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire_gpu(sem) < need) {   // the acquire orders the adds below
                            if (*abort || globaltimer_ns() - t0 > lim) {
                                *abort = 1;
                                report_error(4);
                                got = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    if (got && !*abort) {
                        tma_reduce_add_2d(&tmAcc, box, 32 * w, row0 + 32 * h);
                        bulk_commit();
                    }
                }
                __syncwarp();
                if (*abort) { run = false; break; }
            }
            if (sem && lane == 0 && run) {
                // release the previous tile's semaphore one tile late, once its reductions (not
                // only their reads) are complete: at most this tile's two groups are pending
                if (pending) {
                    bulk_wait_le2_complete();
                    red_release_gpu_add(pending, 1);
                }
                pending = sem;
            }
            __syncwarp();
        }
        if (lane == 0) {
            bulk_wait_all();
            if (pending && !*abort) red_release_gpu_add(pending, 1);
        }
        __syncwarp();
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
        // ---------------------------------------------------------------- compute warpgroups
        const int x = warp >> 2;                           // query tiles of parity x
        const int r = (warp & 3) * 32 + lane;              // key row = TMEM lane
        const int kidx = j * 128 + r;
        // queries that see key kidx: [qmin, qmax] (empty for a key past the end)
        int qmin = 1, qmax = 0;
        if (kidx < nk) {
            qmin = mk.wr < 0 ? -0x7fffffff : clamp_int(kidx - mk.off - mk.wr);
            qmax = mk.wl < 0 ? 0x7fffffff : clamp_int(kidx - mk.off + mk.wl);
        }
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + COL_S + 64 * x;
        const uint32_t tDP = tmem + lane_base + COL_DP + 64 * x;
        uint8_t* ds_row = sdS + x * DS_BYTES + r * 128;
        const float sl2 = p.scale_log2;
        auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
            return __all_sync(0xffffffffu, bounded_wait(bar, par, abort, lim));
        };
        float pr[64];
        bool ok = true;

        for (int it = x; it < NTT; it += 2) {
            const int i = i_begin + it % NT;
            const int st = it % STAGES;
            const uint32_t ph = static_cast<uint32_t>((it >> 1) & 1);
            const float* L2 = sL2 + st * 64;
            const float* Dv = sDv + st * 64;
            // ---- P^T = exp2(S^T·scale·log2e - LSE·log2e), masked; bf16 into TMEM over S^T
            if (!(ok = wait_all(&bars->s_full[x], ph))) break;
            tc_fence_after();
            bool edge;
            {   // every key of the tile visible to every query of the tile: no mask needed
                long long flo, fhi;
                visible_keys(mk, static_cast<long long>(i) * BQ + BQ - 1,
                             static_cast<long long>(i) * BQ, flo, fhi);
                edge = !(flo <= j * 128LL && j * 128LL + 127 <= fhi);
            }
            {   // the whole S^T row of the tile (64 columns): two loads, one wait
                uint32_t u[64];
                tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
                tmem_ld_wait();
                reg_fence<64>(u);
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const float4 l4 = *reinterpret_cast<const float4*>(L2 + c);
                    pr[c] = ex2_approx(fmaf(__uint_as_float(u[c]), sl2, -l4.x));
                    pr[c + 1] = ex2_approx(fmaf(__uint_as_float(u[c + 1]), sl2, -l4.y));
                    pr[c + 2] = ex2_approx(fmaf(__uint_as_float(u[c + 2]), sl2, -l4.z));
                    pr[c + 3] = ex2_approx(fmaf(__uint_as_float(u[c + 3]), sl2, -l4.w));
                }
            }
            if (edge) {
                const int q0 = i * BQ;
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (q0 + c < qmin || q0 + c > qmax) pr[c] = 0.f;
            }
            {
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) w[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
                tmem_st32(tS, w);                          // query q at column q/2
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&bars->p_full[x]);
            // ---- dS^T = P^T ∘ (dP^T - D) -> bf16 into shared memory (row r, swizzled)
            if (!(ok = wait_all(&bars->dp_full[x], ph))) break;
            if (it >= 2 && !(ok = wait_all(&bars->ds_free[x], ph ^ 1u))) break;
            tc_fence_after();
            uint32_t du[64];                                   // the dP^T row, one wait
            tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&du[0]));
            tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&du[32]));
            tmem_ld_wait();
            reg_fence<64>(du);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t* u = du + 32 * h;
                uint32_t w[16];
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                    const float4 d4 = *reinterpret_cast<const float4*>(Dv + 32 * h + 2 * c);
                    w[c] = pack_bf16x2(pr[32 * h + 2 * c] * (__uint_as_float(u[2 * c]) - d4.x),
                                       pr[32 * h + 2 * c + 1] * (__uint_as_float(u[2 * c + 1]) - d4.y));
                    w[c + 1] = pack_bf16x2(pr[32 * h + 2 * c + 2] * (__uint_as_float(u[2 * c + 2]) - d4.z),
                                           pr[32 * h + 2 * c + 3] * (__uint_as_float(u[2 * c + 3]) - d4.w));
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int unit = 4 * h + t;                // queries 8·unit .. 8·unit+7
                    *reinterpret_cast<uint4*>(ds_row + ((unit ^ (r & 7)) << 4)) =
                        make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_full[x]);
        }
        // ---- epilogue: warpgroup x writes head-dim columns 64x .. 64x+63 of dV and dK
        if (ok && NTT == 0) {
            // no query sees these keys: dK = dV = 0
            if (kidx < nk && !ACC) {     // (accumulating: nothing to add)
                const size_t orow = (static_cast<size_t>(kvbh) * nk + kidx) * D + x * 64;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    reinterpret_cast<uint4*>(p.dk + orow)[c] = make_uint4(0u, 0u, 0u, 0u);
                    reinterpret_cast<uint4*>(p.dv + orow)[c] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            ok = false;
        }
        if (ok) ok = wait_all(&bars->dkv_done, 0);
        if (ok) {
            tc_fence_after();
            const size_t orow = (static_cast<size_t>(kvbh) * nk + kidx) * D + x * 64;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t tacc = tmem + lane_base + (which == 0 ? COL_DV : COL_DK) + x * 64;
                const float mul = which == 0 ? 1.f : p.scale;
                __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + orow;
#pragma unroll 1
                for (int cc = 0; cc < 64; cc += 32) {
                    uint32_t u[32];
                    tmem_ld32(tacc + cc, u);
                    tmem_ld_wait();
                    reg_fence<32>(u);
                    if constexpr (ACC) {
                        if (kidx < nk)
                            add_row_f32<32>((which == 0 ? acc.dv : acc.dk) +
                                                (static_cast<size_t>(kvbh) * acc.rows + kidx) * D +
                                                x * 64 + cc,
                                            u, mul);
                    } else {
                        uint32_t w[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            w[c] = pack_bf16x2(__uint_as_float(u[2 * c]) * mul,
                                               __uint_as_float(u[2 * c + 1]) * mul);
                        if (kidx < nk) {
                            uint4* o = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                o[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t stream) {
    using C = BwdCfg<D>;
    const int BH = a.B * a.H;
    // query rows per head in the workspace (this launch's rows start at a.q_row0 within them)
    const int n_pad = ((a.ws_rows > 0 ? a.ws_rows : a.nq) + 127) / 128 * 128;
    const int nkt = (a.nk + 127) / 128;
    const int nk_pad = nkt * 128;
    // Main-kernel CTAs run per K/V head. Heads per group: a K/V head's K and V (4·nk·d bytes) and
    // its g query heads' Q, dO (4·nq·d each) and fp32 dQ rows (4·nq·d each); keep a group within
    // ~48 MB of L2
    const int BHkv = a.B * a.Hkv;
    const int kvg = a.H / a.Hkv;
    int group;
    {
        const long long per_head = (4LL * nk_pad + 8LL * kvg * n_pad) * D;
        long long g = (48LL << 20) / (per_head > 0 ? per_head : 1);
        group = static_cast<int>(g < 1 ? 1 : (g > BHkv ? BHkv : g));
    }
    cudaError_t e;
    const cudaEvent_t* ev = a.phase_events;
    if (ev && ev[0] && (e = cudaEventRecord(ev[0], stream)) != cudaSuccess) return e;
    // 1. preprocess
    if (a.phases & 1) {
        const long long rows = static_cast<long long>(BH) * n_pad;
        const int rpw = 32 / (D / 8);
        long long blocks = (rows + (8 * rpw) - 1) / (8 * rpw);
        if (blocks > 148 * 16) blocks = 148 * 16;
        const int n_sems = a.deterministic ? BH * (n_pad / 64) * 4 : 0;
        bwd_preprocess_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dO), a.lse,
            a.L2vec, a.Dvec, a.dq_acc, a.deterministic ? a.sems : nullptr, a.nq, n_pad, rows,
            n_sems);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 2. main
    if (a.phases & 2) {
        if (a.deterministic && !(a.phases & 1)) {
            // the semaphores count this launch's partials from zero (the accumulator keeps its sums)
            const size_t n_sems = static_cast<size_t>(BH) * (n_pad / 64) * 4;
            if ((e = cudaMemsetAsync(a.sems, 0, n_sems * sizeof(int), stream)) != cudaSuccess) return e;
        }
        const AccOut acc{a.dk_acc32, a.dv_acc32, a.kv_rows > 0 ? a.kv_rows : a.nk};
        BwdKParams kp;
        kp.lse = a.lse;
        // the workspace rows of this launch's first query, in every head
        kp.Dvec = a.Dvec + a.q_row0;
        kp.L2vec = a.L2vec + a.q_row0;
        kp.dq_acc = a.dq_acc + static_cast<size_t>(a.q_row0) * D;
        // semaphores count one launch's partials (zeroed by the preprocess or just above), so
        // every launch indexes them from its own first query tile
        kp.sems = a.sems;
        kp.dk = static_cast<__nv_bfloat16*>(a.dk);
        kp.dv = static_cast<__nv_bfloat16*>(a.dv);
        kp.n_pad = n_pad;
        kp.BH = BHkv;
        kp.nkt = nkt;
        kp.kv_group = kvg;
        kp.deterministic = a.deterministic;
        kp.group = group;
        kp.mask = MaskSpec{a.nq, a.nk, a.wl, a.wr, static_cast<long long>(a.nk) - a.nq};
        kp.scale = a.scale;
        kp.scale_log2 = a.scale * kBwdLog2e;
        kp.timeout_ns = a.timeout_ns;
        const long long grid = static_cast<long long>(nkt) * BHkv;
        if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        const int qbox = D == 128 ? q64::BQ : 128;
        CUtensorMap mq, mk, mv, mdo;
        if ((e = make_tmap_bf16(&mq, a.q, BH, a.nq, D, qbox, a.q_rows)) != cudaSuccess) return e;
        if ((e = make_tmap_bf16(&mk, a.k, BHkv, a.nk, D, 128, a.kv_rows)) != cudaSuccess) return e;
        if ((e = make_tmap_bf16(&mv, a.v, BHkv, a.nk, D, 128, a.kv_rows)) != cudaSuccess) return e;
        if ((e = make_tmap_bf16(&mdo, a.dO, BH, a.nq, D, qbox, a.q_rows)) != cudaSuccess) return e;
        if constexpr (D == 128) {
            CUtensorMap macc;   // the fp32 dQ accumulator as (B·H·n_pad) rows x 128 columns
            if ((e = make_tmap_acc(&macc, kp.dq_acc,
                                   static_cast<long long>(BH) * n_pad - a.q_row0, D)) != cudaSuccess)
                return e;
            const auto kern = acc.dk ? bwd_main_q64_kernel<true> : bwd_main_q64_kernel<false>;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, q64::SMEM);
            if (e != cudaSuccess) return e;
            if (ev && ev[1] && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess) return e;
            kern<<<static_cast<unsigned>(grid), q64::kThreads, q64::SMEM, stream>>>(
                mq, mk, mv, mdo, macc, kp, acc);
        } else {
            const auto kern = acc.dk ? bwd_main_kernel<D, true> : bwd_main_kernel<D, false>;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
            if (e != cudaSuccess) return e;
            if (ev && ev[1] && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess) return e;
            kern<<<static_cast<unsigned>(grid), kBwdThreads, C::SMEM, stream>>>(mq, mk, mv, mdo, kp,
                                                                                acc);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (ev && ev[2] && (e = cudaEventRecord(ev[2], stream)) != cudaSuccess) return e;
    }
    // 3. dQ convert
    if (a.phases & 4) {
        const long long total8 = static_cast<long long>(BH) * a.nq * (D / 8);
        long long blocks = (total8 + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        bwd_dq_convert_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            a.dq_acc, static_cast<__nv_bfloat16*>(a.dq), a.nq, n_pad, total8, a.scale);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (ev && ev[3] && (e = cudaEventRecord(ev[3], stream)) != cudaSuccess) return e;
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
