// Forward pass on the sm_100a tensor cores: bf16 in / bf16 out, or E4M3 (fp8) in / bf16 out, with
// fp32 accumulation.
//
// The method is the tiled forward pass with online softmax: Q, K and V are split into tiles held
// on chip, each tile updates a running row max m and row sum l, and the running output is
// rescaled when m grows, so the n x n score matrix never reaches device memory ("Attention
// Mechanism: Revolusi Representasi Sequence", §13 "FlashAttention — How It Works"; "Flash
// Attention Nedir?", sections "Tiling (Blok Bölümleme)" and "Online Softmax"). The output update
// carries the factor exp(m_old - m_new) on the old term; the division by l is deferred to the
// end (the same value in exact arithmetic).
//
// B200 mapping (one CTA per pair of 128-row query tiles of one (b,h)):
//   warp 8      TMA producer: Q tiles once, then K_j / V_j tiles through a STAGES-deep ring.
//   warp 9      issues every tcgen05.mma (the whole warp runs the loop, one lane chosen by
//               elect.sync issues): S_g = Q_g·K_j^T (SMEM x SMEM -> TMEM) and O_g += P_g·V_j
//               (P from TMEM, V from SMEM), and signals through tcgen05.commit.
//   warps 0-3   softmax of query tile 0, warps 4-7 softmax of query tile 1: one thread per row
//               (= one TMEM lane). They read S from TMEM, apply the mask on tiles that straddle
//               its boundary, update m/l, rescale O in TMEM when m grows, and write P (bf16)
//               back over S.
//   The two query tiles alternate, so the tensor cores run one tile's MMAs while the other tile's
//   softmax runs. TMEM (512 columns): O_0 | O_1 | S_0 (P_0) | S_1 (P_1), 128 columns each.
//   FP8 variant ("Flash Attention Nedir?" and "Apa itu FlashAttention": FlashAttention-3 runs the
//   same method in FP8 on Hopper): Q, K, V are E4M3 with one dequantisation factor per tensor;
//   both products run as kind::f8f6f4 MMAs (32 keys or features per instruction), S is scaled by
//   scale·q_descale·k_descale, P is rounded to E4M3 (values up to 2^8 under the lazy rescale,
//   within E4M3's range of 448) and O is multiplied by v_descale in the epilogue. An E4M3 tile with
//   d = 128 has the byte layout of a bf16 tile with d = 64 (rows of 128 bytes).
//   Masks (causal, sliding window, query/key lengths that differ; see MaskSpec): each query tile
//   visits only the key tiles that hold a key it can see; the two tiles of a pair stream the
//   union of their ranges once. A row that sees no key gets O = 0 and LSE = -inf.
#include <cooperative_groups.h>

#include <atomic>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

constexpr int kFwdThreads = 384;   // 3 warpgroups
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

template <int D, bool F8>
struct FwdCfg {
    static constexpr int EB = F8 ? 1 : 2;                // bytes per element
    static constexpr int BM = 128;                       // query rows per tile
    static constexpr int BN = 128;                       // keys per tile
    static constexpr int CW = D * EB >= 128 ? 128 / EB : D;   // elements per swizzle row
    static constexpr int NCH = D / CW;                   // swizzle chunks per tile row
    static constexpr int SWB = CW * EB;                  // swizzle width in bytes (128 or 64)
    static constexpr uint32_t SWZ = SWB == 128 ? 2u : 4u;
    static constexpr int KSTEP = 32 / EB;                // K elements per MMA instruction
    static constexpr int CHUNK = 128 * SWB;              // bytes of one [128 rows x CW] chunk
    static constexpr int TILE = NCH * CHUNK;             // bytes of one 128 x D tile
    static constexpr int STAGES = TILE >= 32768 ? 2 : 3;
    static constexpr int STAGING = (2 + 2 * STAGES) * TILE;    // Q tiles, K and V rings
    static constexpr int SMEM = STAGING + 512;
    // The split kernels' partials (2 x 128 rows x (D + 4) fp32, then 256 x (m, l)) are written
    // over the staging memory once every copy and MMA of the CTA is complete. bf16 staging always
    // holds them; E4M3 staging (half the bytes) may not, so the split kernels place the barrier
    // block after whichever is larger.
    static constexpr int PARTIALS = (2 * BM * (D + 4) + 2 * 2 * BM) * 4;
    static constexpr int BARS_SPLIT = STAGING > PARTIALS ? STAGING : PARTIALS;
    static constexpr int SMEM_SPLIT = BARS_SPLIT + 512;
    static_assert(F8 || PARTIALS <= STAGING, "bf16 partials fit in the staging memory");
    static_assert(SMEM_SPLIT <= 232448, "dynamic shared memory per block");
    static_assert(SWB == 128 || SWB == 64, "tile rows of 64 or 128 bytes");
};

struct FwdBars {
    uint64_t q_full;
    uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
    uint64_t s_full[2], p_half[2], p_full[2], o_done[2];
    uint64_t teardown;
    uint32_t tmem_base;
    int abort;
};

struct FwdKParams {
    void* o;
    float* lse;
    int BH, n_pairs, group;
    int kv_group;     // query heads per K/V head (grouped-query attention); 1 for MHA
    MaskSpec mask;
    float scale_log2;
    float o_scale;    // output multiplier (v_descale for E4M3 inputs, 1 for bf16)
    uint64_t timeout_ns;
    int split;        // key shares per tile pair (cluster size of the split kernel; else 1)
};

// Every thread of every CTA of the cluster arrives, then waits (release / acquire ordering of
// shared-memory writes across the cluster). Threads of a warp may arrive at different times.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire;\n" ::: "memory");
}

// Bounded wait that ignores the abort flag: used while draining in-flight copies/MMAs on the
// way out, so that nothing is left writing into shared memory or TMEM after the CTA exits.
__device__ __forceinline__ void drain_wait_fwd(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) {
            report_error(4);
            return;
        }
}

// Single-lane commit for a converged warp (see elect_one).
#define FMMA_COMMIT(bar) do { if (elect_one()) mma_commit(bar); } while (0)

// Writes P of columns c, c+1 over the raw scores in u (c even, loop unrolled): bf16 pairs fill
// u[c/2]; E4M3 quadruples fill u[c/4] (columns c, c+1 in the low half when c % 4 == 0). Only
// entries at or below c/2 are written, all already consumed.
template <bool F8>
__device__ __forceinline__ void store_p(uint32_t* u, int c, float p0, float p1) {
    if constexpr (F8) {
        const uint32_t h = pack_e4m3x2(p0, p1);
        if ((c & 2) == 0) u[c / 4] = h;
        else u[c / 4] |= h << 16;
    } else {
        u[c / 2] = pack_bf16x2(p0, p1);
    }
}

// SPLIT: the CTAs of a cluster share the key tiles of one tile pair (small grids); each keeps its
// unnormalised O and (m, l) for its share, and the cluster merges them through distributed
// shared memory with the rule that joins two softmax blocks (weights 2^(m_s - M)).
// ACC: p.o and p.lse are a running fp32 result (o_acc, and lse_acc in natural log) over earlier
// key sets, into which this launch folds its own (acc_first: initialised instead of read); their
// heads start acc_rows rows apart.
template <int D, bool F8, bool SPLIT, bool ACC = false>
__device__ __forceinline__ void fwd_body(const CUtensorMap* tmQ_, const CUtensorMap* tmK_,
                                         const CUtensorMap* tmV_, const FwdKParams& p,
                                         int acc_first = 0, long long acc_rows = 0) {
    using C = FwdCfg<D, F8>;
    static_assert(!(ACC && (F8 || SPLIT)), "accumulating launches: bf16 without key split");
    const CUtensorMap& tmQ = *tmQ_;
    const CUtensorMap& tmK = *tmK_;
    const CUtensorMap& tmV = *tmV_;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sQ = smem;                                   // 2 tiles
    uint8_t* sK = smem + 2 * C::TILE;                     // STAGES tiles
    uint8_t* sV = sK + C::STAGES * C::TILE;               // STAGES tiles
    FwdBars* bars = reinterpret_cast<FwdBars*>(smem + (SPLIT ? C::BARS_SPLIT : C::STAGING));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Heads are processed in groups of p.group (sized so that a group's K and V stay in L2);
    // within a group, tile pairs go from the last to the first (longest first under a causal
    // mask) across the group's heads.
    const int L = SPLIT ? static_cast<int>(blockIdx.x) / p.split : static_cast<int>(blockIdx.x);
    const int gbase = (L / (p.group * p.n_pairs)) * p.group;
    const int gsize = min(p.group, p.BH - gbase);
    const int r_in = L - gbase * p.n_pairs;
    const int pair = p.n_pairs - 1 - r_in / gsize;
    const int bh = gbase + r_in % gsize;
    const int kvbh = bh / p.kv_group;                     // (b, h / g) = (b·H + h) / g
    const MaskSpec& mk = p.mask;
    const int nq = mk.nq;
    // key tiles [J0[g], J0[g] + T[g]) of query tile g; the pair streams [Jmin, Jmin + U) once
    int J0[2], T[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const long long a = static_cast<long long>(2 * pair + g) * C::BM;
        J0[g] = 0;
        T[g] = 0;
        if (a < nq) {
            long long lo, hi;
            visible_keys(mk, a, min(a + C::BM - 1, static_cast<long long>(nq - 1)), lo, hi);
            if (lo <= hi) {
                J0[g] = static_cast<int>(lo / C::BN);
                T[g] = static_cast<int>(hi / C::BN) + 1 - J0[g];
            }
        }
    }
    if constexpr (SPLIT) {
        // this CTA's share (its rank in the cluster) of each tile's key tiles
        const int rank = static_cast<int>(blockIdx.x) % p.split;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int a0 = T[g] * rank / p.split, a1 = T[g] * (rank + 1) / p.split;
            J0[g] += a0;
            T[g] = a1 - a0;
        }
    }
    const int Jmin = T[0] > 0 ? (T[1] > 0 ? min(J0[0], J0[1]) : J0[0]) : J0[1];
    const int U = (T[0] > 0 || T[1] > 0)
                      ? max(T[0] > 0 ? J0[0] + T[0] : 0, T[1] > 0 ? J0[1] + T[1] : 0) - Jmin
                      : 0;

    if (threadIdx.x == 0) {
        if ((smem_addr(smem) & 1023u) != 0) report_error(3);
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(&bars->s_full[g], 1);
            mbar_init(&bars->p_half[g], 128);
            mbar_init(&bars->p_full[g], 128);
            mbar_init(&bars->o_done[g], 1);
        }
        mbar_init(&bars->teardown, 1);
        bars->abort = ((smem_addr(smem) & 1023u) != 0) ? 1 : 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 9) tmem_alloc(&bars->tmem_base, 512);
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int* abort = &bars->abort;
    const uint64_t lim = p.timeout_ns;

    if (warp >= 8) {
    // The producer warpgroup (loader, MMA issuer, two idle warps) hands most of its registers
    // to the softmax warpgroups: 2·128·208 + 128·80 = 63488 <= 384·168, the launch allocation.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && !*abort && U > 0) {
            uint32_t qbytes = (T[0] > 0 ? C::TILE : 0) + (T[1] > 0 ? C::TILE : 0);
            mbar_arrive_expect_tx(&bars->q_full, qbytes);
            for (int g = 0; g < 2; ++g)
                if (T[g] > 0)
                    for (int ch = 0; ch < C::NCH; ++ch)
                        tma_load_3d(sQ + g * C::TILE + ch * C::CHUNK, &tmQ, &bars->q_full,
                                    ch * C::CW, (2 * pair + g) * C::BM, bh);
            int issued = 0;
            for (int u = 0; u < U; ++u) {
                const int s = u % C::STAGES;
                const int f = u / C::STAGES;
                const int krow = (Jmin + u) * C::BN;
                if (f > 0 && !bounded_wait(&bars->k_empty[s], (f - 1) & 1, abort, lim)) break;
                mbar_arrive_expect_tx(&bars->k_full[s], C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch)
                    tma_load_3d(sK + s * C::TILE + ch * C::CHUNK, &tmK, &bars->k_full[s],
                                ch * C::CW, krow, kvbh);
                issued = 2 * u + 1;
                if (f > 0 && !bounded_wait(&bars->v_empty[s], (f - 1) & 1, abort, lim)) break;
                mbar_arrive_expect_tx(&bars->v_full[s], C::TILE);
                for (int ch = 0; ch < C::NCH; ++ch)
                    tma_load_3d(sV + s * C::TILE + ch * C::CHUNK, &tmV, &bars->v_full[s],
                                ch * C::CW, krow, kvbh);
                issued = 2 * u + 2;
            }
            if (*abort) {
                // let every copy issued so far land before the CTA can exit
                drain_wait_fwd(&bars->q_full, 0, 100000000ull);
                for (int x = 0; x < issued; ++x) {
                    const int u = x >> 1;
                    const int s = u % C::STAGES;
                    drain_wait_fwd((x & 1) ? &bars->v_full[s] : &bars->k_full[s],
                               (u / C::STAGES) & 1, 100000000ull);
                }
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        // The whole warp runs this loop (warp-uniform state) and waits together; one elected
        // lane issues each batch of MMAs with its commit. (A vote per instruction would cost the
        // issuing warp ~100 cycles per tcgen05.mma, more than the tensor pipe needs for one.)
        {
            constexpr uint32_t idS = F8 ? idesc_e4m3_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idPV = F8 ? idesc_e4m3_f32(128, D, 0, 1) : idesc_bf16_f32(128, D, 0, 1);
            // issue helpers: called by the elected lane only
            auto mss = [](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
                if constexpr (F8) mma_ss_f8(d, a, b, id, acc);
                else mma_ss(d, a, b, id, acc);
            };
            auto mts = [](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
                if constexpr (F8) mma_ts_f8(d, a, b, id, acc);
                else mma_ts(d, a, b, id, acc);
            };
            const uint32_t sQa = smem_addr(sQ), sKa = smem_addr(sK), sVa = smem_addr(sV);
            bool ok = U > 0 && bounded_wait_warp(&bars->q_full, 0, abort, lim);
            tc_fence_after();
            int k_ready = -1;
            auto wait_k = [&](int u) -> bool {     // u: index in the pair's key-tile stream
                if (k_ready >= u) return true;
                if (!bounded_wait_warp(&bars->k_full[u % C::STAGES], (u / C::STAGES) & 1, abort,
                                  lim))
                    return false;
                tc_fence_after();
                k_ready = u;
                return true;
            };
            // Lean issue path: descriptors per operand tile computed once, each k-step adds a
            // constant to the low word, loops fully unrolled. The issuing lane shares its SM
            // sub-partition with two busy softmax warps, so every instruction here costs.
            // (tile offsets are added to the start-address field: no descriptor arrays, so no
            // local-memory indexing on the issue path)
            const SDesc dQ0 = sdesc(sQa, 16, 8 * C::SWB, C::SWZ);
            const SDesc dK0 = sdesc(sKa, 16, 8 * C::SWB, C::SWZ);
            const SDesc dV0 = sdesc(sVa, C::CHUNK, 8 * C::SWB, C::SWZ);
            auto tile_of = [](SDesc d, int idx) {
                return SDesc{d.lo + static_cast<uint32_t>(idx) * (C::TILE >> 4), d.hi};
            };
            auto issue_s = [&](int g, int u) {
                const SDesc a = tile_of(dQ0, g), b = tile_of(dK0, u % C::STAGES);
                const uint32_t d = tmem + 256 + g * 128;
#pragma unroll
                for (int ks = 0; ks < D / C::KSTEP; ++ks) {
                    const uint32_t off = static_cast<uint32_t>(
                        (((ks * C::KSTEP) / C::CW) * C::CHUNK + ((ks * C::KSTEP) % C::CW) * C::EB) >> 4);
                    mss(d, sdesc_at(a, off), sdesc_at(b, off), idS, ks > 0 ? 1u : 0u);
                }
            };
            // O += P·V over keys [64·half, 64·half + 64) of the tile
            auto issue_pv = [&](int g, int u, int half, bool accumulate) {
                const SDesc b = tile_of(dV0, u % C::STAGES);
                const uint32_t d = tmem + g * 128, a = tmem + 256 + g * 128;
                constexpr int KH = C::BN / C::KSTEP / 2;   // instructions per half
                // one instruction takes KSTEP keys: 8 TMEM columns of P, KSTEP rows of V
#pragma unroll
                for (int ks = half * KH; ks < half * KH + KH; ++ks)
                    mts(d, a + ks * 8,
                        sdesc_at(b, static_cast<uint32_t>((ks * C::KSTEP * C::SWB) >> 4)), idPV,
                        (accumulate || ks > 0) ? 1u : 0u);
            };
            // Stream step u holds key tile Jmin + u. Query tile g uses steps [J0[g] - Jmin,
            // J0[g] - Jmin + T[g]); its S for step u+1 is issued during step u (or, for its first
            // tile, before the loop / at the end of step u), so every S reading K tile u+1 is
            // issued before k_empty of that tile is committed.
            const int s0[2] = {J0[0] - Jmin, J0[1] - Jmin};
            auto active = [&](int g, int u) { return T[g] > 0 && u >= s0[g] && u < s0[g] + T[g]; };
            if (ok) ok = wait_k(0);
            if (ok) {
                if (elect_one()) {
                    for (int g = 0; g < 2; ++g)
                        if (T[g] > 0 && s0[g] == 0) {
                            issue_s(g, 0);
                            mma_commit(&bars->s_full[g]);
                        }
                    mma_commit(&bars->k_empty[0]);
                }
                __syncwarp();
            }
            for (int u = 0; ok && u < U; ++u) {
                bool v_ready = false;
                auto wait_v = [&]() -> bool {
                    if (v_ready) return true;
                    if (!bounded_wait_warp(&bars->v_full[u % C::STAGES], (u / C::STAGES) & 1,
                                           abort, lim))
                        return false;
                    tc_fence_after();
                    v_ready = true;
                    return true;
                };
                for (int g = 0; g < 2 && ok; ++g) {
                    if (!active(g, u)) continue;
                    const int t = u - s0[g];
                    // the softmax hands over P in two halves of 64 keys: the first half's P·V
                    // runs while the second half's exponentials are computed
                    if (!bounded_wait_warp(&bars->p_half[g], t & 1, abort, lim)) { ok = false; break; }
                    tc_fence_after();
                    if (!wait_v()) { ok = false; break; }
                    if (elect_one()) issue_pv(g, u, 0, t > 0);
                    __syncwarp();
                    if (!bounded_wait_warp(&bars->p_full[g], t & 1, abort, lim)) { ok = false; break; }
                    tc_fence_after();
                    const bool more = t + 1 < T[g];
                    if (elect_one()) {
                        issue_pv(g, u, 1, true);
                        if (!more) mma_commit(&bars->o_done[g]);
                    }
                    __syncwarp();
                    if (more) {
                        if (!wait_k(u + 1)) { ok = false; break; }
                        if (elect_one()) {
                            issue_s(g, u + 1);
                            mma_commit(&bars->s_full[g]);
                        }
                        __syncwarp();
                    }
                }
                if (!ok) break;
                if (u + 1 < U) {
                    for (int g = 0; g < 2 && ok; ++g)
                        if (T[g] > 0 && s0[g] == u + 1) {      // first tile of g is the next one
                            if (!wait_k(u + 1)) { ok = false; break; }
                            if (elect_one()) {
                                issue_s(g, u + 1);
                                mma_commit(&bars->s_full[g]);
                            }
                            __syncwarp();
                        }
                    if (!ok || !(ok = wait_k(u + 1))) break;
                }
                if (!(ok = wait_v())) break;     // every loaded V tile is consumed before reuse
                FMMA_COMMIT(&bars->v_empty[u % C::STAGES]);
                if (u + 1 < U) FMMA_COMMIT(&bars->k_empty[(u + 1) % C::STAGES]);
            }
            // all MMAs of this CTA complete before TMEM is released
            FMMA_COMMIT(&bars->teardown);
            drain_wait_fwd(&bars->teardown, 0, 100000000ull);
        }
        __syncwarp();
    }
    if constexpr (SPLIT) {   // the producer warpgroup takes part in the two cluster barriers
        cluster_sync_all();
        cluster_sync_all();
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 208;");
        // ---------------------------------------------------------------- softmax warpgroups
        const int g = warp >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;                     // row within the tile = TMEM lane
        const int qt = 2 * pair + g;
        const int qidx = qt * C::BM + r;
        const long long a = static_cast<long long>(qt) * C::BM;
        // visible keys of this row: [klo, khi]
        long long klo_l, khi_l;
        visible_keys(mk, qidx, qidx, klo_l, khi_l);
        const int klo = clamp_int(klo_l), khi = clamp_int(khi_l);
        // keys seen by every row of the tile: [flo, fhi] (the last row's lower bound, the first
        // row's upper bound); a key tile starting at kb needs no mask iff flo <= kb, kb+127 <= fhi
        long long flo, fhi;
        visible_keys(mk, a + C::BM - 1, a, flo, fhi);
        const int full_lo = clamp_int(flo);
        const int full_hi = clamp_int(fhi - (C::BN - 1));
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + 256 + g * 128;
        const uint32_t tO = tmem + lane_base + g * 128;
        const float sl2 = p.scale_log2;
        float m = -INFINITY;   // running max of scale*log2(e)*s
        float l = 0.f;         // running sum of exp2(.. - m)
        bool ok = true;
        for (int t = 0; t < T[g]; ++t) {
            const int jj = J0[g] + t;
            ok = bounded_wait(&bars->s_full[g], t & 1, abort, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            // S row of this tile: four 32-column loads, one wait
            uint32_t u[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
            tmem_ld_wait();
            reg_fence<128>(u);
            const int kbase = jj * C::BN;
            const bool edge = kbase < full_lo || kbase > full_hi;
            if (edge) {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    const int kidx = kbase + c;
                    if (kidx < klo || kidx > khi) u[c] = __float_as_uint(-INFINITY);
                }
            }
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
                mx0 = fmax3(mx0, __uint_as_float(u[c]), __uint_as_float(u[c + 1]));
                mx1 = fmax3(mx1, __uint_as_float(u[c + 2]), __uint_as_float(u[c + 3]));
                mx2 = fmax3(mx2, __uint_as_float(u[c + 4]), __uint_as_float(u[c + 5]));
                mx3 = fmax3(mx3, __uint_as_float(u[c + 6]), __uint_as_float(u[c + 7]));
            }
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
            // Lazy rescaling: the reference max m only moves when the tile max exceeds it by more
            // than 8 (a factor 2^8 on P); otherwise P = exp2(s·c - m) is simply allowed to exceed
            // 1. The final O/l and LSE = m + log2 l use the same m, so the result is unchanged.
            if (t == 0) {
                m = m_tile;
            } else if (__any_sync(0xffffffffu, m_tile > m + 8.f)) {
                float alpha = 1.f;
                if (m_tile > m + 8.f) {
                    alpha = ex2_approx(m - m_tile);
                    m = m_tile;
                    l *= alpha;
                }
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_ld_wait();
                    reg_fence<32>(o);
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                    tmem_st32(tO + c * 32, o);
                }
            }
            const float m_use = (m == -INFINITY) ? 0.f : m;
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            const uint64_t nm2 = f2_pack(-m_use, -m_use);
            uint64_t rsa = f2_pack(0.f, 0.f), rsb = f2_pack(0.f, 0.f);
            // P = exp2(s·c - m) on the MUFU (masked -inf scores give exact zeros), two row-sum
            // accumulators to shorten the add chain. P goes to TMEM in two halves of 64 keys
            // (32 columns of bf16 pairs or 16 of E4M3 quadruples each), the first signalled as
            // soon as it is stored so that its P·V overlaps the second half's exponentials.
            constexpr int PW = F8 ? 16 : 32;                // P words per half
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int c = 64 * hh; c < 64 * hh + 64; c += 2) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(u[c]), __uint_as_float(u[c + 1])),
                                     sl2x2, nm2), x0, x1);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    if (c & 2) rsb = f2_add(rsb, f2_pack(p0, p1));
                    else rsa = f2_add(rsa, f2_pack(p0, p1));
                    store_p<F8>(u, c, p0, p1);
                }
                if constexpr (F8)
                    tmem_st16(tS + hh * PW, *reinterpret_cast<uint32_t(*)[16]>(&u[hh * PW]));
                else
                    tmem_st32(tS + hh * PW, *reinterpret_cast<uint32_t(*)[32]>(&u[hh * PW]));
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(hh == 0 ? &bars->p_half[g] : &bars->p_full[g]);
            }
            float ra0, ra1, rb0, rb1;
            f2_unpack(rsa, ra0, ra1);
            f2_unpack(rsb, rb0, rb1);
            const float rs0 = ra0 + rb0, rs1 = ra1 + rb1;
            l += rs0 + rs1;
        }
        if constexpr (SPLIT) {
            // Partial of this share: unnormalised O (fp32, rows padded to D + 4 floats) and
            // (m, l) per row, written over the Q/K/V staging memory once both tiles' MMAs are
            // complete; a row with no key in this share has m = -inf, l = 0.
            bool have = ok && T[g] > 0;
            if (have) {
                have = bounded_wait(&bars->o_done[g], 0, abort, lim);
                have = __all_sync(0xffffffffu, have);
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");   // both softmax warpgroups
            tc_fence_after();
            constexpr int OP = D + 4;
            float* Ob = reinterpret_cast<float*>(smem);
            float* ML = Ob + 2 * C::BM * OP;
            const int row = g * C::BM + r;
            if (have) {
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + c * 32, u);
                    tmem_ld_wait();
                    float4* dst = reinterpret_cast<float4*>(Ob + row * OP + c * 32);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        dst[x] = make_float4(__uint_as_float(u[4 * x]), __uint_as_float(u[4 * x + 1]),
                                             __uint_as_float(u[4 * x + 2]),
                                             __uint_as_float(u[4 * x + 3]));
                }
            }
            ML[2 * row] = have ? m : -INFINITY;
            ML[2 * row + 1] = have ? l : 0.f;
            cluster_sync_all();
            // Merge: this CTA finishes rows [rank*R, rank*R + R) of the pair's 256 rows.
            namespace cg = cooperative_groups;
            cg::cluster_group cluster = cg::this_cluster();
            const int split = p.split;
            const int rank = static_cast<int>(blockIdx.x) % split;
            const int R = 2 * C::BM / split;
            constexpr int C4 = D / 4;
            for (int idx = static_cast<int>(threadIdx.x); idx < R * C4; idx += 256) {
                const int rw = rank * R + idx / C4, c4 = idx % C4;
                const int qi = (2 * pair + rw / C::BM) * C::BM + rw % C::BM;
                if (qi >= nq) continue;
                float M = -INFINITY;
                for (int s2 = 0; s2 < split; ++s2)
                    M = fmaxf(M, cluster.map_shared_rank(ML, s2)[2 * rw]);
                float Lsum = 0.f;
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int s2 = 0; s2 < split; ++s2) {
                    const float* mls = cluster.map_shared_rank(ML, s2);
                    const float ms = mls[2 * rw];
                    if (ms == -INFINITY) continue;
                    const float w = ex2_approx(ms - M);
                    Lsum = fmaf(w, mls[2 * rw + 1], Lsum);
                    const float4 t = *reinterpret_cast<const float4*>(
                        cluster.map_shared_rank(Ob, s2) + rw * OP + c4 * 4);
                    o.x = fmaf(w, t.x, o.x);
                    o.y = fmaf(w, t.y, o.y);
                    o.z = fmaf(w, t.z, o.z);
                    o.w = fmaf(w, t.w, o.w);
                }
                const float inv = Lsum > 0.f ? p.o_scale / Lsum : 0.f;
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                                      (static_cast<size_t>(bh) * nq + qi) * D;
                *reinterpret_cast<uint2*>(orow + c4 * 4) =
                    make_uint2(pack_bf16x2(o.x * inv, o.y * inv), pack_bf16x2(o.z * inv, o.w * inv));
                if (c4 == 0)
                    p.lse[static_cast<size_t>(bh) * nq + qi] =
                        Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
            }
            cluster_sync_all();   // peers may still be reading this CTA's shared memory
        } else if constexpr (ACC) {
            // Fold this launch's rows into the running result: with la the running LSE and lb
            // this launch's (natural log, -inf where no key was seen), L = log(e^la + e^lb),
            // o_acc = e^(la-L)·o_acc + e^(lb-L)·O/l, lse_acc = L; acc_first: la = -inf.
            const size_t arow = static_cast<size_t>(bh) * acc_rows + qidx;
            float* oacc = static_cast<float*>(p.o) + arow * D;
            const bool row = qidx < nq;
            float a[D];                                 // running row, loaded before O is ready
            if (row && !acc_first) {
#pragma unroll
                for (int x = 0; x < D / 4; ++x) {
                    const float4 t = reinterpret_cast<const float4*>(oacc)[x];
                    a[4 * x] = t.x; a[4 * x + 1] = t.y; a[4 * x + 2] = t.z; a[4 * x + 3] = t.w;
                }
            }
            const bool have = ok && T[g] > 0;
            if (have) {
                ok = bounded_wait(&bars->o_done[g], 0, abort, lim);
                ok = __all_sync(0xffffffffu, ok);
            }
            if (ok && have) tc_fence_after();
            const bool seen = ok && have && l > 0.f;
            const float lb = seen ? (m + __log2f(l)) * kLn2 : -INFINITY;
            const float la = (!row || acc_first) ? -INFINITY : p.lse[arow];
            const float mx = fmaxf(la, lb);
            float L = -INFINITY, wa = 0.f, wb = 0.f;
            if (mx != -INFINITY) {
                const float ea = expf(la - mx), eb = expf(lb - mx);
                L = mx + logf(ea + eb);
                wa = ea / (ea + eb);
                wb = seen ? eb / (ea + eb) / l : 0.f;   // includes the 1/l of O/l
            }
            if (ok && (have || acc_first)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    if (have) {
                        tmem_ld32(tO + c * 32, u);
                        tmem_ld_wait();
                    }
                    if (row) {
                        float4* dst = reinterpret_cast<float4*>(oacc + c * 32);
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            float v4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int k = c * 32 + 4 * x + e;
                                const float pa = (wa == 0.f || acc_first) ? 0.f : wa * a[k];
                                const float pb = wb == 0.f ? 0.f : wb * __uint_as_float(u[4 * x + e]);
                                v4[e] = pa + pb;
                            }
                            dst[x] = make_float4(v4[0], v4[1], v4[2], v4[3]);
                        }
                    }
                }
                if (row) p.lse[arow] = L;
            }
        } else if (ok && T[g] > 0) {
            ok = bounded_wait(&bars->o_done[g], 0, abort, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                // a row that saw no key has l = 0 and an all-zero accumulator
                const float inv_l = l > 0.f ? p.o_scale / l : 0.f;
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                                      (static_cast<size_t>(bh) * nq + qidx) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + c * 32, u);
                    tmem_ld_wait();
                    uint32_t w[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        w[x] = pack_bf16x2(__uint_as_float(u[2 * x]) * inv_l,
                                           __uint_as_float(u[2 * x + 1]) * inv_l);
                    if (qidx < nq) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
                    }
                }
                if (qidx < nq)
                    p.lse[static_cast<size_t>(bh) * nq + qidx] =
                        l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
            }
        } else if (ok && T[g] == 0 && qidx < nq) {
            // the whole tile sees no key: O = 0, LSE = -inf
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.o) +
                                                  (static_cast<size_t>(bh) * nq + qidx) * D);
#pragma unroll
            for (int x = 0; x < D / 8; ++x) dst[x] = make_uint4(0u, 0u, 0u, 0u);
            p.lse[static_cast<size_t>(bh) * nq + qidx] = -INFINITY;
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
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdKParams p) {
    fwd_body<D, false, false>(&tmQ, &tmK, &tmV, p);
}

// Folds its result into a running fp32 (o_acc, lse_acc) over earlier key sets (see fwd_body).
struct FwdAccP {
    int first;
    long long rows;   // rows between consecutive heads of o_acc and lse_acc
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_bf16_acc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const FwdKParams p,
                        const FwdAccP acc) {
    fwd_body<D, false, false, true>(&tmQ, &tmK, &tmV, p, acc.first, acc.rows);
}

// Small grids: launched in clusters of p.split CTAs that share each tile pair's key tiles.
template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_bf16_split_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const FwdKParams p) {
    fwd_body<D, false, true>(&tmQ, &tmK, &tmV, p);
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdKParams p) {
    fwd_body<D, true, false>(&tmQ, &tmK, &tmV, p);
}

// E4M3 inputs on small grids: clusters of p.split CTAs as fwd_bf16_split_kernel.
template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_fp8_split_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const FwdKParams p) {
    fwd_body<D, true, true>(&tmQ, &tmK, &tmV, p);
}

// The split kernel of an input type.
template <int D, bool F8>
constexpr auto split_kernel() {
    if constexpr (F8) return fwd_fp8_split_kernel<D>;
    else return fwd_bf16_split_kernel<D>;
}

// Clusters of `split` CTAs of a split kernel that the GPU holds at once (each CTA takes a whole
// SM, and a cluster must fit in one GPC); queried once per (device, d, split) and kept in a
// per-device table of atomics, so concurrent host threads and GPUs of different layouts each see
// their own device's answer. While `stream` is being captured into a graph the query is not made
// and half of SMs / split is assumed.
constexpr int kClusterCacheDevices = 64;

template <int D, bool F8>
int max_active_clusters(int split, int sms, cudaStream_t stream) {
    static std::atomic<int> cache[kClusterCacheDevices][4];
    const int slot = split == 2 ? 0 : split == 4 ? 1 : split == 8 ? 2 : 3;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    std::atomic<int>* entry =
        (dev >= 0 && dev < kClusterCacheDevices) ? &cache[dev][slot] : nullptr;
    if (entry) {
        const int known = entry->load(std::memory_order_relaxed);
        if (known > 0) return known;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        (void)cudaGetLastError();
        return sms / (2 * split);
    }
    if (cap != cudaStreamCaptureStatusNone) return sms / (2 * split);
    using C = FwdCfg<D, F8>;
    constexpr auto kern = split_kernel<D, F8>();
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_SPLIT) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(split * 256));
    cfg.blockDim = dim3(kFwdThreads);
    cfg.dynamicSmemBytes = C::SMEM_SPLIT;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    if (entry) entry->store(n, std::memory_order_relaxed);
    return n;
}

// Key shares per tile pair for the forward: 1 when the pairs alone fill half the SMs, else the
// largest power of two (at most 8, at most the largest number of key tiles a query tile sees)
// that keeps the grid within one CTA per SM and every cluster resident at once.
template <int D, bool F8>
int choose_fwd_split(const MaskSpec& mk, int qtiles, long long pairs_total, cudaStream_t stream) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
    if (pairs_total * 2 > sms) return 1;
    int max_tiles = 0;
    for (int t = 0; t < qtiles; ++t) {
        long long lo, hi;
        const long long a = static_cast<long long>(t) * 128;
        visible_keys(mk, a, a + 127 < mk.nq - 1 ? a + 127 : mk.nq - 1, lo, hi);
        if (lo <= hi) {
            const int c = static_cast<int>(hi / 128 - lo / 128 + 1);
            if (c > max_tiles) max_tiles = c;
        }
    }
    int s = 1;
    while (s < 8 && pairs_total * s * 2 <= sms && s * 2 <= max_tiles &&
           pairs_total <= max_active_clusters<D, F8>(s * 2, sms, stream))
        s *= 2;
    return s;
}

template <int D, bool F8>
cudaError_t launch_fwd_d(const FwdArgs& a, cudaStream_t stream) {
    using C = FwdCfg<D, F8>;
    CUtensorMap mq, mk, mv;
    const int BH = a.B * a.H;
    const int esize = F8 ? 1 : 2;
    cudaError_t e;
    if ((e = make_tmap(&mq, a.q, esize, BH, a.nq, D, 128, a.q_rows)) != cudaSuccess) return e;
    const int BHkv = a.B * a.Hkv;
    if ((e = make_tmap(&mk, a.k, esize, BHkv, a.nk, D, 128, a.kv_rows)) != cudaSuccess) return e;
    if ((e = make_tmap(&mv, a.v, esize, BHkv, a.nk, D, 128, a.kv_rows)) != cudaSuccess) return e;
    void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const FwdKParams);
    if constexpr (F8) kern = fwd_fp8_kernel<D>;
    else kern = fwd_bf16_kernel<D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    FwdKParams kp;
    kp.o = a.o;
    kp.lse = a.lse;
    kp.BH = BH;
    const int qtiles = (a.nq + 127) / 128;
    kp.n_pairs = (qtiles + 1) / 2;
    kp.mask = MaskSpec{a.nq, a.nk, a.wl, a.wr, static_cast<long long>(a.nk) - a.nq};
    kp.kv_group = a.H / a.Hkv;
    // heads per group: K and V of one head take 4·nk·d bytes; keep a group's within ~32 MB of L2
    {
        const long long per_head = 4LL * a.nk * D;
        long long g = (32LL << 20) / (per_head > 0 ? per_head : 1);
        kp.group = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
    }
    kp.scale_log2 = a.scale * kLog2e * (F8 ? a.q_descale * a.k_descale : 1.f);
    kp.o_scale = F8 ? a.v_descale : 1.f;
    kp.timeout_ns = a.timeout_ns;
    const long long pairs_total = static_cast<long long>(kp.n_pairs) * BH;
    if constexpr (!F8) {
        if (a.acc_first >= 0) {      // accumulating launch: one CTA per tile pair
            kp.split = 1;
            if (pairs_total > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
            constexpr auto akern = fwd_bf16_acc_kernel<D>;
            e = cudaFuncSetAttribute(akern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
            if (e != cudaSuccess) return e;
            const FwdAccP acc{a.acc_first, a.q_rows > 0 ? a.q_rows : a.nq};
            akern<<<static_cast<unsigned>(pairs_total), kFwdThreads, C::SMEM, stream>>>(
                mq, mk, mv, kp, acc);
            return cudaGetLastError();
        }
    }
    kp.split = choose_fwd_split<D, F8>(kp.mask, qtiles, pairs_total, stream);
    const long long grid = pairs_total * kp.split;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (kp.split == 1) {
        kern<<<static_cast<unsigned>(grid), kFwdThreads, C::SMEM, stream>>>(mq, mk, mv, kp);
        return cudaGetLastError();
    }
    constexpr auto skern = split_kernel<D, F8>();
    e = cudaFuncSetAttribute(skern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_SPLIT);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kFwdThreads);
    cfg.dynamicSmemBytes = C::SMEM_SPLIT;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(kp.split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, skern, mq, mk, mv, kp);
}

}  // namespace

cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t stream) {
    switch (a.d) {
        case 32: return launch_fwd_d<32, false>(a, stream);
        case 64: return launch_fwd_d<64, false>(a, stream);
        case 128: return launch_fwd_d<128, false>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_fwd_fp8(const FwdArgs& a, cudaStream_t stream) {
    switch (a.d) {
        case 64: return launch_fwd_d<64, true>(a, stream);
        case 128: return launch_fwd_d<128, true>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
