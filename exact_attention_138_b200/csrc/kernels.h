// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace attn {

// Which keys each query sees. Query i (of nq) is aligned with key i + off, off = nk - nq (the last
// query with the last key); key j is visible iff  i + off - wl <= j <= i + off + wr, a negative
// wl or wr meaning unbounded on that side. (wl, wr) = (-1, 0) with nq = nk is the causal mask,
// (-1, -1) no mask, (w, w) the sliding window of "Attention Mechanism ...", §4.5.
// Because both bounds grow with i, the keys seen by a block of consecutive queries form one
// contiguous range, and the queries that see a block of keys do too; host and device derive the
// tile ranges of both passes from the functions below, so the passes agree on which (query tile,
// key tile) pairs meet.
struct MaskSpec {
    int nq, nk;
    int wl, wr;
    long long off;
};

__host__ __device__ inline long long floor_div(long long a, long long b) {
    return a >= 0 ? a / b : -((-a + b - 1) / b);
}

// Keys [lo, hi] (clipped to [0, nk)) seen by some query in rows [a, b] (b < nq); lo > hi if none.
__host__ __device__ inline void visible_keys(const MaskSpec& m, long long a, long long b,
                                             long long& lo, long long& hi) {
    lo = m.wl < 0 ? 0 : a + m.off - m.wl;
    hi = m.wr < 0 ? m.nk - 1 : b + m.off + m.wr;
    if (lo < 0) lo = 0;
    if (hi > m.nk - 1) hi = m.nk - 1;
}

// Query tiles [i0, i1) of `bq` rows that meet keys [c, e] (e < nk); i0 >= i1 if none.
__host__ __device__ inline void visible_query_tiles(const MaskSpec& m, long long c, long long e,
                                                    int bq, int& i0, int& i1) {
    const long long ntiles = (m.nq + bq - 1) / bq;
    long long t0 = 0, t1 = ntiles;
    if (m.wr >= 0) {
        const long long x = c - m.off - m.wr;   // first query whose window reaches key c
        if (x > m.nq - 1) t0 = ntiles;
        else if (x > 0) t0 = x / bq;
    }
    if (m.wl >= 0) {
        const long long y = e - m.off + m.wl;   // last query whose window reaches back to key e
        if (y < 0) t1 = 0;
        else if (y / bq + 1 < t1) t1 = y / bq + 1;
    }
    i0 = static_cast<int>(t0);
    i1 = static_cast<int>(t1 > t0 ? t1 : t0);
}

// First key tile of `bk` keys met by the query tile starting at row a.
__host__ __device__ inline int first_key_tile(const MaskSpec& m, long long a, int bk) {
    if (m.wl < 0) return 0;
    const long long lo = a + m.off - m.wl;
    return lo <= 0 ? 0 : static_cast<int>(lo / bk);
}

// Last key tile of `bk` keys met by the query tile of rows [a, a + bq) (clipped to nq); only
// meaningful when the tile meets some key.
__host__ __device__ inline int last_key_tile(const MaskSpec& m, long long a, int bq, int bk) {
    long long lo, hi;
    const long long b = a + bq - 1 < m.nq - 1 ? a + bq - 1 : m.nq - 1;
    visible_keys(m, a, b, lo, hi);
    return hi < 0 ? 0 : static_cast<int>(hi / bk);
}

__host__ __device__ inline int clamp_int(long long x) {
    return x < -0x7fffffffLL ? -0x7fffffff : (x > 0x7fffffffLL ? 0x7fffffff : static_cast<int>(x));
}

struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    int B, H, nq, nk, d;  // query rows, key rows
    int Hkv;          // K/V heads; query head h reads K/V head h / (H / Hkv)
    float scale;
    int wl, wr;       // visible window (see MaskSpec)
    float q_descale, k_descale, v_descale;   // E4M3 inputs only: real value = stored · descale
    uint64_t timeout_ns;
    // >= 0: o and lse are a running fp32 result (o_acc, lse_acc) that the launch folds its own
    // into (bf16 inputs); 1: the first such launch (initialise, do not read)
    int acc_first = -1;
    // rows between consecutive heads of q (and, accumulating, of o_acc / lse_acc) and of k, v;
    // 0: nq / nk (packed)
    long long q_rows = 0, kv_rows = 0;
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
    int B, H, nq, nk, d;  // query rows, key rows
    int Hkv;          // K/V heads (dk, dv have Hkv heads)
    float scale;
    int wl, wr;       // visible window (see MaskSpec)
    int deterministic;
    // n_pad = nq rounded up to a multiple of 128
    float* Dvec;      // workspace: B*H*n_pad, D_i = rowsum(dO∘O) (0 on padding rows)
    float* L2vec;     // workspace: B*H*n_pad, LSE_i·log2(e) (+inf on padding rows and on rows
                      // that see no key)
    float* dq_acc;    // workspace: B*H*n_pad*d
    int* sems;        // workspace: B*H*(n_pad/64)*4, deterministic mode only
    uint64_t timeout_ns;
    const cudaEvent_t* phase_events;   // 4 events or nullptr (measurement hook)
    // Kernels to run: 1 the preprocess (D, LSE·log2 e, zeroed dQ accumulator and semaphores),
    // 2 the main kernel, 4 the dQ conversion. With dk_acc32 / dv_acc32 set, the main kernel adds
    // dK and dV (fp32, (B, Hkv, nk, d)) into them instead of writing dk, dv.
    int phases = 7;
    float* dk_acc32 = nullptr;
    float* dv_acc32 = nullptr;
    // Views (main kernel only): rows between consecutive heads of q, dO and of k, v, dk_acc32,
    // dv_acc32 (0: nq / nk); the workspace holds ws_rows query rows per head (0: nq) and this
    // launch's queries are its rows [q_row0, q_row0 + nq) (q_row0 a multiple of 64).
    long long q_rows = 0, kv_rows = 0;
    int ws_rows = 0, q_row0 = 0;
};

// Encodes a 3-D tensor map over a (B*H, n, d) tensor of `esize`-byte elements (2: bf16, 1: 8-bit)
// with a box of (chunk, box_rows, 1), chunk = min(d, 128 / esize) elements, and the swizzle that
// matches the chunk's bytes (128: 128-byte, 64: 64-byte). Consecutive heads start head_rows rows
// apart (0: n, packed; a view of rows of a longer sequence otherwise).
cudaError_t make_tmap(CUtensorMap* map, const void* base, int esize, int BH, int n, int d,
                      int box_rows = 128, long long head_rows = 0);
inline cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int BH, int n, int d,
                                  int box_rows = 128, long long head_rows = 0) {
    return make_tmap(map, base, 2, BH, n, d, box_rows, head_rows);
}

// Encodes a 2-D tensor map over the fp32 dQ accumulator: `rows` rows of `d` fp32 values, box of
// 32 rows x 32 columns, no swizzle (the backward's drain adds [32 queries][32 columns] boxes).
cudaError_t make_tmap_acc(CUtensorMap* map, float* base, long long rows, int d);

cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_fwd_fp8(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint64_t timeout_ns, cudaStream_t stream);

}  // namespace attn
