/*
 * attn.h — C ABI of libattn.so: exact scaled dot-product attention on one NVIDIA B200 (sm_100a).
 *
 * The operation (forward):
 *     O = softmax(scale · Q·K^T + M) · V,     LSE_i = ln sum_j exp(scale · q_i·k_j + M_ij)
 *   "Attention Mechanism: Revolusi Representasi Sequence", §3 "Scaled Dot-Product Attention:
 *   Formula Inti" (Steps 1-4: scores, scaling, row softmax, weighted sum of V rows) and §4.4
 *   "Causal / Masked Attention" (M_ij = 0 for j <= i, -inf for j > i). The row log-sum-exp is the
 *   statistic of "Flash Attention Nedir?", section "Online Softmax"; it is returned in the natural
 *   log so that the backward pass can rebuild P = exp(scale·q·k - LSE) tile by tile ("Apa itu
 *   FlashAttention", "Cara kerja teknik Tiling dan Recomputation", item 2).
 *   Q, K, V tiles are processed on chip with an online softmax, so the n x n score matrix of
 *   "Calculateur de mémoire d'attention" ("La formule") is never written to device memory.
 *
 * The operation (backward), the exact derivative of the forward definition:
 *     P = exp(scale·Q·K^T + M - LSE),  dV = P^T·dO,  dP = dO·V^T,  D_i = sum_c dO_ic·O_ic,
 *     dS = P∘(dP - D),  dQ = scale·dS·K,  dK = scale·dS^T·Q.
 *
 * Layout and ownership (all calls):
 *   - q, k, v, o, dO, dq, dk, dv: caller-owned DEVICE memory, contiguous row-major (B, H, n, d):
 *     element (b, h, i, c) at offset ((b*H + h)*n + i)*d + c. bf16 (ATTN_BF16) or fp32
 *     (ATTN_FP32) elements. Base addresses must be 16-byte aligned (TMA requirement).
 *   - lse: caller-owned DEVICE memory, fp32, (B, H, n), 16-byte aligned.
 *   - attn_fwd / attn_bwd: query and key lengths are both n; d is the head dimension of Q, K
 *     and V alike. Other lengths, masks and K/V head counts: the *_gqa and *_ex entry points.
 *   - scale: the factor applied to Q·K^T (normally 1/sqrt(d)); any finite positive value.
 *   - stream: a cudaStream_t (NULL = the legacy default stream). Every call is asynchronous on
 *     that stream and allocates nothing; the library's only device memory is the fixed scratch
 *     array of attn_bwd_noalloc (see there). Calls are capturable into CUDA graphs (make one
 *     call outside capture first, so that one-time driver lookups happen there).
 *
 * Errors: each call validates its arguments before launching anything and returns ATTN_OK or
 *   ATTN_ERR_INVALID   null pointer, B, H or n < 1, n > 2^31 - 257, misaligned pointer,
 *                      non-finite or <= 0 scale,
 *                      workspace pointer null or not 256-byte aligned;
 *   ATTN_ERR_UNSUPPORTED  d not in {32, 64, 128}; fp32 backward; an unknown dtype;
 *   ATTN_ERR_WORKSPACE    ws_bytes smaller than attn_bwd_workspace_bytes();
 *   ATTN_ERR_CUDA      a launch or encode error reported by the CUDA runtime / driver;
 *   ATTN_ERR_TIMEOUT   reported by attn_get_device_status(): a device-side wait ran past its
 *                      limit and the kernel returned early (outputs are then undefined).
 */
#ifndef ATTN_H
#define ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ATTN_BF16 = 0, ATTN_FP32 = 1 } attn_dtype;

enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID = 1,
    ATTN_ERR_UNSUPPORTED = 2,
    ATTN_ERR_CUDA = 3,
    ATTN_ERR_TIMEOUT = 4,
    ATTN_ERR_WORKSPACE = 5
};

/* Library ABI version (major*100 + minor). */
int attn_version(void);

/* Forward pass. Writes o (same dtype as q) and lse (fp32).
 *   dtype ATTN_BF16: tcgen05 tensor-core kernel, fp32 accumulation, P rounded to bf16 before P·V,
 *                    O rounded to bf16 (round-to-nearest-even). Small grids (fewer pairs of
 *                    128-row query tiles than half the SMs) split each pair's keys over a cluster
 *                    of 2-8 CTAs merged on chip; one launch, no library memory.
 *   dtype ATTN_FP32: exact fp32 kernel on the FMA pipes (no TF32), for the pages' float32 cases.
 *                    When B*H*ceil(n/64) query tiles would leave the SMs under-filled, each tile's
 *                    keys are split over a thread-block cluster of up to 8 CTAs whose partial
 *                    (max, sum, O) are merged on chip; still one launch and no library memory.
 * causal != 0 applies the mask M of §4.4 (query i sees keys 0..i). */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int n, int d, float scale, int causal, int dtype, void* stream);

/* Grouped-query attention ("Attention Mechanism: Revolusi Representasi Sequence", §12 "GQA vs
 * MQA — KV Cache Optimization"): k and v have Hkv heads, (B, Hkv, n, d); query head h (of H) uses
 * K/V head h / (H / Hkv), exactly as if K and V were expanded with repeat_interleave(H/Hkv, dim=1)
 * (no copy is made). Hkv = H is attn_fwd; Hkv = 1 is multi-query attention. H must be a multiple
 * of Hkv (else ATTN_ERR_INVALID). Everything else as attn_fwd. */
int attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int Hkv, int n, int d, float scale, int causal, int dtype,
                 void* stream);

/* Forward pass over one key set folded into a running result over earlier key sets (ring
 * attention: one call per hop; "Attention Mechanism: Revolusi Representasi Sequence", §16 "Long
 * Context Training", Ring Attention). The launch computes this key set's O_b, LSE_b exactly as
 * attn_fwd_ex (q, k, v bf16; same shapes and masks) and, in the same kernel, combines them with
 * the running o_acc (B, H, nq, d) fp32 and lse_acc (B, H, nq) fp32 (natural log), row by row:
 *     L = log(exp(lse_acc) + exp(LSE_b)),
 *     o_acc = exp(lse_acc - L)·o_acc + exp(LSE_b - L)·O_b,   lse_acc = L,
 * which is exact because each result is normalised by its own exp(LSE) (the rule of
 * attn_ring_merge, without the rounding of O_b to bf16). first != 0: o_acc and lse_acc are not
 * read (they are set to this key set's result). A row that sees no key in any call so far has
 * o_acc = 0, lse_acc = -inf.
 *   Views of longer sequences: the heads of q, o_acc and lse_acc start q_head_rows rows apart and
 *   those of k and v kv_head_rows rows apart (0: nq / nk, the packed layouts); so rows
 *   [r0, r0 + nq) of (B, H, N, d) tensors are passed as the pointers to row r0 with
 *   q_head_rows = N.
 * Errors as attn_fwd_ex; null or misaligned (16-byte) o_acc / lse_acc, or head_rows below the
 * row count -> ATTN_ERR_INVALID. */
int attn_fwd_accumulate(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc,
                        int B, int H, int Hkv, int nq, int nk, int d, long long q_head_rows,
                        long long kv_head_rows, float scale, int window_left, int window_right,
                        int first, void* stream);

/* FP8 forward pass ("Flash Attention Nedir?" and "Apa itu FlashAttention": FlashAttention-3 runs
 * the method in FP8 on Hopper). q, k, v hold E4M3 bytes (OCP FP8 E4M3: 1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, max 448) in the layouts of attn_fwd_ex; the real
 * inputs are q·q_descale, k·k_descale and v·v_descale (one positive, finite factor per tensor).
 * o receives bf16 (B, H, nq, d); lse (B, H, nq) fp32 is the natural-log row statistic of
 * scale·Q·K^T over the visible keys, as for attn_fwd. Masks (window_left, window_right), query /
 * key lengths and K/V head counts as attn_fwd_ex.
 * Both products run on the tensor cores with E4M3 operands and fp32 accumulation; the softmax
 * weights P are rounded to E4M3 before P·V (relative error up to 2^-4 for weights >= 2^-6,
 * absolute error up to 2^-10 below), so the result is not within the bf16 path's tolerance: an
 * element differs from the exact attention of the dequantised inputs by up to 2^-4·max|V| from the
 * normal-range weights, plus 2^-10·max|V|/l per subnormal weight (l >= 1 is the row's sum of
 * weights), plus bf16 output rounding.
 * d must be 64 or 128 (else ATTN_ERR_UNSUPPORTED); other errors as attn_fwd_ex, and a descale that
 * is not positive and finite is ATTN_ERR_INVALID. */
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int Hkv, int nq, int nk, int d, float scale,
                 int window_left, int window_right,
                 float q_descale, float k_descale, float v_descale, void* stream);

/* Bytes of device workspace attn_bwd needs for these sizes: the D vector and the LSE·log2(e)
 * vector (B·H·n fp32 each, padded per head to a multiple of 128 rows) and the fp32 dQ accumulator
 * (B·H·n·d fp32, padded the same way), each rounded up to 256 bytes; with deterministic != 0 also
 * four int semaphores per 64 query rows. */
size_t attn_bwd_workspace_bytes(int B, int H, int n, int d, int deterministic);

/* Masked and cross-length attention. Sliding window: "Attention Mechanism: Revolusi
 * Representasi Sequence", §4.5 "Sparse Attention" (each token attends only to neighbours within
 * ±w); cross-attention: same page, §4.2 (queries from one sequence, keys and values from another,
 * so nq and nk differ).
 *   q, o: (B, H, nq, d); k, v: (B, Hkv, nk, d); lse: (B, H, nq); layouts and dtypes as attn_fwd.
 *   Query i is aligned with key i + (nk - nq) (the last query with the last key). Key j is
 *   visible to query i iff  i + (nk - nq) - window_left <= j <= i + (nk - nq) + window_right;
 *   a negative window_left / window_right means unbounded on that side. So (-1, 0) with nq == nk
 *   is attn_fwd's causal mask, (-1, -1) no mask, (w, w) the page's ±w window, (w, 0) a causal
 *   window of w + 1 keys.
 *   A query that sees no key (possible when nq > nk or with a window that falls outside the keys)
 *   gets o = 0 and lse = -inf.
 * Errors as attn_fwd; nk < 1 is ATTN_ERR_INVALID. */
int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int H, int Hkv, int nq, int nk, int d, float scale,
                int window_left, int window_right, int dtype, void* stream);

/* Backward pass (bf16 only). Inputs q, k, v, o, dO (bf16) and lse (fp32, from attn_fwd with the
 * same scale and causal flag). Writes dq, dk, dv (bf16). The workspace (caller-owned device
 * memory of at least attn_bwd_workspace_bytes() bytes, 256-byte aligned) is overwritten.
 *   deterministic == 0: dQ partial tiles are added to the fp32 accumulator with atomic adds, so
 *                       the rounding order (and the last bits of dq) can vary between runs.
 *   deterministic != 0: each query tile's partials are added in decreasing key-tile order, so
 *                       repeated runs give identical bits. */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, void* dq, void* dk, void* dv,
             int B, int H, int n, int d, float scale, int causal, int dtype, int deterministic,
             void* workspace, size_t ws_bytes, void* stream);

/* Backward pass of attn_fwd_gqa: k, v, dk, dv have Hkv heads; dk and dv of a K/V head are the sums
 * over its H/Hkv query heads (the gradient through the expansion). The workspace is
 * attn_bwd_workspace_bytes(B, H, n, d, deterministic) with the QUERY head count H. Everything
 * else as attn_bwd. */
int attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv,
                 int B, int H, int Hkv, int n, int d, float scale, int causal, int dtype,
                 int deterministic, void* workspace, size_t ws_bytes, void* stream);

/* Backward pass of attn_fwd_ex (bf16 only): dq (B, H, nq, d); dk, dv (B, Hkv, nk, d), summed over
 * the query heads of each K/V head. Keys that no query sees get dk = dv = 0. The workspace is
 * attn_bwd_workspace_bytes(B, H, nq, d, deterministic) (query rows). Everything else as attn_bwd;
 * the deterministic mode adds the dQ partials of a query tile in decreasing key-tile order,
 * starting from the last key tile that the tile meets. */
int attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dO,
                const float* lse, void* dq, void* dk, void* dv,
                int B, int H, int Hkv, int nq, int nk, int d, float scale,
                int window_left, int window_right, int dtype, int deterministic,
                void* workspace, size_t ws_bytes, void* stream);

/* Backward pass without a caller workspace, for callers that cannot allocate device memory where
 * they run it (e.g. code inside a host framework that owns all device allocations, or a loop that
 * must not call cudaMalloc). The pages have no counterpart to this entry point.
 * Same arguments, validation, kernels and results as attn_bwd, except that the scratch memory is a
 * fixed 32 MiB device array owned by the library: it is reserved on every GPU where the library's
 * device code is loaded, until the process exits, and nothing is allocated or freed per call.
 * Returns ATTN_ERR_WORKSPACE, launching nothing, when attn_bwd_workspace_bytes(B, H, n, d,
 * deterministic) exceeds 32 MiB (33,554,432 bytes). All calls on a device share the array and
 * leave their contents in it; each call rewrites or zeroes what it reads, but calls whose kernels
 * overlap on the GPU (unordered streams, concurrent host threads) race and give wrong results.
 * Arguments and the size limit are checked before any CUDA call. Outside stream capture each call
 * looks up the array's device address on the current device (cudaGetSymbolAddress); while the
 * stream is being captured the address found by the latest uncaptured call on that device is
 * used, so make one call on each device before capturing (otherwise ATTN_ERR_CUDA). */
int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                     const float* lse, void* dq, void* dk, void* dv,
                     int B, int H, int n, int d, float scale, int causal, int dtype,
                     int deterministic, void* stream);

/* The backward pass in three parts, for gradients summed over several key sets with the same
 * queries (ring attention: one call of attn_bwd_accumulate per hop, each with the K/V chunk that
 * the hop holds; "Attention Mechanism: Revolusi Representasi Sequence", §16 "Long Context
 * Training", Ring Attention). Because P = exp(scale·q·k - LSE) uses the final LSE over all keys and
 * D = rowsum(dO∘O) the final O (the recomputation of "Flash Attention Nedir?", Recomputation),
 * each key set's contribution to dQ, dK and dV is independent of the others and the sums are the
 * gradients of attention over all keys together. bf16 inputs only (else ATTN_ERR_UNSUPPORTED).
 * The workspace is attn_bwd_workspace_bytes(B, H, nq, d, deterministic), 256-byte aligned; it
 * carries D, LSE·log2(e) and the fp32 dQ sum from one call to the next, so the calls of one
 * sequence use the same workspace, sizes and deterministic flag, in stream order.
 *
 * attn_bwd_prepare: o, dO (B, H, nq, d) bf16 and lse (B, H, nq) fp32 of the whole forward pass;
 *   computes D and LSE·log2(e) and zeroes the dQ sum.
 * attn_bwd_accumulate: adds the gradients of attention of q, dO (B, H, nq, d) over the keys
 *   k, v (B, Hkv, nk, d) with the visible window of attn_fwd_ex: dQ into the workspace's fp32
 *   sum, and dK, dV (scale included, summed over the query heads of each K/V head) into the
 *   caller's fp32 arrays dk_acc, dv_acc (B, Hkv, nk, d), which the caller zeroes before the first
 *   call. Keys that no query sees add nothing. deterministic != 0: each call adds a query tile's
 *   partials in decreasing key-tile order, so the whole sequence of calls repeats bit for bit.
 *   Views: the heads of q and dO start q_head_rows rows apart, those of k, v, dk_acc and dv_acc
 *   kv_head_rows apart (0: nq / nk, packed). The workspace was prepared for ws_rows query rows
 *   (0: nq) and this call's queries are its rows [q_row0, q_row0 + nq), q_row0 a multiple of
 *   64; either they end at ws_rows or nq is a multiple of 128 (else ATTN_ERR_INVALID).
 * attn_bwd_finish: writes dq (B, H, nq, d) bf16 = scale · the dQ sum.
 * Errors: null or misaligned (16-byte) pointer, or sizes as attn_bwd_ex -> ATTN_ERR_INVALID; a
 *   workspace that is null or not 256-byte aligned -> ATTN_ERR_INVALID, too small ->
 *   ATTN_ERR_WORKSPACE; a failed launch -> ATTN_ERR_CUDA. Arguments are checked before anything
 *   is launched. */
int attn_bwd_prepare(const void* o, const void* dO, const float* lse, int B, int H, int nq, int d,
                     int dtype, int deterministic, void* workspace, size_t ws_bytes,
                     void* stream);
int attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* dO,
                        float* dk_acc, float* dv_acc, int B, int H, int Hkv, int nq, int nk, int d,
                        long long q_head_rows, long long kv_head_rows, int ws_rows, int q_row0,
                        float scale, int window_left, int window_right, int dtype,
                        int deterministic, void* workspace, size_t ws_bytes, void* stream);
int attn_bwd_finish(void* dq, int B, int H, int nq, int d, float scale, int dtype,
                    int deterministic, void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then returns and clears the sticky device status word: ATTN_OK, or
 * ATTN_ERR_TIMEOUT if a kernel's bounded wait expired since the last call, or ATTN_ERR_CUDA if
 * the synchronisation itself failed. */
int attn_get_device_status(void* stream);

/* Sets the limit of every device-side wait, in microseconds (default 2,000,000 = 2 s). Values
 * below 100 are raised to 100. Returns the previous value. */
unsigned attn_set_wait_timeout_us(unsigned us);

/* Self-test of the bounded-wait path: launches one CTA that waits on an mbarrier no thread ever
 * arrives on, with a limit of `timeout_us` microseconds, so the wait expires and the kernel sets
 * ATTN_ERR_TIMEOUT and returns. Returns the launch status; read the result with
 * attn_get_device_status(). Never faults or hangs the device. */
int attn_selftest_wait_timeout(unsigned timeout_us, void* stream);

/* Ring attention building blocks ("Attention Mechanism: Revolusi Representasi Sequence", §16 "Long
 * Context Training", Ring Attention: the sequence is split across GPUs and attention over all
 * chunks is computed by passing K/V chunks around a ring). Each hop attends the local queries to
 * one K/V chunk (attn_fwd_ex / attn_bwd_ex); these two calls combine the hops. Both are
 * elementwise, asynchronous on `stream`, and validate before launching.
 *
 * attn_ring_merge: folds one hop's partial result into a running one, row by row:
 *     LSE = log(exp(lse_acc) + exp(lse_part)),
 *     o_acc = exp(lse_acc - LSE)·o_acc + exp(lse_part - LSE)·o_part,   lse_acc = LSE,
 *   which is exact because each partial output is normalised by its own exp(LSE). A row with
 *   lse = -inf (no visible key in that chunk) has weight 0; rows with no key anywhere stay o = 0,
 *   lse = -inf.
 *   o_acc: rows x d fp32 (caller-owned device memory, 16-byte aligned); lse_acc: rows fp32;
 *   o_part: rows x d in part_dtype (ATTN_BF16 or ATTN_FP32); lse_part: rows fp32 (natural log).
 *   first != 0: o_acc / lse_acc are not read (they are initialised from the partial).
 *   o_out != NULL: the merged rows are also written there in out_dtype (the final hop's output).
 *   Errors: null pointer or rows < 1 -> ATTN_ERR_INVALID; d not in {32, 64, 128} or an unknown
 *   dtype -> ATTN_ERR_UNSUPPORTED; misaligned pointer -> ATTN_ERR_INVALID. */
int attn_ring_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                    long long rows, int d, int part_dtype, int first, void* o_out, int out_dtype,
                    void* stream);

/* attn_ring_accumulate: acc (count fp32) = (first ? 0 : acc) + part, where part (count elements
 * in part_dtype) may be NULL (no addition); with out != NULL the sum is also written there in
 * out_dtype. Used for the gradients of ring attention: dQ accumulates over the hops of the local
 * queries, dK / dV accumulate while travelling with their K / V chunk.
 *   count must be a positive multiple of 8; pointers 16-byte aligned (else ATTN_ERR_INVALID). */
int attn_ring_accumulate(float* acc, const void* part, long long count, int part_dtype, int first,
                         void* out, int out_dtype, void* stream);

/* Measurement hook. `events` is NULL (recording off, the default) or an array of 4 cudaEvent_t
 * created by the caller. While set, every attn_bwd call records, on its stream, events[0] before
 * its preprocess kernel (D = rowsum(dO∘O)), events[1] before its main kernel, events[2] after
 * the main kernel and events[3] after the dQ conversion kernel, so that a caller can time the
 * three kernels separately with cudaEventElapsedTime. NULL entries are skipped. The array is
 * copied; the events must stay valid while recording is on. Process-wide setting; not meant for concurrent callers. */
void attn_set_bwd_phase_events(void* const* events);

/* Static string for an error code. */
const char* attn_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
