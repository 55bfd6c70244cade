// C-ABI entry points of libattn.so (declared in include/attn.h): argument validation, tensor-map
// encoding, workspace carving and kernel launches on the caller's stream.
#include <cudaTypedefs.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "../../include/attn.h"
#include "kernels.h"
#include "ring.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace {

std::atomic<unsigned> g_timeout_us{2000000u};
cudaEvent_t g_phase_events[4];
std::atomic<bool> g_phase_on{false};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int to_code(cudaError_t e) { return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA; }

__global__ void wait_selftest_kernel(uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Nobody arrives on `bar`: the wait runs out, records ATTN_ERR_TIMEOUT and returns.
    if (threadIdx.x == 0) bounded_wait(&bar, 0, &abort_flag, timeout_ns);
    __syncthreads();
}

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
    size_t d_off, l2_off, acc_off, sem_off, total;
};

// D (fp32) | LSE·log2e (fp32) | dQ accumulator (fp32, d per row) | semaphores (four per 64 rows),
// every per-row array padded per head to a multiple of 128 rows.
WsLayout ws_layout(int B, int H, int n, int d, int deterministic) {
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t n_pad = (static_cast<size_t>(n) + 127) / 128 * 128;
    WsLayout w;
    w.d_off = 0;
    w.l2_off = round_up(BH * n_pad * sizeof(float));
    w.acc_off = w.l2_off + round_up(BH * n_pad * sizeof(float));
    w.sem_off = w.acc_off + round_up(BH * n_pad * d * sizeof(float));
    w.total = w.sem_off + (deterministic ? round_up(BH * (n_pad / 64) * 4 * sizeof(int)) : 0);
    return w;
}

// Longest sequence accepted: tile and row arithmetic runs in 32-bit integers up to the length
// rounded up to a multiple of 128 (plus one tile).
constexpr int kMaxSeq = 0x7fffffff - 256;

int validate_common(int B, int H, int n, int d, float scale, int dtype) {
    if (B < 1 || H < 1 || n < 1 || n > kMaxSeq) return ATTN_ERR_INVALID;
    if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID;
    if (static_cast<long long>(B) * H > 0x7fffffffLL) return ATTN_ERR_INVALID;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP32) return ATTN_ERR_UNSUPPORTED;
    if (d != 32 && d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

}  // namespace

cudaError_t make_tmap(CUtensorMap* map, const void* base, int esize, int BH, int n, int d,
                      int box_rows, long long head_rows) {
    if (head_rows <= 0) head_rows = n;
    if (head_rows < n) return cudaErrorInvalidValue;
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const int chunk = d * esize >= 128 ? 128 / esize : d;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize,
                             static_cast<cuuint64_t>(d) * esize * static_cast<cuuint64_t>(head_rows)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(chunk), static_cast<cuuint32_t>(box_rows), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    const int chunk_bytes = chunk * esize;
    if (chunk_bytes != 128 && chunk_bytes != 64) return cudaErrorInvalidValue;
    const CUtensorMapSwizzle swz =
        chunk_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapDataType dt =
        esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Argument checks of the backward entry points, everything but the workspace: null and
// misaligned pointers, sizes, scale, head counts and dtype.
int validate_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, const void* dq, const void* dk, const void* dv, int B, int H,
                 int Hkv, int nq, int nk, int d, float scale, int dtype) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, scale, dtype);
    if (rc) return rc;
    if (nk < 1 || nk > kMaxSeq) return ATTN_ERR_INVALID;
    if (Hkv < 1 || H % Hkv != 0) return ATTN_ERR_INVALID;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv};
    for (const void* p : ptrs)
        if (!aligned16(p)) return ATTN_ERR_INVALID;
    return ATTN_OK;
}

cudaError_t make_tmap_acc(CUtensorMap* map, float* base, long long rows, int d) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (rows < 1 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;   // 32-bit box coordinates
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * sizeof(float)};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_wait_selftest(uint64_t timeout_ns, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(timeout_ns);
    return cudaGetLastError();
}

}  // namespace attn

using namespace attn;

extern "C" {

int attn_version(void) { return 100; }

const char* attn_error_string(int code) {
    switch (code) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_CUDA: return "CUDA error";
        case ATTN_ERR_TIMEOUT: return "device-side wait timed out";
        case ATTN_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown error";
    }
}

unsigned attn_set_wait_timeout_us(unsigned us) {
    if (us < 100u) us = 100u;
    return g_timeout_us.exchange(us);
}

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int Hkv, int nq, int nk, int d, float scale, int wl, int wr, int dtype,
                    void* stream) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, scale, dtype);
    if (rc) return rc;
    if (nk < 1 || nk > kMaxSeq) return ATTN_ERR_INVALID;
    if (Hkv < 1 || H % Hkv != 0) return ATTN_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID;
    FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.H = H; a.nq = nq; a.nk = nk; a.d = d; a.Hkv = Hkv;
    a.scale = scale;
    a.wl = wl < 0 ? -1 : wl;
    a.wr = wr < 0 ? -1 : wr;
    a.q_descale = a.k_descale = a.v_descale = 1.f;
    a.timeout_ns = static_cast<uint64_t>(g_timeout_us.load()) * 1000ull;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = (dtype == ATTN_BF16) ? launch_fwd_bf16(a, s) : launch_fwd_f32(a, s);
    return to_code(e);
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int n, int d, float scale, int causal, int dtype, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, H, n, n, d, scale, -1, causal ? 0 : -1, dtype, stream);
}

int attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Hkv, int n, int d, float scale, int causal, int dtype, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, Hkv, n, n, d, scale, -1, causal ? 0 : -1, dtype,
                    stream);
}

int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int Hkv, int nq, int nk, int d, float scale, int window_left, int window_right,
                int dtype, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, Hkv, nq, nk, d, scale, window_left, window_right, dtype,
                    stream);
}

int attn_fwd_accumulate(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc,
                        int B, int H, int Hkv, int nq, int nk, int d, long long q_head_rows,
                        long long kv_head_rows, float scale, int window_left, int window_right,
                        int first, void* stream) {
    if (!q || !k || !v || !o_acc || !lse_acc) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, scale, ATTN_BF16);
    if (rc) return rc;
    if (nk < 1 || nk > kMaxSeq) return ATTN_ERR_INVALID;
    if (Hkv < 1 || H % Hkv != 0) return ATTN_ERR_INVALID;
    if ((q_head_rows != 0 && q_head_rows < nq) || (kv_head_rows != 0 && kv_head_rows < nk) ||
        q_head_rows < 0 || kv_head_rows < 0 || q_head_rows > kMaxSeq || kv_head_rows > kMaxSeq)
        return ATTN_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_acc) || !aligned16(lse_acc))
        return ATTN_ERR_INVALID;
    FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o_acc; a.lse = lse_acc;
    a.B = B; a.H = H; a.nq = nq; a.nk = nk; a.d = d; a.Hkv = Hkv;
    a.scale = scale;
    a.wl = window_left < 0 ? -1 : window_left;
    a.wr = window_right < 0 ? -1 : window_right;
    a.q_descale = a.k_descale = a.v_descale = 1.f;
    a.timeout_ns = static_cast<uint64_t>(g_timeout_us.load()) * 1000ull;
    a.acc_first = first ? 1 : 0;
    a.q_rows = q_head_rows;
    a.kv_rows = kv_head_rows;
    return to_code(launch_fwd_bf16(a, static_cast<cudaStream_t>(stream)));
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Hkv, int nq, int nk, int d, float scale, int window_left, int window_right,
                 float q_descale, float k_descale, float v_descale, void* stream) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, scale, ATTN_BF16);
    if (rc) return rc;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (nk < 1 || nk > kMaxSeq || Hkv < 1 || H % Hkv != 0) return ATTN_ERR_INVALID;
    const float ds[3] = {q_descale, k_descale, v_descale};
    for (float x : ds)
        if (!(x > 0.f) || !isfinite(x)) return ATTN_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID;
    FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.H = H; a.nq = nq; a.nk = nk; a.d = d; a.Hkv = Hkv;
    a.scale = scale;
    a.wl = window_left < 0 ? -1 : window_left;
    a.wr = window_right < 0 ? -1 : window_right;
    a.q_descale = q_descale;
    a.k_descale = k_descale;
    a.v_descale = v_descale;
    a.timeout_ns = static_cast<uint64_t>(g_timeout_us.load()) * 1000ull;
    return to_code(launch_fwd_fp8(a, static_cast<cudaStream_t>(stream)));
}

size_t attn_bwd_workspace_bytes(int B, int H, int n, int d, int deterministic) {
    if (B < 1 || H < 1 || n < 1 || d < 1) return 0;
    return ws_layout(B, H, n, d, deterministic).total;
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dO,
                    const float* lse, void* dq, void* dk, void* dv, int B, int H, int Hkv, int nq,
                    int nk, int d, float scale, int wl, int wr, int dtype, int deterministic,
                    void* workspace, size_t ws_bytes, void* stream) {
    int rc = validate_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, nq, nk, d, scale, dtype);
    if (rc) return rc;
    WsLayout w = ws_layout(B, H, nq, d, deterministic);
    if (!workspace) return ATTN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_INVALID;
    if (ws_bytes < w.total) return ATTN_ERR_WORKSPACE;
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.dO = dO; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.B = B; a.H = H; a.nq = nq; a.nk = nk; a.d = d; a.Hkv = Hkv;
    a.scale = scale;
    a.wl = wl < 0 ? -1 : wl;
    a.wr = wr < 0 ? -1 : wr;
    a.deterministic = deterministic ? 1 : 0;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.Dvec = reinterpret_cast<float*>(ws + w.d_off);
    a.L2vec = reinterpret_cast<float*>(ws + w.l2_off);
    a.dq_acc = reinterpret_cast<float*>(ws + w.acc_off);
    a.sems = deterministic ? reinterpret_cast<int*>(ws + w.sem_off) : nullptr;
    a.timeout_ns = static_cast<uint64_t>(g_timeout_us.load()) * 1000ull;
    a.phase_events = g_phase_on.load() ? g_phase_events : nullptr;
    return to_code(launch_bwd_bf16(a, static_cast<cudaStream_t>(stream)));
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, void* dq, void* dk, void* dv, int B, int H, int n, int d,
             float scale, int causal, int dtype, int deterministic, void* workspace,
             size_t ws_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, H, H, n, n, d, scale, -1, causal ? 0 : -1,
                    dtype, deterministic, workspace, ws_bytes, stream);
}

int attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int Hkv, int n,
                 int d, float scale, int causal, int dtype, int deterministic, void* workspace,
                 size_t ws_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, n, n, d, scale, -1,
                    causal ? 0 : -1, dtype, deterministic, workspace, ws_bytes, stream);
}

int attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dO,
                const float* lse, void* dq, void* dk, void* dv, int B, int H, int Hkv, int nq,
                int nk, int d, float scale, int window_left, int window_right, int dtype,
                int deterministic, void* workspace, size_t ws_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, nq, nk, d, scale, window_left,
                    window_right, dtype, deterministic, workspace, ws_bytes, stream);
}

// Workspace arguments shared by the backward entry points: present, 256-byte aligned, large
// enough for (B, H, nq, d, deterministic).
static int check_ws(const void* workspace, size_t ws_bytes, int B, int H, int nq, int d,
                    int deterministic, WsLayout* w) {
    *w = ws_layout(B, H, nq, d, deterministic);
    if (!workspace) return ATTN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_INVALID;
    if (ws_bytes < w->total) return ATTN_ERR_WORKSPACE;
    return ATTN_OK;
}

static void set_ws(BwdArgs& a, void* workspace, const WsLayout& w, int deterministic) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.Dvec = reinterpret_cast<float*>(ws + w.d_off);
    a.L2vec = reinterpret_cast<float*>(ws + w.l2_off);
    a.dq_acc = reinterpret_cast<float*>(ws + w.acc_off);
    a.sems = deterministic ? reinterpret_cast<int*>(ws + w.sem_off) : nullptr;
    a.timeout_ns = static_cast<uint64_t>(g_timeout_us.load()) * 1000ull;
    a.phase_events = nullptr;
}

int attn_bwd_prepare(const void* o, const void* dO, const float* lse, int B, int H, int nq,
                     int d, int dtype, int deterministic, void* workspace, size_t ws_bytes,
                     void* stream) {
    if (!o || !dO || !lse) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, 1.f, dtype);
    if (rc) return rc;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(o) || !aligned16(dO) || !aligned16(lse)) return ATTN_ERR_INVALID;
    WsLayout w;
    if ((rc = check_ws(workspace, ws_bytes, B, H, nq, d, deterministic, &w))) return rc;
    BwdArgs a = {};
    a.o = o; a.dO = dO; a.lse = lse;
    a.B = B; a.H = H; a.Hkv = H; a.nq = nq; a.nk = nq; a.d = d;
    a.scale = 1.f;
    a.wl = -1; a.wr = -1;
    a.deterministic = deterministic ? 1 : 0;
    set_ws(a, workspace, w, a.deterministic);
    a.phases = 1;
    return to_code(launch_bwd_bf16(a, static_cast<cudaStream_t>(stream)));
}

int attn_bwd_accumulate(const void* q, const void* k, const void* v, const void* dO,
                        float* dk_acc, float* dv_acc, int B, int H, int Hkv, int nq, int nk, int d,
                        long long q_head_rows, long long kv_head_rows, int ws_rows, int q_row0,
                        float scale, int window_left, int window_right, int dtype,
                        int deterministic, void* workspace, size_t ws_bytes, void* stream) {
    if (!q || !k || !v || !dO || !dk_acc || !dv_acc) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, scale, dtype);
    if (rc) return rc;
    if (nk < 1 || nk > kMaxSeq) return ATTN_ERR_INVALID;
    if (Hkv < 1 || H % Hkv != 0) return ATTN_ERR_INVALID;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    const void* ptrs[] = {q, k, v, dO, dk_acc, dv_acc};
    for (const void* p : ptrs)
        if (!aligned16(p)) return ATTN_ERR_INVALID;
    if (ws_rows == 0) ws_rows = nq;
    if ((q_head_rows != 0 && q_head_rows < nq) || (kv_head_rows != 0 && kv_head_rows < nk) ||
        q_head_rows < 0 || kv_head_rows < 0 || q_head_rows > kMaxSeq || kv_head_rows > kMaxSeq)
        return ATTN_ERR_INVALID;
    // the first query sits on a 64-row boundary of the workspace (its fp32 rows are moved by bulk
    // copies), and the rows after this launch's last query tile are padding or there are none
    if (ws_rows < 1 || ws_rows > kMaxSeq || q_row0 < 0 || q_row0 % 64 != 0 ||
        q_row0 > ws_rows - nq || (q_row0 + nq != ws_rows && nq % 128 != 0))
        return ATTN_ERR_INVALID;
    WsLayout w;
    if ((rc = check_ws(workspace, ws_bytes, B, H, ws_rows, d, deterministic, &w))) return rc;
    BwdArgs a = {};
    a.q = q; a.k = k; a.v = v; a.dO = dO;
    a.B = B; a.H = H; a.Hkv = Hkv; a.nq = nq; a.nk = nk; a.d = d;
    a.scale = scale;
    a.wl = window_left < 0 ? -1 : window_left;
    a.wr = window_right < 0 ? -1 : window_right;
    a.deterministic = deterministic ? 1 : 0;
    set_ws(a, workspace, w, a.deterministic);
    a.phases = 2;
    a.dk_acc32 = dk_acc;
    a.dv_acc32 = dv_acc;
    a.q_rows = q_head_rows;
    a.kv_rows = kv_head_rows;
    a.ws_rows = ws_rows;
    a.q_row0 = q_row0;
    return to_code(launch_bwd_bf16(a, static_cast<cudaStream_t>(stream)));
}

int attn_bwd_finish(void* dq, int B, int H, int nq, int d, float scale, int dtype,
                    int deterministic, void* workspace, size_t ws_bytes, void* stream) {
    if (!dq) return ATTN_ERR_INVALID;
    int rc = validate_common(B, H, nq, d, scale, dtype);
    if (rc) return rc;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(dq)) return ATTN_ERR_INVALID;
    WsLayout w;
    if ((rc = check_ws(workspace, ws_bytes, B, H, nq, d, deterministic, &w))) return rc;
    BwdArgs a = {};
    a.dq = dq;
    a.B = B; a.H = H; a.Hkv = H; a.nq = nq; a.nk = nq; a.d = d;
    a.scale = scale;
    a.wl = -1; a.wr = -1;
    a.deterministic = deterministic ? 1 : 0;
    set_ws(a, workspace, w, a.deterministic);
    a.phases = 4;
    return to_code(launch_bwd_bf16(a, static_cast<cudaStream_t>(stream)));
}

int attn_ring_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                    long long rows, int d, int part_dtype, int first, void* o_out, int out_dtype,
                    void* stream) {
    if (!o_acc || !lse_acc || !o_part || !lse_part || rows < 1) return ATTN_ERR_INVALID;
    if (d != 32 && d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if ((part_dtype != ATTN_BF16 && part_dtype != ATTN_FP32) ||
        (o_out && out_dtype != ATTN_BF16 && out_dtype != ATTN_FP32))
        return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(o_acc) || !aligned16(o_part) || (o_out && !aligned16(o_out)))
        return ATTN_ERR_INVALID;
    return to_code(launch_ring_merge(o_acc, lse_acc, o_part, lse_part, rows, d,
                                     part_dtype == ATTN_BF16, first ? 1 : 0, o_out,
                                     out_dtype == ATTN_BF16, static_cast<cudaStream_t>(stream)));
}

int attn_ring_accumulate(float* acc, const void* part, long long count, int part_dtype, int first,
                         void* out, int out_dtype, void* stream) {
    if (!acc || count < 1 || count % 8 != 0) return ATTN_ERR_INVALID;
    if ((part && part_dtype != ATTN_BF16 && part_dtype != ATTN_FP32) ||
        (out && out_dtype != ATTN_BF16 && out_dtype != ATTN_FP32))
        return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(acc) || (part && !aligned16(part)) || (out && !aligned16(out)))
        return ATTN_ERR_INVALID;
    return to_code(launch_ring_accumulate(acc, part, count, part_dtype == ATTN_BF16,
                                          first ? 1 : 0, out, out_dtype == ATTN_BF16,
                                          static_cast<cudaStream_t>(stream)));
}

void attn_set_bwd_phase_events(void* const* events) {
    if (!events) {
        g_phase_on.store(false);
        return;
    }
    for (int i = 0; i < 4; ++i) g_phase_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_phase_on.store(true);
}

int attn_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return v;
}

int attn_selftest_wait_timeout(unsigned timeout_us, void* stream) {
    if (timeout_us == 0 || timeout_us > 10000000u) return ATTN_ERR_INVALID;
    return to_code(launch_wait_selftest(static_cast<uint64_t>(timeout_us) * 1000ull,
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
