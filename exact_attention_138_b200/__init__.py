"""exact_attention_138_b200 — exact scaled dot-product attention on one B200 (sm_100a).

Python binding of the C ABI in ``include/attn.h`` (``libattn.so``, built in-tree by
``python exact_attention_138_b200/build.py``). This module only marshals arguments: device
memory and streams come from PyTorch, every step of the computation runs in the library's
CUDA kernels. There is no CPU fallback: if the library is missing the import fails.

    O = softmax(scale · Q·K^T + M) · V      ("Attention Mechanism: Revolusi Representasi
    Sequence", §3 Steps 1-4; causal mask M of §4.4, sliding window of §4.5, cross-attention
    with different query / key lengths of §4.2)

Raw entry points keep the C names (``attn_fwd``, ``attn_fwd_gqa``, ``attn_fwd_ex``, ``attn_bwd``,
``attn_bwd_gqa``, ``attn_bwd_ex``, ``attn_bwd_workspace_bytes``,
``attn_get_device_status``, ``attn_set_wait_timeout_us``, ``attn_selftest_wait_timeout``,
``attn_error_string``, ``attn_version``); ``forward`` / ``backward`` wrap them for torch tensors.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "attn.h")

ATTN_BF16, ATTN_FP32 = 0, 1
ATTN_OK, ATTN_ERR_INVALID, ATTN_ERR_UNSUPPORTED = 0, 1, 2
ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT, ATTN_ERR_WORKSPACE = 3, 4, 5

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python exact_attention_138_b200/build.py` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_lib.attn_version.restype = _i
_lib.attn_version.argtypes = []
_lib.attn_error_string.restype = ctypes.c_char_p
_lib.attn_error_string.argtypes = [_i]
_lib.attn_fwd.restype = _i
_lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]
_lib.attn_fwd_gqa.restype = _i
_lib.attn_fwd_gqa.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _vp]
_lib.attn_bwd_gqa.restype = _i
_lib.attn_bwd_gqa.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f,
                              _i, _i, _i, _vp, _sz, _vp]
_lib.attn_fwd_ex.restype = _i
_lib.attn_fwd_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp]
_lib.attn_bwd_ex.restype = _i
_lib.attn_bwd_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                             _f, _i, _i, _i, _i, _vp, _sz, _vp]
_ll = ctypes.c_longlong
_lib.attn_fwd_fp8.restype = _i
_lib.attn_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _f, _f,
                              _f, _vp]
_lib.attn_ring_merge.restype = _i
_lib.attn_ring_merge.argtypes = [_vp, _vp, _vp, _vp, _ll, _i, _i, _i, _vp, _i, _vp]
_lib.attn_ring_accumulate.restype = _i
_lib.attn_ring_accumulate.argtypes = [_vp, _vp, _ll, _i, _i, _vp, _i, _vp]
_lib.attn_bwd_workspace_bytes.restype = _sz
_lib.attn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
_lib.attn_bwd.restype = _i
_lib.attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                          _i, _i, _vp, _sz, _vp]
_lib.attn_fwd_accumulate.restype = _i
_lib.attn_fwd_accumulate.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _ll, _ll, _f,
                                     _i, _i, _i, _vp]
_lib.attn_bwd_prepare.restype = _i
_lib.attn_bwd_prepare.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
_lib.attn_bwd_accumulate.restype = _i
_lib.attn_bwd_accumulate.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _ll,
                                     _ll, _i, _i, _f, _i, _i, _i, _i, _vp, _sz, _vp]
_lib.attn_bwd_finish.restype = _i
_lib.attn_bwd_finish.argtypes = [_vp, _i, _i, _i, _i, _f, _i, _i, _vp, _sz, _vp]
_lib.attn_get_device_status.restype = _i
_lib.attn_get_device_status.argtypes = [_vp]
_lib.attn_set_wait_timeout_us.restype = ctypes.c_uint
_lib.attn_set_wait_timeout_us.argtypes = [ctypes.c_uint]
_lib.attn_selftest_wait_timeout.restype = _i
_lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp]
_lib.attn_set_bwd_phase_events.restype = None
_lib.attn_set_bwd_phase_events.argtypes = [_vp]


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {attn_error_string(code)} (code {code})")


def library():
    """The loaded ctypes library (for tests that check exported symbols)."""
    return _lib


def declared_functions():
    """Names of the functions declared in include/attn.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


# ---------------------------------------------------------------- raw C entry points
def attn_version() -> int:
    return _lib.attn_version()


def attn_error_string(code: int) -> str:
    return _lib.attn_error_string(int(code)).decode()


def attn_fwd(q, k, v, o, lse, B, H, n, d, scale, causal, dtype, stream) -> int:
    return _lib.attn_fwd(q, k, v, o, lse, B, H, n, d, scale, causal, dtype, stream)


def attn_fwd_gqa(q, k, v, o, lse, B, H, Hkv, n, d, scale, causal, dtype, stream) -> int:
    return _lib.attn_fwd_gqa(q, k, v, o, lse, B, H, Hkv, n, d, scale, causal, dtype, stream)


def attn_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, n, d, scale, causal, dtype,
                 deterministic, workspace, ws_bytes, stream) -> int:
    return _lib.attn_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, n, d, scale, causal,
                             dtype, deterministic, workspace, ws_bytes, stream)


def attn_fwd_ex(q, k, v, o, lse, B, H, Hkv, nq, nk, d, scale, window_left, window_right, dtype,
                stream) -> int:
    return _lib.attn_fwd_ex(q, k, v, o, lse, B, H, Hkv, nq, nk, d, scale, window_left,
                            window_right, dtype, stream)


def attn_bwd_ex(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, nq, nk, d, scale, window_left,
                window_right, dtype, deterministic, workspace, ws_bytes, stream) -> int:
    return _lib.attn_bwd_ex(q, k, v, o, dO, lse, dq, dk, dv, B, H, Hkv, nq, nk, d, scale,
                            window_left, window_right, dtype, deterministic, workspace, ws_bytes,
                            stream)


def attn_fwd_fp8(q, k, v, o, lse, B, H, Hkv, nq, nk, d, scale, window_left, window_right,
                 q_descale, k_descale, v_descale, stream) -> int:
    return _lib.attn_fwd_fp8(q, k, v, o, lse, B, H, Hkv, nq, nk, d, scale, window_left,
                             window_right, q_descale, k_descale, v_descale, stream)


def attn_ring_merge(o_acc, lse_acc, o_part, lse_part, rows, d, part_dtype, first, o_out,
                    out_dtype, stream) -> int:
    return _lib.attn_ring_merge(o_acc, lse_acc, o_part, lse_part, rows, d, part_dtype, first,
                                o_out, out_dtype, stream)


def attn_ring_accumulate(acc, part, count, part_dtype, first, out, out_dtype, stream) -> int:
    return _lib.attn_ring_accumulate(acc, part, count, part_dtype, first, out, out_dtype, stream)


def attn_bwd_workspace_bytes(B, H, n, d, deterministic) -> int:
    return _lib.attn_bwd_workspace_bytes(B, H, n, d, deterministic)


def attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, n, d, scale, causal, dtype, deterministic,
             workspace, ws_bytes, stream) -> int:
    return _lib.attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, n, d, scale, causal, dtype,
                         deterministic, workspace, ws_bytes, stream)


def attn_fwd_accumulate(q, k, v, o_acc, lse_acc, B, H, Hkv, nq, nk, d, q_head_rows,
                        kv_head_rows, scale, window_left, window_right, first, stream) -> int:
    return _lib.attn_fwd_accumulate(q, k, v, o_acc, lse_acc, B, H, Hkv, nq, nk, d, q_head_rows,
                                    kv_head_rows, scale, window_left, window_right, first, stream)


def attn_bwd_prepare(o, dO, lse, B, H, nq, d, dtype, deterministic, workspace, ws_bytes,
                     stream) -> int:
    return _lib.attn_bwd_prepare(o, dO, lse, B, H, nq, d, dtype, deterministic, workspace,
                                 ws_bytes, stream)


def attn_bwd_accumulate(q, k, v, dO, dk_acc, dv_acc, B, H, Hkv, nq, nk, d, q_head_rows,
                        kv_head_rows, ws_rows, q_row0, scale, window_left, window_right, dtype,
                        deterministic, workspace, ws_bytes, stream) -> int:
    return _lib.attn_bwd_accumulate(q, k, v, dO, dk_acc, dv_acc, B, H, Hkv, nq, nk, d,
                                    q_head_rows, kv_head_rows, ws_rows, q_row0, scale,
                                    window_left, window_right, dtype, deterministic, workspace,
                                    ws_bytes, stream)


def attn_bwd_finish(dq, B, H, nq, d, scale, dtype, deterministic, workspace, ws_bytes,
                    stream) -> int:
    return _lib.attn_bwd_finish(dq, B, H, nq, d, scale, dtype, deterministic, workspace, ws_bytes,
                                stream)


def attn_get_device_status(stream=None) -> int:
    return _lib.attn_get_device_status(stream)


def attn_set_wait_timeout_us(us: int) -> int:
    return _lib.attn_set_wait_timeout_us(int(us))


def attn_selftest_wait_timeout(timeout_us: int, stream=None) -> int:
    return _lib.attn_selftest_wait_timeout(int(timeout_us), stream)


def attn_set_bwd_phase_events(events) -> None:
    """events: None, or 4 torch.cuda.Event objects (created with enable_timing=True)."""
    if events is None:
        _lib.attn_set_bwd_phase_events(None)
        return
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _lib.attn_set_bwd_phase_events(ctypes.cast(arr, ctypes.c_void_p))


# ---------------------------------------------------------------- torch-tensor wrappers
def _dims(q):
    if q.dim() == 2:
        return 1, 1, q.shape[0], q.shape[1]
    if q.dim() != 4:
        raise ValueError("expected (B, H, n, d) or (n, d) tensors")
    return tuple(q.shape)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float32:
        return ATTN_FP32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _head_rows(*ts):
    """Rows between consecutive heads shared by (B, H, n, d) tensors / (B, H, n) row vectors that
    may be views of rows of longer sequences (0 when packed); raises for other layouts."""
    rows = None
    for t in ts:
        if t.dim() == 4:
            B, H, n, d = t.shape
            e = d                                   # elements per row
            ok = t.stride(3) == 1 and t.stride(2) == d
        else:
            B, H, n = t.shape
            e = 1
            ok = t.stride(2) == 1
        # rows between heads: from the head stride, or from the batch stride when H == 1 (the
        # stride of a dimension of size 1 carries no layout)
        hs = t.stride(1) if H > 1 else (t.stride(0) if B > 1 else None)
        if hs is None:
            r = n if rows is None else rows         # a single head: any row count fits
        else:
            ok = ok and hs % e == 0 and (B == 1 or H == 1 or t.stride(0) == H * hs)
            r = hs // e
        if not ok or r < n or (rows is not None and r != rows):
            raise ValueError("expected packed (B, H, n, d) tensors or views of rows of a longer "
                             "sequence with one layout")
        rows = r
    return 0 if rows is None or rows == ts[0].shape[2] else rows


def _packed(where, *ts):
    """The entry points without view support take packed CUDA tensors on one device: a host
    tensor's pointer must never reach a kernel, and a strided one would be read as packed."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{where}: tensors must be on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{where}: tensors must be on one device")
        if not t.is_contiguous():
            raise ValueError(f"{where}: tensors must be contiguous")


def _shaped(where, pairs):
    """(tensor, expected shape, expected dtype or None) triples: a buffer the kernels write or read
    must have the size they assume (the C ABI only sees pointers)."""
    for t, shape, dtype in pairs:
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{where}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{where}: expected {dtype}, got {t.dtype}")


def _on_device(where, dev, *ts):
    """Views are allowed (their layout is checked by _head_rows), host tensors are not."""
    for t in ts:
        if not t.is_cuda:
            raise ValueError(f"{where}: tensors must be on a CUDA device")
        if t.device != dev:
            raise ValueError(f"{where}: tensors must be on one device ({dev})")


def _check(rc, where):
    if rc != ATTN_OK:
        raise AttnError(rc, where)


def _kv_heads(q, k, v):
    """(K/V head count, key length): heads equal to q's (multi-head) or a divisor of it
    (grouped-query); k and v of shape (B, Hkv, nk, d)."""
    B, H, n, d = _dims(q)
    kd = _dims(k)
    if k.dim() != q.dim() or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must match each other and q's dtype")
    if kd[0] != B or kd[3] != d or H % kd[1] != 0:
        raise ValueError("k, v must be (B, Hkv, nk, d) with H a multiple of Hkv")
    return kd[1], kd[2]


def _window(causal, window):
    """(window_left, window_right): None -> causal (-1, 0) or none (-1, -1); causal=True with a
    window caps the right side at 0. Negative = unbounded."""
    if window is None:
        return (-1, 0) if causal else (-1, -1)
    wl, wr = (int(window[0]), int(window[1]))
    wl = -1 if wl < 0 else wl
    wr = -1 if wr < 0 else wr
    if causal:
        wr = 0
    return wl, wr


def forward(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None, window=None):
    """O, LSE = attention(q, k, v). q: contiguous CUDA tensor (B,H,n,d) or (n,d), bf16 or fp32;
    k, v: same shape, or (B,Hkv,nk,d) for grouped-query attention and / or another key length
    (cross-attention). window=(left, right): key j visible to query i iff
    i+nk-nq-left <= j <= i+nk-nq+right (negative = unbounded); causal=True is (-1, 0).
    Returns O (same dtype/shape as q) and LSE (fp32, (B,H,nq)); a query that sees no key gets
    O = 0 and LSE = -inf."""
    import torch
    B, H, n, d = _dims(q)
    Hkv, nk = _kv_heads(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    _packed("forward", q, k, v, out, lse)
    _shaped("forward", [(out, q.shape, q.dtype), (lse, (B, H, n) if q.dim() == 4 else (n,),
                                                  torch.float32)])
    if nk != n or window is not None:
        wl, wr = _window(causal, window)
        rc = attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, n, nk, d,
                         float(scale), wl, wr, _dtype_code(q), _stream_handle(stream))
    elif Hkv == H:
        rc = attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, n, d, float(scale),
                      int(bool(causal)), _dtype_code(q), _stream_handle(stream))
    else:
        rc = attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, n, d,
                          float(scale), int(bool(causal)), _dtype_code(q), _stream_handle(stream))
    _check(rc, "attn_fwd")
    return out, lse


def forward_accumulate(q, k, v, o_acc, lse_acc, first=False, causal=False, scale=None,
                       window=None, stream=None):
    """Fold attention of q (bf16) over the keys k, v into the running fp32 o_acc (q's shape) and
    lse_acc ((B, H, nq), natural log) in place (attn_fwd_accumulate); first=True initialises
    them. Masks as `forward`."""
    import torch
    B, H, n, d = _dims(q)
    Hkv, nk = _kv_heads(q, k, v)
    if o_acc.shape != q.shape or o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32:
        raise ValueError("o_acc must be fp32 with q's shape, lse_acc fp32 (B, H, nq)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    wl, wr = _window(causal, window)
    _on_device("forward_accumulate", q.device, q, k, v, o_acc, lse_acc)
    q_rows, kv_rows = _head_rows(q, o_acc, lse_acc), _head_rows(k, v)
    rc = attn_fwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(o_acc), _ptr(lse_acc), B, H, Hkv, n,
                             nk, d, q_rows, kv_rows, float(scale), wl, wr, int(bool(first)),
                             _stream_handle(stream))
    _check(rc, "attn_fwd_accumulate")


def backward(q, k, v, o, do, lse, causal=False, scale=None, deterministic=False, dq=None,
             dk=None, dv=None, workspace=None, stream=None, window=None):
    """dQ, dK, dV of attention given dO (bf16 tensors, lse from `forward` with the same causal /
    window arguments). dK, dV have k's (B, Hkv, nk, d) shape and, for grouped-query inputs, sum
    over each group's query heads."""
    import torch
    B, H, n, d = _dims(q)
    Hkv, nk = _kv_heads(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = attn_bwd_workspace_bytes(B, H, n, d, int(bool(deterministic)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _packed("backward", q, k, v, o, do, lse, dq, dk, dv, workspace)
    lse_shape = (B, H, n) if q.dim() == 4 else (n,)
    _shaped("backward", [(o, q.shape, q.dtype), (do, q.shape, q.dtype),
                         (lse, lse_shape, torch.float32), (dq, q.shape, q.dtype),
                         (dk, k.shape, k.dtype), (dv, v.shape, v.dtype)])
    ws_bytes = workspace.numel() * workspace.element_size()
    if nk != n or window is not None:
        wl, wr = _window(causal, window)
        rc = attn_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                         _ptr(dk), _ptr(dv), B, H, Hkv, n, nk, d, float(scale), wl, wr,
                         _dtype_code(q), int(bool(deterministic)), _ptr(workspace), ws_bytes,
                         _stream_handle(stream))
    elif Hkv == H:
        rc = attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                      _ptr(dv), B, H, n, d, float(scale), int(bool(causal)), _dtype_code(q),
                      int(bool(deterministic)), _ptr(workspace), ws_bytes, _stream_handle(stream))
    else:
        rc = attn_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                          _ptr(dk), _ptr(dv), B, H, Hkv, n, d, float(scale), int(bool(causal)),
                          _dtype_code(q), int(bool(deterministic)), _ptr(workspace), ws_bytes,
                          _stream_handle(stream))
    _check(rc, "attn_bwd")
    return dq, dk, dv


class BackwardSum:
    """The backward pass of one set of queries, summed over several key sets (attn_bwd_prepare /
    attn_bwd_accumulate / attn_bwd_finish): construct with the final o, dO, lse of the queries,
    call `add` once per key set (dK, dV added into fp32 arrays the caller zeroed), then `finish`
    for dQ. The workspace it holds is reused by `reset` for another pass of the same sizes."""

    def __init__(self, o, do, lse, deterministic=False, stream=None):
        import torch
        self.B, self.H, self.n, self.d = _dims(o)
        self.det = int(bool(deterministic))
        need = attn_bwd_workspace_bytes(self.B, self.H, self.n, self.d, self.det)
        self.ws = torch.empty(need, dtype=torch.uint8, device=o.device)
        self.reset(o, do, lse, stream)

    def reset(self, o, do, lse, stream=None):
        import torch
        if _dims(o) != (self.B, self.H, self.n, self.d):
            raise ValueError("reset needs the sizes the workspace was made for")
        _packed("BackwardSum", o, do, lse, self.ws)
        _shaped("BackwardSum", [(do, o.shape, o.dtype), (lse, o.shape[:-1], torch.float32)])
        rc = attn_bwd_prepare(_ptr(o), _ptr(do), _ptr(lse), self.B, self.H, self.n, self.d,
                              _dtype_code(o), self.det, _ptr(self.ws), self.ws.numel(),
                              _stream_handle(stream))
        _check(rc, "attn_bwd_prepare")

    def add(self, q, k, v, do, dk_acc, dv_acc, scale=None, causal=False, window=None,
            stream=None, q_row0=0):
        """dQ sum += and dk_acc, dv_acc (fp32, k's shape) += the gradients over keys k, v. q, dO
        may be rows [q_row0, q_row0 + nq) of the queries (views of them; q_row0 a multiple of
        64), k, v, dk_acc, dv_acc views of rows of longer key sequences."""
        import torch
        Hkv, nk = _kv_heads(q, k, v)
        for t in (dk_acc, dv_acc):
            if t.shape != k.shape or t.dtype != torch.float32:
                raise ValueError("dk_acc, dv_acc must be fp32 with k's shape")
        if (q.dim() != 4 or q.shape[0] != self.B or q.shape[1] != self.H or q.shape[3] != self.d
                or q.shape[2] + int(q_row0) > self.n or int(q_row0) < 0 or int(q_row0) % 64):
            raise ValueError("q must be (B, H, nq, d) rows of the queries this sum was made for")
        _shaped("BackwardSum.add", [(do, q.shape, q.dtype)])
        _on_device("BackwardSum.add", self.ws.device, q, k, v, do, dk_acc, dv_acc)
        if scale is None:
            scale = 1.0 / math.sqrt(self.d)
        wl, wr = _window(causal, window)
        nq = q.shape[2]
        q_rows, kv_rows = _head_rows(q, do), _head_rows(k, v, dk_acc, dv_acc)
        rc = attn_bwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dk_acc), _ptr(dv_acc),
                                 self.B, self.H, Hkv, nq, nk, self.d, q_rows, kv_rows, self.n,
                                 int(q_row0), float(scale), wl, wr, _dtype_code(q), self.det,
                                 _ptr(self.ws), self.ws.numel(), _stream_handle(stream))
        _check(rc, "attn_bwd_accumulate")

    def finish(self, dq=None, scale=None, stream=None):
        """dQ (bf16, (B, H, n, d)) = scale · the dQ sum."""
        import torch
        if dq is None:
            dq = torch.empty((self.B, self.H, self.n, self.d), dtype=torch.bfloat16,
                             device=self.ws.device)
        if scale is None:
            scale = 1.0 / math.sqrt(self.d)
        _packed("BackwardSum.finish", dq, self.ws)
        _shaped("BackwardSum.finish", [(dq, (self.B, self.H, self.n, self.d), torch.bfloat16)])
        rc = attn_bwd_finish(_ptr(dq), self.B, self.H, self.n, self.d, float(scale),
                             _dtype_code(dq), self.det, _ptr(self.ws), self.ws.numel(),
                             _stream_handle(stream))
        _check(rc, "attn_bwd_finish")
        return dq


def device_status(stream=None) -> int:
    """Synchronise and return/clear the device status word (ATTN_OK or ATTN_ERR_TIMEOUT)."""
    return attn_get_device_status(_stream_handle(stream))


def ring_merge(o_acc, lse_acc, o_part, lse_part, first=False, out=None, stream=None):
    """Fold a partial (o_part, lse_part) into the running fp32 (o_acc, lse_acc) in place; with
    `out` also write the merged output there (see attn_ring_merge)."""
    import torch
    d = o_acc.shape[-1]
    rows = lse_acc.numel()
    _packed("ring_merge", o_acc, lse_acc, o_part, lse_part, out)
    _shaped("ring_merge", [(o_acc, tuple(lse_acc.shape) + (d,), torch.float32),
                           (lse_acc, lse_acc.shape, torch.float32), (o_part, o_acc.shape, None),
                           (lse_part, lse_acc.shape, torch.float32)]
            + ([(out, o_acc.shape, None)] if out is not None else []))
    rc = attn_ring_merge(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part), rows, d,
                         _dtype_code(o_part), int(bool(first)),
                         _ptr(out) if out is not None else None,
                         _dtype_code(out) if out is not None else ATTN_BF16,
                         _stream_handle(stream))
    _check(rc, "attn_ring_merge")


def ring_accumulate(acc, part=None, first=False, out=None, stream=None):
    """acc (fp32) = (0 if first else acc) + part; with `out` also write the sum there."""
    import torch
    _packed("ring_accumulate", acc, part, out)
    _shaped("ring_accumulate", [(acc, acc.shape, torch.float32)]
            + [(t, acc.shape, None) for t in (part, out) if t is not None])
    rc = attn_ring_accumulate(_ptr(acc), _ptr(part) if part is not None else None, acc.numel(),
                              _dtype_code(part) if part is not None else ATTN_BF16,
                              int(bool(first)), _ptr(out) if out is not None else None,
                              _dtype_code(out) if out is not None else ATTN_BF16,
                              _stream_handle(stream))
    _check(rc, "attn_ring_accumulate")


def forward_fp8(q, k, v, q_descale=1.0, k_descale=1.0, v_descale=1.0, causal=False, scale=None,
                out=None, lse=None, stream=None, window=None):
    """O (bf16), LSE of attention with E4M3 inputs: q, k, v are torch.float8_e4m3fn (or uint8
    holding E4M3 bytes) CUDA tensors (B,H,nq,d) / (B,Hkv,nk,d), d in {64, 128}; the real inputs
    are q·q_descale, k·k_descale, v·v_descale. Masks as `forward`."""
    import torch
    for t in (q, k, v):
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise ValueError("forward_fp8 expects float8_e4m3fn (or uint8) tensors")
    B, H, n, d = _dims(q)
    kd = _dims(k)
    if v.shape != k.shape or kd[0] != B or kd[3] != d or H % kd[1] != 0:
        raise ValueError("k, v must be (B, Hkv, nk, d) with H a multiple of Hkv")
    Hkv, nk = kd[1], kd[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    _packed("forward_fp8", q, k, v, out, lse)
    _shaped("forward_fp8", [(out, q.shape, torch.bfloat16),
                            (lse, (B, H, n) if q.dim() == 4 else (n,), torch.float32)])
    wl, wr = _window(causal, window)
    rc = attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, n, nk, d,
                      float(scale), wl, wr, float(q_descale), float(k_descale), float(v_descale),
                      _stream_handle(stream))
    _check(rc, "attn_fwd_fp8")
    return out, lse
