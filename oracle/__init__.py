"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm may
import this package. It shares no code with the CUDA library (``exact_attention_138_b200``) and
neither imports the other.

The arithmetic lives in ``attn_oracle.c`` (plain loops, fp64, OpenMP over independent rows);
this module builds it with gcc when needed and marshals numpy arrays through ctypes. One
function, ``bwd_key_rows_batched``, is numpy instead: the same derivative with fp64 matrix
products over batches of query rows, for sequences where the C loops would take days. Inputs are
passed as float32 arrays: fp32 inputs and bf16-rounded inputs are both represented exactly in
float32 and are widened to float64 inside the C code.

Sources of each function are cited in ``attn_oracle.c``:
  * "Attention Mechanism: Revolusi Representasi Sequence", §3 Steps 1-4 and §4.4 (definition,
    causal mask), §13 "FlashAttention — How It Works" (online softmax recurrence);
  * "Efficient Attention", efficient_attention.py part 3 (row tiling in 128-row blocks);
  * "Flash Attention Nedir?", "Online Softmax" (log-sum-exp statistic);
  * "Apa itu FlashAttention", "Cara kerja teknik Tiling dan Recomputation" (backward recomputes
    the softmax; the gradient formulas are the exact derivative of the definition);
  * "Calculateur de mémoire d'attention", "La formule" (score-matrix bytes B·H·n²·e).
  * "Attention Mechanism ...", §12 "GQA vs MQA — KV Cache Optimization": query heads in groups of
    g = H / H_kv share one K/V head; the page expands K and V with repeat_interleave(g, dim=1)
    and then runs standard attention, which is exactly what fwd_gqa / bwd_gqa do.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so (plain -O2, portable x86-64/aarch64 code)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        try:
            lib = ctypes.CDLL(build())
        except OSError:
            lib = ctypes.CDLL(build(force=True))
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        I, D = ctypes.c_int, ctypes.c_double
        lib.oracle_fwd.argtypes = [f32p, f32p, f32p, I, I, I, I, D, I, f64p, f64p]
        lib.oracle_fwd_rowtiled.argtypes = [f32p, f32p, f32p, I, I, I, I, D, I, I, f64p, f64p]
        lib.oracle_fwd_online.argtypes = [f32p, f32p, f32p, I, I, I, I, D, I, I, I, f64p, f64p]
        lib.oracle_fwd_rows.argtypes = [f32p, f32p, f32p, I, I, I, I, D, I, i64p, I, f64p, f64p]
        lib.oracle_bwd.argtypes = [f32p, f32p, f32p, f32p, I, I, I, I, D, I, f64p, f64p, f64p,
                                   f64p]
        lib.oracle_bwd_query_rows.argtypes = [f32p, f32p, f32p, f32p, I, I, I, I, D, I, i64p, I,
                                              f64p, f64p]
        lib.oracle_bwd_key_rows.argtypes = [f32p, f32p, f32p, f32p, I, I, I, I, D, I,
                                            ctypes.c_long, i32p, I, f64p, f64p]
        lib.oracle_fwd_ex.argtypes = [f32p, f32p, f32p, I, I, I, I, I, D, I, I, f64p, f64p]
        lib.oracle_bwd_ex.argtypes = [f32p, f32p, f32p, f32p, I, I, I, I, I, D, I, I, f64p, f64p,
                                      f64p]
        lib.oracle_score_matrix_bytes.argtypes = [D, D, D, D]
        lib.oracle_score_matrix_bytes.restype = D
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        for name in ("oracle_fwd", "oracle_fwd_rowtiled", "oracle_fwd_online", "oracle_fwd_rows",
                     "oracle_bwd", "oracle_bwd_query_rows", "oracle_bwd_key_rows", "oracle_fwd_ex",
                     "oracle_bwd_ex"):
            getattr(lib, name).restype = I
        _lib = lib
        return lib


def _f32(x) -> np.ndarray:
    """Accept numpy arrays or CPU torch tensors (fp32 or bf16); return contiguous float32."""
    if hasattr(x, "detach"):  # torch tensor: widen exactly to fp32 on the CPU
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _shape4(q):
    if q.ndim == 2:
        return 1, 1, q.shape[0], q.shape[1]
    if q.ndim != 4:
        raise ValueError("expected (B,H,n,d) or (n,d)")
    return q.shape


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed with code {rc}")


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(t: int) -> None:
    _load().oracle_set_num_threads(int(t))


def score_matrix_bytes(B, H, n, e) -> int:
    """Bytes of the materialised score matrix, B·H·n²·e."""
    return int(round(_load().oracle_score_matrix_bytes(B, H, n, e)))


def fwd(q, k, v, scale, causal=False):
    """Definition with the full score matrix of each (b,h). Returns (O fp64, LSE fp64)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, n, d = _shape4(q)
    o = np.empty(q.shape, np.float64)
    lse = np.empty(q.shape[:-1], np.float64)
    _check(_load().oracle_fwd(q, k, v, B, H, n, d, float(scale), int(bool(causal)), o, lse),
           "oracle_fwd")
    return o, lse


def fwd_rowtiled(q, k, v, scale, causal=False, block_rows=128):
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, n, d = _shape4(q)
    o = np.empty(q.shape, np.float64)
    lse = np.empty(q.shape[:-1], np.float64)
    _check(_load().oracle_fwd_rowtiled(q, k, v, B, H, n, d, float(scale), int(bool(causal)),
                                       int(block_rows), o, lse), "oracle_fwd_rowtiled")
    return o, lse


def fwd_online(q, k, v, scale, causal=False, block_cols=128, literal_page_form=False):
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, n, d = _shape4(q)
    o = np.empty(q.shape, np.float64)
    lse = np.empty(q.shape[:-1], np.float64)
    _check(_load().oracle_fwd_online(q, k, v, B, H, n, d, float(scale), int(bool(causal)),
                                     int(block_cols), int(bool(literal_page_form)), o, lse),
           "oracle_fwd_online")
    return o, lse


def fwd_rows(q, k, v, scale, causal, rows):
    """O and LSE for flat row indices rows[t] = (b*H + h)*n + i."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, n, d = _shape4(q)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((len(rows), d), np.float64)
    lse = np.empty(len(rows), np.float64)
    _check(_load().oracle_fwd_rows(q, k, v, B, H, n, d, float(scale), int(bool(causal)), rows,
                                   len(rows), o, lse), "oracle_fwd_rows")
    return o, lse


def bwd(q, k, v, do, scale, causal=False):
    """Exact derivative. Returns (dQ, dK, dV, D) in fp64."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, H, n, d = _shape4(q)
    dq = np.empty(q.shape, np.float64)
    dk = np.empty(q.shape, np.float64)
    dv = np.empty(q.shape, np.float64)
    D = np.empty(q.shape[:-1], np.float64)
    _check(_load().oracle_bwd(q, k, v, do, B, H, n, d, float(scale), int(bool(causal)), dq, dk,
                              dv, D), "oracle_bwd")
    return dq, dk, dv, D


def bwd_query_rows(q, k, v, do, scale, causal, rows):
    """dQ (and D) for flat query rows rows[t] = bh*n + i."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, H, n, d = _shape4(q)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dq = np.empty((len(rows), d), np.float64)
    D = np.empty(len(rows), np.float64)
    _check(_load().oracle_bwd_query_rows(q, k, v, do, B, H, n, d, float(scale),
                                         int(bool(causal)), rows, len(rows), dq, D),
           "oracle_bwd_query_rows")
    return dq, D


def bwd_key_rows(q, k, v, do, scale, causal, bh, keys):
    """dK and dV for key rows `keys` (indices within one head) of head bh = b*H + h."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, H, n, d = _shape4(q)
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int32))
    dk = np.empty((len(keys), d), np.float64)
    dv = np.empty((len(keys), d), np.float64)
    _check(_load().oracle_bwd_key_rows(q, k, v, do, B, H, n, d, float(scale), int(bool(causal)),
                                       int(bh), keys, len(keys), dk, dv), "oracle_bwd_key_rows")
    return dk, dv


def bwd_key_rows_batched(q, k, v, do, scale, causal, bh, keys, block_rows=256):
    """dK and dV for key rows `keys` of head bh, for sequences too long for ``bwd_key_rows``.

    Same derivative as ``bwd_key_rows`` (the exact gradient of "Attention Mechanism ...", §3
    Steps 1-4 with the causal mask of §4.4; the pages only say that the backward pass recomputes
    the softmax: "Apa itu FlashAttention", "Cara kerja teknik Tiling dan Recomputation", item 2),
    but every query row's score row, softmax and dP row come from an fp64 matrix product
    (numpy matmul, a library primitive) over a batch of `block_rows` query rows at a time — the
    row batching of "Efficient Attention" (efficient_attention.py, part 3), which changes no
    row's arithmetic. The C loops of ``bwd_key_rows`` stream all of K for every query row, which
    at n = 131072 is petabytes of memory traffic; this form does the same steps in minutes.

    Per batch of query rows i in [r0, r1), in fp64:
      1. S = scale · Q_rows · K^T over keys j < r1 under the causal mask (keys j >= r1 are masked
         for every row of the batch: their P entries are exactly 0 and drop out of every sum);
         over all keys otherwise; then S_ij = -inf for j > i when causal.
      2. m_i = max_j S_ij, P_ij = exp(S_ij - m_i) / sum_j exp(S_ij - m_i)   (full rows).
      3. dP = dO_rows · V^T;  D_i = sum_j P_ij dP_ij;  dS = P ∘ (dP - D).
      4. for each sampled key t: dK_t += scale · sum_i dS_it q_i,  dV_t += sum_i P_it dO_i.
    Returns (dK rows, dV rows), each (len(keys), d) fp64.
    """
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, H, n, d = _shape4(q)
    bh = int(bh)
    if not (0 <= bh < B * H):
        raise ValueError("head index out of range")
    keys = np.asarray(keys, dtype=np.int64)
    if keys.size < 1 or keys.min() < 0 or keys.max() >= n:
        raise ValueError("key index out of range")
    Q = q.reshape(B * H, n, d)[bh].astype(np.float64)
    K = k.reshape(B * H, n, d)[bh].astype(np.float64)
    V = v.reshape(B * H, n, d)[bh].astype(np.float64)
    dO = do.reshape(B * H, n, d)[bh].astype(np.float64)
    dk = np.zeros((keys.size, d), np.float64)
    dv = np.zeros((keys.size, d), np.float64)
    r_start = int(keys.min()) if causal else 0      # rows i < min key see none of the keys
    for r0 in range(r_start, n, block_rows):
        r1 = min(n, r0 + block_rows)
        kend = r1 if causal else n
        S = (Q[r0:r1] @ K[:kend].T) * scale                              # step 1
        if causal:
            rows = np.arange(r0, r1)[:, None]
            S[np.arange(kend)[None, :] > rows] = -np.inf
        m = S.max(axis=1, keepdims=True)                                 # step 2
        P = np.exp(S - m)
        P /= P.sum(axis=1, keepdims=True)
        dP = dO[r0:r1] @ V[:kend].T                                      # step 3
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        sel = keys < kend                                                # step 4
        if sel.any():
            cols = keys[sel]
            dk[sel] += scale * (dS[:, cols].T @ Q[r0:r1])
            dv[sel] += P[:, cols].T @ dO[r0:r1]
    return dk, dv


# ---------------------------------------------------------------------------------------------
# Grouped-query attention ("Attention Mechanism ...", §12): K, V have H_kv heads; query head h
# uses K/V head h // (H // H_kv). Forward and backward run on the expanded K/V (the page's
# repeat_interleave step); the gradient of a shared K/V head is the sum over its query heads.
# ---------------------------------------------------------------------------------------------
def _expand_kv(x, H):
    x = _f32(x)
    B, Hkv = x.shape[0], x.shape[1]
    if H % Hkv != 0:
        raise ValueError("H must be a multiple of H_kv")
    return np.ascontiguousarray(np.repeat(x, H // Hkv, axis=1))


def fwd_gqa(q, k, v, scale, causal=False):
    q = _f32(q)
    H = q.shape[1]
    return fwd(q, _expand_kv(k, H), _expand_kv(v, H), scale, causal)


def bwd_gqa(q, k, v, do, scale, causal=False):
    """Returns (dQ with H heads, dK and dV with H_kv heads, D)."""
    q = _f32(q)
    B, H, n, d = q.shape
    Hkv = _f32(k).shape[1]
    dq, dk, dv, D = bwd(q, _expand_kv(k, H), _expand_kv(v, H), do, scale, causal)
    g = H // Hkv
    dk = dk.reshape(B, Hkv, g, n, d).sum(axis=2)
    dv = dv.reshape(B, Hkv, g, n, d).sum(axis=2)
    return dq, dk, dv, D


# ---------------------------------------------------------------------------------------------
# Mask and shape variants ("Attention Mechanism ...", §4.5 sliding window ±w; §4.2 cross-attention
# with different query / key lengths). Query i is aligned with key i + (nk - nq); key j is visible
# iff (i + off) - wl <= j <= (i + off) + wr, negative = unbounded. Rows that see no key: O = 0,
# LSE = -inf. Optional kv heads (grouped-query) follow the repeat_interleave recipe.
# ---------------------------------------------------------------------------------------------
def fwd_ex(q, k, v, scale, window_left=-1, window_right=-1):
    q = _f32(q)
    H = q.shape[1]
    k, v = _expand_kv(k, H), _expand_kv(v, H)
    B, _, nq, d = q.shape
    nk = k.shape[2]
    o = np.empty(q.shape, np.float64)
    lse = np.empty(q.shape[:-1], np.float64)
    _check(_load().oracle_fwd_ex(q, k, v, B, H, nq, nk, d, float(scale), int(window_left),
                                 int(window_right), o, lse), "oracle_fwd_ex")
    return o, lse


def bwd_ex(q, k, v, do, scale, window_left=-1, window_right=-1):
    """(dQ, dK, dV): dK, dV with k's head count (summed over grouped query heads)."""
    q, do = _f32(q), _f32(do)
    B, H, nq, d = q.shape
    Hkv = _f32(k).shape[1]
    ke, ve = _expand_kv(k, H), _expand_kv(v, H)
    nk = ke.shape[2]
    dq = np.empty(q.shape, np.float64)
    dk = np.empty(ke.shape, np.float64)
    dv = np.empty(ke.shape, np.float64)
    _check(_load().oracle_bwd_ex(q, ke, ve, do, B, H, nq, nk, d, float(scale), int(window_left),
                                 int(window_right), dq, dk, dv), "oracle_bwd_ex")
    g = H // Hkv
    return dq, dk.reshape(B, Hkv, g, nk, d).sum(2), dv.reshape(B, Hkv, g, nk, d).sum(2)
