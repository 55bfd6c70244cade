"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function that
include/attn.h declares, and rejects bad arguments before touching the device."""
import ctypes

import pytest

import exact_attention_138_b200 as ea

FAKE = 1 << 20          # an aligned, never-dereferenced pointer value (validation fails first)


def test_every_declared_function_is_exported():
    names = ea.declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_fwd_gqa", "attn_bwd_gqa", "attn_bwd_noalloc",
            "attn_fwd_ex", "attn_bwd_ex", "attn_fwd_fp8", "attn_ring_merge",
            "attn_ring_accumulate",
            "attn_bwd_workspace_bytes", "attn_get_device_status",
            "attn_error_string", "attn_version", "attn_set_wait_timeout_us",
            "attn_selftest_wait_timeout"} <= set(names)
    lib = ea.library()
    for name in names:
        assert hasattr(lib, name), name


def test_version_and_error_strings():
    assert ea.attn_version() >= 100
    for code in range(6):
        assert ea.attn_error_string(code) and ea.attn_error_string(code) != "unknown error"
    assert ea.attn_error_string(99) == "unknown error"


def test_workspace_size_formula():
    # D and LSE·log2e (fp32, per-head rows padded to 128) + dQ accumulator (fp32, same rows x d)
    n_pad = 256
    want = 2 * (2 * 3 * n_pad * 4) + 2 * 3 * n_pad * 64 * 4
    assert ea.attn_bwd_workspace_bytes(2, 3, 200, 64, 0) == want
    # deterministic: four int semaphores per 64 query rows, 6 heads x 4 tiles x 4 = 384 B -> 512
    assert ea.attn_bwd_workspace_bytes(2, 3, 200, 64, 1) == want + 512
    assert ea.attn_bwd_workspace_bytes(0, 3, 200, 64, 0) == 0


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, n=128, d=64, scale=0.125,
             causal=0, dtype=ea.ATTN_BF16, stream=None)
    a.update(kw)
    return ea.attn_fwd(*(ctypes.c_void_p(a[x]) if x in "q k v o lse".split() else a[x]
                         for x in "q k v o lse B H n d scale causal dtype stream".split()))


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), ea.ATTN_ERR_INVALID),
    (dict(lse=0), ea.ATTN_ERR_INVALID),
    (dict(n=0), ea.ATTN_ERR_INVALID),
    (dict(n=2**31 - 200), ea.ATTN_ERR_INVALID),     # tile arithmetic would overflow
    (dict(B=0), ea.ATTN_ERR_INVALID),
    (dict(H=-1), ea.ATTN_ERR_INVALID),
    (dict(scale=0.0), ea.ATTN_ERR_INVALID),
    (dict(scale=float("inf")), ea.ATTN_ERR_INVALID),
    (dict(scale=float("nan")), ea.ATTN_ERR_INVALID),
    (dict(d=48), ea.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), ea.ATTN_ERR_UNSUPPORTED),
    (dict(dtype=7), ea.ATTN_ERR_UNSUPPORTED),
    (dict(v=FAKE + 8), ea.ATTN_ERR_INVALID),       # not 16-byte aligned
    (dict(o=FAKE + 2), ea.ATTN_ERR_INVALID),
])
def test_forward_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


def _bwd(**kw):
    a = dict(B=1, H=2, n=300, d=128, scale=0.1, causal=1, dtype=ea.ATTN_BF16, det=0)
    a.update(kw)
    ptrs = [ctypes.c_void_p(kw.get(p, FAKE)) for p in "q k v o dO lse dq dk dv".split()]
    need = ea.attn_bwd_workspace_bytes(a["B"], a["H"], a["n"], a["d"], a["det"]) if a["B"] > 0 else 0
    ws = kw.get("ws", FAKE)
    ws_bytes = kw.get("ws_bytes", need)
    return ea.attn_bwd(*ptrs, a["B"], a["H"], a["n"], a["d"], a["scale"], a["causal"], a["dtype"],
                       a["det"], ctypes.c_void_p(ws), ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dO=0), ea.ATTN_ERR_INVALID),
    (dict(dv=0), ea.ATTN_ERR_INVALID),
    (dict(dtype=ea.ATTN_FP32), ea.ATTN_ERR_UNSUPPORTED),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(ws=0), ea.ATTN_ERR_INVALID),
    (dict(ws=FAKE + 16), ea.ATTN_ERR_INVALID),      # workspace must be 256-byte aligned
    (dict(ws_bytes=1000), ea.ATTN_ERR_WORKSPACE),
    (dict(n=0), ea.ATTN_ERR_INVALID),
    (dict(dq=FAKE + 4), ea.ATTN_ERR_INVALID),
])
def test_backward_rejects_bad_arguments(kw, code):
    assert _bwd(**kw) == code


def test_selftest_rejects_bad_limit():
    assert ea.attn_selftest_wait_timeout(0) == ea.ATTN_ERR_INVALID
    assert ea.attn_selftest_wait_timeout(20_000_000) == ea.ATTN_ERR_INVALID


def test_timeout_setter_roundtrip():
    old = ea.attn_set_wait_timeout_us(5)
    assert ea.attn_set_wait_timeout_us(old) == 100      # raised to the 100 us floor


def test_gqa_rejects_head_counts_that_do_not_divide():
    a = [ctypes.c_void_p(FAKE)] * 5
    assert ea.attn_fwd_gqa(*a, 1, 6, 4, 128, 64, 0.125, 0, ea.ATTN_BF16, None) == ea.ATTN_ERR_INVALID
    assert ea.attn_fwd_gqa(*a, 1, 6, 0, 128, 64, 0.125, 0, ea.ATTN_BF16, None) == ea.ATTN_ERR_INVALID
    need = ea.attn_bwd_workspace_bytes(1, 6, 128, 64, 0)
    b = [ctypes.c_void_p(FAKE)] * 9
    assert ea.attn_bwd_gqa(*b, 1, 6, 4, 128, 64, 0.125, 0, ea.ATTN_BF16, 0, ctypes.c_void_p(FAKE),
                           need, None) == ea.ATTN_ERR_INVALID


def test_ex_rejects_bad_lengths_and_heads():
    a = [ctypes.c_void_p(FAKE)] * 5
    f = lambda B, H, Hkv, nq, nk, d=64: ea.attn_fwd_ex(*a, B, H, Hkv, nq, nk, d, 0.125, 4, 4,
                                                       ea.ATTN_BF16, None)
    assert f(1, 2, 2, 128, 0) == ea.ATTN_ERR_INVALID
    assert f(1, 2, 2, 128, 2**31 - 1) == ea.ATTN_ERR_INVALID
    assert f(1, 2, 2, 0, 128) == ea.ATTN_ERR_INVALID
    assert f(1, 6, 4, 128, 128) == ea.ATTN_ERR_INVALID
    assert f(1, 2, 2, 128, 64, d=80) == ea.ATTN_ERR_UNSUPPORTED
    b = [ctypes.c_void_p(FAKE)] * 9
    need = ea.attn_bwd_workspace_bytes(1, 2, 128, 64, 0)
    g = lambda nq, nk, ws_bytes=need, dtype=ea.ATTN_BF16: ea.attn_bwd_ex(
        *b, 1, 2, 2, nq, nk, 64, 0.125, -1, 0, dtype, 0, ctypes.c_void_p(FAKE), ws_bytes, None)
    assert g(128, 0) == ea.ATTN_ERR_INVALID
    assert g(128, 64, dtype=ea.ATTN_FP32) == ea.ATTN_ERR_UNSUPPORTED
    # the workspace follows the query length
    assert g(300, 64) == ea.ATTN_ERR_WORKSPACE


def test_fp8_and_ring_entry_points_validate_before_launch():
    a = [ctypes.c_void_p(FAKE)] * 5
    fp8 = lambda d=128, qs=1.0, nk=128: ea.attn_fwd_fp8(*a, 1, 2, 2, 128, nk, d, 0.1, -1, 0, qs,
                                                        1.0, 1.0, None)
    assert fp8(d=32) == ea.ATTN_ERR_UNSUPPORTED
    assert fp8(qs=0.0) == ea.ATTN_ERR_INVALID
    assert fp8(qs=float("nan")) == ea.ATTN_ERR_INVALID
    assert fp8(nk=0) == ea.ATTN_ERR_INVALID
    f = ctypes.c_void_p(FAKE)
    assert ea.attn_ring_merge(f, f, f, f, 0, 64, ea.ATTN_BF16, 1, None, 0, None) == ea.ATTN_ERR_INVALID
    assert ea.attn_ring_merge(f, f, f, f, 8, 48, ea.ATTN_BF16, 1, None, 0, None) == ea.ATTN_ERR_UNSUPPORTED
    assert ea.attn_ring_merge(f, f, f, f, 8, 64, 9, 1, None, 0, None) == ea.ATTN_ERR_UNSUPPORTED
    assert ea.attn_ring_accumulate(f, f, 12, ea.ATTN_BF16, 0, None, 0, None) == ea.ATTN_ERR_INVALID
    assert ea.attn_ring_accumulate(ctypes.c_void_p(FAKE + 4), None, 16, 0, 0, None, 0, None) == \
        ea.ATTN_ERR_INVALID


def test_noalloc_validates_before_touching_the_device():
    # Argument errors and the 32 MiB scratch limit are reported before any CUDA call, so these
    # return their own codes on a host without a GPU.
    fn = ea.library().attn_bwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 4 + [ctypes.c_float] + \
        [ctypes.c_int] * 3 + [ctypes.c_void_p]

    def call(ptrs, B=1, H=2, n=300, d=128, scale=0.1, dtype=ea.ATTN_BF16, det=0):
        return fn(*[ctypes.c_void_p(p) for p in ptrs], B, H, n, d, scale, 1, dtype, det, None)

    ok = [FAKE] * 9
    assert call([0] + ok[1:]) == ea.ATTN_ERR_INVALID
    assert call(ok[:6] + [FAKE + 4] + ok[7:]) == ea.ATTN_ERR_INVALID
    assert call(ok, d=48) == ea.ATTN_ERR_UNSUPPORTED
    assert call(ok, dtype=ea.ATTN_FP32) == ea.ATTN_ERR_UNSUPPORTED
    assert call(ok, scale=0.0) == ea.ATTN_ERR_INVALID
    assert ea.attn_bwd_workspace_bytes(1, 64, 8192, 128, 0) > (32 << 20)
    assert call(ok, B=1, H=64, n=8192) == ea.ATTN_ERR_WORKSPACE


def _parts(which, **kw):
    """One of the three backward-part entry points with valid fake arguments, `kw` overriding."""
    a = dict(B=1, H=2, Hkv=1, nq=300, nk=500, d=128, scale=0.1, wl=-1, wr=0,
             dtype=ea.ATTN_BF16, det=1, q_rows=0, kv_rows=0, ws_rows=0, q_row0=0)
    a.update(kw)
    ws_rows = a["ws_rows"] or a["nq"]
    need = (ea.attn_bwd_workspace_bytes(a["B"], a["H"], ws_rows, a["d"], a["det"])
            if a["B"] > 0 and ws_rows > 0 else 0)
    ws = ctypes.c_void_p(kw.get("ws", FAKE))
    ws_bytes = kw.get("ws_bytes", need)
    P = lambda name: ctypes.c_void_p(kw.get(name, FAKE))
    if which == "prepare":
        return ea.attn_bwd_prepare(P("o"), P("dO"), P("lse"), a["B"], a["H"], a["nq"], a["d"],
                                   a["dtype"], a["det"], ws, ws_bytes, None)
    if which == "accumulate":
        return ea.attn_bwd_accumulate(P("q"), P("k"), P("v"), P("dO"), P("dk_acc"), P("dv_acc"),
                                      a["B"], a["H"], a["Hkv"], a["nq"], a["nk"], a["d"],
                                      a["q_rows"], a["kv_rows"], a["ws_rows"], a["q_row0"],
                                      a["scale"], a["wl"], a["wr"], a["dtype"], a["det"], ws,
                                      ws_bytes, None)
    return ea.attn_bwd_finish(P("dq"), a["B"], a["H"], a["nq"], a["d"], a["scale"], a["dtype"],
                              a["det"], ws, ws_bytes, None)


@pytest.mark.parametrize("which,kw,code", [
    ("prepare", dict(o=0), ea.ATTN_ERR_INVALID),
    ("prepare", dict(lse=FAKE + 4), ea.ATTN_ERR_INVALID),
    ("prepare", dict(dtype=ea.ATTN_FP32), ea.ATTN_ERR_UNSUPPORTED),
    ("prepare", dict(ws_bytes=1000), ea.ATTN_ERR_WORKSPACE),
    ("prepare", dict(ws=FAKE + 16), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(dk_acc=0), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(dv_acc=FAKE + 8), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(Hkv=3), ea.ATTN_ERR_INVALID),          # H not a multiple of Hkv
    ("accumulate", dict(nk=0), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(scale=-1.0), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(d=48), ea.ATTN_ERR_UNSUPPORTED),
    ("accumulate", dict(ws=0), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(ws_bytes=4096), ea.ATTN_ERR_WORKSPACE),
    ("accumulate", dict(q_rows=299), ea.ATTN_ERR_INVALID),     # heads closer than nq rows
    ("accumulate", dict(kv_rows=499), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(ws_rows=600, q_row0=301), ea.ATTN_ERR_INVALID),   # past the workspace
    ("accumulate", dict(ws_rows=600, q_row0=0), ea.ATTN_ERR_INVALID),     # ragged, not at the end
    ("accumulate", dict(q_row0=-1), ea.ATTN_ERR_INVALID),
    ("accumulate", dict(ws_rows=332, q_row0=32), ea.ATTN_ERR_INVALID),    # off a 64-row boundary
    ("finish", dict(dq=0), ea.ATTN_ERR_INVALID),
    ("finish", dict(nq=0), ea.ATTN_ERR_INVALID),
    ("finish", dict(det=0, ws_bytes=100), ea.ATTN_ERR_WORKSPACE),
])
def test_backward_parts_reject_bad_arguments(which, kw, code):
    assert _parts(which, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(o_acc=0), ea.ATTN_ERR_INVALID),
    (dict(lse_acc=FAKE + 4), ea.ATTN_ERR_INVALID),
    (dict(nk=0), ea.ATTN_ERR_INVALID),
    (dict(Hkv=3), ea.ATTN_ERR_INVALID),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), ea.ATTN_ERR_INVALID),
    (dict(q_rows=100), ea.ATTN_ERR_INVALID),
    (dict(kv_rows=-5), ea.ATTN_ERR_INVALID),
])
def test_forward_accumulate_rejects_bad_arguments(kw, code):
    a = dict(B=1, H=2, Hkv=1, nq=300, nk=500, d=128, scale=0.1, q_rows=0, kv_rows=0)
    a.update(kw)
    P = lambda name: ctypes.c_void_p(kw.get(name, FAKE))
    assert ea.attn_fwd_accumulate(P("q"), P("k"), P("v"), P("o_acc"), P("lse_acc"), a["B"], a["H"],
                                  a["Hkv"], a["nq"], a["nk"], a["d"], a["q_rows"], a["kv_rows"],
                                  a["scale"], -1, 0, 1, None) == code


def test_head_rows_of_views():
    """Rows between heads that the binding passes for views of longer sequences (0 = packed)."""
    import torch
    x = torch.zeros(2, 4, 100, 64)
    assert ea._head_rows(x) == 0
    assert ea._head_rows(x[:, :, 50:]) == 100
    assert ea._head_rows(x[:, :, :30], torch.zeros(2, 4, 100)[:, :, :30]) == 100
    assert ea._head_rows(torch.zeros(3, 1, 100, 32)[:, :, 10:20]) == 100    # H = 1: batch stride
    assert ea._head_rows(torch.zeros(1, 1, 7, 32)) == 0
    for bad in ((x.transpose(1, 2),), (x[:, :, 50:], x[:, :, :30].contiguous()),
                (x[..., :32],)):
        with pytest.raises(ValueError):
            ea._head_rows(*bad)


def test_bindings_refuse_host_and_strided_tensors():
    """The binding stops host tensors (a host pointer must never reach a kernel), strided tensors
    where the entry point takes packed ones, and buffers of the wrong size, before any C call."""
    import torch
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ea.forward(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        ea.backward(q, q, q, q, q, torch.zeros(1, 2, 64))
    with pytest.raises(ValueError, match="CUDA"):
        ea.forward_accumulate(q, q, q, torch.zeros(1, 2, 64, 64), torch.zeros(1, 2, 64))
    with pytest.raises(ValueError):
        ea.ring_accumulate(torch.zeros(16), torch.zeros(8))
    with pytest.raises(ValueError):
        ea.forward_fp8(q.to(torch.uint8), q.to(torch.uint8), q.to(torch.uint8))
    # the layout and size checks themselves
    with pytest.raises(ValueError, match="contiguous"):
        ea._packed("t", torch.zeros(4, 4).t().cuda() if torch.cuda.is_available() else _FakeCuda())
    with pytest.raises(ValueError, match="shape"):
        ea._shaped("t", [(torch.zeros(2, 3), (3, 2), None)])
    with pytest.raises(ValueError, match="expected torch.float32"):
        ea._shaped("t", [(torch.zeros(2, 3, dtype=torch.bfloat16), (2, 3), torch.float32)])


class _FakeCuda:
    """A stand-in with the attributes _packed reads: on a CUDA device, not contiguous."""
    is_cuda = True
    device = "cuda:0"

    def is_contiguous(self):
        return False
