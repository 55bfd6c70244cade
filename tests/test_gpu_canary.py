"""Out-of-bounds write check without a sanitizer: every output (O, LSE, dQ, dK, dV, and the
backward workspace) is placed inside a larger buffer whose guard bands before and after it hold a
fixed byte pattern; after the call the guard bands must be untouched. Odd and ragged shapes,
every head dimension, masks, grouped-query heads and the FP8 and ring entry points."""
import math

import pytest
import torch

import attn_inputs

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402

GUARD = 4096            # bytes on each side (a multiple of 256, so alignment is kept)
PATTERN = 0xA5


def _guarded(shape, dtype, dev):
    """A tensor of `shape` inside a buffer with GUARD bytes of PATTERN before and after it."""
    itemsize = torch.empty((), dtype=dtype).element_size()
    numel = math.prod(shape)
    raw = torch.full((2 * GUARD + numel * itemsize,), PATTERN, dtype=torch.uint8, device=dev)
    inner = raw[GUARD:GUARD + numel * itemsize].view(dtype).view(shape)
    return raw, inner


def _guards_intact(raw):
    return bool(torch.all(raw[:GUARD] == PATTERN)) and bool(torch.all(raw[-GUARD:] == PATTERN))


CASES = [  # (B, H, Hkv, nq, nk, d, window)
    (1, 1, 1, 1, 1, 128, (-1, 0)), (1, 2, 2, 2, 2, 64, (-1, -1)), (2, 1, 1, 17, 17, 32, (-1, 0)),
    (1, 3, 3, 127, 127, 128, (-1, -1)), (1, 2, 2, 129, 129, 64, (-1, 0)),
    (1, 2, 1, 1000, 1000, 128, (30, 5)), (1, 2, 2, 300, 77, 32, (-1, 0)),
    (1, 4, 2, 77, 300, 128, (-1, -1)), (1, 2, 2, 640, 640, 64, (0, 0)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}kv{}_q{}k{}_d{}".format(*c[:6]))
@pytest.mark.parametrize("det", [False, True])
def test_no_write_outside_outputs(cuda_device, case, det):
    B, H, Hkv, nq, nk, d, window = case
    dev = torch.device("cuda:0")
    q, do = (x.to(dev) for x in attn_inputs.random_draws((B, H, nq, d), seed=nq, count=2))
    k, v = (x.to(dev) for x in attn_inputs.random_draws((B, Hkv, nk, d), seed=nk + 1, count=2))
    ro, o = _guarded((B, H, nq, d), torch.bfloat16, dev)
    rl, lse = _guarded((B, H, nq), torch.float32, dev)
    ea.forward(q, k, v, window=window, out=o, lse=lse)
    rdq, dq = _guarded((B, H, nq, d), torch.bfloat16, dev)
    rdk, dk = _guarded((B, Hkv, nk, d), torch.bfloat16, dev)
    rdv, dv = _guarded((B, Hkv, nk, d), torch.bfloat16, dev)
    need = ea.attn_bwd_workspace_bytes(B, H, nq, d, int(det))
    rws, ws = _guarded((need,), torch.uint8, dev)
    ea.backward(q, k, v, o, do, lse, window=window, deterministic=det, dq=dq, dk=dk, dv=dv,
                workspace=ws)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    for name, raw in (("o", ro), ("lse", rl), ("dq", rdq), ("dk", rdk), ("dv", rdv), ("ws", rws)):
        assert _guards_intact(raw), name
    assert torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()


@pytest.mark.parametrize("d", [64, 128])
def test_no_write_outside_outputs_fp8_and_fp32(cuda_device, d):
    dev = torch.device("cuda:0")
    shape = (1, 2, 333, d)
    x8 = (torch.randn(shape, device=dev) * 4).to(torch.float8_e4m3fn)
    ro, o = _guarded(shape, torch.bfloat16, dev)
    rl, lse = _guarded(shape[:3], torch.float32, dev)
    ea.forward_fp8(x8, x8, x8, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert _guards_intact(ro) and _guards_intact(rl)
    q, k, v = (x.to(dev) for x in attn_inputs.random_draws(shape, dtype="fp32", seed=d, count=3))
    ro32, o32 = _guarded(shape, torch.float32, dev)
    rl32, l32 = _guarded(shape[:3], torch.float32, dev)
    ea.forward(q, k, v, causal=True, out=o32, lse=l32)
    torch.cuda.synchronize()
    assert _guards_intact(ro32) and _guards_intact(rl32)
    assert ea.device_status() == ea.ATTN_OK


def test_no_write_outside_ring_buffers(cuda_device):
    dev = torch.device("cuda:0")
    rows, d = 300, 64
    racc, acc = _guarded((rows, d), torch.float32, dev)
    rlse, lacc = _guarded((rows,), torch.float32, dev)
    rout, out = _guarded((rows, d), torch.bfloat16, dev)
    part = torch.randn(rows, d, device=dev).to(torch.bfloat16)
    lpart = torch.randn(rows, device=dev)
    ea.ring_merge(acc, lacc, part, lpart, first=True)
    ea.ring_merge(acc, lacc, part, lpart, first=False, out=out)
    rsum, s = _guarded((rows * d,), torch.float32, dev)
    ea.ring_accumulate(s, part.reshape(-1), first=True, out=None)
    torch.cuda.synchronize()
    for raw in (racc, rlse, rout, rsum):
        assert _guards_intact(raw)
