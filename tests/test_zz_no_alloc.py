"""GPU test of attn_bwd_noalloc, the backward entry point that needs no caller workspace (for
callers that cannot allocate device memory where they run the backward pass). It must give the
same gradients as attn_bwd, call after call, since its fixed scratch array keeps the previous
call's contents. This file is collected last on purpose."""
import ctypes
import math

import numpy as np
import pytest
import torch

import attn_inputs
import exact_attention_138_b200 as ea
from parity_util import TOL_GRAD_REL, rel_fro

pytestmark = pytest.mark.gpu

_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


def _noalloc():
    fn = ea.library().attn_bwd_noalloc
    fn.restype = _i
    fn.argtypes = [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _i, _i, _vp]
    return fn


@pytest.mark.parametrize("shape,causal,det", [((1, 2, 300, 128), True, 0), ((2, 1, 200, 64), False, 1)])
def test_noalloc_matches_workspace_entry_point(cuda_device, shape, causal, det):
    q, k, v, do = (t.to(cuda_device) for t in attn_inputs.random_draws(shape, seed=21, count=4))
    B, H, n, d = shape
    scale = 1.0 / math.sqrt(d)
    o, lse = ea.forward(q, k, v, causal=causal, scale=scale)
    ref = ea.backward(q, k, v, o, do, lse, causal=causal, scale=scale, deterministic=bool(det))
    fn = _noalloc()
    stream = _vp(torch.cuda.current_stream().cuda_stream)
    P = lambda t: _vp(t.data_ptr())
    for _ in range(2):        # two calls in a row: the shared array holds the previous call's data
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        rc = fn(P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv), B, H, n, d, scale,
                int(causal), ea.ATTN_BF16, det, stream)
        assert rc == ea.ATTN_OK
        assert ea.device_status() == ea.ATTN_OK
        for got, want in zip((dq, dk, dv), ref):
            g = got.float().cpu().numpy().astype(np.float64)
            w = want.float().cpu().numpy().astype(np.float64)
            assert np.isfinite(g).all()
            assert rel_fro(g, w) <= TOL_GRAD_REL


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    # 1 x 64 x 8192 x 128 needs ~270 MB of scratch, far more than the 32 MiB array: rejected
    # before any launch (the pointers are never dereferenced).
    assert ea.attn_bwd_workspace_bytes(1, 64, 8192, 128, 0) > (32 << 20)
    fake = _vp(1 << 20)
    rc = _noalloc()(*([fake] * 9), 1, 64, 8192, 128, 0.088, 1, ea.ATTN_BF16, 0, None)
    assert rc == ea.ATTN_ERR_WORKSPACE
