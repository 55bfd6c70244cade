"""GPU test of attn_bwd_noalloc, the backward entry point that needs no caller workspace (for
callers that cannot allocate device memory where they run the backward pass, such as a plug-in
whose host framework owns every allocation). Its scratch is one fixed array that keeps the
previous call's contents, so the test checks call after call: against the fp64 oracle, against
attn_bwd with a workspace (bit for bit in the deterministic mode, which fixes the order of every
addition), and across calls of different sizes and modes whose leftovers (semaphores, padded D /
LSE rows, accumulator rows) sit where the next call's data goes. Outputs are NaN-filled before
each call, so a row the call fails to write shows up. This file is collected last on purpose."""
import ctypes
import math

import numpy as np
import pytest
import torch

import attn_inputs
import exact_attention_138_b200 as ea
import oracle
from parity_util import TOL_GRAD_REL, grad_close, rel_fro, to_np

pytestmark = pytest.mark.gpu

_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


def _noalloc():
    fn = ea.library().attn_bwd_noalloc
    fn.restype = _i
    fn.argtypes = [_vp] * 9 + [_i, _i, _i, _i, _f, _i, _i, _i, _vp]
    return fn


class Case:
    """Inputs on the GPU, the forward outputs, the oracle's gradients and attn_bwd's."""

    def __init__(self, device, shape, causal, det, seed):
        host = attn_inputs.random_draws(shape, seed=seed, count=4)
        self.shape, self.causal, self.det = shape, causal, det
        self.scale = 1.0 / math.sqrt(shape[-1])
        self.q, self.k, self.v, self.do = (t.to(device) for t in host)
        self.o, self.lse = ea.forward(self.q, self.k, self.v, causal=causal, scale=self.scale)
        self.want = oracle.bwd(*host, self.scale, causal)[:3]
        self.ws_result = [t.clone() for t in ea.backward(
            self.q, self.k, self.v, self.o, self.do, self.lse, causal=causal, scale=self.scale,
            deterministic=bool(det))]
        torch.cuda.synchronize()
        assert ea.device_status() == ea.ATTN_OK

    def run_noalloc(self):
        B, H, n, d = self.shape
        grads = [torch.full_like(self.q, float("nan")) for _ in range(3)]
        P = lambda t: _vp(t.data_ptr())   # noqa: E731
        rc = _noalloc()(P(self.q), P(self.k), P(self.v), P(self.o), P(self.do), P(self.lse),
                        *(P(g) for g in grads), B, H, n, d, self.scale, int(self.causal),
                        ea.ATTN_BF16, self.det, _vp(torch.cuda.current_stream().cuda_stream))
        assert rc == ea.ATTN_OK
        assert ea.device_status() == ea.ATTN_OK
        return grads

    def check(self, grads):
        for got, want, ref in zip(grads, self.want, self.ws_result):
            g = to_np(got)
            assert np.isfinite(g).all()
            assert grad_close(g, want)                      # the oracle
            if self.det:
                assert torch.equal(got, ref)                # same order of additions
            else:
                assert rel_fro(g, to_np(ref)) <= TOL_GRAD_REL


@pytest.mark.parametrize("shape,causal,det", [((1, 2, 300, 128), True, 0),
                                              ((2, 1, 200, 64), False, 1)])
def test_noalloc_matches_oracle_and_workspace_entry_point(cuda_device, shape, causal, det):
    case = Case(cuda_device, shape, causal, det, seed=21)
    for _ in range(2):        # two calls in a row: the shared array holds the previous call's data
        case.check(case.run_noalloc())


def test_noalloc_leftovers_of_other_sizes_do_not_leak(cuda_device):
    # A larger deterministic call fills semaphores, padded rows and accumulator rows far past
    # where the smaller calls that follow put theirs; the smaller ones change the layout (heads,
    # lengths, d, mask, dQ mode), and the first call is repeated at the end.
    big = Case(cuda_device, (1, 4, 2048, 128), True, 1, seed=22)
    small_atomic = Case(cuda_device, (2, 1, 300, 64), False, 0, seed=23)
    mid_det = Case(cuda_device, (1, 3, 1000, 128), True, 1, seed=24)
    assert ea.attn_bwd_workspace_bytes(1, 4, 2048, 128, 1) <= (32 << 20)
    first = big.run_noalloc()
    big.check(first)
    for case in (small_atomic, mid_det, small_atomic):
        case.check(case.run_noalloc())
    again = big.run_noalloc()
    big.check(again)
    for a, b in zip(first, again):
        assert torch.equal(a, b)


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    # 1 x 64 x 8192 x 128 needs ~270 MB of scratch, far more than the 32 MiB array: rejected
    # before any launch (the pointers are never dereferenced).
    assert ea.attn_bwd_workspace_bytes(1, 64, 8192, 128, 0) > (32 << 20)
    fake = _vp(1 << 20)
    rc = _noalloc()(*([fake] * 9), 1, 64, 8192, 128, 0.088, 1, ea.ATTN_BF16, 0, None)
    assert rc == ea.ATTN_ERR_WORKSPACE
