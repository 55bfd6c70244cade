"""GPU parity of the backward pass against the fp64 oracle (exact derivative)."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_GRAD_REL, cuda_backward, cuda_forward, grad_close, rel_fro, to_np

pytestmark = pytest.mark.gpu

SHAPES = [(1, 2, 1, 64), (2, 1, 2, 32), (1, 1, 17, 128), (1, 3, 127, 64), (2, 2, 129, 128),
          (1, 2, 300, 32), (1, 1, 1000, 128), (1, 2, 256, 128), (1, 1, 383, 64)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_backward_small_shapes(cuda_device, shape, causal):
    q, k, v, do = attn_inputs.random_draws(shape, seed=(hash(shape) + 7) % 1000, count=4)
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse, dev = cuda_forward(q, k, v, causal, scale)
    dq, dk, dv = cuda_backward(dev, o, lse, do, causal, scale)
    rq, rk, rv, _ = oracle.bwd(q, k, v, do, scale, causal)
    assert grad_close(to_np(dq), rq)
    assert grad_close(to_np(dk), rk)
    assert grad_close(to_np(dv), rv)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_deterministic_mode_is_bitwise_stable(cuda_device, causal):
    q, k, v, do = attn_inputs.random_draws((1, 4, 1000, 128), seed=11, count=4)
    scale = 1 / math.sqrt(128)
    o, lse, dev = cuda_forward(q, k, v, causal, scale)
    a = cuda_backward(dev, o, lse, do, causal, scale, deterministic=True)
    b = cuda_backward(dev, o, lse, do, causal, scale, deterministic=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    rq, rk, rv, _ = oracle.bwd(q, k, v, do, scale, causal)
    for got, want in zip(a, (rq, rk, rv)):
        assert rel_fro(to_np(got), want) <= TOL_GRAD_REL


@pytest.fixture(scope="module", params=["causal_bf16_1x32x4096x128", "causal_bf16_2x32x8192x128",
                                        "causal_bf16_1x8x131072x128"])
def full_run(request, cuda_device):
    w = attn_inputs.WORKLOADS[request.param]
    q, k, v, do = attn_inputs.workload_inputs(w)
    o, lse, dev = cuda_forward(q, k, v, True, w.scale)
    dq, dk, dv = cuda_backward(dev, o, lse, do, True, w.scale)
    yield w, (q, k, v, do), (dq, dk, dv)
    del o, lse, dev, dq, dk, dv
    torch.cuda.empty_cache()


def test_backward_full_size_sampled_query_rows(full_run):
    w, (q, k, v, do), (dq, _, _) = full_run
    rows = attn_inputs.sampled_rows(w, count=256)
    rq, _ = oracle.bwd_query_rows(q, k, v, do, w.scale, True, rows)
    idx = torch.tensor(rows, device=dq.device)
    got = to_np(dq.reshape(-1, w.d).index_select(0, idx))
    assert rel_fro(got, rq) <= TOL_GRAD_REL


def test_backward_full_size_sampled_key_rows(full_run):
    w, (q, k, v, do), (_, dk, dv) = full_run
    g = torch.Generator().manual_seed(attn_inputs.SEED)
    heads = [0, w.B * w.H - 1]
    # at n = 131072 only the last 256 keys are sampled (their queries are few enough to
    # recompute in full); elsewhere keys are drawn across the whole sequence
    lo = w.n - 256 if w.n > 16384 else 0
    got_k, got_v, want_k, want_v = [], [], [], []
    for bh in heads:
        keys = sorted(set(torch.randint(lo, w.n, (12,), generator=g).tolist() + [w.n - 1]))
        rk, rv = oracle.bwd_key_rows(q, k, v, do, w.scale, True, bh, keys)
        kk = torch.tensor(keys, device=dk.device)
        got_k.append(to_np(dk.reshape(-1, w.n, w.d)[bh].index_select(0, kk)))
        got_v.append(to_np(dv.reshape(-1, w.n, w.d)[bh].index_select(0, kk)))
        want_k.append(rk)
        want_v.append(rv)
    assert rel_fro(np.concatenate(got_k), np.concatenate(want_k)) <= TOL_GRAD_REL
    assert rel_fro(np.concatenate(got_v), np.concatenate(want_v)) <= TOL_GRAD_REL


def test_backward_full_size_invariants(full_run):
    # sum_j dV_j = sum_i dO_i (P rows sum to 1) and sum_j dK_j = 0 (dS rows sum to 0), per head
    w, (q, k, v, do), (dq, dk, dv) = full_run
    sdv = dv.float().sum(2)
    sdo = do.to(dv.device).float().sum(2)
    assert (torch.linalg.norm(sdv - sdo) / torch.linalg.norm(sdo)).item() <= TOL_GRAD_REL
    sdk = dk.float().sum(2)
    scale_ref = dk.float().abs().sum(2)
    assert (torch.linalg.norm(sdk) / torch.linalg.norm(scale_ref)).item() <= TOL_GRAD_REL
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()


@pytest.mark.parametrize("shape,Hkv,causal,det", [((1, 4, 300, 128), 2, True, False),
                                                  ((2, 8, 256, 128), 1, True, False),
                                                  ((1, 6, 200, 64), 3, False, False),
                                                  ((1, 4, 383, 128), 2, True, True),
                                                  ((1, 4, 129, 32), 4, True, False)])
def test_gqa_forward_backward(cuda_device, shape, Hkv, causal, det):
    # grouped-query attention ("Attention Mechanism ...", §12): K/V with Hkv heads, no copy
    B, H, n, d = shape
    q, do = attn_inputs.random_draws(shape, seed=31, count=2)
    k, v = attn_inputs.random_draws((B, Hkv, n, d), seed=32, count=2)
    scale = 1.0 / math.sqrt(d)
    o, lse, dev = cuda_forward(q, k, v, causal, scale)
    ro, rlse = oracle.fwd_gqa(q, k, v, scale, causal)
    assert np.abs(to_np(o) - ro).max() <= 1e-2
    assert np.abs(to_np(lse) - rlse).max() <= 1e-3
    dq, dk, dv = cuda_backward(dev, o, lse, do, causal, scale, deterministic=det)
    assert tuple(dk.shape) == (B, Hkv, n, d) and tuple(dv.shape) == (B, Hkv, n, d)
    rq, rk, rv, _ = oracle.bwd_gqa(q, k, v, do, scale, causal)
    assert grad_close(to_np(dq), rq)
    assert grad_close(to_np(dk), rk)
    assert grad_close(to_np(dv), rv)
