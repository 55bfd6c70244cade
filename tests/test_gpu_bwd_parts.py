"""GPU parity of the backward in parts (attn_bwd_prepare / attn_bwd_accumulate / attn_bwd_finish):
with the final O and LSE, the gradients of attention over all keys are the sums of the
gradients over disjoint key sets ("Attention Mechanism ...", §16 Ring Attention; the
recomputation of "Flash Attention Nedir?"). The keys are cut into uneven ranges, each range
gets the part of the causal mask that falls on it, and the sums are compared with the oracle's
gradients over the whole sequence."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import grad_close, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402


def _run(q, k, v, do, cuts, causal, deterministic):
    """dq (bf16) and fp32 dk, dv from one prepare, one accumulate per key range, one finish."""
    n, nk = q.shape[2], k.shape[2]
    scale = 1.0 / math.sqrt(q.shape[-1])
    window = (-1, 0) if causal else None
    o, lse = ea.forward(q, k, v, scale=scale, window=window)
    bs = ea.BackwardSum(o, do, lse, deterministic=deterministic)
    dks, dvs = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        ks, vs = k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous()
        dk = torch.zeros(ks.shape, dtype=torch.float32, device=q.device)
        dv = torch.zeros_like(dk)
        # query i sees global key a + j iff a + j <= i + (nk - n): within the range that is
        # j <= i + (b - a) - n + (nk - b), i.e. window_right = nk - b
        bs.add(q, ks, vs, do, dk, dv, scale=scale, window=(-1, nk - b) if causal else None)
        dks.append(dk)
        dvs.append(dv)
    dq = bs.finish(scale=scale)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    return dq, torch.cat(dks, 2), torch.cat(dvs, 2)


@pytest.mark.parametrize("B,H,Hkv,n,nk,d,cuts,causal", [
    (1, 2, 2, 640, 640, 128, [0, 128, 300, 640], True),
    (2, 2, 2, 1000, 1000, 128, [0, 512, 1000], True),
    (1, 4, 2, 300, 300, 64, [0, 100, 101, 300], True),
    (1, 2, 1, 257, 400, 32, [0, 200, 400], False),
    (1, 2, 2, 384, 384, 128, [0, 384], False),
])
def test_parts_sum_to_the_whole_gradient(cuda_device, B, H, Hkv, n, nk, d, cuts, causal):
    q, do = attn_inputs.random_draws((B, H, n, d), seed=n + d, count=2)
    k, v = attn_inputs.random_draws((B, Hkv, nk, d), seed=n + d + 1, count=2)
    dev = torch.device("cuda:0")
    gq, gk, gv, gdo = (x.to(dev) for x in (q, k, v, do))
    for det in (False, True):
        dq, dk, dv = _run(gq, gk, gv, gdo, cuts, causal, det)
        rq, rk, rv = oracle.bwd_ex(q, k, v, do, 1.0 / math.sqrt(d), -1, 0 if causal else -1)
        assert grad_close(to_np(dq), rq)
        assert grad_close(to_np(dk), rk)
        assert grad_close(to_np(dv), rv)


def test_parts_deterministic_repeat_is_bitwise(cuda_device):
    q, k, v, do = attn_inputs.random_draws((1, 2, 1024, 128), seed=77, count=4)
    dev = torch.device("cuda:0")
    args = [x.to(dev) for x in (q, k, v, do)]
    first = _run(*args, [0, 256, 700, 1024], True, True)
    again = _run(*args, [0, 256, 700, 1024], True, True)
    for a, b in zip(first, again):
        assert torch.equal(a, b)


def test_parts_match_the_single_call(cuda_device):
    """One key range with the whole mask is attn_bwd itself (same kernels, fp32 dK / dV)."""
    q, k, v, do = attn_inputs.random_draws((1, 2, 700, 64), seed=78, count=4)
    dev = torch.device("cuda:0")
    gq, gk, gv, gdo = (x.to(dev) for x in (q, k, v, do))
    dq, dk, dv = _run(gq, gk, gv, gdo, [0, 700], True, True)
    o, lse = ea.forward(gq, gk, gv, causal=True)
    rq, rk, rv = ea.backward(gq, gk, gv, o, gdo, lse, causal=True, deterministic=True)
    torch.cuda.synchronize()
    assert torch.equal(dq, rq)
    assert torch.equal(dk.to(torch.bfloat16), rk)
    assert torch.equal(dv.to(torch.bfloat16), rv)


@pytest.mark.parametrize("d", [64, 128])
def test_parts_on_views_of_the_whole_sequence(cuda_device, d):
    """Query and key row ranges passed as views (no copies): the first 256 queries against each
    key half, the last 256 against all keys (workspace rows from 256), unmasked; the sums equal
    the whole gradient, and the folded forward on the same views equals the whole forward."""
    n = 512
    q, k, v, do = attn_inputs.random_draws((2, 2, n, d), seed=90 + d, count=4)
    dev = torch.device("cuda:0")
    gq, gk, gv, gdo = (x.to(dev) for x in (q, k, v, do))
    scale = 1.0 / math.sqrt(d)
    o_acc = torch.empty(gq.shape, dtype=torch.float32, device=dev)
    lse_acc = torch.empty(gq.shape[:3], dtype=torch.float32, device=dev)
    h = n // 2
    plan = [(0, h, 0, h), (0, h, h, n), (h, n, 0, n)]
    first = {0: True, h: True}
    for a0, a1, b0, b1 in plan:
        ea.forward_accumulate(gq[:, :, a0:a1], gk[:, :, b0:b1], gv[:, :, b0:b1],
                              o_acc[:, :, a0:a1], lse_acc[:, :, a0:a1], first=first[a0],
                              scale=scale)
        first[a0] = False
    torch.cuda.synchronize()
    ro, rlse = oracle.fwd_ex(q, k, v, scale, -1, -1)
    assert np.abs(to_np(o_acc) - ro).max() <= 1e-2
    assert np.abs(to_np(lse_acc) - rlse).max() <= 1e-3
    o = o_acc.to(torch.bfloat16)
    for det in (False, True):
        bs = ea.BackwardSum(o, gdo, lse_acc, deterministic=det)
        dk = torch.zeros(gk.shape, dtype=torch.float32, device=dev)
        dv = torch.zeros_like(dk)
        for a0, a1, b0, b1 in plan:
            bs.add(gq[:, :, a0:a1], gk[:, :, b0:b1], gv[:, :, b0:b1], gdo[:, :, a0:a1],
                   dk[:, :, b0:b1], dv[:, :, b0:b1], scale=scale, q_row0=a0)
        dq = bs.finish(scale=scale)
        torch.cuda.synchronize()
        assert ea.device_status() == ea.ATTN_OK
        rq, rk, rv = oracle.bwd_ex(q, k, v, do, scale, -1, -1)
        assert grad_close(to_np(dq), rq)
        assert grad_close(to_np(dk), rk)
        assert grad_close(to_np(dv), rv)
