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


@pytest.mark.parametrize("d,H,Hkv", [(32, 2, 2), (64, 2, 2), (128, 2, 2), (128, 4, 2), (64, 4, 1)])
def test_parts_on_views_of_the_whole_sequence(cuda_device, d, H, Hkv):
    """Query and key row ranges passed as views (no copies): the first 256 queries against each
    key half, the last 256 against all keys (workspace rows from 256), unmasked; the sums equal
    the whole gradient, and the folded forward on the same views equals the whole forward. Also
    with grouped-query heads (dK, dV summed over each group)."""
    n = 512
    q, do = attn_inputs.random_draws((2, H, n, d), seed=90 + d + H, count=2)
    k, v = attn_inputs.random_draws((2, Hkv, n, d), seed=91 + d + Hkv, count=2)
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


@pytest.mark.parametrize("d,H,Hkv", [(32, 3, 3), (64, 3, 1), (128, 3, 3)])
def test_query_block_that_starts_64_rows_in(cuda_device, d, H, Hkv):
    """Queries [0, 64) see keys [0, 64), queries [64, 256) all 256 keys: one launch of every
    query against the first 64 keys, one of the last 192 queries (workspace rows from 64, so a
    128-row query tile reaches 64 rows past the head's workspace rows, into the next head's and,
    for the last head, past the end) against the other keys. A query block's gradient is that of
    its own attention, so the oracle takes the two blocks apart and dK, dV are the sums; dQ of
    every head must be untouched by its neighbour's tiles."""
    n, m = 256, 64
    q, do = attn_inputs.random_draws((1, H, n, d), seed=70 + d + H, count=2)
    k, v = attn_inputs.random_draws((1, Hkv, n, d), seed=71 + d + Hkv, count=2)
    scale = 1.0 / math.sqrt(d)
    oa, la = oracle.fwd_ex(q[:, :, :m], k[:, :, :m], v[:, :, :m], scale, -1, -1)
    ob, lb = oracle.fwd_ex(q[:, :, m:], k, v, scale, -1, -1)
    dev = torch.device("cuda:0")
    gq, gk, gv, gdo = (x.to(dev) for x in (q, k, v, do))
    o = torch.from_numpy(np.concatenate([oa, ob], 2)).to(dev, torch.bfloat16)
    lse = torch.from_numpy(np.concatenate([la, lb], 2)).to(dev, torch.float32)
    aq, ak, av = oracle.bwd_ex(q[:, :, :m], k[:, :, :m], v[:, :, :m], do[:, :, :m], scale, -1, -1)
    bq, bk, bv = oracle.bwd_ex(q[:, :, m:], k, v, do[:, :, m:], scale, -1, -1)
    rq = np.concatenate([aq, bq], 2)
    rk, rv = bk.copy(), bv.copy()
    rk[:, :, :m] += ak
    rv[:, :, :m] += av
    for det in (False, True):
        bs = ea.BackwardSum(o, gdo, lse, deterministic=det)
        dk = torch.zeros(gk.shape, dtype=torch.float32, device=dev)
        dv = torch.zeros_like(dk)
        for a0, b0, b1 in ((0, 0, m), (m, m, n)):
            bs.add(gq[:, :, a0:], gk[:, :, b0:b1], gv[:, :, b0:b1], gdo[:, :, a0:],
                   dk[:, :, b0:b1], dv[:, :, b0:b1], scale=scale, q_row0=a0)
        dq = bs.finish(scale=scale)
        torch.cuda.synchronize()
        assert ea.device_status() == ea.ATTN_OK
        for h in range(H):
            assert grad_close(to_np(dq[:, h]), rq[:, h])
        assert grad_close(to_np(dk), rk)
        assert grad_close(to_np(dv), rv)


def test_query_rows_off_a_64_row_boundary_are_refused(cuda_device):
    q, k, v, do = (x.to("cuda:0") for x in attn_inputs.random_draws((1, 1, 256, 64), seed=3,
                                                                     count=4))
    o, lse = ea.forward(q, k, v)
    bs = ea.BackwardSum(o, do, lse)
    dk = torch.zeros(k.shape, dtype=torch.float32, device=q.device)
    with pytest.raises(ValueError):
        bs.add(q[:, :, 32:], k, v, do[:, :, 32:], dk, torch.zeros_like(dk), q_row0=32)
