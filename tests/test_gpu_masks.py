"""GPU parity of the mask and shape variants against the fp64 oracle: sliding windows
("Attention Mechanism ...", §4.5 "Sparse Attention"), cross-attention with different query and
key lengths (§4.2), causal masks on unequal lengths (last query aligned with the last key), and
their combination with grouped-query heads. Element-by-element over the whole output, forward
(bf16 and fp32) and backward (bf16, atomic and deterministic dQ)."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_LSE, TOL_O, grad_close, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402  (after the marker: GPU tests only)

# (B, H, Hkv, nq, nk, d, window_left, window_right)
CASES = [
    (1, 2, 2, 300, 300, 64, 5, 5),          # the page's ±w window, tiny w
    (1, 2, 2, 700, 700, 128, 100, 100),
    (1, 2, 2, 640, 640, 128, 128, 0),       # causal window of 129 keys, tile-aligned
    (1, 1, 1, 1000, 1000, 64, 0, 0),        # each query sees only its own key
    (1, 2, 2, 513, 513, 32, 127, 130),
    (2, 2, 2, 256, 777, 128, -1, 0),        # cross lengths, bottom-right causal
    (1, 2, 2, 777, 256, 128, -1, 0),        # more queries than keys: first 521 rows see nothing
    (1, 2, 2, 200, 900, 64, -1, -1),        # cross-attention, no mask
    (1, 2, 2, 900, 200, 128, -1, -1),
    (1, 2, 2, 100, 1000, 128, 20, 3),       # most keys seen by no query
    (1, 2, 2, 1000, 100, 64, 3, 20),
    (1, 4, 2, 600, 600, 128, 64, 64),       # grouped-query heads with a window
    (1, 4, 1, 333, 1111, 64, 50, 0),        # multi-query, cross lengths, causal window
    (1, 2, 2, 1, 1, 128, -1, 0),
    (1, 2, 2, 1, 500, 128, 10, 10),         # one query, a window in the middle of the keys
]


def _ids(c):
    return "B{}H{}kv{}_q{}k{}_d{}_w{}_{}".format(*c)


def _inputs(c, dtype="bf16"):
    B, H, Hkv, nq, nk, d, wl, wr = c
    q, do = attn_inputs.random_draws((B, H, nq, d), dtype=dtype, seed=nq + 7, count=2)
    k, v = attn_inputs.random_draws((B, Hkv, nk, d), dtype=dtype, seed=nk + 11, count=2)
    return q, k, v, do, 1.0 / math.sqrt(d)


def _run_fwd(q, k, v, scale, wl, wr):
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    o, lse = ea.forward(qd, kd, vd, scale=scale, window=(wl, wr))
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    return o, lse, (qd, kd, vd)


def _check_lse(lse, rlse, tol):
    got = to_np(lse)
    empty = np.isneginf(rlse)
    assert np.array_equal(np.isneginf(got), empty)
    assert np.abs(got[~empty] - rlse[~empty]).max(initial=0.0) <= tol


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_masked_forward(cuda_device, case, dtype):
    q, k, v, _, scale = _inputs(case, dtype)
    wl, wr = case[6], case[7]
    o, lse, _ = _run_fwd(q, k, v, scale, wl, wr)
    ro, rlse = oracle.fwd_ex(q, k, v, scale, wl, wr)
    assert np.abs(to_np(o) - ro).max() <= TOL_O[dtype]
    _check_lse(lse, rlse, TOL_LSE[dtype])


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_masked_backward(cuda_device, case, det):
    q, k, v, do, scale = _inputs(case)
    wl, wr = case[6], case[7]
    o, lse, dev = _run_fwd(q, k, v, scale, wl, wr)
    dq, dk, dv = ea.backward(*dev, o, do.to(dev[0].device).contiguous(), lse, scale=scale,
                             deterministic=det, window=(wl, wr))
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    assert tuple(dk.shape) == tuple(k.shape) and tuple(dq.shape) == tuple(q.shape)
    rq, rk, rv = oracle.bwd_ex(q, k, v, do, scale, wl, wr)
    assert grad_close(to_np(dq), rq)
    assert grad_close(to_np(dk), rk)
    assert grad_close(to_np(dv), rv)
    # keys that no query sees have exactly zero gradient, and so do queries that see no key
    nq, nk = case[3], case[4]
    i = np.arange(nq)[:, None] + (nk - nq)
    j = np.arange(nk)[None, :]
    vis = np.ones((nq, nk), bool)
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    for got, dead in ((dq, ~vis.any(1)), (dk, ~vis.any(0)), (dv, ~vis.any(0))):
        assert not torch.any(got[:, :, torch.from_numpy(dead).to(got.device)])


def test_deterministic_masked_backward_is_bitwise_repeatable(cuda_device):
    case = (1, 4, 2, 900, 1300, 128, 200, 50)
    q, k, v, do, scale = _inputs(case)
    o, lse, dev = _run_fwd(q, k, v, scale, 200, 50)
    dod = do.to(dev[0].device).contiguous()
    first = ea.backward(*dev, o, dod, lse, scale=scale, deterministic=True, window=(200, 50))
    for _ in range(3):
        again = ea.backward(*dev, o, dod, lse, scale=scale, deterministic=True, window=(200, 50))
        for a, b in zip(first, again):
            assert torch.equal(a, b)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK


@pytest.mark.parametrize("d", [32, 64, 128])
def test_ex_entry_with_causal_window_equals_causal_entry(cuda_device, d):
    # (-1, 0) on equal lengths through attn_fwd_ex / attn_bwd_ex is the causal path, bit for bit
    q, k, v, do = attn_inputs.random_draws((1, 2, 517, d), seed=d, count=4)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (x.to(dev).contiguous() for x in (q, k, v, do))
    o1, l1 = ea.forward(qd, kd, vd, causal=True)
    o2, l2 = ea.forward(qd, kd, vd, window=(-1, 0))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = ea.backward(qd, kd, vd, o1, dod, l1, causal=True, deterministic=True)
    g2 = ea.backward(qd, kd, vd, o2, dod, l2, window=(-1, 0), deterministic=True)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_sliding_window_long_sequence(cuda_device):
    # a long sequence with a narrow causal window: most (query tile, key tile) pairs are skipped
    B, H, n, d, w = 1, 4, 16384, 128, 512
    q, k, v, do = attn_inputs.random_draws((B, H, n, d), seed=77, count=4)
    scale = 1.0 / math.sqrt(d)
    o, lse, dev = _run_fwd(q, k, v, scale, w, 0)
    # compare a block of rows in the middle and the first rows against the oracle on the keys
    # they can see (rows r0..r1 see keys r0-w..r1; align the sub-problem's last query to its last key)
    for r0, r1 in ((0, 300), (9000, 9300), (n - 200, n)):
        k0 = max(0, r0 - w)
        ro, rlse = oracle.fwd_ex(q[:, :, r0:r1], k[:, :, k0:r1], v[:, :, k0:r1], scale, w, 0)
        assert np.abs(to_np(o[:, :, r0:r1]) - ro).max() <= TOL_O["bf16"]
        _check_lse(lse[:, :, r0:r1], rlse, TOL_LSE["bf16"])
    dq, dk, dv = ea.backward(*dev, o, do.to(dev[0].device).contiguous(), lse, scale=scale,
                             window=(w, 0))
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    # dQ of rows r0..r1 depends only on keys r0-w..r1; dK/dV of keys c0..c1 only on queries c0..c1+w
    r0, r1 = 9000, 9200
    k0 = r0 - w
    rq, _, _ = oracle.bwd_ex(q[:, :, r0:r1], k[:, :, k0:r1], v[:, :, k0:r1], do[:, :, r0:r1], scale,
                             w, 0)
    assert grad_close(to_np(dq[:, :, r0:r1]), rq)
    c0, c1 = 4000, 4150
    qs = slice(c0, c1 + w)
    # sub-problem: queries c0..c1+w, keys c0-w..c1+w; keep only the key rows c0..c1 (whose every
    # query lies inside the sub-problem)
    ks = slice(c0 - w, c1 + w)
    _, rk, rv = oracle.bwd_ex(q[:, :, qs], k[:, :, ks], v[:, :, ks], do[:, :, qs], scale, w, 0)
    assert grad_close(to_np(dk[:, :, c0:c1]), rk[:, :, w:w + (c1 - c0)])
    assert grad_close(to_np(dv[:, :, c0:c1]), rv[:, :, w:w + (c1 - c0)])
