"""GPU parity of the forward pass folded over key sets (attn_fwd_accumulate): attention over
disjoint key ranges, each folded into the running fp32 (O, LSE) inside the forward kernel, must
equal the oracle's attention over all keys ("Attention Mechanism ...", §16 Ring Attention; the
running-maximum rescaling of "Flash Attention Nedir?", Online Softmax, applied across launches)."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_LSE, TOL_O, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402


def _fold(q, k, v, cuts, causal, order=None):
    n, nk = q.shape[2], k.shape[2]
    scale = 1.0 / math.sqrt(q.shape[-1])
    o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    ranges = list(zip(cuts[:-1], cuts[1:]))
    for idx, r in enumerate(order or range(len(ranges))):
        a, b = ranges[r]
        # query i sees global key a + j iff a + j <= i + (nk - n): window_right = nk - b
        ea.forward_accumulate(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), o_acc,
                              lse_acc, first=(idx == 0), scale=scale,
                              window=(-1, nk - b) if causal else None)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    return o_acc, lse_acc


@pytest.mark.parametrize("B,H,Hkv,n,nk,d,cuts,causal,order", [
    (1, 2, 2, 640, 640, 128, [0, 128, 300, 640], True, None),
    (2, 2, 2, 1000, 1000, 128, [0, 512, 1000], True, [1, 0]),   # later keys first
    (1, 4, 2, 300, 300, 64, [0, 100, 101, 300], True, [2, 0, 1]),
    (1, 2, 1, 257, 400, 32, [0, 200, 400], False, None),
    (1, 2, 2, 384, 384, 128, [0, 384], False, None),
])
def test_folded_forward_equals_whole_attention(cuda_device, B, H, Hkv, n, nk, d, cuts, causal,
                                               order):
    q = attn_inputs.random_draws((B, H, n, d), seed=n + d, count=1)[0]
    k, v = attn_inputs.random_draws((B, Hkv, nk, d), seed=n + d + 1, count=2)
    dev = torch.device("cuda:0")
    o, lse = _fold(q.to(dev), k.to(dev), v.to(dev), cuts, causal, order)
    ro, rlse = oracle.fwd_ex(q, k, v, 1.0 / math.sqrt(d), -1, 0 if causal else -1)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["bf16"]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["bf16"]


def test_rows_without_keys_stay_empty(cuda_device):
    """A key range that a query row never sees leaves that row's running result alone; rows
    that see no key at all end with O = 0, LSE = -inf."""
    n, d = 256, 64
    q, k, v = attn_inputs.random_draws((1, 1, n, d), seed=3, count=3)
    dev = torch.device("cuda:0")
    gq, gk, gv = q.to(dev), k.to(dev), v.to(dev)
    o_acc = torch.empty((1, 1, n, d), dtype=torch.float32, device=dev)
    lse_acc = torch.empty((1, 1, n), dtype=torch.float32, device=dev)
    # keys [128, 256) under a causal mask: rows 0..127 see none of them
    ea.forward_accumulate(gq, gk[:, :, 128:].contiguous(), gv[:, :, 128:].contiguous(), o_acc,
                          lse_acc, first=True, window=(-1, 0))
    torch.cuda.synchronize()
    assert torch.all(o_acc[0, 0, :128] == 0)
    assert torch.all(torch.isneginf(lse_acc[0, 0, :128]))
    before = o_acc.clone()
    # then keys [0, 128): every row sees some; rows 128.. combine both ranges
    ea.forward_accumulate(gq, gk[:, :, :128].contiguous(), gv[:, :, :128].contiguous(), o_acc,
                          lse_acc, first=False, window=(-1, 128))
    torch.cuda.synchronize()
    ro, rlse = oracle.fwd_ex(q, k, v, 1.0 / math.sqrt(d), -1, 0)
    assert np.abs(to_np(o_acc) - ro).max() <= TOL_O["bf16"]
    assert np.abs(to_np(lse_acc) - rlse).max() <= TOL_LSE["bf16"]
    assert not torch.equal(before, o_acc)
