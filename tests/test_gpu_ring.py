"""GPU parity of ring attention's kernels: the ring schedule for N ranks run in one process
(chunks indexed instead of sent; no kernel waits on another) must equal the oracle's attention
over the whole sequence ("Attention Mechanism ...", §16 Ring Attention), forward and backward;
the merge and accumulate kernels are also checked on their own."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_LSE, TOL_O, grad_close, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402
from exact_attention_138_b200 import ring  # noqa: E402


def _split(x, world, zigzag=False):
    """Each rank's tensor: chunk p (contiguous) or chunks p and 2N-1-p (zigzag)."""
    if not zigzag:
        return [c.contiguous() for c in torch.chunk(x, world, dim=2)]
    c = torch.chunk(x, 2 * world, dim=2)
    return [torch.cat([c[p], c[2 * world - 1 - p]], dim=2).contiguous() for p in range(world)]


def _unsplit(parts, world, zigzag=False):
    if not zigzag:
        return torch.cat(parts, 2)
    halves = [torch.chunk(t, 2, dim=2) for t in parts]
    return torch.cat([halves[p][0] for p in range(world)] +
                     [halves[p][1] for p in reversed(range(world))], 2)


@pytest.mark.parametrize("world,causal,H,Hkv,n_chunk,d,zigzag", [
    (2, True, 2, 2, 384, 128, False), (4, True, 2, 2, 256, 128, False),
    (3, False, 2, 2, 300, 64, False), (4, True, 4, 2, 200, 64, False),
    (2, False, 2, 1, 512, 32, False), (8, True, 1, 1, 128, 128, False),
    (2, True, 2, 2, 384, 128, True), (4, True, 4, 2, 256, 64, True),
    (3, False, 2, 2, 300, 128, True), (8, True, 1, 1, 128, 128, True),
    (2, True, 2, 2, 256, 32, True), (4, True, 4, 1, 128, 64, True)])
def test_emulated_ring_equals_full_attention(cuda_device, world, causal, H, Hkv, n_chunk, d,
                                             zigzag):
    n = world * n_chunk
    q, do = attn_inputs.random_draws((1, H, n, d), seed=world * 10 + d, count=2)
    k, v = attn_inputs.random_draws((1, Hkv, n, d), seed=world * 10 + d + 1, count=2)
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    qs, ks, vs, dos = (_split(x.to(dev), world, zigzag) for x in (q, k, v, do))
    os_, lses = ring.ring_forward_emulated(qs, ks, vs, causal=causal, scale=scale, zigzag=zigzag)
    dqs, dks, dvs = ring.ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=causal,
                                                scale=scale, zigzag=zigzag)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    o, lse = _unsplit(os_, world, zigzag), _unsplit(lses, world, zigzag)
    dq, dk, dv = (_unsplit(x, world, zigzag) for x in (dqs, dks, dvs))
    wr = 0 if causal else -1
    ro, rlse = oracle.fwd_ex(q, k, v, scale, -1, wr)
    rq, rk, rv = oracle.bwd_ex(q, k, v, do, scale, -1, wr)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["bf16"]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["bf16"]
    assert grad_close(to_np(dq), rq)
    assert grad_close(to_np(dk), rk)
    assert grad_close(to_np(dv), rv)


@pytest.mark.parametrize("zigzag", [False, True])
def test_emulated_ring_deterministic_is_bitwise_repeatable(cuda_device, zigzag):
    world, n_chunk, d = 4, 256, 128
    q, k, v, do = attn_inputs.random_draws((1, 2, world * n_chunk, d), seed=5, count=4)
    dev = torch.device("cuda:0")
    qs, ks, vs, dos = (_split(x.to(dev), world, zigzag) for x in (q, k, v, do))
    os_, lses = ring.ring_forward_emulated(qs, ks, vs, causal=True, zigzag=zigzag)
    first = ring.ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=True, deterministic=True,
                                        zigzag=zigzag)
    again = ring.ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=True, deterministic=True,
                                        zigzag=zigzag)
    for a_list, b_list in zip(first, again):
        for a, b in zip(a_list, b_list):
            assert torch.equal(a, b)
    # and the deterministic sums are the gradients (against the oracle over the whole sequence)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = (_unsplit(x, world, zigzag) for x in first)
    rq, rk, rv = oracle.bwd_ex(q, k, v, do, scale, -1, 0)
    assert grad_close(to_np(dq), rq)
    assert grad_close(to_np(dk), rk)
    assert grad_close(to_np(dv), rv)


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("part_dtype", [torch.bfloat16, torch.float32])
def test_merge_kernel_of_two_key_halves_is_the_whole(cuda_device, d, part_dtype):
    # attention over keys [0, m) and [m, n) merged with the LSE rule = attention over [0, n)
    n, m = 700, 260
    dtype = "bf16" if part_dtype == torch.bfloat16 else "fp32"
    q, k, v = attn_inputs.random_draws((1, 3, 200, d), dtype=dtype, seed=d, count=1) + \
        attn_inputs.random_draws((1, 3, n, d), dtype=dtype, seed=d + 1, count=2)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    halves = [(kd[:, :, :m].contiguous(), vd[:, :, :m].contiguous()),
              (kd[:, :, m:].contiguous(), vd[:, :, m:].contiguous())]
    o_acc = torch.empty(qd.shape, dtype=torch.float32, device=dev)
    lse_acc = torch.empty(qd.shape[:-1], dtype=torch.float32, device=dev)
    out = torch.empty_like(qd)
    for i, (kk, vv) in enumerate(halves):
        o_p, l_p = ea.forward(qd, kk, vv, window=(-1, -1))
        ea.ring_merge(o_acc, lse_acc, o_p, l_p, first=(i == 0), out=out if i == 1 else None)
    torch.cuda.synchronize()
    ro, rlse = oracle.fwd_ex(q, k, v, 1.0 / math.sqrt(d), -1, -1)
    assert np.abs(to_np(out) - ro).max() <= TOL_O[dtype] * (2 if dtype == "fp32" else 1)
    assert np.abs(to_np(lse_acc) - rlse).max() <= TOL_LSE[dtype]
    assert np.abs(to_np(o_acc) - ro).max() <= TOL_O[dtype] * (2 if dtype == "fp32" else 1)


def test_merge_kernel_handles_empty_partials(cuda_device):
    dev = torch.device("cuda:0")
    rows, d = 64, 64
    o_acc = torch.empty(rows, d, device=dev)
    lse_acc = torch.empty(rows, device=dev)
    part = torch.randn(rows, d, device=dev)
    lse_p = torch.randn(rows, device=dev)
    lse_p[:16] = -float("inf")              # rows 0-15: nothing visible in the first part
    ea.ring_merge(o_acc, lse_acc, torch.zeros_like(part).masked_fill(
        torch.isinf(lse_p)[:, None], 0.0), lse_p, first=True)
    part2 = torch.randn(rows, d, device=dev)
    lse2 = torch.full((rows,), -float("inf"), device=dev)
    lse2[:8] = 0.5                           # rows 0-7 see keys only in the second part
    ea.ring_merge(o_acc, lse_acc, part2, lse2, first=False)
    torch.cuda.synchronize()
    assert torch.equal(o_acc[:8], part2[:8]) and torch.all(lse_acc[:8] == 0.5)
    assert torch.all(o_acc[8:16] == 0) and torch.all(torch.isneginf(lse_acc[8:16]))
    assert torch.isfinite(o_acc).all()


def test_accumulate_kernel(cuda_device):
    dev = torch.device("cuda:0")
    acc = torch.randn(4096, device=dev)
    part = torch.randn(4096, device=dev).to(torch.bfloat16)
    want = acc + part.float()
    out = torch.empty(4096, dtype=torch.bfloat16, device=dev)
    ea.ring_accumulate(acc, part, out=out)
    torch.cuda.synchronize()
    assert torch.equal(acc, want)
    assert torch.equal(out, want.to(torch.bfloat16))
    ea.ring_accumulate(acc, part, first=True)
    assert torch.equal(acc, part.float())
