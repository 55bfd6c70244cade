"""The C-ABI calls are stream-ordered and allocate nothing (the backward's workspace comes from the
caller), so a whole training-style step — forward, backward — can be captured into a CUDA graph
and replayed. The replay must reproduce the eagerly computed outputs bit for bit (deterministic
backward) and keep matching the oracle."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_O, grad_close, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402


@pytest.mark.parametrize("d,causal,window", [(128, True, None), (64, False, None),
                                             (128, False, (100, 20))])
def test_captured_step_replays_bitwise(cuda_device, d, causal, window):
    shape = (1, 2, 700, d)
    q, k, v, do = attn_inputs.random_draws(shape, seed=d + 3, count=4)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (x.to(dev).contiguous() for x in (q, k, v, do))
    scale = 1.0 / math.sqrt(d)
    o, lse = torch.empty_like(qd), torch.empty(shape[:3], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(*shape, 1), dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream()

    def step():
        ea.forward(qd, kd, vd, causal=causal, scale=scale, out=o, lse=lse, window=window,
                   stream=s)
        ea.backward(qd, kd, vd, o, dod, lse, causal=causal, scale=scale, deterministic=True,
                    dq=dq, dk=dk, dv=dv, workspace=ws, stream=s, window=window)

    with torch.cuda.stream(s):
        step()                                  # eager (also resolves one-time lookups)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (o, lse, dq, dk, dv)]
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    for a, b in zip(eager, (o, lse, dq, dk, dv)):
        assert torch.equal(a, b)
    wl, wr = window if window is not None else (-1, 0 if causal else -1)
    ro, _ = oracle.fwd_ex(q, k, v, scale, wl, wr)
    rq, rk, rv = oracle.bwd_ex(q, k, v, do, scale, wl, wr)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["bf16"]
    assert grad_close(to_np(dq), rq) and grad_close(to_np(dk), rk) and grad_close(to_np(dv), rv)
