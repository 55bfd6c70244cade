"""The bench workload (2x32x8192x128) in the modes the bench line does not time: no mask (sampled
forward rows and dQ rows against the oracle, computed one by one over all 8192 keys) and the
deterministic backward (bitwise-repeatable, and within the gradient tolerance of the atomic
mode)."""
import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_GRAD_REL, TOL_LSE, TOL_O, rel_fro, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402

W = "causal_bf16_2x32x8192x128"


@pytest.fixture(scope="module")
def inputs(cuda_device):
    w = attn_inputs.WORKLOADS[W]
    host = attn_inputs.workload_inputs(w)
    dev = tuple(t.to(cuda_device) for t in host)
    return w, host, dev


def test_no_mask_full_size_sampled_rows(inputs):
    w, (q, k, v, do), (qd, kd, vd, dod) = inputs
    o, lse = ea.forward(qd, kd, vd, causal=False, scale=w.scale)
    dq, dk, dv = ea.backward(qd, kd, vd, o, dod, lse, causal=False, scale=w.scale)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    rows = attn_inputs.sampled_rows(w, count=96)
    ro, rlse = oracle.fwd_rows(q, k, v, w.scale, False, rows)
    idx = torch.tensor(rows, device=o.device)
    assert np.abs(to_np(o.reshape(-1, w.d).index_select(0, idx)) - ro).max() <= TOL_O["bf16"]
    assert np.abs(to_np(lse.reshape(-1).index_select(0, idx)) - rlse).max() <= TOL_LSE["bf16"]
    rq, _ = oracle.bwd_query_rows(q, k, v, do, w.scale, False, rows[:48])
    got = to_np(dq.reshape(-1, w.d).index_select(0, idx[:48]))
    assert rel_fro(got, rq) <= TOL_GRAD_REL
    # unmasked: sum_j dV_j = sum_i dO_i per head
    sdv, sdo = dv.float().sum(2), dod.float().sum(2)
    assert (torch.linalg.norm(sdv - sdo) / torch.linalg.norm(sdo)).item() <= TOL_GRAD_REL


def test_deterministic_full_size(inputs):
    w, _, (qd, kd, vd, dod) = inputs
    o, lse = ea.forward(qd, kd, vd, causal=True, scale=w.scale)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(*w.shape, 1), dtype=torch.uint8, device=qd.device)
    first = [t.clone() for t in ea.backward(qd, kd, vd, o, dod, lse, causal=True, scale=w.scale,
                                            deterministic=True, workspace=ws)]
    again = ea.backward(qd, kd, vd, o, dod, lse, causal=True, scale=w.scale, deterministic=True,
                        workspace=ws)
    atomic = ea.backward(qd, kd, vd, o, dod, lse, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    for a, b, c in zip(first, again, atomic):
        assert torch.equal(a, b)
        assert rel_fro(to_np(a), to_np(c)) <= 1e-2
