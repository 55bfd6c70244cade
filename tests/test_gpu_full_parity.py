"""Whole-tensor parity with the fp64 oracle at the pages' full-size causal workloads.

  * 1x32x4096x128 (the "Exemple chiffré" size of "Calculateur de mémoire d'attention"): O and LSE
    element by element and dQ, dK, dV as per-tensor Frobenius relative errors, over all 32 heads.
  * 2x32x8192x128 (inputs x0.5): the same on four whole heads spread over both sequences.
  * 1x8x131072x128: dK / dV at sixteen keys of one head spread over the whole sequence (the
    first key is seen by all 131,072 queries), against rows stored by
    tests/golden/make_long_context_key_rows.py (the oracle's fp64 values), in both dQ modes; the
    deterministic mode is also repeated bit for bit and its dQ compared on 256 sampled rows.

Tolerances: O max-abs 1e-2, LSE 1e-3, gradients relative Frobenius error 2e-2 (bf16 inputs,
fp32 accumulation, P and dS rounded to bf16 on the tensor-core path).
"""
import json
import os

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_GRAD_REL, TOL_LSE, TOL_O, rel_fro, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

import exact_attention_138_b200 as ea  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "long_context_key_rows.json")


def _gpu_fwd_bwd(w, host, device, deterministic=False):
    q, k, v, do = (t.to(device) for t in host)
    o, lse = ea.forward(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = ea.backward(q, k, v, o, do, lse, causal=True, scale=w.scale,
                             deterministic=deterministic)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    return o, lse, dq, dk, dv


def test_whole_tensors_1x32x4096x128(cuda_device):
    w = attn_inputs.WORKLOADS["causal_bf16_1x32x4096x128"]
    q, k, v, do = attn_inputs.workload_inputs(w)
    o, lse, dq, dk, dv = (to_np(t) for t in _gpu_fwd_bwd(w, (q, k, v, do), cuda_device))
    torch.cuda.empty_cache()
    ro, rlse = oracle.fwd(q, k, v, w.scale, True)
    assert np.abs(o - ro).max() <= TOL_O["bf16"]
    assert np.abs(lse - rlse).max() <= TOL_LSE["bf16"]
    rq, rk, rv, _ = oracle.bwd(q, k, v, do, w.scale, True)
    for name, got, want in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = rel_fro(got, want)
        worst = max(rel_fro(got[0, h], want[0, h]) for h in range(w.H))
        assert err <= TOL_GRAD_REL, (name, err, worst)


def test_whole_heads_2x32x8192x128(cuda_device):
    w = attn_inputs.WORKLOADS["causal_bf16_2x32x8192x128"]
    q, k, v, do = attn_inputs.workload_inputs(w)
    o, lse, dq, dk, dv = _gpu_fwd_bwd(w, (q, k, v, do), cuda_device)
    heads = [(0, 0), (0, 21), (1, 10), (1, 31)]     # four heads over both sequences
    got = {name: [] for name in ("dq", "dk", "dv")}
    want = {name: [] for name in ("dq", "dk", "dv")}
    for b, h in heads:
        sl = lambda t: t[b:b + 1, h:h + 1].contiguous()   # noqa: E731
        hq, hk, hv, hdo = (sl(t) for t in (q, k, v, do))
        ro, rlse = oracle.fwd(hq, hk, hv, w.scale, True)
        assert np.abs(to_np(o[b, h]) - ro[0, 0]).max() <= TOL_O["bf16"], (b, h)
        assert np.abs(to_np(lse[b, h]) - rlse[0, 0]).max() <= TOL_LSE["bf16"], (b, h)
        rq, rk, rv, _ = oracle.bwd(hq, hk, hv, hdo, w.scale, True)
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            gh = to_np(g[b, h])
            assert rel_fro(gh, r[0, 0]) <= TOL_GRAD_REL, (name, b, h, rel_fro(gh, r[0, 0]))
            got[name].append(gh)
            want[name].append(r[0, 0])
    for name in got:
        assert rel_fro(np.stack(got[name]), np.stack(want[name])) <= TOL_GRAD_REL, name


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def long_context(cuda_device):
    w = attn_inputs.WORKLOADS["causal_bf16_1x8x131072x128"]
    host = attn_inputs.workload_inputs(w)
    g = _golden()
    assert g["workload"] == w.name and g["shape"] == list(w.shape)
    # the stored rows belong to these inputs: the head's sums must match the draws
    for t, s in zip(host, g["input_sums_q_k_v_do"]):
        x = t.float().reshape(-1, w.n, w.d)[g["head"]].numpy().astype(np.float64).sum()
        assert x == pytest.approx(s, rel=1e-12, abs=1e-9)
    yield w, host, g
    torch.cuda.empty_cache()


def _check_golden_keys(g, dk, dv):
    keys = torch.tensor(g["keys"], device=dk.device)
    head = g["head"]
    gk = to_np(dk.reshape(-1, dk.shape[-2], dk.shape[-1])[head].index_select(0, keys))
    gv = to_np(dv.reshape(-1, dv.shape[-2], dv.shape[-1])[head].index_select(0, keys))
    assert rel_fro(gk, np.array(g["dk"])) <= TOL_GRAD_REL
    assert rel_fro(gv, np.array(g["dv"])) <= TOL_GRAD_REL
    # key 0 alone (the longest accumulation: every query of the sequence adds to it)
    assert rel_fro(gk[0], np.array(g["dk"][0])) <= TOL_GRAD_REL
    assert rel_fro(gv[0], np.array(g["dv"][0])) <= TOL_GRAD_REL


def test_long_context_key_rows_across_sequence(long_context, cuda_device):
    w, host, g = long_context
    _, _, _, dk, dv = _gpu_fwd_bwd(w, host, cuda_device)
    _check_golden_keys(g, dk, dv)


def test_long_context_deterministic(long_context, cuda_device):
    w, host, g = long_context
    q, k, v, do = (t.to(cuda_device) for t in host)
    o, lse = ea.forward(q, k, v, causal=True, scale=w.scale)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(*w.shape, 1), dtype=torch.uint8,
                     device=cuda_device)
    first = [t.clone() for t in ea.backward(q, k, v, o, do, lse, causal=True, scale=w.scale,
                                            deterministic=True, workspace=ws)]
    again = ea.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, deterministic=True,
                        workspace=ws)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    for a, b in zip(first, again):
        assert torch.equal(a, b)
    dq, dk, dv = first
    _check_golden_keys(g, dk, dv)
    rows = attn_inputs.sampled_rows(w, count=256)
    rq, _ = oracle.bwd_query_rows(*host, w.scale, True, rows)
    idx = torch.tensor(rows, device=dq.device)
    assert rel_fro(to_np(dq.reshape(-1, w.d).index_select(0, idx)), rq) <= TOL_GRAD_REL
