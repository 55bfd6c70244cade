"""GPU parity of the forward pass against the fp64 oracle.

Small and ragged shapes are compared element by element over the whole output; the pages'
full-size workloads are compared on seeded sampled rows (each computed one by one by the
oracle) plus whole-output properties."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_LSE, TOL_O, cuda_forward, to_np

pytestmark = pytest.mark.gpu

SHAPES = [(1, 2, 1, 64), (2, 1, 2, 32), (1, 1, 17, 128), (1, 3, 127, 64), (2, 2, 129, 128),
          (1, 2, 300, 32), (1, 1, 1000, 128), (1, 2, 256, 128), (1, 1, 383, 64), (1, 1, 640, 32)]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_forward_small_shapes(cuda_device, shape, causal, dtype):
    q, k, v = attn_inputs.random_draws(shape, dtype=dtype, seed=hash(shape) % 1000, count=3)
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse, _ = cuda_forward(q, k, v, causal, scale)
    ro, rlse = oracle.fwd(q, k, v, scale, causal)
    assert np.abs(to_np(o) - ro).max() <= TOL_O[dtype]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE[dtype]


def test_forward_p1_fp32_workload(cuda_device):
    # (2,3,128,32) fp32, seed-9 draws of efficient_attention.py; atol 1e-5 as on the page
    w = attn_inputs.WORKLOADS["p1_fp32_2x3x128x32"]
    q, k, v, _ = attn_inputs.workload_inputs(w)
    o, lse, _ = cuda_forward(q, k, v, False, w.scale)
    ro, rlse = oracle.fwd(q, k, v, w.scale, False)
    assert np.abs(to_np(o) - ro).max() <= 1e-5
    assert np.abs(to_np(lse) - rlse).max() <= 1e-5


@pytest.mark.parametrize("name", ["rowtile_fp32_4096x64", "rowtile_bf16_4096x64"])
def test_forward_rowtile_workload(cuda_device, name):
    w = attn_inputs.WORKLOADS[name]
    q, k, v, _ = attn_inputs.workload_inputs(w)
    o, lse, _ = cuda_forward(q, k, v, False, w.scale)
    ro, rlse = oracle.fwd(q, k, v, w.scale, False)
    rt, _ = oracle.fwd_rowtiled(q, k, v, w.scale, False, 128)
    assert np.array_equal(ro, rt)          # the oracle's own full == row-tiled claim
    assert np.abs(to_np(o) - ro).max() <= TOL_O[w.dtype]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE[w.dtype]


@pytest.mark.parametrize("name", ["causal_bf16_1x32x4096x128", "causal_bf16_2x32x8192x128",
                                  "causal_bf16_1x8x131072x128"])
def test_forward_full_size_sampled_rows(cuda_device, name):
    w = attn_inputs.WORKLOADS[name]
    q, k, v, _ = attn_inputs.workload_inputs(w)
    o, lse, _ = cuda_forward(q, k, v, True, w.scale)
    rows = attn_inputs.sampled_rows(w)
    ro, rlse = oracle.fwd_rows(q, k, v, w.scale, True, rows)
    idx = torch.tensor(rows, device=o.device)
    go = to_np(o.reshape(-1, w.d).index_select(0, idx))
    glse = to_np(lse.reshape(-1).index_select(0, idx))
    assert np.abs(go - ro).max() <= TOL_O["bf16"]
    assert np.abs(glse - rlse).max() <= TOL_LSE["bf16"]
    # whole-output properties: finite, and every row a convex combination of value rows
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    vmax = v.float().abs().amax().item()
    assert o.float().abs().amax().item() <= vmax + 1e-2
    # causal row 0 of every head equals v[0] (rounded to bf16)
    assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0])


def test_forward_large_magnitude_stays_finite(cuda_device):
    q, k, v = attn_inputs.random_draws((1, 2, 512, 128), dtype="bf16", factor=30.0, seed=5,
                                       count=3)
    for causal in (False, True):
        o, lse, _ = cuda_forward(q, k, v, causal, 1 / math.sqrt(128))
        ro, rlse = oracle.fwd(q, k, v, 1 / math.sqrt(128), causal)
        assert torch.isfinite(o).all()
        # |V| reaches ~120 here, where one bf16 ulp of O is 0.5: the O bound scales with max|V|
        # (1e-2 of it, about 5x the bf16 rounding of O and P); LSE (~|s| ~ 1e3) relative 1e-5
        vmax = float(v.float().abs().max())
        assert np.abs(to_np(o) - ro).max() <= TOL_O["bf16"] * vmax
        assert np.abs(to_np(lse) - rlse).max() <= 1e-5 * np.abs(rlse).max()


def test_forward_repeatable(cuda_device):
    q, k, v = attn_inputs.random_draws((1, 4, 1024, 128), seed=3, count=3)
    o1, l1, _ = cuda_forward(q, k, v, True, 0.1)
    o2, l2, _ = cuda_forward(q, k, v, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("Hkv", [1, 2])
def test_gqa_forward_fp32(cuda_device, Hkv):
    q = attn_inputs.random_draws((1, 4, 200, 64), dtype="fp32", seed=41, count=1)[0]
    k, v = attn_inputs.random_draws((1, Hkv, 200, 64), dtype="fp32", seed=42, count=2)
    o, lse, _ = cuda_forward(q, k, v, True, 0.125)
    ro, rlse = oracle.fwd_gqa(q, k, v, 0.125, True)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["fp32"]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["fp32"]


# fp32 grids on both sides of the key split. The launcher picks the query-tile height (64 rows
# down to 32 in steps of 4; 2 threads per row, so heights that are not multiples of 16 leave the
# CTA's last warp partial) and the key split (1-8 CTAs of a cluster, merging their (m, l, O) on
# chip) from a cost model over resident CTAs and clusters. With a B200's counts these shapes give
# 56-row tiles without a split (2,8,1000,64), 60-row tiles in pairs (1,12,1000,128), 64-row tiles
# in 8 shares, some empty under the causal mask (1,1,1000,128), and 4 uneven shares of 11 key
# tiles (2,3,700,32).
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(2, 8, 1000, 64), (1, 12, 1000, 128), (1, 1, 1000, 128),
                                   (2, 3, 700, 32)], ids=lambda s: "x".join(map(str, s)))
def test_forward_fp32_split_and_unsplit_grids(cuda_device, shape, causal):
    q, k, v = attn_inputs.random_draws(shape, dtype="fp32", seed=sum(shape), count=3)
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse, _ = cuda_forward(q, k, v, causal, scale)
    ro, rlse = oracle.fwd(q, k, v, scale, causal)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["fp32"]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["fp32"]
