"""Forward parity on grids that fill the GPU (more tile pairs than the SMs hold at once), where
the library runs one CTA per pair of query tiles with no key split; most of the other forward
tests have small grids, which take the kernels that split each pair's keys over a cluster. Whole
tensors against the oracle, element by element, with the masks and head layouts of the pages
("Attention Mechanism ...", §4.2, §4.4, §4.5, §12)."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_LSE, TOL_O, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402


@pytest.mark.parametrize("H,Hkv,nq,nk,window", [
    (40, 40, 2048, 2048, (-1, 0)),       # causal
    (40, 40, 2000, 2000, (-1, 0)),       # causal, ragged last tile
    (40, 40, 2048, 2048, None),          # no mask
    (40, 40, 2048, 2048, (300, 0)),      # causal window of 301 keys
    (40, 8, 2048, 2048, (-1, 0)),        # grouped-query heads
    (40, 40, 1900, 3000, (-1, 0)),       # more keys than queries, bottom-right aligned
])
def test_forward_on_full_grids(cuda_device, H, Hkv, nq, nk, window):
    d = 128
    # inputs scaled by 0.5 as in the pages' 2x32x8192x128 workload: |O| stays below 2, where one
    # bf16 rounding of the output is at most 2^-8, inside the 1e-2 bound
    q = attn_inputs.random_draws((1, H, nq, d), factor=0.5, seed=nq + H, count=1)[0]
    k, v = attn_inputs.random_draws((1, Hkv, nk, d), factor=0.5, seed=nk + Hkv, count=2)
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    o, lse = ea.forward(q.to(dev), k.to(dev), v.to(dev), scale=scale, window=window)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    wl, wr = window if window is not None else (-1, -1)
    ro, rlse = oracle.fwd_ex(q, k, v, scale, wl, wr)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["bf16"]
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["bf16"]
