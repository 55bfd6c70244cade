"""Failure detection on the GPU without faulting it: a bounded device-side wait that nobody
satisfies runs out, reports ATTN_ERR_TIMEOUT through the status word, and leaves the context
usable."""
import math

import pytest
import torch

import attn_inputs
import exact_attention_138_b200 as ea
from parity_util import cuda_forward

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(cuda_device):
    assert ea.device_status() == ea.ATTN_OK
    assert ea.attn_selftest_wait_timeout(2000) == ea.ATTN_OK      # 2 ms limit
    assert ea.device_status() == ea.ATTN_ERR_TIMEOUT
    assert ea.device_status() == ea.ATTN_OK                         # the word was cleared
    q, k, v = attn_inputs.random_draws((1, 1, 256, 64), seed=1, count=3)
    o, lse, _ = cuda_forward(q, k, v, True, 1 / math.sqrt(64))
    assert torch.isfinite(o).all()
