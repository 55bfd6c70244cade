"""A forward captured into a CUDA graph in a fresh process, before any eager call: the small-grid
bf16 launch then picks its key split without the occupancy query (which is not made while a
stream is being captured). The replay must match the oracle like an eager call."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = textwrap.dedent("""
    import math, sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
    import attn_inputs, oracle
    import exact_attention_138_b200 as ea
    from parity_util import TOL_O, TOL_LSE, to_np
    shape = (1, 2, 1000, 64)
    q, k, v = attn_inputs.random_draws(shape, seed=77, count=3)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ea.forward(qd, kd, vd, causal=True, scale=0.125, out=o, lse=lse, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    ro, rl = oracle.fwd(q, k, v, 0.125, True)
    assert np.abs(to_np(o) - ro).max() <= TOL_O["bf16"]
    assert np.abs(to_np(lse) - rl).max() <= TOL_LSE["bf16"]
    print("cold capture ok")
""")


def test_forward_captured_before_any_eager_call(cuda_device):
    code = SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "cold capture ok" in r.stdout
