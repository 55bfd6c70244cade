"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds no attention arithmetic: it only draws random numbers and names the
workloads. Both the CUDA path and the CPU oracle consume what it returns.

Workloads (all entries iid N(0,1) unless a factor is given):
  * ``p1_script``: the two draws of efficient_attention.py ("Efficient Attention", section
    "Mengapa Memori Attention Tumbuh Kuadratik"): torch.manual_seed(9), then q, k, v of shape
    (2,3,128,32), then q2, k2, v2 of shape (4096,64), in that order, from torch's CPU stream.
  * bf16 workloads: a CPU ``torch.Generator`` seeded with 9 draws fp32 q, k, v, dO in that order,
    each multiplied by the workload's factor and then rounded to bf16 (round-to-nearest-even).
    Drawing on the CPU makes the same inputs available to the oracle without a GPU.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

SEED = 9


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n: int
    d: int
    causal: bool
    dtype: str          # "fp32" or "bf16"
    backward: bool
    factor: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.n, self.d)


# The five workloads of the pages: (2,3,128,32) fp32; (4096,64) fp32 and bf16 (single head);
# causal bf16 fwd+bwd at (1,32,4096,128), (2,32,8192,128) with inputs x0.5, and (1,8,131072,128).
WORKLOADS = {
    "p1_fp32_2x3x128x32": Workload("p1_fp32_2x3x128x32", 2, 3, 128, 32, False, "fp32", False),
    "rowtile_fp32_4096x64": Workload("rowtile_fp32_4096x64", 1, 1, 4096, 64, False, "fp32", False),
    "rowtile_bf16_4096x64": Workload("rowtile_bf16_4096x64", 1, 1, 4096, 64, False, "bf16", False),
    "causal_bf16_1x32x4096x128": Workload("causal_bf16_1x32x4096x128", 1, 32, 4096, 128, True,
                                          "bf16", True),
    "causal_bf16_2x32x8192x128": Workload("causal_bf16_2x32x8192x128", 2, 32, 8192, 128, True,
                                          "bf16", True, 0.5),
    "causal_bf16_1x8x131072x128": Workload("causal_bf16_1x8x131072x128", 1, 8, 131072, 128, True,
                                           "bf16", True),
}

HEADLINE = "causal_bf16_2x32x8192x128"


def p1_script_draws():
    """(q, k, v) of shape (2,3,128,32) and (q2, k2, v2) of shape (4096,64), fp32, CPU."""
    state = torch.random.get_rng_state()
    try:
        torch.manual_seed(SEED)
        q = torch.randn(2, 3, 128, 32)
        k = torch.randn(2, 3, 128, 32)
        v = torch.randn(2, 3, 128, 32)
        q2 = torch.randn(4096, 64)
        k2 = torch.randn(4096, 64)
        v2 = torch.randn(4096, 64)
    finally:
        torch.random.set_rng_state(state)
    return (q, k, v), (q2, k2, v2)


def bf16_draws(shape, factor=1.0, seed=SEED, count=4):
    """`count` tensors (q, k, v, dO, ...) drawn in that order, scaled by factor, rounded to bf16."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = []
    for _ in range(count):
        t = torch.randn(*shape, generator=g, dtype=torch.float32)
        if factor != 1.0:
            t.mul_(factor)
        out.append(t.to(torch.bfloat16))
    return out


def random_draws(shape, dtype="bf16", factor=1.0, seed=SEED, count=4):
    """Generic seeded draws for odd-shaped test cases (fp32 or bf16)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = []
    for _ in range(count):
        t = torch.randn(*shape, generator=g, dtype=torch.float32) * factor
        out.append(t.to(torch.bfloat16) if dtype == "bf16" else t)
    return out


def workload_inputs(w: Workload):
    """CPU inputs of a named workload: (q, k, v, dO) with dO None for forward-only workloads."""
    if w.name == "p1_fp32_2x3x128x32":
        (q, k, v), _ = p1_script_draws()
        return q, k, v, None
    if w.name.startswith("rowtile_"):
        _, (q2, k2, v2) = p1_script_draws()
        shp = (1, 1, 4096, 64)
        q2, k2, v2 = (t.reshape(shp) for t in (q2, k2, v2))
        if w.dtype == "bf16":
            q2, k2, v2 = (t.to(torch.bfloat16) for t in (q2, k2, v2))
        return q2, k2, v2, None
    q, k, v, do = bf16_draws(w.shape, factor=w.factor)
    return q, k, v, do


def sampled_rows(w: Workload, count=256, seed=SEED):
    """Flat query-row indices (bh*n + i): `count` uniform draws plus i = 0 and i = n-1 of the
    first and last head, sorted and de-duplicated."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    total = w.B * w.H * w.n
    r = torch.randint(0, total, (count,), generator=g).tolist()
    last = w.B * w.H - 1
    r += [0, w.n - 1, last * w.n, last * w.n + w.n - 1]
    return sorted(set(r))
