"""Writes long_context_key_rows.json: oracle dK / dV rows of the long-context workload.

    python tests/golden/make_long_context_key_rows.py [--out PATH]

Workload: causal bf16 attention over one 131,072-token sequence, 8 heads, d = 128, inputs q, k,
v, dO drawn by attn_inputs (seed 9, N(0,1), rounded to bf16) — the long-context row of
"Attention Mechanism: Revolusi Representasi Sequence" (§6 complexity table, §16 "Long Context
Training"). For one head and sixteen keys spread over the whole sequence (the first key, which
every one of the 131,072 queries sees, keys around n/2, tile edges and the last key), the fp64
oracle computes the exact dK and dV rows (oracle.bwd_key_rows_batched: every query row's full
softmax recomputed, as "Flash Attention Nedir?", section "Recomputation", describes).

Only oracle/ and attn_inputs (seeded draws, no attention arithmetic) are called. The file also
stores fp64 sums of the head's inputs, so that a test can tell when the draws have changed.
About 5-10 minutes on 8 host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import attn_inputs  # noqa: E402
import oracle  # noqa: E402

WORKLOAD = "causal_bf16_1x8x131072x128"
HEAD = 5
KEYS = [0, 1, 127, 128, 4096, 16383, 32768, 45000, 65535, 65536, 81921, 98304, 114687, 122880,
        130944, 131071]
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "long_context_key_rows.json")


def head_sums(tensors, head, n, d):
    """fp64 sums of one head of each input (bf16 values are exact in fp64)."""
    out = []
    for t in tensors:
        x = t.float().reshape(-1, n, d)[head].numpy().astype(np.float64)
        out.append(float(x.sum()))
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=OUT)
    args = ap.parse_args()
    w = attn_inputs.WORKLOADS[WORKLOAD]
    q, k, v, do = attn_inputs.workload_inputs(w)
    t0 = time.time()
    dk, dv = oracle.bwd_key_rows_batched(q, k, v, do, w.scale, True, HEAD, KEYS)
    secs = time.time() - t0
    rec = {
        "_about": ("Exact fp64 dK / dV rows of the causal long-context workload at sixteen keys "
                   "of one head, written by the oracle (not by the CUDA library). Inputs: "
                   "attn_inputs.workload_inputs for the workload below. Tolerance in the test: "
                   "relative Frobenius error 2e-2 per tensor over the stored rows."),
        "command": "python tests/golden/make_long_context_key_rows.py",
        "oracle_function": "oracle.bwd_key_rows_batched",
        "workload": WORKLOAD,
        "shape": list(w.shape),
        "scale": w.scale,
        "causal": True,
        "head": HEAD,
        "keys": KEYS,
        "input_sums_q_k_v_do": head_sums((q, k, v, do), HEAD, w.n, w.d),
        "oracle_seconds": round(secs, 1),
        "dk": [[float(f"{x:.9e}") for x in row] for row in dk],
        "dv": [[float(f"{x:.9e}") for x in row] for row in dv],
    }
    with open(args.out, "w") as f:
        json.dump(rec, f, indent=0)
        f.write("\n")
    print(f"wrote {args.out} in {secs:.0f} s")


if __name__ == "__main__":
    main()
