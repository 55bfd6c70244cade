#!/usr/bin/env python3
"""Benchmark: exact attention forward + backward TFLOPS on B200 (bf16, causal).

One step = one forward (attn_fwd) and one backward (attn_bwd) pass over one batch of the
workload B=2, H=32, n=8192, d=128, causal, bf16, inputs iid N(0,1) x 0.5 drawn from a seeded
CPU generator. FLOPs per step follow the convention forward = 4·B·H·n²·d (two matmuls), halved
for the causal mask, backward = 2.5 x forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line on rank 0. With N > 1 (launched by torchrun, one process per GPU) every
rank runs its own batch: the units are independent (b,h) problems, so the shards need no
collective; time is the max over ranks (weak scaling). `--impl reference` times the fp64 CPU
oracle on a bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOPS at 1 B200 (bf16, causal) and % of dense bf16 peak"
WORKLOAD = "causal_bf16_2x32x8192x128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def step_flops(B, H, n, d, causal=True):
    fwd = 4.0 * B * H * n * n * d * (0.5 if causal else 1.0)
    return fwd, 2.5 * fwd


def rank_seed(rank):
    """Each rank draws its own batch: seed 9 + rank (rank 0 reproduces the single-GPU inputs)."""
    return 9 + rank


def max_over_ranks(value, dist=None, device="cpu"):
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def whole_job_tflops(flops_per_rank, world, ms_per_step):
    """Weak scaling: every rank processes its own batch; the job's rate is all ranks' FLOPs over
    the slowest rank's time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Sources that determine each profiled kernel: its own file plus the shared headers.
KERNEL_SOURCES = {
    "bwd_main_q64_kernel": ("bwd_bf16.cu", "kernels.h", "sm100_ptx.cuh"),
    "fwd_bf16_kernel": ("fwd_bf16.cu", "kernels.h", "sm100_ptx.cuh"),
}


def csrc_digest(kernel=None):
    """Hash of the CUDA sources of `kernel` (all of csrc/ when None)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "exact_attention_138_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(d))
    for name in sorted(names):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the committed ncu
    summary, if the kernel sources have not changed since the counters were taken; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(kernel)
    if (not entry or entry.get("csrc_sha") != csrc_digest(kernel)
            or entry.get("workload") != workload):
        return None
    return entry.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [x for x in sm if smax and x >= 0.3 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "reasons": reasons, "samples": len(rows)}


def oracle_sample(seconds_target, q, k, v, do, w, rng_seed=9):
    """Time the fp64 oracle on a bounded sample of the workload's query rows: forward rows
    (O, LSE) and backward dQ rows, in batches of uniformly drawn rows until about
    `seconds_target` seconds have been spent. Returns (TFLOPS credited, seconds, rows, threads);
    each row is credited with the workload's average algorithmic FLOPs per query row."""
    import numpy as np
    import oracle
    B, H, n, d = w.B, w.H, w.n, w.d
    total_rows = B * H * n
    fwd, bwd = step_flops(B, H, n, d)
    per_row = (fwd + bwd) / total_rows
    rng = np.random.default_rng(rng_seed)
    qf, kf, vf, dof = (oracle._f32(t) for t in (q, k, v, do))   # widen once, outside the timing
    rows_done, spent, batch = 0, 0.0, 64
    while spent < seconds_target:
        rows = np.sort(rng.choice(total_rows, size=batch, replace=False))
        t0 = time.perf_counter()
        oracle.fwd_rows(qf, kf, vf, w.scale, True, rows)
        oracle.bwd_query_rows(qf, kf, vf, dof, w.scale, True, rows)
        spent += time.perf_counter() - t0
        rows_done += batch
        batch = min(batch * 2, 2048)
    return per_row * rows_done / spent / 1e12, spent, rows_done, oracle.num_threads()


def run_reference(args, w):
    """Reference arm: the fp64 CPU oracle (as it stands) on the machine's host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import attn_inputs
    q, k, v, do = attn_inputs.workload_inputs(w)
    times, flops_rate, rows_used, threads = [], [], 0, 1
    # each step is a bounded sample, sized so that the whole run stays within ~2 minutes
    per_step = min(args.ref_seconds, 120.0 / (args.warmup + args.steps))
    for i in range(args.warmup + args.steps):
        rate, dt, rows_n, threads = oracle_sample(per_step, q, k, v, do, w, 9 + i)
        if i >= args.warmup:
            times.append(dt)
            flops_rate.append(rate)
            rows_used = rows_n
    value = statistics.mean(flops_rate)
    sample = (f"{rows_used} uniformly drawn query rows of {w.B}x{w.H}x{w.n}x{w.d} per step "
              f"(forward O/LSE rows + backward dQ rows, fp64); TFLOPS credited at the "
              f"workload's average FLOPs per query row")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "d": w.d,
                   "causal": True, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# The pages' small forward-only cases: short n (2x3x128x32 fp32) and small d (1x1x4096x64 fp32
# and bf16). They fill a small fraction of the GPU, so they are timed per launch with L2 flushed
# in between and reported as achieved HBM bandwidth beside the FLOP rate.
SMALL_CASES = ("p1_fp32_2x3x128x32", "rowtile_fp32_4096x64", "rowtile_bf16_4096x64")
L2_FLUSH_BYTES = 256 << 20          # written between timed launches (L2 is 126 MB)
SM_COUNT = 148


def roofline_peak(burst, sustained, timed_ms, clk, peak_src):
    """Dense bf16 peak that a kernel timed in this run is held against, and why.

    The burst figure (a GEMM timed alone, at the maximum clock) applies unless the timed region
    lasted over a second AND the sampled clock record shows the power cap active, which is when
    the sustained figure (a GEMM looped for seconds under the cap) describes the conditions."""
    reasons = clk.get("reasons") or []
    long_run = timed_ms > 1000.0
    capped = "sw_power_cap" in reasons
    if long_run and capped:
        return sustained, (f"bf16_tflops_sustained ({peak_src}): timed region {timed_ms:.0f} ms "
                           f"> 1 s with sw_power_cap active")
    why = (f"timed region {timed_ms:.0f} ms <= 1 s" if not long_run
           else "no sw_power_cap in the clock record")
    return burst, f"bf16_tflops ({peak_src}, burst): {why}"


def bwd_main_bytes(w):
    """Algorithmic DRAM bytes of one backward main-kernel launch: Q, K, V, dO read, dK, dV
    written (bf16), LSE·log2e and D read (fp32), the fp32 dQ accumulator read and written once."""
    rows = w.B * w.H * w.n
    return rows * w.d * 2 * 6 + rows * 4 * 2 + rows * w.d * 4 * 2


def fwd_case_bytes(w):
    """Algorithmic HBM bytes of one forward launch: q, k, v read once, O written, fp32 LSE
    written."""
    e = 4 if w.dtype == "fp32" else 2
    return 4 * w.B * w.H * w.n * w.d * e + 4 * w.B * w.H * w.n


def fwd_case_query_tiles(w):
    """Query tiles of one forward launch: 64 rows in fp32, 128 rows in bf16 (the fp32 kernel may
    split each tile's keys over a cluster of CTAs; the bf16 kernel runs tiles in pairs)."""
    rows = 64 if w.dtype == "fp32" else 128
    return w.B * w.H * ((w.n + rows - 1) // rows)


def time_forward_case(ea, w, dev, stream, iters, warmup, hbm_peak, fma_peak, e4m3=False):
    """Median device time of one forward launch of workload `w` over `iters` launches, each
    preceded by a write of a buffer larger than L2 so that q, k, v come from HBM. With e4m3 the
    workload's inputs are quantised to E4M3 (descale 2^-4) and run through the FP8 forward."""
    import torch
    import attn_inputs
    q, k, v, _ = attn_inputs.workload_inputs(w)
    q, k, v = (t.to(dev) for t in (q, k, v))
    desc = 2.0 ** -4
    if e4m3:
        q, k, v = ((t.float() / desc).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
                   for t in (q, k, v))
    o = torch.empty(q.shape, dtype=torch.bfloat16 if e4m3 else q.dtype, device=dev)
    lse = torch.empty((w.B, w.H, w.n), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd():
        if e4m3:
            ea.forward_fp8(q, k, v, desc, desc, desc, causal=w.causal, scale=w.scale, out=o,
                           lse=lse, stream=stream)
        else:
            ea.forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)

    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    with torch.cuda.stream(stream):
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fwd()
            b.record(stream)
    torch.cuda.synchronize()
    if ea.device_status() != ea.ATTN_OK:
        raise SystemExit(f"device status not OK in the {w.name} forward timings")
    us = statistics.median(a.elapsed_time(b) * 1e3 for a, b in ev)
    nbytes = fwd_case_bytes(w) if not e4m3 else 3 * q.numel() + 2 * q.numel() + 4 * lse.numel()
    flops = 4.0 * w.B * w.H * w.n * w.n * w.d * (0.5 if w.causal else 1.0)
    gbs = nbytes / (us * 1e-6) / 1e9
    tflops = flops / (us * 1e-6) / 1e12
    out = {"us": us, "launches": iters, "bytes": nbytes, "hbm_gbs": gbs,
           "hbm_frac": gbs / hbm_peak, "tflops": tflops, "query_tiles": fwd_case_query_tiles(w),
           "sms": SM_COUNT, "dtype": "e4m3" if e4m3 else w.dtype,
           "l2": f"{L2_FLUSH_BYTES >> 20} MiB written before every launch"}
    if w.dtype == "fp32":
        out["fma_frac"] = tflops / fma_peak
    return out


def fma_peak_tflops(sm_max_mhz):
    """fp32 FFMA peak: SMs x 128 lanes x 2 FLOP x the maximum SM clock."""
    return SM_COUNT * 128 * 2 * sm_max_mhz * 1e6 / 1e12


def run_forward_case(args, w):
    """One forward-only workload (the pages' small cases): one JSON line with its per-launch time,
    achieved HBM bandwidth and FLOP rate. A profiling and reporting mode; the headline run carries
    the same numbers under `small_cases`."""
    import torch
    if int(os.environ.get("WORLD_SIZE", "1")) != 1:
        raise SystemExit("forward-only workloads run on one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    import exact_attention_138_b200 as ea
    peaks, peak_src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    stream = torch.cuda.current_stream()
    with ClockSampler(0) as clocks:
        r = time_forward_case(ea, w, dev, stream, args.steps, args.warmup, hbm,
                              fma_peak_tflops(1965.0))
    clk = clocks.summary()
    fma = fma_peak_tflops(clk["sm_max_mhz"] or 1965.0)
    if "fma_frac" in r:
        r["fma_frac"] = r["tflops"] / fma
    line = {
        "metric": "attention forward latency and achieved HBM bandwidth (small case)",
        "value": r["us"], "unit": "us", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": False, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "d": w.d,
                   "causal": w.causal, "l2": r["l2"]},
        "roofline": {"bound": "hbm", "achieved": r["hbm_gbs"], "peak": hbm, "unit": "GB/s",
                     "frac": r["hbm_frac"], "peak_kind": f"hbm_gbs ({peak_src})",
                     "traffic": None},
        "case": r, "gpu_launches": args.steps, "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def visible_pairs(nq, nk, wl, wr):
    """Number of (query, key) pairs a mask leaves visible (query i aligned with key i + nk - nq;
    key j visible iff i + off - wl <= j <= i + off + wr, negative = unbounded)."""
    total, off = 0, nk - nq
    for i in range(nq):
        lo = 0 if wl < 0 else max(0, i + off - wl)
        hi = nk - 1 if wr < 0 else min(nk - 1, i + off + wr)
        total += max(0, hi - lo + 1)
    return total


def time_variants(args, w, ea, q, k, v, do, ws, stream, causal_flops):
    """fwd+bwd time of grouped-query, sliding-window and (emulated) ring attention on the bench
    tensors. TFLOPS count only visible (query, key) pairs: 4·d FLOP per pair forward, 2.5 times
    that backward."""
    import torch
    from exact_attention_138_b200 import ring

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.variant_steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        if ea.device_status() != ea.ATTN_OK:
            raise SystemExit("device status not OK in the variant timings")
        return a.elapsed_time(b) / args.variant_steps

    per_pair = 3.5 * 4 * w.d          # forward 4·d FLOP per visible pair, backward 2.5x
    out = {"steps": args.variant_steps, "flops": "3.5 x 4·d per visible (query, key) pair"}
    B, H, n = w.B, w.H, w.n
    # grouped-query: 8 K/V heads (the first 8 of each batch's K and V)
    kv_heads = 8
    kg, vg = (t[:, :kv_heads].contiguous() for t in (k, v))

    def gqa():
        o, lse = ea.forward(q, kg, vg, causal=True, scale=w.scale, stream=stream)
        ea.backward(q, kg, vg, o, do, lse, causal=True, scale=w.scale, workspace=ws,
                    stream=stream)
    ms = timed(gqa)
    out["gqa_kv8"] = {"ms": ms, "tflops": causal_flops / (ms * 1e-3) / 1e12,
                      "config": f"H={H}, Hkv={kv_heads}, causal"}
    # no mask: every (query, key) pair (twice the causal FLOPs)
    def full():
        o, lse = ea.forward(q, k, v, causal=False, scale=w.scale, stream=stream)
        ea.backward(q, k, v, o, do, lse, causal=False, scale=w.scale, workspace=ws, stream=stream)
    ms = timed(full)
    out["no_mask"] = {"ms": ms, "tflops": B * H * n * n * per_pair / (ms * 1e-3) / 1e12,
                      "config": "unmasked (cross-attention shape with n_q = n_k)"}
    # sliding window: causal, 1024 keys to the left
    win = (1024, 0)
    pairs = B * H * visible_pairs(n, n, *win)

    def window():
        o, lse = ea.forward(q, k, v, scale=w.scale, window=win, stream=stream)
        ea.backward(q, k, v, o, do, lse, scale=w.scale, window=win, workspace=ws, stream=stream)
    ms = timed(window)
    out["window_1024"] = {"ms": ms, "tflops": pairs * per_pair / (ms * 1e-3) / 1e12,
                          "config": "causal window of 1025 keys (left 1024, right 0)"}
    # ring attention, 4 ranks emulated in one process (zigzag chunks): the whole job's kernels
    ranks = 4
    c = torch.chunk
    chunks = [c(t, 2 * ranks, dim=2) for t in (q, k, v, do)]
    per_rank = [[torch.cat([x[p], x[2 * ranks - 1 - p]], dim=2).contiguous() for p in range(ranks)]
                for x in chunks]
    rq, rk, rv, rdo = per_rank
    ops = ring.CudaOps()        # one set of buffers and workspaces for every step
    os_, lses = ring.ring_forward_emulated(rq, rk, rv, causal=True, scale=w.scale, zigzag=True,
                                           ops=ops)

    def ring_step():
        o_, l_ = ring.ring_forward_emulated(rq, rk, rv, causal=True, scale=w.scale, zigzag=True,
                                            ops=ops)
        ring.ring_backward_emulated(rq, rk, rv, o_, rdo, l_, causal=True, scale=w.scale,
                                    zigzag=True, ops=ops)
    ms = timed(ring_step)
    out["ring_zigzag_4"] = {"ms": ms, "tflops": causal_flops / (ms * 1e-3) / 1e12,
                            "config": "4 ranks emulated on one GPU, each on its own CUDA "
                                      "stream (hop r+1 of rank p waits for hop r of rank p-1), "
                                      "zigzag chunks of 1024 rows, one launch per hop; same "
                                      "FLOPs as the bench step"}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the extra timing of the FP8 (E4M3) forward pass")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the extra timings of grouped-query, sliding-window and ring "
                         "attention on the bench inputs")
    ap.add_argument("--variant-steps", type=int, default=20)
    ap.add_argument("--no-small-cases", action="store_true",
                    help="skip the per-launch timings of the small forward-only cases")
    ap.add_argument("--small-case-launches", type=int, default=50)
    ap.add_argument("--deterministic", action="store_true",
                    help="time the backward with deterministic (ordered) dQ accumulation")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="named workload of attn_inputs.WORKLOADS (profiling runs use a smaller "
                         "one; the headline is the default)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    import attn_inputs
    w = attn_inputs.WORKLOADS[args.workload]
    if not w.backward:
        if args.impl == "reference":
            ap.error("the reference arm times the forward+backward workloads")
        return run_forward_case(args, w)
    if not (w.causal and w.dtype == "bf16"):
        ap.error("the bench workload must be a causal bf16 forward+backward workload")
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import exact_attention_138_b200 as ea
    stream = torch.cuda.current_stream()

    # --- the pages' small forward-only cases, per launch with L2 flushed in between. They run
    # before the long step, whose power draw can leave the SM clock below its maximum for a
    # while; the clock they saw is recorded beside them.
    small = None
    if not args.no_small_cases and world == 1:
        hbm = load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        fma = fma_peak_tflops(1965.0)
        with ClockSampler(local) as small_clocks:
            small = {name: time_forward_case(ea, attn_inputs.WORKLOADS[name], dev, stream,
                                             args.small_case_launches, args.warmup, hbm, fma)
                     for name in SMALL_CASES}
            # the row-tiling case's bf16 inputs quantised to E4M3, through the FP8 forward
            small["rowtile_e4m3_4096x64"] = time_forward_case(
                ea, attn_inputs.WORKLOADS["rowtile_bf16_4096x64"], dev, stream,
                args.small_case_launches, args.warmup, hbm, fma, e4m3=True)
        small["peaks"] = {"hbm_gbs": hbm, "fp32_fma_tflops": fma,
                          "fp32_fma_kind": "148 SMs x 128 lanes x 2 FLOP x 1965 MHz"}
        small["clocks"] = small_clocks.summary()

    # --- inputs: each rank draws its own batch (seed 9 + rank), rounded to bf16 on the host
    q_h, k_h, v_h, do_h = attn_inputs.bf16_draws(w.shape, factor=w.factor, seed=rank_seed(rank))
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.n), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    det = bool(args.deterministic)
    ws = torch.empty(ea.attn_bwd_workspace_bytes(w.B, w.H, w.n, w.d, int(det)), dtype=torch.uint8,
                     device=dev)

    def step():
        ea.forward(q, k, v, causal=True, scale=w.scale, out=o, lse=lse, stream=stream)
        ea.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, dq=dq, dk=dk, dv=dv,
                    workspace=ws, stream=stream, deterministic=det)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ea.device_status() != ea.ATTN_OK:
        raise SystemExit("device status not OK after warm-up")

    # --- timed region: K steps; per-kernel events for the roofline
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for row in ev:              # torch creates the CUDA event at its first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for s in range(args.steps):
            e = ev[s]
            e[0].record(stream)
            ea.forward(q, k, v, causal=True, scale=w.scale, out=o, lse=lse, stream=stream)
            ea.attn_set_bwd_phase_events(e[1:5])
            ea.backward(q, k, v, o, do, lse, causal=True, scale=w.scale, dq=dq, dk=dk, dv=dv,
                        workspace=ws, stream=stream, deterministic=det)
            ea.attn_set_bwd_phase_events(None)
            e[5].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    if ea.device_status() != ea.ATTN_OK:
        raise SystemExit("device status not OK after the timed region")
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    pre_ms = [e[1].elapsed_time(e[2]) for e in ev]
    main_ms = [e[2].elapsed_time(e[3]) for e in ev]
    conv_ms = [e[3].elapsed_time(e[4]) for e in ev]
    bwd_ms = [e[1].elapsed_time(e[4]) for e in ev]
    total_ms = max_over_ranks(total_ms, dist, dev)

    fwd_flops, bwd_flops = step_flops(w.B, w.H, w.n, w.d)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(fwd_flops + bwd_flops, world, ms_per_step)
    peaks, peak_src = load_peaks()
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    fwd_tf = fwd_flops / (statistics.mean(fwd_ms) * 1e-3) / 1e12
    bwd_tf = bwd_flops / (statistics.mean(bwd_ms) * 1e-3) / 1e12
    main_tf = bwd_flops / (statistics.mean(main_ms) * 1e-3) / 1e12

    # --- extra: the FP8 (E4M3) forward pass on the same inputs, quantised with descale 2^-4
    fp8 = None
    if w.d in (64, 128) and not args.no_fp8:
        desc = 2.0 ** -4
        q8, k8, v8 = ((t.float() / desc).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
                      for t in (q, k, v))

        def fwd8():
            ea.forward_fp8(q8, k8, v8, desc, desc, desc, causal=True, scale=w.scale, out=o,
                           lse=lse, stream=stream)

        for _ in range(args.warmup):
            fwd8()
        torch.cuda.synchronize()
        barrier()
        a8 = torch.cuda.Event(enable_timing=True)
        b8 = torch.cuda.Event(enable_timing=True)
        a8.record(stream)
        for _ in range(args.steps):
            fwd8()
        b8.record(stream)
        torch.cuda.synchronize()
        if ea.device_status() != ea.ATTN_OK:
            raise SystemExit("device status not OK after the FP8 forward")
        ms8 = max_over_ranks(a8.elapsed_time(b8) / args.steps, dist, dev)
        tf8 = fwd_flops / (ms8 * 1e-3) / 1e12
        fp8 = {"ms": ms8, "tflops": tf8, "peak": 2 * burst,
               "peak_kind": "bf16_tflops x 2 (nominal fp8 / bf16 dense ratio)",
               "pct_of_peak": 100 * tf8 / (2 * burst),
               "inputs": "the workload's q, k, v quantised to E4M3 with descale 2^-4",
               "steps": args.steps}
        del q8, k8, v8

    # --- extra: the next rows on the same inputs (fwd + bwd per step, short runs)
    variants = None
    if not args.no_variants and world == 1:
        variants = time_variants(args, w, ea, q, k, v, do, ws, stream, fwd_flops + bwd_flops)

    # --- end to end through the public API with host buffers (pinned), copies inside the timing.
    # Three streams run as a pipeline: while step k computes, step k+1's inputs travel host ->
    # device and step k-1's results device -> host (two device buffer sets; every step copies
    # its full inputs in and its outputs and LSE out).
    pin = [t.pin_memory() for t in (q_h, k_h, v_h, do_h)]
    outs_h = [torch.empty(w.shape, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    lse_h = torch.empty((w.B, w.H, w.n), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin)
    d2h = sum(t.numel() * t.element_size() for t in outs_h) + lse_h.numel() * 4
    ins = [(q, k, v, do), tuple(torch.empty_like(t) for t in (q, k, v, do))]
    outs = [(o, dq, dk, dv, lse),
            (torch.empty_like(o), torch.empty_like(dq), torch.empty_like(dk), torch.empty_like(dv),
             torch.empty_like(lse))]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n_steps):
        for e in ev_comp + ev_out:          # all buffers free at the start
            e.record(stream)
        for st in range(n_steps):
            b = st % 2
            qb, kb, vb, dob = ins[b]
            ob, dqb, dkb, dvb, lseb = outs[b]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b])          # step st-2 finished reading ins[b]
                for dst, src in zip(ins[b], pin):
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])             # step st-2's results have left outs[b]
            ea.forward(qb, kb, vb, causal=True, scale=w.scale, out=ob, lse=lseb, stream=stream)
            ea.backward(qb, kb, vb, ob, dob, lseb, causal=True, scale=w.scale, dq=dqb, dk=dkb,
                        dv=dvb, workspace=ws, stream=stream, deterministic=det)
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                for dst, src in zip(outs_h, (ob, dqb, dkb, dvb)):
                    dst.copy_(src, non_blocking=True)
                lse_h.copy_(lseb, non_blocking=True)
                ev_out[b].record(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b_end = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    e2e_run(args.e2e_steps)
    stream.wait_stream(s_out)
    b_end.record(stream)
    torch.cuda.synchronize()
    if ea.device_status() != ea.ATTN_OK:
        raise SystemExit("device status not OK after the end-to-end steps")
    e2e_ms = a.elapsed_time(b_end) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    e2e_value = whole_job_tflops(fwd_flops + bwd_flops, world, e2e_ms)

    clk = clocks.summary()
    main_kernel = "bwd_main_q64_kernel" if w.d == 128 else "bwd_main_kernel"
    fwd_kernel = "fwd_bf16_kernel"
    peak, peak_kind = roofline_peak(burst, sustained, total_ms, clk, peak_src)
    fwd_algo_bytes = fwd_case_bytes(w)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "d": w.d, "causal": True,
                   "input_factor": w.factor, "global_batch": w.B * world,
                   "dq_accumulation": "deterministic" if det else "atomic",
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": f"inputs larger than L2 (q,k,v,dO {w.B*w.H*w.n*w.d*2/2**20:.0f} MiB "
                         f"each); no flush"},
        "fwd": {"ms": statistics.mean(fwd_ms), "tflops": fwd_tf,
                "pct_of_burst_peak": 100 * fwd_tf / burst},
        "bwd": {"ms": statistics.mean(bwd_ms), "tflops": bwd_tf,
                "pct_of_burst_peak": 100 * bwd_tf / burst,
                "preprocess_ms": statistics.mean(pre_ms), "main_ms": statistics.mean(main_ms),
                "dq_convert_ms": statistics.mean(conv_ms)},
        "pct_of_burst_peak": 100 * (value / world) / burst,
        "roofline": {"kernel": main_kernel, "bound": "tensor", "achieved": main_tf,
                     "peak": peak, "unit": "TFLOP/s", "frac": main_tf / peak,
                     "peak_kind": peak_kind,
                     "frac_of_burst": main_tf / burst, "frac_of_sustained": main_tf / sustained,
                     "traffic": recorded_traffic(main_kernel, w.name),
                     "algorithmic_bytes": bwd_main_bytes(w)},
        "roofline_fwd": {"kernel": fwd_kernel, "bound": "tensor", "achieved": fwd_tf,
                         "peak": peak, "unit": "TFLOP/s", "frac": fwd_tf / peak,
                         "peak_kind": peak_kind,
                         "frac_of_burst": fwd_tf / burst, "frac_of_sustained": fwd_tf / sustained,
                         "traffic": recorded_traffic(fwd_kernel, w.name),
                         "algorithmic_bytes": fwd_algo_bytes},
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps,
                "schedule": "3-stream pipeline: step k+1 host->device, step k compute, "
                            "step k-1 device->host"},
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
    }
    if fp8 is not None:
        line["fp8_fwd"] = fp8
    if variants is not None:
        line["variants"] = variants
    if small is not None:
        line["small_cases"] = small
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, rows_n, threads = oracle_sample(args.cpu_seconds, q_h, k_h, v_h, do_h, w)
        line["cpu_baseline"] = {
            "value": rate, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"{rows_n} query rows (forward O/LSE + backward dQ, fp64) in {dt:.1f} s; "
                      f"credited at the workload's average FLOPs per query row"}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
