"""Host-side arithmetic of bench.py that needs no GPU: the FLOP convention of the step, the
algorithmic bytes of the small forward-only cases, and the FFMA peak used for the fp32 kernel."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import attn_inputs  # noqa: E402
import bench  # noqa: E402


def test_step_flops_of_the_bench_workload():
    # forward 4·B·H·n²·d halved by the causal mask; backward 2.5 x forward
    fwd, bwd = bench.step_flops(2, 32, 8192, 128)
    assert fwd == 1_099_511_627_776
    assert bwd == 2_748_779_069_440
    fwd_full, _ = bench.step_flops(1, 1, 4096, 64, causal=False)
    assert fwd_full == 4 * 4096 * 4096 * 64


def test_small_case_bytes_and_tiles():
    by_name = {n: attn_inputs.WORKLOADS[n] for n in bench.SMALL_CASES}
    # q, k, v read and O written (4 tensors of B·H·n·d elements) plus the fp32 LSE
    assert bench.fwd_case_bytes(by_name["p1_fp32_2x3x128x32"]) == 4 * 2 * 3 * 128 * 32 * 4 + 4 * 768
    assert bench.fwd_case_bytes(by_name["rowtile_fp32_4096x64"]) == 4_210_688
    assert bench.fwd_case_bytes(by_name["rowtile_bf16_4096x64"]) == 4 * 4096 * 64 * 2 + 4 * 4096
    # 64-row query tiles in fp32, 128-row tiles in bf16
    assert bench.fwd_case_query_tiles(by_name["p1_fp32_2x3x128x32"]) == 12
    assert bench.fwd_case_query_tiles(by_name["rowtile_fp32_4096x64"]) == 64
    assert bench.fwd_case_query_tiles(by_name["rowtile_bf16_4096x64"]) == 32
    assert all(not w.backward for w in by_name.values())


def test_fma_peak():
    # 148 SMs x 128 fp32 lanes x 2 FLOP per FFMA at 1965 MHz
    assert abs(bench.fma_peak_tflops(1965.0) - 74.44992) < 1e-9


def test_roofline_peak_choice():
    # burst unless the timed region is over a second AND the power cap was seen
    burst, sust = 1655.5, 1405.2
    p, why = bench.roofline_peak(burst, sust, 80.0, {"reasons": ["sw_power_cap"]}, "measured")
    assert p == burst and "burst" in why
    p, why = bench.roofline_peak(burst, sust, 5000.0, {"reasons": []}, "measured")
    assert p == burst
    p, why = bench.roofline_peak(burst, sust, 5000.0, {"reasons": ["sw_power_cap"]}, "measured")
    assert p == sust and "sustained" in why


def test_backward_main_algorithmic_bytes():
    # 2x32x8192x128: Q, K, V, dO in and dK, dV out (bf16), LSE·log2e and D (fp32), fp32 dQ
    # accumulator read and written once
    w = attn_inputs.WORKLOADS["causal_bf16_2x32x8192x128"]
    rows = 2 * 32 * 8192
    assert bench.bwd_main_bytes(w) == rows * 128 * 2 * 6 + rows * 8 + rows * 128 * 8
    assert abs(bench.bwd_main_bytes(w) / 1e9 - 1.3465) < 1e-3
