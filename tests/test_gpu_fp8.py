"""GPU check of the FP8 (E4M3) forward pass against the fp64 oracle on the dequantised inputs
("Flash Attention Nedir?" / "Apa itu FlashAttention": FlashAttention-3 runs the method in FP8).

The kernel rounds the softmax weights P to E4M3 before P·V, so the bf16 path's 1e-2 bound does
not apply. The bound used here follows from that rounding: each weight carries a relative error of
at most 2^-4 (3 mantissa bits, round to nearest), and P·V / l is a convex combination, so an
output element moves by at most 2^-4·max|V|; bf16 output rounding adds 2^-9·|O|. Where every
weight is 0 or 1 (Q = 0 under a causal mask) the weights are exact and the bf16 bound holds."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from parity_util import TOL_LSE, TOL_O, to_np

pytestmark = pytest.mark.gpu

import exact_attention_138_b200 as ea  # noqa: E402

E4M3_MAX = 448.0


def _quant(x, descale):
    """fp32 tensor -> (E4M3 tensor, dequantised fp32 values) with real value = e4m3 · descale."""
    q8 = (x.float() / descale).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return q8, q8.float() * descale


def _case(shape_q, shape_kv, seed, desc=(2.0 ** -4, 2.0 ** -4, 2.0 ** -5)):
    q, = attn_inputs.random_draws(shape_q, dtype="fp32", seed=seed, count=1)
    k, v = attn_inputs.random_draws(shape_kv, dtype="fp32", seed=seed + 1, count=2)
    (q8, qd), (k8, kd), (v8, vd) = (_quant(x, s) for x, s in zip((q, k, v), desc))
    return (q8, k8, v8), (qd, kd, vd), desc


def _bound(vd, o_ref):
    return 2.0 ** -4 * float(vd.abs().max()) + 2.0 ** -9 * float(np.abs(o_ref).max()) + 1e-3


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,Hkv,nq,nk", [(1, 2, 2, 300, 300), (2, 2, 1, 129, 129),
                                           (1, 4, 2, 1000, 1000), (1, 2, 2, 200, 700)])
def test_fp8_forward_matches_dequantised_oracle(cuda_device, B, H, Hkv, nq, nk, d, causal):
    (q8, k8, v8), (qd, kd, vd), desc = _case((B, H, nq, d), (B, Hkv, nk, d), seed=nq + d)
    dev = torch.device("cuda:0")
    o, lse = ea.forward_fp8(q8.to(dev), k8.to(dev), v8.to(dev), *desc, causal=causal)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    scale = 1.0 / math.sqrt(d)
    ro, rlse = oracle.fwd_ex(qd.numpy(), kd.numpy(), vd.numpy(), scale, -1, 0 if causal else -1)
    err = np.abs(to_np(o) - ro)
    assert err.max() <= _bound(vd, ro)
    # the rounding errors of the weights are unbiased: the whole-tensor error stays far below the
    # per-element bound
    assert np.linalg.norm(to_np(o) - ro) / np.linalg.norm(ro) <= 3e-2
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["bf16"]


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_forward_exact_weights(cuda_device, d):
    # Q = 0 under a causal mask: row i weighs keys 0..i equally (P = 1 exactly in E4M3), so O is
    # the prefix mean of V and LSE = ln(i+1); this pins the P·V operand layout (including the byte
    # order of P in tensor memory) to within the bf16 bound
    n = 333
    v, = attn_inputs.random_draws((1, 2, n, d), dtype="fp32", seed=d, count=1)
    v8, vd = _quant(v, 2.0 ** -5)
    q8 = torch.zeros((1, 2, n, d), dtype=torch.float8_e4m3fn)
    k8, kd = _quant(attn_inputs.random_draws((1, 2, n, d), dtype="fp32", seed=d + 1, count=1)[0],
                    2.0 ** -4)
    dev = torch.device("cuda:0")
    o, lse = ea.forward_fp8(q8.to(dev), k8.to(dev), v8.to(dev), 1.0, 2.0 ** -4, 2.0 ** -5,
                            causal=True)
    torch.cuda.synchronize()
    want = np.cumsum(vd.numpy().astype(np.float64), axis=2) / np.arange(1, n + 1)[:, None]
    assert np.abs(to_np(o) - want).max() <= TOL_O["bf16"]
    np.testing.assert_allclose(to_np(lse)[0, 0], np.log(np.arange(1, n + 1)), rtol=0, atol=1e-5)


def test_fp8_forward_window_and_empty_rows(cuda_device):
    (q8, k8, v8), (qd, kd, vd), desc = _case((1, 2, 600, 128), (1, 2, 250, 128), seed=3)
    dev = torch.device("cuda:0")
    o, lse = ea.forward_fp8(q8.to(dev), k8.to(dev), v8.to(dev), *desc, window=(40, 0))
    torch.cuda.synchronize()
    ro, rlse = oracle.fwd_ex(qd.numpy(), kd.numpy(), vd.numpy(), 1 / math.sqrt(128), 40, 0)
    empty = np.isneginf(rlse)
    assert empty[0, 0, :350].all() and not empty[0, 0, 350:].any()
    assert np.array_equal(np.isneginf(to_np(lse)), empty)
    assert np.all(to_np(o)[empty] == 0)
    assert np.abs(to_np(o) - ro).max() <= _bound(vd, ro)


def test_fp8_rejects_bad_arguments(cuda_device):
    x = torch.zeros((1, 1, 128, 128), dtype=torch.float8_e4m3fn, device="cuda:0")
    with pytest.raises(ea.AttnError):
        ea.forward_fp8(x, x, x, q_descale=0.0)
    y = torch.zeros((1, 1, 128, 32), dtype=torch.float8_e4m3fn, device="cuda:0")
    with pytest.raises(ea.AttnError):
        ea.forward_fp8(y, y, y)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_small_grid_key_split(cuda_device, causal):
    # 1x1x4096x64, the size of the row-tiling example: 16 pairs of query tiles on 148 SMs, so each
    # pair's keys are split over a thread-block cluster and the shares merged on chip
    (q8, k8, v8), (qd, kd, vd), desc = _case((1, 1, 4096, 64), (1, 1, 4096, 64), seed=77)
    dev = torch.device("cuda:0")
    o, lse = ea.forward_fp8(q8.to(dev), k8.to(dev), v8.to(dev), *desc, causal=causal)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    ro, rlse = oracle.fwd(qd.numpy(), kd.numpy(), vd.numpy(), 1.0 / 8.0, causal)
    got = to_np(o)
    assert np.abs(got - ro).max() <= _bound(vd, ro)
    assert np.linalg.norm(got - ro) / np.linalg.norm(ro) <= 3e-2
    assert np.abs(to_np(lse) - rlse).max() <= TOL_LSE["bf16"]
