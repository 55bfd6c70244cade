"""Helpers shared by the GPU parity tests: run the CUDA path through the binding and compare
with the fp64 oracle on the same (bf16-rounded or fp32) inputs."""
import numpy as np
import torch

# Tolerances. O: max abs 1e-5 (fp32) / 1e-2 (bf16); gradients: Frobenius relative error 2e-2
# per tensor; LSE: 1e-5 (fp32) / 1e-3 (bf16) absolute.
TOL_O = {"fp32": 1e-5, "bf16": 1e-2}
TOL_LSE = {"fp32": 1e-5, "bf16": 1e-3}
TOL_GRAD_REL = 2e-2


def rel_fro(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def grad_close(got, want, tol=TOL_GRAD_REL, zero_atol=1e-4):
    """Frobenius relative error <= tol; where the exact gradient is identically zero (n = 1:
    P = 1 so dS = 0, hence dQ = dK = 0) the result must be zero up to rounding residue."""
    want = np.asarray(want, np.float64)
    if not np.any(want):
        return float(np.abs(np.asarray(got, np.float64)).max()) <= zero_atol
    return rel_fro(got, want) <= tol


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def cuda_forward(q, k, v, causal, scale):
    import exact_attention_138_b200 as ea
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    o, lse = ea.forward(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    return o, lse, (qd, kd, vd)


def cuda_backward(dev_inputs, o, lse, do, causal, scale, deterministic=False):
    import exact_attention_138_b200 as ea
    qd, kd, vd = dev_inputs
    dod = do.to(qd.device).contiguous()
    dq, dk, dv = ea.backward(qd, kd, vd, o, dod, lse, causal=causal, scale=scale,
                             deterministic=deterministic)
    torch.cuda.synchronize()
    assert ea.device_status() == ea.ATTN_OK
    return dq, dk, dv
