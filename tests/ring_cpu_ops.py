"""CPU stand-ins (fp64 numpy) for the per-hop operations of the ring schedule, so that the
multi-rank schedule and its point-to-point exchanges can run as gloo ranks on the CPU. The hop
forward is the oracle's masked definition; the hop backward uses the global LSE and O (as the
CUDA kernels do): P = exp(scale·q·k - LSE), D = rowsum(dO∘O), dS = P∘(dP - D), with dQ summed in
the query chunk's state and dK, dV added into the travelling fp32 accumulators."""
import numpy as np
import torch

import oracle


def _np(t):
    return t.detach().cpu().numpy().astype(np.float64)


def _visible(nq, nk, wl, wr):
    i = np.arange(nq)[:, None] + (nk - nq)
    j = np.arange(nk)[None, :]
    vis = np.ones((nq, nk), bool)
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    return vis


class CpuOps:
    def fwd(self, q, k, v, scale, window):
        o, lse = oracle.fwd_ex(q.float().numpy(), k.float().numpy(), v.float().numpy(), scale,
                               window[0], window[1])
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out):
        la = np.full(lse_part.shape, -np.inf) if first else _np(lse_acc)
        lb = _np(lse_part)
        L = np.logaddexp(la, lb)
        with np.errstate(invalid="ignore"):
            wa = np.where(np.isneginf(la), 0.0, np.exp(la - L))
            wb = np.where(np.isneginf(lb), 0.0, np.exp(lb - L))
        oa = np.zeros(o_acc.shape) if first else _np(o_acc)
        o = wa[..., None] * oa + wb[..., None] * _np(o_part)
        o_acc.copy_(torch.from_numpy(o))
        lse_acc.copy_(torch.from_numpy(L))
        if out is not None:
            out.copy_(torch.from_numpy(o))

    def fwd_fold(self, o_acc, lse_acc, first, q, k, v, scale, window, slot=0):
        o_p, l_p = self.fwd(q, k, v, scale, window)
        self.merge(o_acc, lse_acc, o_p, l_p, first, None)

    def bwd_begin(self, key, o, do, lse, deterministic):
        """State of the rank's queries: D = rowsum(dO∘O), the global LSE and a zero dQ sum."""
        O, dO, L = _np(o), _np(do), _np(lse)
        return {"D": (dO * O).sum(-1), "L": L, "dq": np.zeros(O.shape)}

    def bwd_add(self, st, q, k, v, do, dk_acc, dv_acc, scale, window, q_row0):
        Q, K, V, dO = (_np(x) for x in (q, k, v, do))
        rows = slice(q_row0, q_row0 + Q.shape[2])
        H, Hkv = Q.shape[1], K.shape[1]
        K, V = np.repeat(K, H // Hkv, axis=1), np.repeat(V, H // Hkv, axis=1)
        vis = _visible(Q.shape[2], K.shape[2], *window)
        S = np.einsum("bhid,bhjd->bhij", Q, K) * scale
        P = np.where(vis, np.exp(S - st["L"][:, :, rows][..., None]), 0.0)
        dP = np.einsum("bhid,bhjd->bhij", dO, V)
        dS = P * (dP - st["D"][:, :, rows][..., None])
        st["dq"][:, :, rows] += np.einsum("bhij,bhjd->bhid", dS, K)
        dk = scale * np.einsum("bhij,bhid->bhjd", dS, Q)
        dv = np.einsum("bhij,bhid->bhjd", P, dO)
        B, _, n, d = dk.shape
        dk_acc.copy_(torch.from_numpy(_np(dk_acc) + dk.reshape(B, Hkv, H // Hkv, n, d).sum(2)))
        dv_acc.copy_(torch.from_numpy(_np(dv_acc) + dv.reshape(B, Hkv, H // Hkv, n, d).sum(2)))

    def bwd_finish(self, st, out, scale):
        out.copy_(torch.from_numpy(scale * st["dq"]))
        return out

    def accumulate(self, acc, part, first, out):
        a = np.zeros(acc.shape) if first else _np(acc)
        if part is not None:
            a = a + _np(part)
        acc.copy_(torch.from_numpy(a))
        if out is not None:
            out.copy_(torch.from_numpy(a))
