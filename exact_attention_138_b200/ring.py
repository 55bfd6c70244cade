"""Ring attention: exact attention over a sequence split into chunks, one chunk per rank
("Attention Mechanism: Revolusi Representasi Sequence", §16 "Long Context Training", Ring
Attention; §6, long-context techniques table).

Rank p holds the queries, keys and values of chunk p (all chunks the same length). In hop r it
attends its queries to K/V chunk (p - r) mod N, which arrived from rank p - 1, while sending the
chunk it holds on to rank p + 1; the partial results are folded together with the log-sum-exp
rule (attn_ring_merge). Under a causal mask a hop is either unmasked (an earlier chunk), causal
(its own chunk) or skipped (a later chunk). The backward pass walks the same ring with the final
O and LSE: dQ accumulates locally over the hops, and the dK / dV accumulators travel with their
chunk and arrive back at its owner after the last hop.

Every arithmetic step runs in the library's CUDA kernels (attn_fwd_ex / attn_bwd_ex per hop,
attn_ring_merge / attn_ring_accumulate between hops); this module only schedules them and moves
chunks with torch.distributed point-to-point operations (NCCL on GPUs), which run on NCCL's
stream and overlap the current hop's kernels. `ring_forward_emulated` / `ring_backward_emulated`
run the same schedule for N ranks inside one process (chunks are indexed instead of sent), which
is how the kernels of the multi-rank path are checked on a single GPU.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist


def hop_window(q_chunk: int, kv_chunk: int, causal: bool):
    """(window_left, window_right) for the queries of one chunk against the keys of another, or
    None when no key of that chunk is visible (a later chunk under a causal mask)."""
    if not causal or kv_chunk < q_chunk:
        return (-1, -1)
    if kv_chunk == q_chunk:
        return (-1, 0)
    return None


def _last_hop(rank: int, world: int, causal: bool) -> int:
    # hop r visits chunk (rank - r) mod world; with a causal mask chunks after `rank` are skipped
    return rank if causal else world - 1


class CudaOps:
    """The per-hop operations, all in libattn.so."""

    def __init__(self):
        import exact_attention_138_b200 as ea
        self.ea = ea

    def fwd(self, q, k, v, scale, window):
        return self.ea.forward(q, k, v, scale=scale, window=window)

    def bwd(self, q, k, v, o, do, lse, scale, window, deterministic):
        return self.ea.backward(q, k, v, o, do, lse, scale=scale, window=window,
                                deterministic=deterministic)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out):
        self.ea.ring_merge(o_acc, lse_acc, o_part, lse_part, first=first, out=out)

    def accumulate(self, acc, part, first, out):
        self.ea.ring_accumulate(acc, part, first=first, out=out)


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


class _FwdState:
    def __init__(self, q):
        self.o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        self.lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
        self.out = torch.empty_like(q)
        self.first = True


def _fwd_hop(ops, st, q, k, v, rank, world, r, causal, scale):
    w = hop_window(rank, (rank - r) % world, causal)
    if w is None:
        return
    o_p, l_p = ops.fwd(q, k, v, scale, w)
    last = r == _last_hop(rank, world, causal)
    ops.merge(st.o_acc, st.lse, o_p, l_p, st.first, st.out if last else None)
    st.first = False


class _BwdState:
    def __init__(self, q):
        self.dq_acc = torch.zeros(q.shape, dtype=torch.float32, device=q.device)


def _bwd_hop(ops, st, q, k, v, o, do, lse, dk_acc, dv_acc, rank, world, r, causal, scale, det):
    w = hop_window(rank, (rank - r) % world, causal)
    if w is None:
        return
    dq_p, dk_p, dv_p = ops.bwd(q, k, v, o, do, lse, scale, w, det)
    ops.accumulate(st.dq_acc, dq_p, False, None)
    ops.accumulate(dk_acc, dk_p, False, None)
    ops.accumulate(dv_acc, dv_p, False, None)


def _peers(group):
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    to_global = (lambda x: dist.get_global_rank(group, x)) if group is not None else (lambda x: x)
    return rank, world, to_global((rank + 1) % world), to_global((rank - 1) % world)


def _exchange(tensors, nxt, prv, group):
    """Start sending `tensors` to the next rank and receiving same-shaped ones from the previous
    rank; returns (received tensors, requests)."""
    recv = [torch.empty_like(t) for t in tensors]
    ops = [dist.P2POp(dist.isend, t, nxt, group) for t in tensors]
    ops += [dist.P2POp(dist.irecv, t, prv, group) for t in recv]
    return recv, dist.batch_isend_irecv(ops)


def ring_forward(q, k, v, causal=False, scale=None, group=None, ops=None):
    """O, LSE of attention over the whole sequence for this rank's query chunk. q: (B,H,n,d),
    k, v: (B,Hkv,n,d) chunks of the same length on every rank (chunk index = rank)."""
    ops = ops or CudaOps()
    scale = _scale(q, scale)
    rank, world, nxt, prv = _peers(group)
    st = _FwdState(q)
    cur = [k.contiguous(), v.contiguous()]
    for r in range(world):
        reqs = None
        if r < world - 1:
            nxt_kv, reqs = _exchange(cur, nxt, prv, group)
        _fwd_hop(ops, st, q, cur[0], cur[1], rank, world, r, causal, scale)
        if reqs is not None:
            for req in reqs:
                req.wait()
            cur = nxt_kv
    return st.out, st.lse


def ring_backward(q, k, v, o, do, lse, causal=False, scale=None, group=None, ops=None,
                  deterministic=False):
    """dQ, dK, dV of ring attention for this rank's chunk, given the final O and LSE of
    `ring_forward` and dO."""
    ops = ops or CudaOps()
    scale = _scale(q, scale)
    rank, world, nxt, prv = _peers(group)
    st = _BwdState(q)
    cur = [k.contiguous(), v.contiguous()]
    acc = [torch.zeros(k.shape, dtype=torch.float32, device=k.device),
           torch.zeros(v.shape, dtype=torch.float32, device=v.device)]
    for r in range(world):
        reqs = None
        if r < world - 1:
            nxt_kv, reqs = _exchange(cur, nxt, prv, group)
        _bwd_hop(ops, st, q, cur[0], cur[1], o, do, lse, acc[0], acc[1], rank, world, r, causal,
                 scale, deterministic)
        # the dK / dV accumulators travel on with their chunk; after the last hop each rank holds
        # its own chunk's
        nxt_acc, acc_reqs = _exchange(acc, nxt, prv, group)
        for req in (reqs or []) + acc_reqs:
            req.wait()
        if reqs is not None:
            cur = nxt_kv
        acc = nxt_acc
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ops.accumulate(st.dq_acc, None, False, dq)
    ops.accumulate(acc[0], None, False, dk)
    ops.accumulate(acc[1], None, False, dv)
    return dq, dk, dv


def ring_forward_emulated(qs, ks, vs, causal=False, scale=None, ops=None):
    """The ring_forward schedule for len(qs) ranks in one process (chunk lists, one per rank)."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    states = [_FwdState(q) for q in qs]
    for r in range(world):
        for p in range(world):
            s = (p - r) % world      # the chunk rank p holds in hop r
            _fwd_hop(ops, states[p], qs[p], ks[s], vs[s], p, world, r, causal, scale)
    return [s.out for s in states], [s.lse for s in states]


def ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=False, scale=None, ops=None,
                           deterministic=False):
    """The ring_backward schedule for len(qs) ranks in one process."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    states = [_BwdState(q) for q in qs]
    dk_acc = [torch.zeros(k.shape, dtype=torch.float32, device=k.device) for k in ks]
    dv_acc = [torch.zeros(v.shape, dtype=torch.float32, device=v.device) for v in vs]
    for r in range(world):
        for p in range(world):
            s = (p - r) % world
            _bwd_hop(ops, states[p], qs[p], ks[s], vs[s], os_[p], dos[p], lses[p], dk_acc[s],
                     dv_acc[s], p, world, r, causal, scale, deterministic)
    dqs, dks, dvs = [], [], []
    for p in range(world):
        dq, dk, dv = torch.empty_like(qs[p]), torch.empty_like(ks[p]), torch.empty_like(vs[p])
        ops.accumulate(states[p].dq_acc, None, False, dq)
        ops.accumulate(dk_acc[p], None, False, dk)
        ops.accumulate(dv_acc[p], None, False, dv)
        dqs.append(dq)
        dks.append(dk)
        dvs.append(dv)
    return dqs, dks, dvs
