"""Ring attention: exact attention over a sequence split into chunks held by different ranks
("Attention Mechanism: Revolusi Representasi Sequence", §16 "Long Context Training", Ring
Attention; §6, long-context techniques table).

Layouts. With N ranks the sequence is cut into equal chunks:
  contiguous  N chunks; rank p holds chunk p.
  zigzag      2N chunks; rank p holds chunks p and 2N-1-p (its q, k, v are those two chunks one
              after the other). Under a causal mask every rank then sees the same amount of work
              (the contiguous layout gives rank N-1 N times the work of rank 0).
In hop r a rank attends its query chunks to the K/V chunks of rank (p - r) mod N, which arrived
from rank p - 1, while sending the chunks it holds on to rank p + 1; the partial results of each
query chunk are folded together with the log-sum-exp rule (attn_ring_merge). Under a causal mask
a (query chunk, key chunk) pair is unmasked (earlier key chunk), causal (same chunk) or skipped
(later key chunk). The backward pass walks the same ring with the final O and LSE: dQ accumulates
locally, and the dK / dV accumulators travel with their chunks and arrive back at their owner
after the last hop.

Every arithmetic step runs in the library's CUDA kernels (attn_fwd_ex / attn_bwd_ex per chunk
pair, attn_ring_merge / attn_ring_accumulate between them); this module only schedules them and
moves chunks with torch.distributed point-to-point operations (NCCL on GPUs), which run on NCCL's
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


def rank_chunks(rank: int, world: int, zigzag: bool):
    """Global indices of the chunks rank `rank` holds, in the order its tensors store them."""
    return [rank, 2 * world - 1 - rank] if zigzag else [rank]


class CudaOps:
    """The per-chunk-pair operations, all in libattn.so. One set of per-hop output buffers and one
    backward workspace are kept and reused by every hop of a ring pass (each hop's partials are
    folded into the running results on the same stream before the next hop overwrites them)."""

    def __init__(self):
        import exact_attention_138_b200 as ea
        self.ea = ea
        self._bufs = {}

    def _buf(self, key, shape, dtype, device):
        t = self._bufs.get(key)
        if t is None or tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device:
            t = torch.empty(shape, dtype=dtype, device=device)
            self._bufs[key] = t
        return t

    def fwd(self, q, k, v, scale, window):
        o = self._buf("o", q.shape, q.dtype, q.device)
        lse = self._buf("lse", q.shape[:-1], torch.float32, q.device)
        return self.ea.forward(q, k, v, scale=scale, window=window, out=o, lse=lse)

    def bwd(self, q, k, v, o, do, lse, scale, window, deterministic):
        """(dQ partial, dK and dV partials stacked as one (2, B, Hkv, n, d) tensor)."""
        B, H, n, d = q.shape
        dq = self._buf("dq", q.shape, q.dtype, q.device)
        dkv = self._buf("dkv", (2,) + tuple(k.shape), k.dtype, k.device)
        need = self.ea.attn_bwd_workspace_bytes(B, H, n, d, int(bool(deterministic)))
        ws = self._bufs.get("ws")
        if ws is None or ws.numel() < need or ws.device != q.device:
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            self._bufs["ws"] = ws
        self.ea.backward(q, k, v, o, do, lse, scale=scale, window=window,
                         deterministic=deterministic, dq=dq, dk=dkv[0], dv=dkv[1], workspace=ws)
        return dq, dkv

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out):
        self.ea.ring_merge(o_acc, lse_acc, o_part, lse_part, first=first, out=out)

    def accumulate(self, acc, part, first, out):
        self.ea.ring_accumulate(acc, part, first=first, out=out)


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


def _split(x, parts):
    """The chunks of a rank's (B, H, parts·c, d) tensor as contiguous tensors."""
    if parts == 1:
        return [x.contiguous()]
    return [c.contiguous() for c in torch.chunk(x, parts, dim=2)]


def _join(chunks):
    return chunks[0] if len(chunks) == 1 else torch.cat(chunks, dim=2)


class _FwdState:
    def __init__(self, q):
        self.o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        self.lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
        self.first = True


def _fwd_hop(ops, states, qs, q_ids, kvs, kv_ids, causal, scale):
    """Fold every visible (query chunk, key chunk) pair of one hop into the running results."""
    for qi, q in enumerate(qs):
        for ki, (k, v) in enumerate(kvs):
            w = hop_window(q_ids[qi], kv_ids[ki], causal)
            if w is None:
                continue
            o_p, l_p = ops.fwd(q, k, v, scale, w)
            st = states[qi]
            ops.merge(st.o_acc, st.lse, o_p, l_p, st.first, None)
            st.first = False


def _fwd_outputs(ops, states, qs):
    outs = []
    for st, q in zip(states, qs):
        out = torch.empty_like(q)
        ops.accumulate(st.o_acc, None, False, out)    # fp32 running output -> q's dtype
        outs.append(out)
    return _join(outs), _join([st.lse for st in states])


def _bwd_hop(ops, dq_acc, qs, q_ids, os_, dos, lses, kvs, kv_ids, dkv_acc, causal, scale, det):
    for qi, q in enumerate(qs):
        for ki, (k, v) in enumerate(kvs):
            w = hop_window(q_ids[qi], kv_ids[ki], causal)
            if w is None:
                continue
            dq_p, dkv_p = ops.bwd(q, k, v, os_[qi], dos[qi], lses[qi], scale, w, det)
            ops.accumulate(dq_acc[qi], dq_p, False, None)
            ops.accumulate(dkv_acc[ki], dkv_p, False, None)      # dK and dV in one pass


def _convert(ops, accs, likes):
    outs = []
    for acc, like in zip(accs, likes):
        out = torch.empty_like(like)
        ops.accumulate(acc, None, False, out)
        outs.append(out)
    return _join(outs)


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


def ring_forward(q, k, v, causal=False, scale=None, group=None, ops=None, zigzag=False):
    """O, LSE of attention over the whole sequence for this rank's query chunks. q: (B,H,n,d),
    k, v: (B,Hkv,n,d) holding this rank's chunk(s) of the layout (n = one chunk, or two chunks
    for zigzag); every rank's chunks have the same length."""
    ops = ops or CudaOps()
    scale = _scale(q, scale)
    rank, world, nxt, prv = _peers(group)
    parts = 2 if zigzag else 1
    q_ids = rank_chunks(rank, world, zigzag)
    qs = _split(q, parts)
    states = [_FwdState(c) for c in qs]
    cur = _split(k, parts) + _split(v, parts)          # k chunks, then v chunks
    for r in range(world):
        reqs = None
        if r < world - 1:
            nxt_kv, reqs = _exchange(cur, nxt, prv, group)
        kv_ids = rank_chunks((rank - r) % world, world, zigzag)
        kvs = list(zip(cur[:parts], cur[parts:]))
        _fwd_hop(ops, states, qs, q_ids, kvs, kv_ids, causal, scale)
        if reqs is not None:
            for req in reqs:
                req.wait()
            cur = nxt_kv
    return _fwd_outputs(ops, states, qs)


def ring_backward(q, k, v, o, do, lse, causal=False, scale=None, group=None, ops=None,
                  deterministic=False, zigzag=False):
    """dQ, dK, dV of ring attention for this rank's chunks, given the final O and LSE of
    `ring_forward` (same layout) and dO."""
    ops = ops or CudaOps()
    scale = _scale(q, scale)
    rank, world, nxt, prv = _peers(group)
    parts = 2 if zigzag else 1
    q_ids = rank_chunks(rank, world, zigzag)
    qs, os_, dos = _split(q, parts), _split(o, parts), _split(do, parts)
    lses = [c.contiguous() for c in torch.chunk(lse, parts, dim=2)]
    dq_acc = [torch.zeros(c.shape, dtype=torch.float32, device=c.device) for c in qs]
    ks, vs = _split(k, parts), _split(v, parts)
    cur = ks + vs
    # per K/V chunk: its dK and dV accumulators stacked, (2, B, Hkv, chunk, d) fp32
    acc = [torch.zeros((2,) + tuple(c.shape), dtype=torch.float32, device=c.device) for c in ks]
    for r in range(world):
        reqs = None
        if r < world - 1:
            nxt_kv, reqs = _exchange(cur, nxt, prv, group)
        kv_ids = rank_chunks((rank - r) % world, world, zigzag)
        kvs = list(zip(cur[:parts], cur[parts:]))
        _bwd_hop(ops, dq_acc, qs, q_ids, os_, dos, lses, kvs, kv_ids, acc, causal, scale,
                 deterministic)
        # the dK / dV accumulators travel on with their chunks; after the last hop each rank
        # holds its own chunks'
        nxt_acc, acc_reqs = _exchange(acc, nxt, prv, group)
        for req in (reqs or []) + acc_reqs:
            req.wait()
        if reqs is not None:
            cur = nxt_kv
        acc = nxt_acc
    return (_convert(ops, dq_acc, qs), _convert(ops, [a[0] for a in acc], ks),
            _convert(ops, [a[1] for a in acc], vs))


def ring_forward_emulated(qs, ks, vs, causal=False, scale=None, ops=None, zigzag=False):
    """The ring_forward schedule for len(qs) ranks in one process: qs[p], ks[p], vs[p] are rank
    p's tensors in the chosen layout."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    parts = 2 if zigzag else 1
    q_chunks = [_split(q, parts) for q in qs]
    kv_chunks = [list(zip(_split(k, parts), _split(v, parts))) for k, v in zip(ks, vs)]
    states = [[_FwdState(c) for c in qc] for qc in q_chunks]
    for r in range(world):
        for p in range(world):
            s = (p - r) % world      # the rank whose chunks rank p holds in hop r
            _fwd_hop(ops, states[p], q_chunks[p], rank_chunks(p, world, zigzag), kv_chunks[s],
                     rank_chunks(s, world, zigzag), causal, scale)
    outs = [_fwd_outputs(ops, states[p], q_chunks[p]) for p in range(world)]
    return [o for o, _ in outs], [l for _, l in outs]


def ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=False, scale=None, ops=None,
                           deterministic=False, zigzag=False):
    """The ring_backward schedule for len(qs) ranks in one process."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    parts = 2 if zigzag else 1
    q_chunks = [_split(q, parts) for q in qs]
    o_chunks = [_split(o, parts) for o in os_]
    do_chunks = [_split(x, parts) for x in dos]
    l_chunks = [[c.contiguous() for c in torch.chunk(x, parts, dim=2)] for x in lses]
    kv_chunks = [list(zip(_split(k, parts), _split(v, parts))) for k, v in zip(ks, vs)]
    dq_acc = [[torch.zeros(c.shape, dtype=torch.float32, device=c.device) for c in qc]
              for qc in q_chunks]
    dkv_acc = [[torch.zeros((2,) + tuple(k.shape), dtype=torch.float32, device=k.device)
                for k, _ in kvc] for kvc in kv_chunks]
    for r in range(world):
        for p in range(world):
            s = (p - r) % world
            _bwd_hop(ops, dq_acc[p], q_chunks[p], rank_chunks(p, world, zigzag), o_chunks[p],
                     do_chunks[p], l_chunks[p], kv_chunks[s], rank_chunks(s, world, zigzag),
                     dkv_acc[s], causal, scale, deterministic)
    dqs, dks, dvs = [], [], []
    for p in range(world):
        dqs.append(_convert(ops, dq_acc[p], q_chunks[p]))
        dks.append(_convert(ops, [a[0] for a in dkv_acc[p]], [k for k, _ in kv_chunks[p]]))
        dvs.append(_convert(ops, [a[1] for a in dkv_acc[p]], [v for _, v in kv_chunks[p]]))
    return dqs, dks, dvs
