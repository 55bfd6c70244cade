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
locally (in the fp32 sum of the query chunk's backward workspace), and the fp32 dK / dV
accumulators travel with their chunks, are added to in place by every hop, and arrive back at
their owner after the last hop.

Every arithmetic step runs in the library's CUDA kernels: forward, attn_fwd_accumulate per
chunk pair (it folds the pair into the running result inside the forward kernel); backward,
attn_bwd_prepare once per query chunk, attn_bwd_accumulate per chunk pair and attn_bwd_finish at
the end; attn_ring_accumulate for the final conversions. This module only schedules them and
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
    """The per-chunk-pair operations, all in libattn.so. One set of per-hop forward output buffers
    is reused by every hop (each partial is merged on the same stream before the next hop
    overwrites it), and one backward workspace per query chunk (keyed by the caller) is kept for
    the next pass of the same sizes, so an instance passed to every step allocates nothing after
    the first."""

    def __init__(self):
        import exact_attention_138_b200 as ea
        self.ea = ea
        self._bufs = {}
        self._sums = {}

    def _buf(self, key, shape, dtype, device):
        t = self._bufs.get(key)
        if t is None or tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device:
            t = torch.empty(shape, dtype=dtype, device=device)
            self._bufs[key] = t
        return t

    def fwd(self, q, k, v, scale, window, slot=0):
        """O and LSE of one chunk pair, in buffers of `slot` (one per concurrent caller)."""
        o = self._buf(("o", slot), q.shape, q.dtype, q.device)
        lse = self._buf(("lse", slot), q.shape[:-1], torch.float32, q.device)
        return self.ea.forward(q, k, v, scale=scale, window=window, out=o, lse=lse)

    def bwd_begin(self, key, o, do, lse, deterministic):
        """Backward state of one query chunk (o, dO, lse of the whole forward pass)."""
        st = self._sums.get(key)
        if (st is None or st.det != int(bool(deterministic)) or st.ws.device != o.device
                or (st.B, st.H, st.n, st.d) != tuple(o.shape)):
            st = self.ea.BackwardSum(o, do, lse, deterministic=deterministic)
            self._sums[key] = st
        else:
            st.reset(o, do, lse)
        return st

    def bwd_add(self, st, q, k, v, do, dkv_acc, scale, window):
        """dQ sum of `st` and dkv_acc (fp32 (2, B, Hkv, n_k, d): dK, dV) += this pair's part."""
        st.add(q, k, v, do, dkv_acc[0], dkv_acc[1], scale=scale, window=window)

    def bwd_finish(self, st, out, scale):
        """Writes dQ of `st` into `out` (the query chunk's dtype and shape) and returns it."""
        return st.finish(out, scale=scale)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out):
        self.ea.ring_merge(o_acc, lse_acc, o_part, lse_part, first=first, out=out)

    def fwd_fold(self, o_acc, lse_acc, first, q, k, v, scale, window, slot=0):
        """Fold one chunk pair into the running (o_acc, lse_acc): inside the forward kernel for
        bf16 inputs, else a forward into this slot's buffers and a merge."""
        if q.dtype == torch.bfloat16:
            self.ea.forward_accumulate(q, k, v, o_acc, lse_acc, first=first, scale=scale,
                                       window=window)
            return
        o_p, l_p = self.fwd(q, k, v, scale, window, slot)
        self.merge(o_acc, lse_acc, o_p, l_p, first, None)

    def accumulate(self, acc, part, first, out):
        self.ea.ring_accumulate(acc, part, first=first, out=out)


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


def _wide(x):
    """x viewed with 8-byte elements when its rows allow (copies then move 4x fewer elements)."""
    if x.is_contiguous() and x.dim() == 4 and (x.shape[-1] * x.element_size()) % 8 == 0:
        return x.view(torch.int64)
    return x


def _split(x, parts):
    """The chunks of a rank's (B, H, parts·c, d) tensor as contiguous tensors."""
    if parts == 1:
        return [x.contiguous()]
    w = _wide(x)
    return [c.contiguous().view(x.dtype) for c in torch.chunk(w, parts, dim=2)]


def _join(chunks):
    if len(chunks) == 1:
        return chunks[0]
    return torch.cat([_wide(c) for c in chunks], dim=2).view(chunks[0].dtype)


class _FwdState:
    def __init__(self, q):
        self.o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        self.lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
        self.first = True


def _fwd_hop(ops, states, qs, q_ids, kvs, kv_ids, causal, scale, slot=0):
    """Fold every visible (query chunk, key chunk) pair of one hop into the running results."""
    for qi, q in enumerate(qs):
        for ki, (k, v) in enumerate(kvs):
            w = hop_window(q_ids[qi], kv_ids[ki], causal)
            if w is None:
                continue
            st = states[qi]
            ops.fwd_fold(st.o_acc, st.lse, st.first, q, k, v, scale, w, slot)
            st.first = False


def _fwd_outputs(ops, states, qs):
    outs = []
    for st, q in zip(states, qs):
        out = torch.empty_like(q)
        ops.accumulate(st.o_acc, None, False, out)    # fp32 running output -> q's dtype
        outs.append(out)
    return _join(outs), _join([st.lse for st in states])


def _bwd_hop(ops, sums, qs, q_ids, dos, kvs, kv_ids, dkv_acc, causal, scale):
    for qi, q in enumerate(qs):
        for ki, (k, v) in enumerate(kvs):
            w = hop_window(q_ids[qi], kv_ids[ki], causal)
            if w is None:
                continue
            ops.bwd_add(sums[qi], q, k, v, dos[qi], dkv_acc[ki], scale, w)


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
    sums = [ops.bwd_begin(("local", i), os_[i], dos[i], lses[i], deterministic)
            for i in range(parts)]
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
        _bwd_hop(ops, sums, qs, q_ids, dos, kvs, kv_ids, acc, causal, scale)
        # the dK / dV accumulators travel on with their chunks; after the last hop each rank
        # holds its own chunks'
        nxt_acc, acc_reqs = _exchange(acc, nxt, prv, group)
        for req in (reqs or []) + acc_reqs:
            req.wait()
        if reqs is not None:
            cur = nxt_kv
        acc = nxt_acc
    return (_join([ops.bwd_finish(st, torch.empty_like(c), scale) for st, c in zip(sums, qs)]),
            _convert(ops, [a[0] for a in acc], ks), _convert(ops, [a[1] for a in acc], vs))


class _Lanes:
    """One CUDA stream per emulated rank (as on N GPUs, where ranks run at the same time), or
    nothing on the CPU. `hop_done(p)` marks the end of rank p's hop; `after_previous(p)` makes
    rank p's next hop wait for rank p - 1's last one, which is when the chunks (and the dK / dV
    sums travelling with them) would have arrived from that rank."""

    def __init__(self, world, device):
        self.cuda = device.type == "cuda"
        self.world = world
        if self.cuda:
            self.main = torch.cuda.current_stream(device)
            self.streams = [torch.cuda.Stream(device) for _ in range(world)]
            self.events = [None] * world
            start = torch.cuda.Event()
            start.record(self.main)
            for st in self.streams:
                st.wait_event(start)

    def rank(self, p):
        import contextlib
        return torch.cuda.stream(self.streams[p]) if self.cuda else contextlib.nullcontext()

    def hop_done(self, p):
        if self.cuda:
            ev = torch.cuda.Event()
            ev.record(self.streams[p])
            self.events[p] = ev

    def after_previous(self, p):
        if self.cuda:
            ev = self.events[(p - 1) % self.world]
            if ev is not None:
                self.streams[p].wait_event(ev)

    def join(self):
        if self.cuda:
            for st in self.streams:
                self.main.wait_stream(st)


def ring_forward_emulated(qs, ks, vs, causal=False, scale=None, ops=None, zigzag=False):
    """The ring_forward schedule for len(qs) ranks in one process: qs[p], ks[p], vs[p] are rank
    p's tensors in the chosen layout. Each rank's kernels run on a stream of its own."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    parts = 2 if zigzag else 1
    q_chunks = [_split(q, parts) for q in qs]
    kv_chunks = [list(zip(_split(k, parts), _split(v, parts))) for k, v in zip(ks, vs)]
    states = [[_FwdState(c) for c in qc] for qc in q_chunks]
    outs = [[torch.empty_like(c) for c in qc] for qc in q_chunks]
    lanes = _Lanes(world, qs[0].device)
    for r in range(world):
        for p in range(world):
            s = (p - r) % world      # the rank whose chunks rank p holds in hop r
            with lanes.rank(p):
                _fwd_hop(ops, states[p], q_chunks[p], rank_chunks(p, world, zigzag),
                         kv_chunks[s], rank_chunks(s, world, zigzag), causal, scale, slot=p)
    for p in range(world):
        with lanes.rank(p):
            for st, out in zip(states[p], outs[p]):
                ops.accumulate(st.o_acc, None, False, out)
    lanes.join()
    return ([_join(outs[p]) for p in range(world)],
            [_join([st.lse for st in states[p]]) for p in range(world)])


def ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=False, scale=None, ops=None,
                           deterministic=False, zigzag=False):
    """The ring_backward schedule for len(qs) ranks in one process, each rank on a stream of its
    own; a rank's hop waits for the previous rank's hop before it adds into the dK / dV sums
    that travel from there."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    parts = 2 if zigzag else 1
    q_chunks = [_split(q, parts) for q in qs]
    o_chunks = [_split(o, parts) for o in os_]
    do_chunks = [_split(x, parts) for x in dos]
    l_chunks = [[c.contiguous() for c in torch.chunk(x, parts, dim=2)] for x in lses]
    kv_chunks = [list(zip(_split(k, parts), _split(v, parts))) for k, v in zip(ks, vs)]
    sums = [[ops.bwd_begin((p, i), o_chunks[p][i], do_chunks[p][i], l_chunks[p][i],
                           deterministic) for i in range(parts)] for p in range(world)]
    dkv_acc = [[torch.zeros((2,) + tuple(k.shape), dtype=torch.float32, device=k.device)
                for k, _ in kvc] for kvc in kv_chunks]
    dq_out = [[torch.empty_like(c) for c in qc] for qc in q_chunks]
    dk_out = [[torch.empty_like(k) for k, _ in kvc] for kvc in kv_chunks]
    dv_out = [[torch.empty_like(v) for _, v in kvc] for kvc in kv_chunks]
    lanes = _Lanes(world, qs[0].device)
    for r in range(world):
        for p in range(world):
            s = (p - r) % world
            with lanes.rank(p):
                if r > 0:
                    lanes.after_previous(p)
                _bwd_hop(ops, sums[p], q_chunks[p], rank_chunks(p, world, zigzag), do_chunks[p],
                         kv_chunks[s], rank_chunks(s, world, zigzag), dkv_acc[s], causal, scale)
        for p in range(world):
            lanes.hop_done(p)
    # the last addition to rank p's own chunks' sums is rank p - 1's in the last hop
    for p in range(world):
        with lanes.rank(p):
            lanes.after_previous(p)
            for st, out in zip(sums[p], dq_out[p]):
                ops.bwd_finish(st, out, scale)
            for acc, dk, dv in zip(dkv_acc[p], dk_out[p], dv_out[p]):
                ops.accumulate(acc[0], None, False, dk)
                ops.accumulate(acc[1], None, False, dv)
    lanes.join()
    return ([_join(x) for x in dq_out], [_join(x) for x in dk_out], [_join(x) for x in dv_out])
