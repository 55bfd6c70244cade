"""Ring attention: exact attention over a sequence split into chunks held by different ranks
("Attention Mechanism: Revolusi Representasi Sequence", §16 "Long Context Training", Ring
Attention; §6, long-context techniques table).

Layouts. With N ranks the sequence is cut into equal chunks:
  contiguous  N chunks; rank p holds chunk p.
  zigzag      2N chunks; rank p holds chunks p and 2N-1-p (its q, k, v are those two chunks one
              after the other). Under a causal mask every rank then sees the same amount of work
              (the contiguous layout gives rank N-1 N times the work of rank 0).
In hop r a rank attends its query chunks to the K/V chunks of rank (p - r) mod N, which arrived
from rank p - 1, while sending the chunks it holds on to rank p + 1; the partial results are
folded together with the log-sum-exp rule (attn_ring_merge). Under a causal mask a (query chunk,
key chunk) pair is unmasked (earlier key chunk), causal (same chunk) or skipped (later key
chunk). The visible pairs of a hop are joined into as few launches as the masks allow, each on
row ranges (views) of the rank's whole tensors: with zigzag chunks every hop is one launch (the
rank's own chunks: the causal mask of their concatenation; an earlier rank's: all queries
against its first chunk; a later rank's: the second query chunk against both; the backward's
launches start their queries on 64-row boundaries, so causal zigzag chunks on GPUs are multiples
of 64 rows). The backward pass walks the same ring with the final O and LSE: dQ accumulates
locally (in the fp32 sum of the rank's backward workspace), and the fp32 dK / dV accumulators
travel with their chunks, are added to in place by every hop, and arrive back at their owner
after the last hop.

Every arithmetic step runs in the library's CUDA kernels: forward, attn_fwd_accumulate per
launch (it folds the launch into the running result inside the forward kernel); backward,
attn_bwd_prepare once per rank, attn_bwd_accumulate per launch and attn_bwd_finish at the end;
attn_ring_accumulate for the final conversions. This module only schedules them and
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


def hop_launches(q_ids, kv_ids, causal):
    """The launches of one hop, as (first query chunk, end, first key chunk, end, window) over the
    rank's chunk order: the visible (query chunk, key chunk) pairs, joined into one launch when
    they form the causal mask of the concatenated chunks or a block with no mask, else one
    launch per pair."""
    W = [[hop_window(a, b, causal) for b in kv_ids] for a in q_ids]
    full = (-1, -1)
    if causal and q_ids == kv_ids and q_ids == sorted(q_ids):
        return [(0, len(q_ids), 0, len(kv_ids), (-1, 0))]
    rows = [a for a in range(len(q_ids)) if any(w is not None for w in W[a])]
    cols = [b for b in range(len(kv_ids)) if any(W[a][b] is not None for a in range(len(q_ids)))]
    if (rows and rows == list(range(rows[0], rows[-1] + 1))
            and cols == list(range(cols[0], cols[-1] + 1))
            and all(W[a][b] == full for a in rows for b in cols)):
        return [(rows[0], rows[-1] + 1, cols[0], cols[-1] + 1, full)]
    return [(a, a + 1, b, b + 1, W[a][b]) for a in range(len(q_ids)) for b in range(len(kv_ids))
            if W[a][b] is not None]


class CudaOps:
    """The per-hop operations, all in libattn.so: the forward folded into a running result, and
    the backward in parts (one workspace per rank, kept for the next pass of the same sizes, so
    an instance passed to every step allocates nothing after the first)."""

    def __init__(self):
        import exact_attention_138_b200 as ea
        self.ea = ea
        self._sums = {}

    def fwd_fold(self, o_acc, lse_acc, first, q, k, v, scale, window, slot=0):
        """Fold attention of q over k, v into the running (o_acc, lse_acc) (views allowed)."""
        if q.dtype == torch.bfloat16:
            self.ea.forward_accumulate(q, k, v, o_acc, lse_acc, first=first, scale=scale,
                                       window=window)
            return
        # other input types: a forward on copies and a merge into copies of the running rows
        o_p, l_p = self.ea.forward(q.contiguous(), k.contiguous(), v.contiguous(), scale=scale,
                                   window=window)
        oa, la = o_acc.contiguous(), lse_acc.contiguous()
        self.ea.ring_merge(oa, la, o_p, l_p, first=first)
        o_acc.copy_(oa)
        lse_acc.copy_(la)

    def bwd_begin(self, key, o, do, lse, deterministic):
        """Backward state of the rank's queries (o, dO, lse of the whole forward pass)."""
        st = self._sums.get(key)
        if (st is None or st.det != int(bool(deterministic)) or st.ws.device != o.device
                or (st.B, st.H, st.n, st.d) != tuple(o.shape)):
            st = self.ea.BackwardSum(o, do, lse, deterministic=deterministic)
            self._sums[key] = st
        else:
            st.reset(o, do, lse)
        return st

    def bwd_add(self, st, q, k, v, do, dk_acc, dv_acc, scale, window, q_row0):
        """dQ sum of `st` (its rows from q_row0) and dk_acc, dv_acc += this launch's part."""
        if q_row0 % 64:
            raise ValueError("the backward adds query rows from 64-row boundaries: the chunks of "
                             "a causal zigzag ring must be multiples of 64 rows long")
        st.add(q, k, v, do, dk_acc, dv_acc, scale=scale, window=window, q_row0=q_row0)

    def bwd_finish(self, st, out, scale):
        """Writes dQ of `st` into `out` and returns it."""
        return st.finish(out, scale=scale)

    def accumulate(self, acc, part, first, out):
        self.ea.ring_accumulate(acc, part, first=first, out=out)


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


def _rows(x, lo, hi, c):
    """Rows [lo·c, hi·c) of a (.., n, d) tensor or (.., n) vector: a view, no copy."""
    return x[:, :, lo * c:hi * c]


def _chunk_len(q, parts):
    n = q.shape[2]
    if n % parts:
        raise ValueError("a zigzag rank holds two chunks of equal length")
    return n // parts


def _fwd_hop(ops, o_acc, lse_acc, init, q, k, v, q_ids, kv_ids, causal, scale, slot=0):
    """Fold one hop into the rank's running (o_acc, lse_acc); init[a]: query chunk a has been
    initialised by an earlier launch."""
    c = _chunk_len(q, len(q_ids))
    for a0, a1, b0, b1, w in hop_launches(q_ids, kv_ids, causal):
        first = not init[a0]
        if any(init[a] != init[a0] for a in range(a0, a1)):
            raise RuntimeError("a launch over query chunks in different states")
        ops.fwd_fold(_rows(o_acc, a0, a1, c), _rows(lse_acc, a0, a1, c), first,
                     _rows(q, a0, a1, c), _rows(k, b0, b1, c), _rows(v, b0, b1, c), scale, w,
                     slot)
        for a in range(a0, a1):
            init[a] = True


def _bwd_hop(ops, st, q, do, k, v, dkv_acc, q_ids, kv_ids, causal, scale):
    c = _chunk_len(q, len(q_ids))
    for a0, a1, b0, b1, w in hop_launches(q_ids, kv_ids, causal):
        ops.bwd_add(st, _rows(q, a0, a1, c), _rows(k, b0, b1, c), _rows(v, b0, b1, c),
                    _rows(do, a0, a1, c), _rows(dkv_acc[0], b0, b1, c),
                    _rows(dkv_acc[1], b0, b1, c), scale, w, a0 * c)


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
    q_ids = rank_chunks(rank, world, zigzag)
    o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    init = [False] * len(q_ids)
    cur = [k.contiguous(), v.contiguous()]
    for r in range(world):
        reqs = None
        if r < world - 1:
            nxt_kv, reqs = _exchange(cur, nxt, prv, group)
        kv_ids = rank_chunks((rank - r) % world, world, zigzag)
        _fwd_hop(ops, o_acc, lse_acc, init, q, cur[0], cur[1], q_ids, kv_ids, causal, scale)
        if reqs is not None:
            for req in reqs:
                req.wait()
            cur = nxt_kv
    out = torch.empty_like(q)
    ops.accumulate(o_acc, None, False, out)            # fp32 running output -> q's dtype
    return out, lse_acc


def ring_backward(q, k, v, o, do, lse, causal=False, scale=None, group=None, ops=None,
                  deterministic=False, zigzag=False):
    """dQ, dK, dV of ring attention for this rank's chunks, given the final O and LSE of
    `ring_forward` (same layout) and dO."""
    ops = ops or CudaOps()
    scale = _scale(q, scale)
    rank, world, nxt, prv = _peers(group)
    q_ids = rank_chunks(rank, world, zigzag)
    st = ops.bwd_begin("local", o, do, lse, deterministic)
    cur = [k.contiguous(), v.contiguous()]
    # dK and dV accumulators of the chunks held, stacked: (2, B, Hkv, n, d) fp32
    acc = torch.zeros((2,) + tuple(k.shape), dtype=torch.float32, device=k.device)
    for r in range(world):
        reqs = None
        if r < world - 1:
            nxt_kv, reqs = _exchange(cur, nxt, prv, group)
        kv_ids = rank_chunks((rank - r) % world, world, zigzag)
        _bwd_hop(ops, st, q, do, cur[0], cur[1], acc, q_ids, kv_ids, causal, scale)
        # the dK / dV accumulators travel on with their chunks; after the last hop each rank
        # holds its own chunks'
        (nxt_acc,), acc_reqs = _exchange([acc], nxt, prv, group)
        for req in (reqs or []) + acc_reqs:
            req.wait()
        if reqs is not None:
            cur = nxt_kv
        acc = nxt_acc
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    ops.accumulate(acc[0], None, False, dk)
    ops.accumulate(acc[1], None, False, dv)
    return ops.bwd_finish(st, torch.empty_like(q), scale), dk, dv


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
    o_acc = [torch.empty(q.shape, dtype=torch.float32, device=q.device) for q in qs]
    lse_acc = [torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device) for q in qs]
    outs = [torch.empty_like(q) for q in qs]
    kvs = [(k.contiguous(), v.contiguous()) for k, v in zip(ks, vs)]
    init = [[False] * (2 if zigzag else 1) for _ in range(world)]
    lanes = _Lanes(world, qs[0].device)
    for r in range(world):
        for p in range(world):
            s = (p - r) % world      # the rank whose chunks rank p holds in hop r
            with lanes.rank(p):
                _fwd_hop(ops, o_acc[p], lse_acc[p], init[p], qs[p], kvs[s][0], kvs[s][1],
                         rank_chunks(p, world, zigzag), rank_chunks(s, world, zigzag), causal,
                         scale, slot=p)
    for p in range(world):
        with lanes.rank(p):
            ops.accumulate(o_acc[p], None, False, outs[p])
    lanes.join()
    return outs, lse_acc


def ring_backward_emulated(qs, ks, vs, os_, dos, lses, causal=False, scale=None, ops=None,
                           deterministic=False, zigzag=False):
    """The ring_backward schedule for len(qs) ranks in one process, each rank on a stream of its
    own; a rank's hop waits for the previous rank's hop before it adds into the dK / dV sums
    that travel from there."""
    ops = ops or CudaOps()
    world = len(qs)
    scale = _scale(qs[0], scale)
    kvs = [(k.contiguous(), v.contiguous()) for k, v in zip(ks, vs)]
    sums = [ops.bwd_begin(p, os_[p], dos[p], lses[p], deterministic) for p in range(world)]
    dkv_acc = [torch.zeros((2,) + tuple(k.shape), dtype=torch.float32, device=k.device)
               for k in ks]
    dq_out = [torch.empty_like(q) for q in qs]
    dk_out = [torch.empty_like(k) for k in ks]
    dv_out = [torch.empty_like(v) for v in vs]
    lanes = _Lanes(world, qs[0].device)
    for r in range(world):
        for p in range(world):
            s = (p - r) % world
            with lanes.rank(p):
                if r > 0:
                    lanes.after_previous(p)
                _bwd_hop(ops, sums[p], qs[p], dos[p], kvs[s][0], kvs[s][1], dkv_acc[s],
                         rank_chunks(p, world, zigzag), rank_chunks(s, world, zigzag), causal,
                         scale)
        for p in range(world):
            lanes.hop_done(p)
    # the last addition to rank p's own chunks' sums is rank p - 1's in the last hop
    for p in range(world):
        with lanes.rank(p):
            lanes.after_previous(p)
            ops.bwd_finish(sums[p], dq_out[p], scale)
            ops.accumulate(dkv_acc[p][0], None, False, dk_out[p])
            ops.accumulate(dkv_acc[p][1], None, False, dv_out[p])
    lanes.join()
    return dq_out, dk_out, dv_out
