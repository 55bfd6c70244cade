"""Ring attention's multi-rank schedule on CPU ranks (gloo, point-to-point isend/irecv): each
rank holds one chunk of the sequence, K/V chunks travel around the ring, partial results are
merged and the dK/dV accumulators travel back to their owners. The per-hop arithmetic is the CPU
stand-in of tests/ring_cpu_ops.py; the gathered results must equal the oracle's attention over
the whole sequence ("Attention Mechanism ...", §16 Ring Attention)."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(world, n_chunk, H, Hkv, d):
    g = torch.Generator().manual_seed(41)
    n = world * n_chunk
    q = torch.randn(1, H, n, d, generator=g).double()
    k = torch.randn(1, Hkv, n, d, generator=g).double()
    v = torch.randn(1, Hkv, n, d, generator=g).double()
    do = torch.randn(1, H, n, d, generator=g).double()
    return q, k, v, do


def _layout(world, n_chunk, zigzag):
    """Global row indices of each rank's tensors (contiguous: one chunk; zigzag: chunks p and
    2N-1-p)."""
    if not zigzag:
        return [np.arange(p * n_chunk, (p + 1) * n_chunk) for p in range(world)]
    c = n_chunk // 2
    return [np.concatenate([np.arange(p * c, (p + 1) * c),
                            np.arange((2 * world - 1 - p) * c, (2 * world - p) * c)])
            for p in range(world)]


def _worker(rank, world, port, causal, n_chunk, H, Hkv, d, zigzag, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from exact_attention_138_b200 import ring
    from ring_cpu_ops import CpuOps
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, do = _inputs(world, n_chunk, H, Hkv, d)
        rows = torch.from_numpy(_layout(world, n_chunk, zigzag)[rank])
        mine = [x.index_select(2, rows).contiguous() for x in (q, k, v, do)]
        scale = 1.0 / math.sqrt(d)
        ops = CpuOps()
        o, lse = ring.ring_forward(mine[0], mine[1], mine[2], causal=causal, scale=scale, ops=ops,
                                   zigzag=zigzag)
        dq, dk, dv = ring.ring_backward(mine[0], mine[1], mine[2], o, mine[3], lse, causal=causal,
                                        scale=scale, ops=ops, zigzag=zigzag)
        out[rank] = tuple(x.numpy() for x in (o, lse, dq, dk, dv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,H,Hkv,zigzag", [
    (2, True, 2, 2, False), (2, False, 2, 1, False), (3, True, 4, 2, False),
    (2, True, 2, 2, True), (3, True, 2, 1, True), (3, False, 2, 2, True)])
def test_ring_schedule_on_cpu_ranks_equals_full_attention(world, causal, H, Hkv, zigzag):
    import oracle
    n_chunk, d = 24, 8
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), causal, n_chunk, H, Hkv, d, zigzag,
                                      out),
                       nprocs=world, join=True, start_method="spawn")
    q, k, v, do = _inputs(world, n_chunk, H, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    qf, kf, vf, dof = (x.float().numpy() for x in (q, k, v, do))
    ro, rlse = oracle.fwd_ex(qf, kf, vf, scale, -1, 0 if causal else -1)
    rq, rk, rv = oracle.bwd_ex(qf, kf, vf, dof, scale, -1, 0 if causal else -1)
    order = np.argsort(np.concatenate(_layout(world, n_chunk, zigzag)))
    got = [np.concatenate([out[r][i] for r in range(world)], axis=2)[:, :, order]
           for i in range(5)]
    np.testing.assert_allclose(got[0], ro, rtol=0, atol=1e-5)
    np.testing.assert_allclose(got[1], rlse, rtol=0, atol=1e-5)
    for g, want in zip(got[2:], (rq, rk, rv)):
        np.testing.assert_allclose(g, want, rtol=0, atol=1e-5)


def test_hop_windows():
    from exact_attention_138_b200 import ring
    assert ring.hop_window(3, 1, True) == (-1, -1)
    assert ring.hop_window(2, 2, True) == (-1, 0)
    assert ring.hop_window(1, 2, True) is None
    assert all(ring.hop_window(p, s, False) == (-1, -1) for p in range(3) for s in range(3))


def test_zigzag_layout_balances_causal_work():
    from exact_attention_138_b200 import ring
    world = 4
    for zigzag, balanced in ((False, False), (True, True)):
        work = []
        for p in range(world):
            mine = ring.rank_chunks(p, world, zigzag)
            pairs = 0.0
            for r in range(world):
                for a in mine:
                    for b in ring.rank_chunks((p - r) % world, world, zigzag):
                        w = ring.hop_window(a, b, True)
                        pairs += 0 if w is None else (0.5 if w == (-1, 0) else 1.0)
            work.append(pairs)
        assert (len(set(work)) == 1) == balanced, work


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [True, False])
def test_hop_launches_cover_the_visible_pairs_once(world, causal):
    """Each hop's launches, expanded back to (query chunk, key chunk) pairs with the mask each
    pair gets, must be exactly the visible pairs with their own windows; with zigzag chunks every
    hop is a single launch."""
    from exact_attention_138_b200 import ring
    for zigzag in (False, True):
        for p in range(world):
            q_ids = ring.rank_chunks(p, world, zigzag)
            for r in range(world):
                kv_ids = ring.rank_chunks((p - r) % world, world, zigzag)
                launches = ring.hop_launches(q_ids, kv_ids, causal)
                got = {}
                for a0, a1, b0, b1, w in launches:
                    for a in range(a0, a1):
                        for b in range(b0, b1):
                            assert (a, b) not in got
                            if w == (-1, 0) and (a1 - a0) > 1:
                                # the causal mask of the concatenation, on this pair
                                qa, kb = q_ids[a], kv_ids[b]
                                got[(a, b)] = (-1, 0) if qa == kb else ((-1, -1) if kb < qa else None)
                            else:
                                got[(a, b)] = w
                want = {(a, b): ring.hop_window(qa, kb, causal)
                        for a, qa in enumerate(q_ids) for b, kb in enumerate(kv_ids)}
                for key, w in want.items():
                    assert got.get(key) == w, (p, r, key)
                if zigzag and any(w is not None for w in want.values()):
                    assert len(launches) == 1


def test_gpu_ring_backward_refuses_query_views_off_64_rows():
    """The library's backward adds a launch's queries from 64-row boundaries of the rank's
    queries; a causal zigzag ring whose chunk length is not a multiple of 64 is refused with a
    message before anything is launched (the check needs no GPU)."""
    from exact_attention_138_b200 import ring
    ops = ring.CudaOps()
    with pytest.raises(ValueError, match="64"):
        ops.bwd_add(None, None, None, None, None, None, None, 1.0, None, 150)
