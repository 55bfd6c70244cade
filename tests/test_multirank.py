"""The N > 1 host logic of bench.py on two CPU ranks (gloo): every rank draws its own batch, the
step time is the max over ranks, and the job's rate is all ranks' work over that time (weak
scaling, no collective on the data path)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import attn_inputs
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 3.0 + 2.0 * rank                       # rank 1 is the slow one
        worst = bench.max_over_ranks(my_ms, dist, "cpu")
        q = attn_inputs.bf16_draws((1, 2, 8, 16), seed=bench.rank_seed(rank), count=1)[0]
        gathered = [torch.empty_like(q.float()) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        out[rank] = (worst, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_independent_batches():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 5.0            # both ranks see the slowest rank's time
    assert out[0][1] is False                       # the two ranks' batches differ


def test_whole_job_value_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(3.85e12, 1, 5.0)
    assert bench.whole_job_tflops(3.85e12, 4, 5.0) == pytest.approx(4 * one)
    assert bench.whole_job_tflops(3.85e12, 2, 10.0) == pytest.approx(one)
    assert bench.rank_seed(0) == 9                  # rank 0 reproduces the single-GPU inputs
    assert bench.max_over_ranks(7.0) == 7.0
