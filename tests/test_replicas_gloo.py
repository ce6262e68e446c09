"""The N > 1 path of bench.py (independent replicas) on CPU with gloo, world size 2.

The layer does not shard, so N GPUs run N replicas; the job's value is all
ranks' tokens over the slowest rank's time.  This checks the reduction and the
aggregation that bench.py uses, with two real processes.
"""
import os
import socket

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
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        my_ms = 100.0 + 50.0 * rank              # rank 1 is the slow one
        ms_max = bench.max_over_ranks(my_ms, world, device="cpu")
        out[rank] = (ms_max, bench.job_tokens_per_s(8192, world, 10, ms_max))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1]                       # both ranks agree
    ms_max, value = out[0]
    assert ms_max == 150.0
    assert value == pytest.approx(2 * 8192 * 10 / 0.150)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tokens_per_s(100, 1, 4, 200.0) == pytest.approx(2000.0)
