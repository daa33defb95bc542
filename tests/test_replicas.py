"""Multi-process host logic of bench.py on CPU: world_size-2 gloo ranks.

bench.py runs one independent replica per GPU (the step does not shard); its
only cross-rank step is the max-over-ranks reduction of the timings, and the
whole-job throughput divides every rank's units by that time.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r timed (r + 1) ms for the step and 10 (r + 1) ms end to end
        got = bench.max_over_ranks([1.0 + rank, 10.0 * (1 + rank)])
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1] == [2.0, 20.0]


def test_max_over_ranks_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([3.5, 7.25]) == [3.5, 7.25]


def test_job_throughput_counts_every_rank():
    import bench
    # 2 replicas x 8 queries x 100 steps in 50 ms (the slowest rank's time)
    assert bench.job_throughput(2, 8, 100, 50.0) == pytest.approx(32000.0)
    assert bench.job_throughput(1, 8, 100, 50.0) == pytest.approx(16000.0)
