"""Memory Parallel's exchange on two gloo ranks (CPU): the candidate and partial
all-gathers stack every rank's tensors in rank order, which is the layout the
merge entry points read (part after part). The merges themselves run in libmsa on
the GPU (tests/test_gpu_memory_parallel.py); here each rank checks, with the
oracle's merges, that the gathered stack yields the single-bank result."""
import math
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    from oracle import msa_oracle as O
    from sparse_attention_routed_b200.parallel import exchange_candidates, exchange_partials, shard_ranges
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(0)                      # the same bank on every rank
        n, rows, k, d = 30, 6, 4, 8
        scores = rng.integers(-4, 5, (rows, n)).astype(np.float32) / 4.0
        lo, hi = shard_ranges(n, world)[rank]
        loc = np.stack([O.select_top_k(scores[r, lo:hi], k) for r in range(rows)])
        sc = torch.from_numpy(np.take_along_axis(scores[:, lo:hi], loc, 1).astype(np.float32))
        ix = torch.from_numpy((loc + lo).astype(np.int32))
        all_sc, all_ix = exchange_candidates(sc, ix)
        assert tuple(all_sc.shape) == (world, rows, k) and all_ix.dtype == torch.int32
        for r in range(rows):
            got, _ = O.merge_candidates(list(all_sc[:, r].numpy()), list(all_ix[:, r].numpy()), k)
            want = sorted(range(n), key=lambda j: (-scores[r, j], j))[:k]
            assert list(got) == want
        # partials of one softmax split between the ranks' key sets
        q = rng.standard_normal(d)
        keys = rng.standard_normal((50, d))
        vals = rng.standard_normal((50, d))
        a, b = (0, 20) if rank == 0 else (20, 50)
        po, pl = O.attention_partial(q, keys[a:b], vals[a:b])
        all_o, all_l = exchange_partials(torch.from_numpy(po[None]), torch.tensor([pl], dtype=torch.float64))
        merged, _ = O.merge_partials(list(all_o[:, 0].numpy()), list(all_l[:, 0].numpy()))
        assert np.abs(merged - O.softmax_attention(q, keys, vals)).max() < 1e-12
        out[rank] = 1
    finally:
        dist.destroy_process_group()


def test_exchange_on_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 1, 1: 1}
