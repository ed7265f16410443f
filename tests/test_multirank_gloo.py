"""The multi-rank logic of bench.py on CPU with gloo, world size 2: ranks draw
independent batches (weak scaling, no data-path exchange) and the timing is
combined as the max over ranks, the work as the sum."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench
        import workloads as W
        ms = 10.0 + rank * 5.0
        nbytes = 1000.0 * (rank + 1)
        mx = bench.rank_reduce(ms, "max", world)
        sm = bench.rank_reduce(nbytes, "sum", world)
        seed = bench.rank_seed("gqa8b", rank)
        lens = W.lens_gqa8b(np.random.default_rng(seed))
        results[rank] = (mx, sm, seed, lens.tolist())
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_reductions():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 15.0           # max over ranks
    assert r0[1] == r1[1] == 3000.0         # sum over ranks
    assert r0[2] != r1[2]                   # independent seeds
    assert r0[3] != r1[3]                   # hence independent batches


def test_single_rank_is_identity():
    import bench
    assert bench.rank_reduce(3.5, "max", 1) == 3.5
