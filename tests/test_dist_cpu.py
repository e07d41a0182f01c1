"""Host-side multi-process logic of bench.py on CPU (gloo, world size 2).

With --gpus N the benchmark runs one independent replica per rank and reports
the slowest rank's time; the max-over-ranks reduction and the barrier are the
only collectives.  Here two gloo ranks check that reduction.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank], world)
        bench.barrier(world)
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == [2.0, 10.0] and out[1] == [2.0, 10.0]


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
