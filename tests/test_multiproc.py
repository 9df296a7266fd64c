"""Host-side logic of bench.py for N > 1 ranks, on CPU with gloo.

The bench runs one replica per GPU (weak scaling, no data-path collective);
the only cross-rank steps are the barrier and the max over ranks of the
measured time.  These run here as two gloo processes.
"""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench.barrier(world)
        m = bench.max_over_ranks(1.5 + rank, world)
        q.put((rank, m, bench.rank_seed(0, rank)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_distinct_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [m for _, m, _ in got] == [2.5, 2.5]
    assert got[0][2] != got[1][2]
