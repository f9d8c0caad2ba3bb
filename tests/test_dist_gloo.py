"""The multi-process plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank serves its own batch (no collective on the data path); the only exchange is
the max-over-ranks of the measured time.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    from datetime import timedelta

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(None)
        # rank r measured (r + 1) * 1.5 ms: the job time is the slowest rank's
        results[rank] = bench.max_over_ranks((rank + 1) * 1.5)
        bench.barrier(None)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_gloo(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(results) == {r: world * 1.5 for r in range(world)}


def test_single_process_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    bench.barrier(None)
    assert bench.dist_env()[0] >= 1
