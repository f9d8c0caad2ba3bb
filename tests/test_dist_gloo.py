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


def test_gpus_flag_must_match_launcher():
    import bench
    assert bench.launch_plan(1, {}) == "run"
    assert bench.launch_plan(4, {}) == "spawn"
    assert bench.launch_plan(2, {"WORLD_SIZE": "2"}) == "run"
    with pytest.raises(ValueError):
        bench.launch_plan(8, {"WORLD_SIZE": "1"})
    with pytest.raises(ValueError):
        bench.launch_plan(1, {"WORLD_SIZE": "4"})
    with pytest.raises(ValueError):
        bench.launch_plan(0, {})
    cmd = bench.spawn_command(4, ["--gpus", "4", "--steps", "3"], 29555)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "29555" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]


def test_mismatched_gpus_flag_fails_loudly():
    """A --gpus request that disagrees with the launcher's WORLD_SIZE exits non-zero before
    any GPU work, instead of printing a line with the wrong n_gpus."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "8",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode != 0
    assert "--gpus 8" in r.stderr and r.stdout.strip() == ""
