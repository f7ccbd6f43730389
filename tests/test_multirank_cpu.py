"""The multi-process path of bench.py on the CPU with a world-size-2 gloo
group: replicas time themselves and every rank reports the slowest rank's
time; the reference arm runs on rank 0 only."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank                 # rank 1 is the slow one
        got = bench.max_over_ranks(mine, dist, None)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world2_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup, gpus = "block2b", 1, 0, 2
    assert bench.run_reference(A(), [], 1, {}) is None


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5


if __name__ == "__main__":
    pytest.main([__file__])
