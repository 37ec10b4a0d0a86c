"""The benchmark's multi-rank plumbing on CPU: world_size 2 over gloo.

bench.py reports the slowest rank's time and the sum of all ranks' work;
this runs that reduction in two real processes."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, rank, world)
        ms, units = bench.reduce_step_time(10.0 + 5.0 * rank, 100.0 * (rank + 1))
        bench.barrier()
        q.put((rank, ms, units))
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 15.0, 300.0), (1, 15.0, 300.0)]


def test_single_process_passthrough(monkeypatch):
    import bench
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 0, 1)
    assert bench.reduce_step_time(3.0, 7.0) == (3.0, 7.0)


def test_warmup_rule():
    import bench
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
