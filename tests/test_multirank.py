"""Host logic of the multi-GPU benchmark path, on CPU with two `gloo` ranks.

The path shards into independent replicas (no data-path collective); the only cross-rank step is the
max over ranks of the timed region, and the whole-job rate counts every rank's work over that max.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        secs = [1.5, 2.5][rank]                      # rank 1 is the slow one
        mx = bench.reduce_max(secs)
        rate = bench.whole_job_rate(100.0, steps=10, world=ws, max_seconds=mx)
        q.put((rank, ws, r, local, mx, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, r, local, mx, rate in out:
        assert ws == 2 and r == rank and local == rank
        assert mx == pytest.approx(2.5)                         # the slowest rank's time
        assert rate == pytest.approx(100.0 * 10 * 2 / 2.5)      # all ranks' work over that time


def test_single_process_needs_no_process_group():
    import bench
    assert bench.reduce_max(3.0) == 3.0
    assert bench.whole_job_rate(10.0, 4, 1, 2.0) == pytest.approx(20.0)
