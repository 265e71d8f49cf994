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


def test_launcher_starts_n_ranks_and_passes_rank0_line():
    # bench.launch_ranks is what `python bench.py --gpus N` runs when no process group exists; here
    # it starts two CPU ranks of a stand-in script, which print one line from rank 0 only.
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    probe = os.path.join(root, "tests", "rank_probe.py")
    code = ("import sys; sys.path.insert(0, %r); import bench; "
            "sys.exit(bench.launch_ranks(2, %r, ['--steps', '3']))") % (root, probe)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["max_seconds"] == 2.0 and out["argv"] == ["--steps", "3"]


def test_gpus_must_match_an_existing_process_group():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode == 2 and "does not match" in r.stderr
