"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2): the
job time is the slowest rank's, the rate counts every rank's work, only
rank 0 of the reference arm runs, and a rank that leaves makes the other
rank's next collective end with an error within the process-group timeout
(no hang). The path has no data-path collective (replicas), so this is all
the multi-rank logic there is.

CPU only."""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port, timeout_s):
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _ranks_max(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, port, 30)
    ms = bench.max_over_ranks(1.0 + 2.0 * rank, 2, "cpu")        # rank 0: 1 ms, rank 1: 3 ms
    rate = bench.job_rate(1.5e9, 2, ms)
    with open(os.path.join(out_dir, "r%d" % rank), "w") as f:
        f.write("%r %r" % (ms, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_job_time_is_the_slowest_rank(tmp_path):
    mp.spawn(_ranks_max, args=(_free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in (0, 1):
        ms, rate = (float(x) for x in open(tmp_path / ("r%d" % r)).read().split())
        assert ms == 3.0
        assert rate == pytest.approx(2 * 1.5e9 / 3e-3 / 1e12)      # both ranks' work over the slowest time


def _rank_leaves(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, port, 5)
    bench.max_over_ranks(1.0, 2, "cpu")                              # one step together
    if rank == 1:
        os._exit(0)                                                  # leaves between steps, no collective in flight
    import time
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(1.0, 2, "cpu")
        status = "completed"
    except Exception as e:                                           # the collective must fail, not hang
        status = "error:" + type(e).__name__
    with open(os.path.join(out_dir, "r0"), "w") as f:
        f.write("%s %.1f" % (status, time.monotonic() - t0))
    os._exit(0)


def test_a_rank_that_leaves_ends_the_next_collective_with_an_error(tmp_path):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_leaves, args=(r, port, str(tmp_path))) for r in (0, 1)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
    alive = [pr for pr in procs if pr.is_alive()]
    for pr in alive:
        pr.kill()
    assert not alive, "a rank hung"
    status, secs = open(tmp_path / "r0").read().split()
    assert status.startswith("error:")
    assert float(secs) < 60


def test_reference_arm_runs_on_rank_0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
