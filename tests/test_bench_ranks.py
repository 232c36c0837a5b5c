"""Host logic of bench.py's N-rank run (CPU only, world size 2 over gloo): the timed region's
device time is the max over ranks, the rate counts every rank's tokens, and under a multi-rank
launch the reference arm runs on rank 0 alone (the other ranks exit at once, printing nothing)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, times, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_max = bench.max_over_ranks(times[rank], dist, "cpu")
        rate = bench.whole_job_rate(world, 100, 4, ms_max)
        out_q.put((rank, ms_max, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_gloo():
    world, times = 2, [12.5, 20.0]
    with socket.socket() as sk:  # a free local port for the rendezvous
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, rate in res:
        assert ms_max == 20.0  # the slowest rank's time on every rank
        assert rate == pytest.approx(world * 100 * 4 / 0.020)


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.25, None, "cpu") == 7.25
    assert bench.whole_job_rate(1, 10, 1, 5.0) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
