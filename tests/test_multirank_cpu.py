"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
per rank, as torchrun launches them) agree on the slowest rank's time, the
whole-job rate counts every rank's units, every rank draws its own inputs,
and the reference arm runs on rank 0 only."""
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


def _rank_main(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], torch.device("cpu"), world)
        rate = bench.whole_job_rate(8 * 100, ms, world)
        seed = bench.rank_seed(1000, rank)
        dist.barrier()
        q.put((rank, ms, rate, seed))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_units():
    world, port = 2, _free_port()
    times = [3.0, 5.0]                     # ms: rank 1 is the slower one
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, rate, seed in got:
        assert ms == max(times)                       # every rank reports the max
        assert rate == pytest.approx(8 * 100 * world / (max(times) / 1e3))
    assert got[0][3] != got[1][3]                     # independent inputs per rank


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu"), 1) == 2.5
    assert bench.whole_job_rate(10, 2.0, 1) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only():
    # a rank other than 0 of a torchrun launch exits 0 without output or work
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
