"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun
would start them.  The path has no exchange step (every rank runs an
independent replica), so what is shared between ranks is only the timing:
the step time is the maximum over ranks and the reported value counts every
rank's work.  The reference arm runs on rank 0 alone."""

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.join(os.path.dirname(__file__), "..")
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from exact_io_aware_bwd_b200.workloads import WORKLOADS
        w = WORKLOADS["mha4k"]
        ms = [2.0, 3.5][rank]                       # rank 1 is the slow one
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        seed = bench.rank_seed(w, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        out[rank] = (got, bench.job_tflops(world, 1e12, got), tuple(seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_every_replica():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    for rank in range(world):
        got, tflops, seeds = res[rank]
        assert got == 3.5                            # the slowest rank sets the time
        assert tflops == pytest.approx(2 * 1e12 / 3.5e-3 / 1e12)
        assert seeds[0] != seeds[1]                  # replicas draw different inputs


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1.25, 1, torch.device("cpu")) == 1.25
    assert bench.job_tflops(1, 2e12, 1.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
