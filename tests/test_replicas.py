"""Multi-GPU in this project is replicas only: independent processes, one per
GPU, with no collective on the data path.  The host logic that combines them
(the slowest rank's time, the whole-job throughput) and the reference arm's
rank handling run here on CPU with two gloo ranks."""
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
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], dist, "cpu")
        out[rank] = (ms, bench.whole_job_gbs(world, 1_000_000, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_slowest_rank_sets_the_time():
    world, port = 2, _free_port()
    times = [1.25, 2.5]
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, times, out), nprocs=world, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        ms, gbs = res[rank]
        assert ms == max(times)
        assert gbs == pytest.approx(2 * 1_000_000 / (2.5e-3) / 1e9)


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks(3.0, None, "cpu") == 3.0
    assert bench.whole_job_gbs(1, 2_000_000, 1.0) == pytest.approx(2.0)


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
