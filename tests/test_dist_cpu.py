"""The multi-rank path of bench.py on CPU: world size 2 over gloo.

The benchmark runs replicas (one image per rank, no collective on the data path); the
host logic that spans ranks is the max-over-ranks device time and the whole-job
throughput.  The reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(100.0 + 25.0 * rank, dist, "cpu")
        value, ms_step = bench.job_throughput(50, world, ms)
        dist.barrier()
        out[rank] = (ms, value, ms_step)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, value, ms_step = res[rank]
        assert ms == 125.0                       # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 50 * world / 0.125)
        assert ms_step == pytest.approx(2.5)


def test_throughput_single_process():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5) == 7.5
    v, ms = bench.job_throughput(10, 1, 1000.0)
    assert v == pytest.approx(20.0) and ms == pytest.approx(100.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
