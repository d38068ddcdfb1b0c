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


def _cfg_parallel_worker(rank, world, port, out, cfg):
    """Rank r of the CFG-parallel schedule on CPU: the oracle's single-branch forward and
    guided Euler update stand in for the library's kernels; the exchange is a real gloo
    all-gather."""
    import numpy as np
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from diffusion_transformer_text_block_b200.cfg_parallel import cfg_parallel_loop
    import oracle.moss_oracle as o
    from synth import TINY, make_weights, numpy_weights

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = numpy_weights(make_weights(TINY, 31))
        rng = np.random.default_rng(31)
        tc = rng.standard_normal((16, TINY.hidden))
        tu = rng.standard_normal((5, TINY.hidden))
        steps = 4
        sig = o.sigma_schedule(steps, 5.0)
        x = o.gaussian_noise(8 * 8 * 32, 7).reshape(8, 8, 32)

        def forward(xx, t, uncond, skip):
            text = tu if uncond else tc
            return o.dit_forward(xx, text[None], t, [(1,) if skip else ()], w, TINY.heads)[0].astype(np.float32)

        def exchange(v):
            parts = [torch.empty(v.shape, dtype=torch.float32) for _ in range(2)]
            dist.all_gather(parts, torch.from_numpy(np.ascontiguousarray(v)))
            return parts[0].numpy(), parts[1].numpy()

        def update(xx, v_c, v_u, c, s0, s1):
            xx[...] = o.cfg_euler(xx, v_c, v_u, c, s0, s1)

        res = cfg_parallel_loop(x, sig, steps, cfg, rank, forward, exchange, update,
                                lambda i: o.slg_active(i, steps, 0.01, 1.0))
        out[rank] = res.copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cfg", [3.0, 1.0])
def test_cfg_parallel_schedule_gloo_world2(cfg):
    """Both ranks end with the single-process sampler's latent, bit for bit: rank 0 runs the
    conditional branch, rank 1 the unconditional one with its skip window, one exchange per
    step, the same update on both copies."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import oracle.moss_oracle as o
    from synth import TINY, make_weights, numpy_weights

    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_cfg_parallel_worker, args=(world, port, out, cfg), nprocs=world, join=True)
        res = dict(out)
    w = numpy_weights(make_weights(TINY, 31))
    rng = np.random.default_rng(31)
    tc = rng.standard_normal((16, TINY.hidden))
    tu = rng.standard_normal((5, TINY.hidden))
    ref = o.sample(w, TINY.heads, 64, 64, tc, tu, steps=4, cfg=cfg, shift=5.0, seed=7, uncond_skip_layers=(1,))
    for rank in range(world):
        np.testing.assert_array_equal(res[rank], ref)
