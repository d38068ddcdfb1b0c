"""CFG-parallel sampling (diffusion_transformer_text_block_b200.cfg_parallel) on the GPU: two
processes, one per CFG branch, exchanging velocities each step.  The box this runs on has one GPU,
so both ranks share it and the exchange goes through gloo on the host; no kernel of one rank waits
for the other's.  Both ranks must end with the same latent, within 40 dB of the float64 oracle's
sampler (oracle.sample, which runs the two branches of every step in one process), and equal to
the single-process moss_sample within 1e-6."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(n_u):
    from synth import TINY, make_text, make_weights
    w = {k: v.cuda() for k, v in make_weights(TINY, 121).items()}
    tc = make_text(1, 16, TINY.hidden, 122)[0].cuda()
    tu = make_text(1, max(n_u, 1), TINY.hidden, 123)[0][:n_u].contiguous().cuda()
    return w, tc, tu


def _worker(rank, world, port, out, n_u, cfg):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import diffusion_transformer_text_block_b200 as moss
    from diffusion_transformer_text_block_b200.cfg_parallel import cfg_parallel_sample
    from synth import TINY

    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, tc, tu = _inputs(n_u)
        model = moss.Model(TINY, w, max_tokens=32, max_batch=2, max_latent_hw=64, max_steps=4)
        x = cfg_parallel_sample(model, tc, tu, 64, 64, steps=4, cfg=cfg, seed=5, uncond_skip_layers=[1])
        torch.cuda.synchronize()
        out[rank] = (x.cpu().numpy(), moss.device_status(clear=True))
        model.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_u,cfg", [(16, 3.0), (5, 3.0), (16, 1.0)])
def test_cfg_parallel_matches_oracle_and_moss_sample(n_u, cfg):
    sys.path.insert(0, ROOT)
    import diffusion_transformer_text_block_b200 as moss
    from oracle import moss_oracle as o
    from synth import TINY, to_numpy
    from tests.gpu_common import psnr

    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out, n_u, cfg), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    w, tc, tu = _inputs(n_u)
    model = moss.Model(TINY, w, max_tokens=32, max_batch=2, max_latent_hw=64, max_steps=4)
    ref = model.sample(tc, tu, 64, 64, steps=4, cfg=cfg, seed=5, uncond_skip_layers=[1]).cpu().numpy()
    model.close()
    wn = {k: to_numpy(v) for k, v in w.items()}
    oracle_x = o.sample(wn, TINY.heads, 64, 64, to_numpy(tc), to_numpy(tu), steps=4, cfg=cfg, seed=5,
                        uncond_skip_layers=(1,))
    for rank in range(world):
        x, status = res[rank]
        assert status == 0
        np.testing.assert_array_equal(x, res[0][0])
        err = np.linalg.norm(x.astype(np.float64) - ref) / np.linalg.norm(ref)
        assert err <= 1e-6, err
        assert psnr(oracle_x, x) >= 40.0, psnr(oracle_x, x)
