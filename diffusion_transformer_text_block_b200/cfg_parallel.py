"""CFG-parallel sampling over two ranks (one process per GPU, torch.distributed for plumbing).

SGLang cookbook "OpenMOSS/MOSS-Image", 4. Deployment features: CFG parallelism dispatches the
branches of a step (conditional, unconditional) to different GPUs.  Rank 0 runs the conditional branch,
rank 1 the unconditional one (skipping its layers inside the skip window); after each step's
forward the two velocities are exchanged with one all-gather (2 MB of FP32 at 1024^2) and both
ranks apply the same CFG + Euler kernel to their own copy of the latent, so the copies stay
identical without a second exchange.  At cfg == 1 there is no unconditional pass and each rank
runs the conditional branch alone (no exchange).

Every step of the path runs in the library's kernels (moss_dit_forward, moss_cfg_euler_step,
moss_init_noise); this module only orders the calls and the collective.
"""
from __future__ import annotations

from typing import Callable, Sequence


def cfg_parallel_loop(x, sigmas: Sequence[float], steps: int, cfg: float, rank: int,
                      forward: Callable, exchange: Callable, update: Callable, window: Callable):
    """The schedule of CFG-parallel sampling, independent of the device and the backend.

    forward(x, t, uncond, skip) -> this rank's velocity; exchange(v) -> (v_c, v_u), the same on
    both ranks; update(x, v_c, v_u, cfg, sigma, sigma_next) updates x in place; window(i) -> the
    skip window holds at step i.  rank 0 owns the conditional branch, rank 1 the unconditional.
    """
    for i in range(steps):
        t = float(sigmas[i])
        if cfg == 1.0:
            v = forward(x, t, False, False)
            update(x, v, v, 1.0, sigmas[i], sigmas[i + 1])
            continue
        v = forward(x, t, rank == 1, rank == 1 and window(i))
        v_c, v_u = exchange(v)
        update(x, v_c, v_u, cfg, sigmas[i], sigmas[i + 1])
    return x


def cfg_parallel_sample(model, text_c, text_u, height: int, width: int, steps: int = 50, cfg: float = 3.0,
                        shift: float = 5.0, seed: int = 42, uncond_skip_layers: Sequence[int] = (22,),
                        slg_start: float = 0.01, slg_stop: float = 1.0, group=None):
    """moss_sample split over the two ranks of `group` (the default process group if None).

    Both ranks pass the same arguments; each returns the final latent [height/8, width/8, 32]
    (identical on the two ranks).  text_u is read on rank 1 only."""
    import torch
    import torch.distributed as dist

    import diffusion_transformer_text_block_b200 as moss

    if dist.get_world_size(group) != 2:
        raise ValueError("CFG-parallel sampling needs a group of exactly two ranks")
    rank = dist.get_rank(group)
    x = torch.empty(height // 8, width // 8, 32, device=text_c.device, dtype=torch.float32)
    moss.init_noise(x, seed)
    sig = moss.sigma_schedule(steps, shift)
    skips = list(uncond_skip_layers)
    gathered = torch.empty(2, height // 8, width // 8, 32, device=x.device, dtype=torch.float32)

    def forward(xx, t, uncond, skip):
        text = text_u if uncond else text_c
        return model.forward(xx, text[None], height, width, t, skip_layers=[skips if skip else []])[0]

    staged = dist.get_backend(group) == "gloo"  # gloo gathers host tensors: stage through the host

    def exchange(v):
        if staged:
            parts = [torch.empty(v.shape, dtype=torch.float32) for _ in range(2)]
            dist.all_gather(parts, v.cpu(), group=group)
            gathered.copy_(torch.stack(parts))
        else:
            dist.all_gather(list(gathered.unbind(0)), v.contiguous(), group=group)
        return gathered[0], gathered[1]

    def update(xx, v_c, v_u, c, s0, s1):
        moss.cfg_euler_step(xx, v_c.contiguous(), v_u.contiguous(), c, float(s0), float(s1))

    return cfg_parallel_loop(x, sig, steps, cfg, rank, forward, exchange, update,
                             lambda i: moss.slg_active(i, steps, slg_start, slg_stop))
