"""Shared fixtures of the GPU parity tests: seeded models and inputs on cuda:0, and the
error measures the tolerances are stated in."""
import math

import numpy as np
import torch

import diffusion_transformer_text_block_b200 as moss
from synth import TINY, ModelShape, make_weights, numpy_weights, to_numpy

# One full-width block (hidden 3072, 24 heads of 128, FFN 8192) for the C2 workload.
WIDE1 = ModelShape(layers=1, hidden=3072, heads=24, ffn=8192)


def rel_l2(a, ref) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))


def cuda_weights(shape, seed, layers=None):
    w = make_weights(shape, seed, device="cpu", layers=layers)
    return {k: v.cuda() for k, v in w.items()}, numpy_weights(w)


def make_model(shape, seed, max_tokens, max_batch=2, max_latent_hw=64, max_steps=8, layers=None):
    wg, wn = cuda_weights(shape, seed, layers)
    model = moss.Model(shape, wg, max_tokens=max_tokens, max_batch=max_batch, max_latent_hw=max_latent_hw,
                       max_steps=max_steps)
    return model, wg, wn


def assert_no_device_error():
    assert moss.device_status(clear=True) == 0


def psnr(ref, test) -> float:
    ref = np.asarray(ref, np.float64)
    test = np.asarray(test, np.float64)
    mse = float(np.mean((ref - test) ** 2))
    rng = float(ref.max() - ref.min())
    return float("inf") if mse == 0 else 10 * math.log10(rng * rng / mse)


class LazyLayers:
    """A stacked [L, ...] weight tensor on the GPU that the oracle indexes one layer at a time: each
    index returns that layer as an exact float64 numpy copy.  The full model's 5e9 parameters in
    float64 would need 40 GB of host memory; one layer needs under 1 GB."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __len__(self):
        return self.shape[0]

    def __getitem__(self, l):
        return self.t[l].to(torch.float64).cpu().numpy()


def lazy_numpy_weights(w: dict) -> dict:
    """The oracle's view of a GPU weight dict: stacked per-layer weights stay on the GPU behind
    LazyLayers, the small ones are copied to float64 numpy once."""
    per_layer = {"mod_w", "mod_b", "wqkv", "q_gain", "k_gain", "wo", "wg", "wu", "wd"}
    return {k: LazyLayers(v) if k in per_layer else to_numpy(v) for k, v in w.items()}
