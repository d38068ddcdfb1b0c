"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and lays them out; it holds none of the
DiT's arithmetic.  Both the CPU oracle and the CUDA library consume exactly the
tensors produced here (the oracle after an exact BF16 -> float upcast).

Recipe (what the pages give for the workload, the rest is ours):
  * linear weights and biases ~ N(0, 0.02), rounded to BF16 (round-to-nearest-even,
    torch's ``.to(torch.bfloat16)``);
  * per-head Q/K RMSNorm gains = 1 + N(0, 0.02), kept in FP32;
  * latents, text states and residual streams ~ N(0, 1) in FP32.
Small shapes are drawn on the CPU; the 5B-parameter full model is drawn on the
GPU (``device="cuda"``) because drawing 5e9 normals on the host takes minutes.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Width parameters of the single-stream DiT.

    The full model is 42 joint blocks, hidden 3072, 24 heads of 128, FFN 8192,
    over 2x2 patches of the 32-channel latent (windpaint.ai, "MOSS-Image: specs,
    settings, VRAM and text rendering tested", Architecture and specs table).
    ``c_t`` is the width of the timestep embedding / conditioning vector.
    """

    layers: int
    hidden: int
    heads: int
    ffn: int
    head_dim: int = 128
    c_t: int = 256
    patch: int = 2
    latent_channels: int = 32

    @property
    def patch_dim(self) -> int:
        return self.patch * self.patch * self.latent_channels


FULL = ModelShape(layers=42, hidden=3072, heads=24, ffn=8192)
TINY = ModelShape(layers=2, hidden=256, heads=2, ffn=704)


def _normal(shape, gen, device, std=1.0, dtype=torch.float32):
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_generator(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_weights(shape: ModelShape, seed: int, device: str = "cpu", layers: int | None = None,
                 std: float = 0.02) -> dict:
    """All DiT parameters, stacked over layers.

    Linear weights are stored [out_features, in_features] (row-major, the
    reduction index contiguous).  ``wqkv`` is the fused Q|K|V projection, the
    "proj.qkv" form of the checkpoints (InvokeAI MOSS-Image guide, Transformer
    formats).
    """
    L = shape.layers if layers is None else layers
    D, F, C, d = shape.hidden, shape.ffn, shape.c_t, shape.head_dim
    g = make_generator(seed, device)
    bf = torch.bfloat16
    w = {}
    w["t_w1"] = _normal((C, 256), g, device, std, bf)
    w["t_b1"] = _normal((C,), g, device, std, bf)
    w["t_w2"] = _normal((C, C), g, device, std, bf)
    w["t_b2"] = _normal((C,), g, device, std, bf)
    w["img_w"] = _normal((D, shape.patch_dim), g, device, std, bf)
    w["img_b"] = _normal((D,), g, device, std, bf)
    w["mod_w"] = _normal((L, 6 * D, C), g, device, std, bf)
    w["mod_b"] = _normal((L, 6 * D), g, device, std, bf)
    w["wqkv"] = _normal((L, 3 * D, D), g, device, std, bf)
    w["q_gain"] = 1.0 + _normal((L, d), g, device, std)
    w["k_gain"] = 1.0 + _normal((L, d), g, device, std)
    w["wo"] = _normal((L, D, D), g, device, std, bf)
    w["wg"] = _normal((L, F, D), g, device, std, bf)
    w["wu"] = _normal((L, F, D), g, device, std, bf)
    w["wd"] = _normal((L, D, F), g, device, std, bf)
    w["final_mod_w"] = _normal((2 * D, C), g, device, std, bf)
    w["final_mod_b"] = _normal((2 * D,), g, device, std, bf)
    w["out_w"] = _normal((shape.patch_dim, D), g, device, std, bf)
    w["out_b"] = _normal((shape.patch_dim,), g, device, std, bf)
    return w


TEXT_ENC_DIM = 4096  # width of the text encoder's final-layer states (Qwen3.5-9B)
TEXT_BLOCKS = 2      # text-only refiner blocks


def make_text_weights(shape: ModelShape, seed: int, enc_dim: int = TEXT_ENC_DIM, blocks: int = TEXT_BLOCKS,
                      device: str = "cpu", std: float = 0.02) -> dict:
    """Text path parameters: projection [D, enc_dim] + [D] and `blocks` text-only blocks with the
    joint blocks' linear layers and Q/K gains (stacked like make_weights; no modulation)."""
    D, F, d = shape.hidden, shape.ffn, shape.head_dim
    g = make_generator(seed, device)
    bf = torch.bfloat16
    w = {}
    w["proj_w"] = _normal((D, enc_dim), g, device, std, bf)
    w["proj_b"] = _normal((D,), g, device, std, bf)
    w["wqkv"] = _normal((blocks, 3 * D, D), g, device, std, bf)
    w["q_gain"] = 1.0 + _normal((blocks, d), g, device, std)
    w["k_gain"] = 1.0 + _normal((blocks, d), g, device, std)
    w["wo"] = _normal((blocks, D, D), g, device, std, bf)
    w["wg"] = _normal((blocks, F, D), g, device, std, bf)
    w["wu"] = _normal((blocks, F, D), g, device, std, bf)
    w["wd"] = _normal((blocks, D, F), g, device, std, bf)
    return w


def make_encoder_states(n_txt: int, seed: int, enc_dim: int = TEXT_ENC_DIM, device: str = "cpu") -> torch.Tensor:
    """BF16 final-layer text-encoder states [n_txt, enc_dim] ~ N(0, 1) (stand-in for Qwen3.5-9B's)."""
    return _normal((n_txt, enc_dim), make_generator(seed, device), device, 1.0, torch.bfloat16)


def make_latent(h8: int, w8: int, seed: int, channels: int = 32, device: str = "cpu") -> torch.Tensor:
    """FP32 latent [h8, w8, channels] ~ N(0, 1)."""
    return _normal((h8, w8, channels), make_generator(seed, device), device)


def make_text(batch: int, n_txt: int, hidden: int, seed: int, device: str = "cpu") -> torch.Tensor:
    """FP32 text states [batch, n_txt, hidden] ~ N(0, 1) (stand-in for the refined prompt)."""
    return _normal((batch, n_txt, hidden), make_generator(seed, device), device)


def make_residual(batch: int, n_tok: int, hidden: int, seed: int, device: str = "cpu") -> torch.Tensor:
    """FP32 residual stream [batch, n_tok, hidden] ~ N(0, 1)."""
    return _normal((batch, n_tok, hidden), make_generator(seed, device), device)


def to_numpy(t: torch.Tensor):
    """Exact float copy of a (possibly BF16) tensor as a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()


def numpy_weights(w: dict, layer_slice=None) -> dict:
    """Float64 numpy copies of a weight dict (optionally only some layers)."""
    out = {}
    for k, v in w.items():
        if layer_slice is not None and k in _PER_LAYER:
            v = v[layer_slice]
        out[k] = to_numpy(v)
    return out


_PER_LAYER = {"mod_w", "mod_b", "wqkv", "q_gain", "k_gain", "wo", "wg", "wu", "wd"}
