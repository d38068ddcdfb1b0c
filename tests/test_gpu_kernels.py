"""Operator-level parity of the CUDA kernels with the oracle, through the C ABI.

Tolerances, from the arithmetic:
  * GEMM: exact BF16 inputs, FP32 accumulation over K -> relative L2 <= 1e-5.
  * attention: P is rounded to BF16 before the PV product and O is stored in BF16
    (unit roundoff 2^-9 each); 3/8 of the exponentials come from a cubic with relative error
    <= 1.0e-4, well below that -> relative L2 <= 1e-2.
  * LN-modulate: BF16 output -> relative L2 <= 5e-3.
  * CFG + Euler: FP32, <= 1e-6 relative to the magnitude of the terms (FMA allowed).
  * noise: FP32 Box-Muller on identical integers -> |dz| <= 1e-5 (1 + |z|).
  * modulation: FP32 accumulation of BF16 weights -> relative L2 <= 1e-5.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_text_block_b200 as moss
from oracle import moss_oracle as o
from synth import TINY
from tests.gpu_common import assert_no_device_error, make_model, rel_l2

pytestmark = pytest.mark.gpu


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 512, 320), (1024, 768, 3072), (77, 96, 704),
                                   (2304, 3072, 1024)])
def test_gemm_bf16(M, N, K):
    a, b = _bf16((M, K), 1), _bf16((N, K), 2)
    c = moss.op_gemm_bf16(a.cuda(), b.cuda())
    torch.cuda.synchronize()
    ref = a.double().numpy() @ b.double().numpy().T
    assert rel_l2(c.cpu().numpy(), ref) <= 1e-5
    assert_no_device_error()


@pytest.mark.parametrize("B,N,H,qscale", [(1, 32, 2, 1.0), (2, 200, 2, 1.0), (2, 384, 3, 1.0), (1, 520, 2, 4.0),
                                          (2, 1, 1, 1.0), (1, 300, 1, 32.0), (1, 129, 1, 1.0), (1, 255, 1, 1.0),
                                          (2, 257, 1, 1.0), (1, 511, 2, 1.0),
                                          (2, 100, 80, 1.0), (2, 520, 64, 1.0), (2, 1100, 24, 1.0)])
def test_attention(B, N, H, qscale):
    """Against the oracle; qscale 32 spreads a row's scores over several hundred (log2 units), so
    exponent arguments fall below -126, where the kernel's polynomial exponentials clamp.
    The last three shapes launch more CTAs (256-query block, head, branch) than the GPU has SMs:
    one key step per CTA with 80 heads, a ragged key tail of 8 with 64 heads, and a last query
    block of 76 rows (its tile B entirely past the sequence end) with 24 heads."""
    D = H * 128
    q = _bf16((B, N, D), 3, qscale)
    k = _bf16((B, N, D), 4)
    v = _bf16((B, N, D), 5)
    qkv = torch.cat([q, k, v], dim=2).contiguous()
    out = moss.op_attention(qkv.cuda(), H)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    for b in range(B):
        qh = q[b].double().numpy().reshape(N, H, 128).transpose(1, 0, 2)
        kh = k[b].double().numpy().reshape(N, H, 128).transpose(1, 0, 2)
        vh = v[b].double().numpy().reshape(N, H, 128).transpose(1, 0, 2)
        ref = o.attention(qh, kh, vh).transpose(1, 0, 2).reshape(N, D)
        assert rel_l2(got[b], ref) <= 1e-2, (b, rel_l2(got[b], ref))
    assert_no_device_error()


@pytest.mark.parametrize("rows,dim", [(1, 256), (37, 256), (500, 3072), (9216, 3072)])
def test_ln_modulate(rows, dim):
    g = torch.Generator().manual_seed(6)
    x = torch.randn(rows, dim, generator=g) * 3 + 0.5
    shift = torch.randn(dim, generator=g) * 0.1
    scale = torch.randn(dim, generator=g) * 0.1
    h = moss.op_ln_modulate(x.cuda(), shift.cuda(), scale.cuda())
    torch.cuda.synchronize()
    ref = o.ln_modulate(x.double().numpy(), shift.double().numpy(), scale.double().numpy())
    assert rel_l2(h.float().cpu().numpy(), ref) <= 5e-3
    assert_no_device_error()


@pytest.mark.parametrize("n", [0, 3, 4, 1001, 128 * 128 * 32, 256 * 256 * 32])
def test_cfg_euler(n):
    g = torch.Generator().manual_seed(7)
    x, vc, vu = (torch.randn(n, generator=g) for _ in range(3))
    sig = o.sigma_schedule(50, 5.0)
    s0, s1 = float(sig[3]), float(sig[4])
    xg = x.cuda()
    moss.cfg_euler_step(xg, vc.cuda(), vu.cuda(), 3.0, s0, s1)
    torch.cuda.synchronize()
    ref = o.cfg_euler(x.numpy(), vc.numpy(), vu.numpy(), 3.0, s0, s1)
    if n == 0:
        return
    dt = abs(np.float32(s1) - np.float32(s0))
    scale = np.abs(x.numpy()) + dt * (np.abs(vu.numpy()) + 3.0 * (np.abs(vc.numpy()) + np.abs(vu.numpy())))
    assert np.all(np.abs(xg.cpu().numpy() - ref) <= 1e-6 * scale)
    # cfg = 1 -> the conditional velocity, up to the rounding of v_u + (v_c - v_u)
    x1 = x.cuda()
    moss.cfg_euler_step(x1, vc.cuda(), vu.cuda(), 1.0, s0, s1)
    ref1 = o.euler_update(x.numpy(), vc.numpy(), s0, s1)
    assert np.all(np.abs(x1.cpu().numpy() - ref1) <= 1e-6 * scale)
    # v_u = v_c (what the step passes when no negative branch runs): exactly x + dt v_c
    x2 = x.cuda()
    moss.cfg_euler_step(x2, vc.cuda(), vc.cuda(), 1.0, s0, s1)
    assert np.all(np.abs(x2.cpu().numpy() - ref1) <= 1e-6 * (np.abs(x.numpy()) + dt * np.abs(vc.numpy())))


@pytest.mark.parametrize("n,seed", [(4, 0), (1001, 42), (128 * 128 * 32, 42), (64, (1 << 40) + 3)])
def test_noise_matches_oracle(n, seed):
    x = torch.empty(n, device="cuda")
    moss.init_noise(x, seed)
    torch.cuda.synchronize()
    ref = o.gaussian_noise(n, seed).astype(np.float64)
    got = x.cpu().double().numpy()
    assert np.all(np.abs(got - ref) <= 1e-5 * (1 + np.abs(ref)))


def test_modulation_matches_oracle():
    model, _, wn = make_model(TINY, 21, max_tokens=64)
    for t in (0.0, 0.37, 1.0):
        mod = model.modulation(t).cpu().double().numpy()
        c = o.conditioning(t, wn)
        ref = np.concatenate([o.block_modulation(c, wn["mod_w"][l], wn["mod_b"][l]) for l in range(TINY.layers)] +
                             [o.block_modulation(c, wn["final_mod_w"], wn["final_mod_b"])])
        assert rel_l2(mod, ref) <= 1e-5
    model.close()
    assert_no_device_error()


def test_attention_2048_sampled_rows():
    """The 2048^2 long-sequence shape: 16384 image + 4096 text tokens, batch 2, 24 heads;
    sampled query rows (tile edges, the image/text boundary, random) against the oracle."""
    B, N, H = 2, 16384 + 4096, 24
    D = H * 128
    g = torch.Generator(device="cuda").manual_seed(11)
    qkv = torch.randn(B, N, 3 * D, generator=g, device="cuda").to(torch.bfloat16)
    out = moss.op_attention(qkv, H)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 63, 64, 127, 128, 16383, 16384, N - 1], rng.integers(0, N, 12)]))
    got = out[:, rows].float().cpu().numpy()
    for b in range(B):
        qb = qkv[b].cpu().double().numpy()
        q = qb[rows, :D].reshape(len(rows), H, 128).transpose(1, 0, 2)
        k = qb[:, D:2 * D].reshape(N, H, 128).transpose(1, 0, 2)
        v = qb[:, 2 * D:].reshape(N, H, 128).transpose(1, 0, 2)
        ref = o.attention(q, k, v).transpose(1, 0, 2).reshape(len(rows), D)
        assert rel_l2(got[b], ref) <= 1e-2
    assert_no_device_error()
