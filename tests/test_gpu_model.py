"""Parity of the DiT block, the forward and the sampler with the oracle, through the C ABI.

Bars (the method's stated tolerances): per-block relative L2 <= 1e-2 with BF16 weights
against the float64 oracle, on the block output and on its update y - x (the residual
alone would hide errors); the forward's velocity per branch <= 1e-2; the tiny 4-step
sampling run >= 40 dB PSNR against the oracle's.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_text_block_b200 as moss
from oracle import moss_oracle as o
from synth import TINY, make_latent, make_residual, make_text
from tests.gpu_common import WIDE1, assert_no_device_error, lazy_numpy_weights, make_model, psnr, rel_l2

pytestmark = pytest.mark.gpu


def _block_case(shape, seed, gh, gw, n_txt, batch, t, layer=0, layers=None):
    N = gh * gw + n_txt
    model, wg, wn = make_model(shape, seed, max_tokens=N, max_batch=batch, max_latent_hw=4 * gh * gw,
                               layers=layers)
    x = make_residual(batch, N, shape.hidden, seed + 1)
    xg = x.cuda()
    model.block_forward(layer, xg, gh, gw, n_txt, t)
    torch.cuda.synchronize()
    y = xg.cpu().double().numpy()
    c = o.conditioning(t, wn)
    mod = o.block_modulation(c, wn["mod_w"][layer], wn["mod_b"][layer])
    ang = o.rope_angles(o.token_positions(gh, gw, n_txt))
    lw = o.layer_weights(wn, layer)
    return model, x.double().numpy(), y, lw, mod, ang


@pytest.mark.parametrize("gh,gw,n_txt,batch", [(4, 4, 16, 2), (8, 10, 60, 2), (2, 3, 0, 1), (1, 1, 300, 2)])
def test_block_tiny(gh, gw, n_txt, batch):
    model, x, y, lw, mod, ang = _block_case(TINY, 31, gh, gw, n_txt, batch, 0.5, layer=1)
    for b in range(batch):
        ref = o.block_forward(x[b], lw, mod, ang, TINY.heads)
        assert rel_l2(y[b], ref) <= 1e-2
        assert rel_l2(y[b] - x[b], ref - x[b]) <= 1e-2, rel_l2(y[b] - x[b], ref - x[b])
    model.close()
    assert_no_device_error()


def test_block_full_width_one_block():
    """One full-width block: 256x256 image (256 image tokens) + 128 text tokens, batch 2,
    t = 0.5, FP32 residual stream."""
    model, x, y, lw, mod, ang = _block_case(WIDE1, 41, 16, 16, 128, 2, 0.5)
    for b in range(2):
        ref = o.block_forward(x[b], lw, mod, ang, WIDE1.heads)
        assert rel_l2(y[b], ref) <= 1e-2
        assert rel_l2(y[b] - x[b], ref - x[b]) <= 1e-2, rel_l2(y[b] - x[b], ref - x[b])
    model.close()
    assert_no_device_error()


def test_block_full_size_sampled_rows():
    """The 1024^2 block shape the benchmark times (4096 image + 512 text tokens, batch 2):
    sampled rows against the oracle's row-restricted block."""
    gh = gw = 64
    n_txt = 512
    model, x, y, lw, mod, ang = _block_case(WIDE1, 43, gh, gw, n_txt, 2, 0.83)
    N = gh * gw + n_txt
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 63, 64, 4095, 4096, N - 1], rng.integers(0, N, 25)]))
    for b in range(2):
        ref = o.block_forward_rows(x[b], lw, mod, ang, rows, WIDE1.heads)
        assert rel_l2(y[b][rows], ref) <= 1e-2
        assert rel_l2(y[b][rows] - x[b][rows], ref - x[b][rows]) <= 1e-2
    model.close()
    assert_no_device_error()


def test_forward_tiny_with_uncond_skip():
    model, wg, wn = make_model(TINY, 51, max_tokens=32, max_latent_hw=64)
    lat = make_latent(8, 8, 52)
    txt = make_text(2, 16, TINY.hidden, 53)
    v = model.forward(lat.cuda(), txt.cuda(), 64, 64, 0.3, skip_layers=[[], [1]])
    torch.cuda.synchronize()
    ref = o.dit_forward(lat.numpy(), txt.double().numpy(), 0.3, [(), (1,)], wn, TINY.heads)
    got = v.cpu().double().numpy()
    for b in range(2):
        assert rel_l2(got[b], ref[b]) <= 1e-2, rel_l2(got[b], ref[b])
    # the skipped branch really differs from an unskipped one
    v2 = model.forward(lat.cuda(), txt.cuda(), 64, 64, 0.3, skip_layers=[[], []])
    assert rel_l2(v2.cpu().numpy()[1], got[1]) > 1e-3
    model.close()
    assert_no_device_error()


def test_forward_tiny_skip_all_layers():
    model, wg, wn = make_model(TINY, 55, max_tokens=48, max_latent_hw=4 * 4 * 8 * 4)
    lat = make_latent(8, 16, 56)  # 64 x 128 image: 32 image tokens
    txt = make_text(1, 16, TINY.hidden, 57)
    v = model.forward(lat.cuda(), txt.cuda(), 64, 128, 0.9, skip_layers=[[0, 1]])
    ref = o.dit_forward(lat.numpy(), txt.double().numpy(), 0.9, [(0, 1)], wn, TINY.heads)
    assert rel_l2(v.cpu().numpy()[0], ref[0]) <= 1e-2
    model.close()
    assert_no_device_error()


def test_sample_tiny_psnr():
    """The tiny sampling run: 64x64 image, 4 flow-Euler steps, shift 5, CFG 3, uncond skips
    block 1 inside [0.01, 1.0], seed 0."""
    model, wg, wn = make_model(TINY, 61, max_tokens=32, max_latent_hw=64, max_steps=4)
    tc = make_text(1, 16, TINY.hidden, 62)[0]
    tu = make_text(1, 16, TINY.hidden, 63)[0]
    out = model.sample(tc.cuda(), tu.cuda(), 64, 64, steps=4, cfg=3.0, shift=5.0, seed=0,
                       uncond_skip_layers=[1], slg_start=0.01, slg_stop=1.0)
    torch.cuda.synchronize()
    ref = o.sample(wn, TINY.heads, 64, 64, tc.double().numpy(), tu.double().numpy(), steps=4, cfg=3.0, shift=5.0,
                   seed=0, uncond_skip_layers=(1,), slg_start=0.01, slg_stop=1.0)
    p = psnr(ref, out.cpu().numpy())
    assert p >= 40.0, p
    model.close()
    assert_no_device_error()


def test_denoise_step_cfg1_and_sample_consistency():
    model, wg, wn = make_model(TINY, 71, max_tokens=32, max_latent_hw=64, max_steps=4)
    tc = make_text(1, 16, TINY.hidden, 72)[0].cuda()
    tu = make_text(1, 16, TINY.hidden, 73)[0].cuda()
    # sample == noise + the same denoising steps called one by one (bitwise)
    a = model.sample(tc, tu, 64, 64, steps=3, seed=5, uncond_skip_layers=[1])
    x = torch.empty(8, 8, 32, device="cuda")
    moss.init_noise(x, 5)
    for i in range(3):
        model.denoise_step(x, tc, tu, 64, 64, i, 3, uncond_skip_layers=[1])
    assert torch.equal(a, x)
    # CFG 1 runs no unconditional pass: NaN negative text cannot reach the result
    bad = torch.full_like(tu, float("nan"))
    y = model.sample(tc, bad, 64, 64, steps=2, cfg=1.0, seed=5, uncond_skip_layers=[1])
    assert torch.isfinite(y).all()
    ref = o.sample(wn, TINY.heads, 64, 64, tc.cpu().double().numpy(), None, steps=2, cfg=1.0, seed=5)
    assert psnr(ref, y.cpu().numpy()) >= 40.0
    model.close()
    assert_no_device_error()


def test_denoise_step_schedule_reuse_matches_per_step_modulation():
    """moss_denoise_step computes a schedule's modulation once and reuses it (steps <= max_steps); with
    steps > max_steps each call computes its own step's vectors.  Both give the same steps bit for bit,
    also after a forward call in between has dropped the stored schedule."""
    a, wg, _ = make_model(TINY, 79, max_tokens=32, max_latent_hw=64, max_steps=8)
    b = moss.Model(TINY, wg, max_tokens=32, max_batch=2, max_latent_hw=64, max_steps=4)
    tc = make_text(1, 16, TINY.hidden, 80)[0].cuda()
    tu = make_text(1, 9, TINY.hidden, 81)[0].cuda()
    x0 = make_latent(8, 8, 82).cuda()
    xa, xb = x0.clone(), x0.clone()
    for i in range(8):
        a.denoise_step(xa, tc, tu, 64, 64, i, 8, uncond_skip_layers=[1])
        b.denoise_step(xb, tc, tu, 64, 64, i, 8, uncond_skip_layers=[1])   # 8 > max_steps: per call
        if i == 3:
            a.forward(x0, torch.stack([tc, tc]), 64, 64, 0.5)              # drops the stored schedule
    torch.cuda.synchronize()
    assert torch.equal(xa, xb)
    a.close()
    b.close()
    assert_no_device_error()


def test_denoise_step_host_buffers_match_device_step():
    """moss_denoise_step_host (latent and prompts in host memory, pinned and pageable) gives the
    device-buffer step's result bit for bit, with a ragged negative prompt and at cfg 1."""
    model, wg, wn = make_model(TINY, 75, max_tokens=32, max_latent_hw=64, max_steps=4)
    tc = make_text(1, 16, TINY.hidden, 76)[0]
    tu = make_text(1, 7, TINY.hidden, 77)[0]
    x0 = make_latent(8, 8, 78)
    for cfg, pinned in ((3.0, True), (3.0, False), (1.0, True)):
        xd = x0.cuda()
        for i in range(2):
            model.denoise_step(xd, tc.cuda(), tu.cuda(), 64, 64, i, 4, cfg=cfg, uncond_skip_layers=[1])
        xh = x0.clone().pin_memory() if pinned else x0.clone()
        htc = tc.pin_memory() if pinned else tc
        htu = tu.pin_memory() if pinned else tu
        for i in range(2):
            model.denoise_step_host(xh, htc, htu, 64, 64, i, 4, cfg=cfg, uncond_skip_layers=[1])
        torch.cuda.synchronize()
        assert torch.equal(xh, xd.cpu()), cfg
    with pytest.raises(moss.MossError, match="host"):
        model.denoise_step_host(x0.cuda(), tc, tu, 64, 64, 0, 4)
    model.close()
    assert_no_device_error()


def test_invalid_requests_launch_nothing():
    model, wg, wn = make_model(TINY, 81, max_tokens=32, max_latent_hw=64)
    lat = torch.zeros(8, 8, 32, device="cuda")
    txt = torch.zeros(2, 16, TINY.hidden, device="cuda")
    before = moss.launch_count()
    with pytest.raises(moss.MossError, match="multiples of 16"):
        model.forward(lat, txt, 60, 64, 0.5)
    with pytest.raises(moss.MossError, match="out of range"):
        model.forward(lat, txt, 64, 64, 0.5, skip_layers=[[], [2]])
    with pytest.raises(moss.MossError, match="max_tokens"):
        model.forward(lat, torch.zeros(2, 17, TINY.hidden, device="cuda"), 64, 64, 0.5)
    assert moss.launch_count() == before
    model.close()


@pytest.mark.parametrize("gh,gw", [(128, 128), (256, 64)])
def test_block_2048_sampled_rows(gh, gw):
    """One full-width block at the largest token count the size rule allows (4.2 MP: 16384 image
    + 4096 text tokens, batch 2), square 2048^2 and the 4096 x 1024 extreme (patch rows up to 255):
    sampled rows against the oracle's row-restricted block."""
    n_txt = 4096
    model, x, y, lw, mod, ang = _block_case(WIDE1, 45, gh, gw, n_txt, 2, 0.41)
    N = gh * gw + n_txt
    rows = np.array([0, gw - 1, gw, 16383, 16384, N - 1, 9000])
    for b in range(2):
        ref = o.block_forward_rows(x[b], lw, mod, ang, rows, WIDE1.heads)
        assert rel_l2(y[b][rows], ref) <= 1e-2
        assert rel_l2(y[b][rows] - x[b][rows], ref - x[b][rows]) <= 1e-2
    model.close()
    assert_no_device_error()


@pytest.fixture(scope="module")
def full_model():
    """The 42-block, hidden-3072 DiT with ~5B random BF16 weights (drawn on the GPU), sized for
    the 1024^2 workload: 4096 image + 512 text tokens per branch, up to 3 branches."""
    from synth import FULL, make_weights
    w = make_weights(FULL, 2, device="cuda")
    model = moss.Model(FULL, w, max_tokens=4096 + 512, max_batch=3, max_latent_hw=128 * 128, max_steps=2)
    yield model, w
    model.close()


def test_full_forward_skip_all_layers_matches_oracle(full_model):
    """1024^2, all 42 layers skipped: patch embed, final LN-modulate, output projection and
    unpatchify of the full-size model against the oracle."""
    from synth import FULL, numpy_weights
    model, w = full_model
    lat = make_latent(128, 128, 7, device="cuda")
    txt = make_text(2, 512, FULL.hidden, 8, device="cuda")
    skip = list(range(FULL.layers))
    v = model.forward(lat, txt, 1024, 1024, 0.6, skip_layers=[skip, skip])
    torch.cuda.synchronize()
    small = {k: w[k] for k in ("t_w1", "t_b1", "t_w2", "t_b2", "img_w", "img_b", "final_mod_w", "final_mod_b",
                               "out_w", "out_b")}
    wn = numpy_weights(small)
    c = o.conditioning(0.6, wn)
    img = o.patchify(lat.cpu().double().numpy()) @ wn["img_w"].T + wn["img_b"]
    ref = o.unpatchify(o.final_layer(img, c, wn), 128, 128)
    got = v.cpu().double().numpy()
    for b in range(2):
        assert rel_l2(got[b], ref) <= 1e-2
    assert_no_device_error()


def test_full_forward_branches_and_determinism(full_model):
    """1024^2, 42 layers, uncond skipping layer 22: the CFG batch equals each branch run alone
    (bitwise: every kernel is row-wise or per-branch and free of atomics order effects), and two
    runs are bitwise identical (run-to-run reproducibility)."""
    from synth import FULL
    model, w = full_model
    lat = make_latent(128, 128, 9, device="cuda")
    txt = make_text(2, 512, FULL.hidden, 10, device="cuda")
    v = model.forward(lat, txt, 1024, 1024, 0.77, skip_layers=[[], [22]]).clone()
    v2 = model.forward(lat, txt, 1024, 1024, 0.77, skip_layers=[[], [22]])
    assert torch.equal(v, v2)
    vc = model.forward(lat, txt[:1].contiguous(), 1024, 1024, 0.77, skip_layers=[[]])
    vu = model.forward(lat, txt[1:].contiguous(), 1024, 1024, 0.77, skip_layers=[[22]])
    assert torch.equal(v[0], vc[0]) and torch.equal(v[1], vu[0])
    assert torch.isfinite(v).all()
    # the skipped layer matters
    vn = model.forward(lat, txt[1:].contiguous(), 1024, 1024, 0.77, skip_layers=[[]])
    assert not torch.equal(vn[0], vu[0])
    assert_no_device_error()


def test_full_denoise_step_matches_manual_cfg(full_model):
    """One 1024^2 denoising step (step 1 of 50: uncond skips layer 22) equals the forward of
    both branches followed by the CFG + Euler update."""
    from synth import FULL
    model, w = full_model
    x0 = make_latent(128, 128, 11, device="cuda")
    tc = make_text(1, 512, FULL.hidden, 12, device="cuda")[0].contiguous()
    tu = make_text(1, 512, FULL.hidden, 13, device="cuda")[0].contiguous()
    x = x0.clone()
    model.denoise_step(x, tc, tu, 1024, 1024, 1, 50, 3.0, 5.0, [22], 0.01, 1.0)
    sig = o.sigma_schedule(50, 5.0)
    v = model.forward(x0, torch.stack([tc, tu]), 1024, 1024, float(sig[1]), skip_layers=[[], [22]])
    ref = x0.clone()
    moss.cfg_euler_step(ref, v[0].contiguous(), v[1].contiguous(), 3.0, float(sig[1]), float(sig[2]))
    assert torch.equal(x, ref)
    assert_no_device_error()


def test_full_guided_step_fused_update_matches_forward_and_update(full_model):
    """The guided step applies the CFG + Euler update inside the output projection (one kernel per
    tile of 128 image tokens, both branches).  On a 272^2 image (17 x 17 = 289 image tokens, so the
    last token tile is partial) with a 300-token prompt and a 77-token negative prompt, it equals the
    two branch forwards followed by the standalone CFG + Euler kernel, bit for bit."""
    from synth import FULL
    model, w = full_model
    x0 = make_latent(34, 34, 24, device="cuda")
    tc = make_text(1, 300, FULL.hidden, 25, device="cuda")[0].contiguous()
    tu = make_text(1, 77, FULL.hidden, 26, device="cuda")[0].contiguous()
    x = x0.clone()
    before = moss.launch_count()
    model.denoise_step(x, tc, tu, 272, 272, 7, 50, 3.0, 5.0, [22], 0.01, 1.0)
    fused_launches = moss.launch_count() - before
    sig = o.sigma_schedule(50, 5.0)
    vc = model.forward(x0, tc[None], 272, 272, float(sig[7]), skip_layers=[[]]).clone()
    vu = model.forward(x0, tu[None], 272, 272, float(sig[7]), skip_layers=[[22]]).clone()
    ref = x0.clone()
    moss.cfg_euler_step(ref, vc[0].contiguous(), vu[0].contiguous(), 3.0, float(sig[7]), float(sig[8]))
    torch.cuda.synchronize()
    assert torch.equal(x, ref)
    assert rel_l2(x.cpu().numpy(), x0.cpu().numpy()) > 1e-3
    # the step launched no standalone update kernel: its class saw no launch
    model.profile_enable(True)
    model.denoise_step(x, tc, tu, 272, 272, 8, 50, 3.0, 5.0, [22], 0.01, 1.0)
    prof = model.profile_read()
    model.profile_enable(False)
    assert prof["cfg_euler"][0] == 0 and prof["gemm_qkv"][0] > 0
    assert fused_launches > 0
    assert_no_device_error()


def test_full_guided_step_2048_fused_update(full_model):
    """The long-sequence stress shape (2048^2: 16384 image tokens, a 4096-token prompt -- the pages'
    maximum -- and a 77-token negative prompt) with the full model: the guided step, whose fused update
    runs 256 work units over at most 148 CTAs, equals the two branch forwards followed by the
    standalone CFG + Euler kernel, bit for bit."""
    from synth import FULL
    _, w = full_model
    model = moss.Model(FULL, w, max_tokens=16384 + 4096, max_batch=2, max_latent_hw=256 * 256, max_steps=10)
    x0 = make_latent(256, 256, 27, device="cuda")
    tc = make_text(1, 4096, FULL.hidden, 28, device="cuda")[0].contiguous()
    tu = make_text(1, 77, FULL.hidden, 29, device="cuda")[0].contiguous()
    x = x0.clone()
    model.denoise_step(x, tc, tu, 2048, 2048, 1, 10, 3.0, 5.0, [22], 0.01, 1.0)
    sig = o.sigma_schedule(10, 5.0)
    vc = model.forward(x0, tc[None], 2048, 2048, float(sig[1]), skip_layers=[[]]).clone()
    vu = model.forward(x0, tu[None], 2048, 2048, float(sig[1]), skip_layers=[[22]]).clone()
    ref = x0.clone()
    moss.cfg_euler_step(ref, vc[0].contiguous(), vu[0].contiguous(), 3.0, float(sig[1]), float(sig[2]))
    torch.cuda.synchronize()
    assert torch.equal(x, ref)
    assert torch.isfinite(x).all() and rel_l2(x.cpu().numpy(), x0.cpu().numpy()) > 1e-3
    model.close()
    assert_no_device_error()


def test_guided_step_fused_update_with_more_tiles_than_sms():
    """The fused update on a 2000 x 1936 image (125 x 121 = 15125 image tokens: 119 token tiles, the last
    partial, so 238 work units over at most 148 CTAs, each CTA taking several): tiny model, a 16-token
    prompt and a 3-token negative prompt; bit for bit against the two forwards and the standalone update."""
    h, w = 2000, 1936
    n_img = (h // 16) * (w // 16)
    model, wg, wn = make_model(TINY, 151, max_tokens=n_img + 16, max_latent_hw=(h // 8) * (w // 8))
    x0 = make_latent(h // 8, w // 8, 152).cuda()
    tc = make_text(1, 16, TINY.hidden, 153)[0].cuda()
    tu = make_text(1, 3, TINY.hidden, 154)[0].cuda()
    x = x0.clone()
    model.denoise_step(x, tc, tu, h, w, 2, 10, 3.0, 5.0, [1], 0.01, 1.0)
    sig = o.sigma_schedule(10, 5.0)
    vc = model.forward(x0, tc[None], h, w, float(sig[2]), skip_layers=[[]]).clone()
    vu = model.forward(x0, tu[None], h, w, float(sig[2]), skip_layers=[[1]]).clone()
    ref = x0.clone()
    moss.cfg_euler_step(ref, vc[0].contiguous(), vu[0].contiguous(), 3.0, float(sig[2]), float(sig[3]))
    torch.cuda.synchronize()
    assert torch.equal(x, ref)
    assert rel_l2(x.cpu().numpy(), x0.cpu().numpy()) > 1e-3
    model.close()
    assert_no_device_error()


@pytest.mark.parametrize("n_u", [5, 0])
def test_sample_tiny_short_negative_prompt(n_u):
    """Branches of different text lengths (n_u = 0: the empty negative prompt): the tiny
    4-step run against the oracle, which runs each branch on its own tokens."""
    model, wg, wn = make_model(TINY, 65, max_tokens=32, max_latent_hw=64, max_steps=4)
    tc = make_text(1, 16, TINY.hidden, 66)[0]
    tu = make_text(1, max(n_u, 1), TINY.hidden, 67)[0][:n_u].contiguous()
    out = model.sample(tc.cuda(), tu.cuda(), 64, 64, steps=4, cfg=3.0, shift=5.0, seed=3,
                       uncond_skip_layers=[1], slg_start=0.01, slg_stop=1.0)
    torch.cuda.synchronize()
    ref = o.sample(wn, TINY.heads, 64, 64, tc.double().numpy(), tu.double().numpy(), steps=4, cfg=3.0, shift=5.0,
                   seed=3, uncond_skip_layers=(1,), slg_start=0.01, slg_stop=1.0)
    assert psnr(ref, out.cpu().numpy()) >= 40.0
    model.close()
    assert_no_device_error()


def test_full_denoise_step_short_negative_prompt(full_model):
    """1024^2 step with a 512-token prompt and a 77-token negative prompt, packed back to back,
    equals the two branches run one at a time followed by the CFG + Euler update."""
    from synth import FULL
    model, w = full_model
    x0 = make_latent(128, 128, 21, device="cuda")
    tc = make_text(1, 512, FULL.hidden, 22, device="cuda")[0].contiguous()
    tu = make_text(1, 77, FULL.hidden, 23, device="cuda")[0].contiguous()
    x = x0.clone()
    model.denoise_step(x, tc, tu, 1024, 1024, 3, 50, 3.0, 5.0, [22], 0.01, 1.0)
    sig = o.sigma_schedule(50, 5.0)
    vc = model.forward(x0, tc[None], 1024, 1024, float(sig[3]), skip_layers=[[]]).clone()
    vu = model.forward(x0, tu[None], 1024, 1024, float(sig[3]), skip_layers=[[22]]).clone()
    ref = x0.clone()
    moss.cfg_euler_step(ref, vc[0].contiguous(), vu[0].contiguous(), 3.0, float(sig[3]), float(sig[4]))
    assert rel_l2(x.cpu().numpy(), ref.cpu().numpy()) <= 1e-6
    assert_no_device_error()


def test_full_accelerators(full_model):
    """1024^2, 2 steps of the full model: moss_sample_ex with the accelerators off equals
    moss_sample; CFG truncation at 0.5 equals a CFG step followed by a conditional-only step;
    the step cache with a huge threshold reuses the second step with a finite change."""
    from synth import FULL
    model, w = full_model
    tc = make_text(1, 512, FULL.hidden, 31, device="cuda")[0].contiguous()
    tu = make_text(1, 77, FULL.hidden, 32, device="cuda")[0].contiguous()
    kw = dict(steps=2, cfg=3.0, shift=5.0, seed=9, uncond_skip_layers=[22], slg_start=0.0, slg_stop=1.0)
    plain = model.sample(tc, tu, 1024, 1024, **kw).clone()
    off, cached, change = model.sample_accelerated(tc, tu, 1024, 1024, **kw)
    assert torch.equal(off, plain) and cached == [False, False]
    trunc, _, _ = model.sample_accelerated(tc, tu, 1024, 1024, cfg_truncation=0.5, **kw)
    x = torch.empty(128, 128, 32, device="cuda")
    moss.init_noise(x, 9)
    model.denoise_step(x, tc, tu, 1024, 1024, 0, 2, 3.0, 5.0, [22], 0.0, 1.0)
    model.denoise_step(x, tc, tu, 1024, 1024, 1, 2, 1.0, 5.0, [22], 0.0, 1.0)
    assert torch.equal(trunc, x)
    cache, cached, change = model.sample_accelerated(tc, tu, 1024, 1024, step_cache_threshold=1e9, **kw)
    torch.cuda.synchronize()
    assert cached == [False, True] and 0.0 < change[1] < 1.0
    assert torch.isfinite(cache).all() and not torch.equal(cache, plain)
    assert_no_device_error()


def test_full_three_pass_slg(full_model):
    """1024^2, one step from the seed's noise, three-pass SLG (reading R24) with a 77-token
    negative prompt: the packed three-branch call equals three single-branch forwards combined
    in FP32.  (One step only: a second step would feed the two results' last-ulp differences
    through the BF16 patch embedding, which magnifies them.)"""
    from synth import FULL
    model, w = full_model
    tc = make_text(1, 512, FULL.hidden, 41, device="cuda")[0].contiguous()
    tu = make_text(1, 77, FULL.hidden, 42, device="cuda")[0].contiguous()
    out, _, _ = model.sample_accelerated(tc, tu, 1024, 1024, steps=1, cfg=3.0, shift=5.0, seed=11,
                                         uncond_skip_layers=[22], slg_start=0.0, slg_stop=1.0, slg_scale=2.0)
    x = torch.empty(128, 128, 32, device="cuda")
    moss.init_noise(x, 11)
    sig = o.sigma_schedule(1, 5.0)
    t = float(sig[0])
    vc = model.forward(x, tc[None], 1024, 1024, t, skip_layers=[[]]).clone()[0]
    vcs = model.forward(x, tc[None], 1024, 1024, t, skip_layers=[[22]]).clone()[0]
    vu = model.forward(x, tu[None], 1024, 1024, t, skip_layers=[[22]]).clone()[0]
    v = vu + 3.0 * (vc - vu) + 2.0 * (vc - vcs)
    ref = x + (float(np.float32(sig[1])) - float(np.float32(sig[0]))) * v
    torch.cuda.synchronize()
    assert rel_l2(out.cpu().numpy(), ref.cpu().numpy()) <= 1e-6
    assert rel_l2(out.cpu().numpy(), x.cpu().numpy()) > 1e-2      # the step moved the latent
    assert_no_device_error()


@pytest.mark.parametrize("h,w", [(64, 128), (128, 48), (48, 80)])
def test_forward_tiny_non_square_matches_oracle(h, w):
    """Non-square images: the patch grid's rows and columns enter the RoPE positions, the patch
    order and the unpatchify differently, so a transposed index shows up here."""
    gh, gw = h // 16, w // 16
    model, wg, wn = make_model(TINY, 131, max_tokens=gh * gw + 16, max_latent_hw=(h // 8) * (w // 8))
    lat = make_latent(h // 8, w // 8, 132)
    txt = make_text(2, 16, TINY.hidden, 133)
    v = model.forward(lat.cuda(), txt.cuda(), h, w, 0.6, skip_layers=[[], [1]])
    torch.cuda.synchronize()
    ref = o.dit_forward(lat.numpy(), txt.double().numpy(), 0.6, [(), (1,)], wn, TINY.heads)
    for b in range(2):
        assert rel_l2(v.cpu().numpy()[b], ref[b]) <= 1e-2
    model.close()
    assert_no_device_error()


def test_sample_tiny_non_square_psnr():
    model, wg, wn = make_model(TINY, 141, max_tokens=4 * 8 + 16, max_latent_hw=8 * 16, max_steps=4)
    tc = make_text(1, 16, TINY.hidden, 142)[0]
    tu = make_text(1, 16, TINY.hidden, 143)[0]
    out = model.sample(tc.cuda(), tu.cuda(), 64, 128, steps=4, cfg=3.0, shift=5.0, seed=2, uncond_skip_layers=[1])
    torch.cuda.synchronize()
    ref = o.sample(wn, TINY.heads, 64, 128, tc.double().numpy(), tu.double().numpy(), steps=4, cfg=3.0, shift=5.0,
                   seed=2, uncond_skip_layers=(1,))
    assert psnr(ref, out.cpu().numpy()) >= 40.0
    model.close()
    assert_no_device_error()


# ---------------------------------------------------------------------------- full depth and width
# Each block meets the per-block bar (relative L2 <= 1e-2 on output and update) on its own; the tests
# below check that stacking all 42 of them keeps the velocity within the same 1e-2 per branch and the
# sampled latent within 40 dB of the float64 oracle.  The GPU rounds the activations that feed each
# GEMM (LN-modulate output, Q/K/V, attention output, SwiGLU product) to BF16, a relative error of at
# most 2^-9 per element; these roundings are independent from block to block, so their effect on
# the stream adds up like a random walk over the blocks rather than compounding, and the final
# LayerNorm of the output layer removes the stream's scale.

def test_full_depth_forward_matches_oracle(full_model, capsys):
    """42 blocks at hidden 3072 (24x128 heads, FFN 8192; windpaint.ai, Architecture and specs) on a
    256^2 image: 256 image + 128 text tokens per branch, CFG batch 2, the unconditional branch
    skipping layer 22, against oracle.dit_forward."""
    from synth import FULL
    model, w = full_model
    lat = make_latent(32, 32, 15, device="cuda")
    txt = make_text(2, 128, FULL.hidden, 16, device="cuda")
    t = 0.8
    v = model.forward(lat, txt, 256, 256, t, skip_layers=[[], [22]])
    torch.cuda.synchronize()
    got = v.cpu().double().numpy()
    ref = o.dit_forward(lat.cpu().numpy(), txt.cpu().double().numpy(), t, [(), (22,)], lazy_numpy_weights(w),
                        FULL.heads)
    errs = [rel_l2(got[b], ref[b]) for b in range(2)]
    with capsys.disabled():
        print(f"\nfull-depth forward 256^2: velocity rel L2 cond {errs[0]:.3e} uncond {errs[1]:.3e}")
    assert max(errs) <= 1e-2, errs
    assert rel_l2(ref[0], ref[1]) > 1e-2        # the two branches really differ
    assert_no_device_error()


def test_full_depth_two_step_sample_matches_oracle(full_model, capsys):
    """moss_sample with the full model on a 256^2 image, 2 steps of the shift-5 schedule at CFG 3 with
    128-token prompts, seed 42: step 0 runs full CFG and step 1 skips layer 22 in the unconditional
    branch (slg window [0.01, 1.0]); against oracle.sample at >= 40 dB."""
    from synth import FULL
    model, w = full_model
    tc = make_text(1, 128, FULL.hidden, 17, device="cuda")[0].contiguous()
    tu = make_text(1, 128, FULL.hidden, 18, device="cuda")[0].contiguous()
    out = model.sample(tc, tu, 256, 256, steps=2, cfg=3.0, shift=5.0, seed=42, uncond_skip_layers=[22],
                       slg_start=0.01, slg_stop=1.0)
    torch.cuda.synchronize()
    ref = o.sample(lazy_numpy_weights(w), FULL.heads, 256, 256, tc.cpu().double().numpy(), tu.cpu().double().numpy(),
                   steps=2, cfg=3.0, shift=5.0, seed=42, uncond_skip_layers=(22,), slg_start=0.01, slg_stop=1.0)
    p = psnr(ref, out.cpu().numpy())
    x0 = o.gaussian_noise(32 * 32 * 32, 42).reshape(32, 32, 32)
    with capsys.disabled():
        print(f"\nfull-depth 2-step sample 256^2: PSNR {p:.2f} dB, latent rel L2 {rel_l2(out.cpu().numpy(), ref):.3e}")
    assert p >= 40.0, p
    assert rel_l2(ref, x0) > 1e-2                 # the steps moved the latent
    assert_no_device_error()


def test_full_width_1024_first_two_layers_match_oracle(full_model, capsys):
    """The 1024^2 workload's own shape (4096 image + 512 text tokens per branch, CFG batch 2) through
    layers 0 and 1 with layers 2..41 skipped on both branches, against oracle.dit_forward."""
    from synth import FULL
    model, w = full_model
    lat = make_latent(128, 128, 19, device="cuda")
    txt = make_text(2, 512, FULL.hidden, 20, device="cuda")
    skip = list(range(2, FULL.layers))
    v = model.forward(lat, txt, 1024, 1024, 0.35, skip_layers=[skip, skip])
    torch.cuda.synchronize()
    got = v.cpu().double().numpy()
    ref = o.dit_forward(lat.cpu().numpy(), txt.cpu().double().numpy(), 0.35, [tuple(skip), tuple(skip)],
                        lazy_numpy_weights(w), FULL.heads)
    errs = [rel_l2(got[b], ref[b]) for b in range(2)]
    with capsys.disabled():
        print(f"\n1024^2 two-layer forward: velocity rel L2 cond {errs[0]:.3e} uncond {errs[1]:.3e}")
    assert max(errs) <= 1e-2, errs
    assert_no_device_error()
