"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to what the pages print, to a closed form, to an
invariant, or to an independent library routine (torch / einops / scipy, which the
oracle itself never calls), so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails here.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn
from einops import rearrange
from scipy import stats

from oracle import moss_oracle as o
from synth import FULL, TINY, make_weights, numpy_weights

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FACTS = json.load(open(os.path.join(GOLD, "pages_facts.json")))


# ---------------------------------------------------------------- noise generator
def test_philox_known_answers():
    kat = json.load(open(os.path.join(GOLD, "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        ctr = np.array([int(x, 16) for x in v["ctr"]], dtype=np.uint64).reshape(4, 1)
        key = [int(x, 16) for x in v["key"]]
        out = o.philox4x32_10(ctr, key)[:, 0]
        assert [int(x) for x in out] == [int(x, 16) for x in v["out"]]


def test_uniform23_open_interval_and_exact():
    bits = np.array([0, 511, 512, 0xFFFFFFFF], dtype=np.uint32)
    u = o.uniform23(bits)
    assert u[0] == 0.5 / 2**23 and u[1] == u[0]
    assert u[2] == 1.5 / 2**23
    assert u[3] == (2**23 - 0.5) / 2**23 < 1.0
    assert np.all(u.astype(np.float32).astype(np.float64) == u)  # exact in FP32


def test_gaussian_noise_is_standard_normal():
    z = o.gaussian_noise(1 << 20, seed=42).astype(np.float64)
    assert z.dtype == np.float64 and z.shape == (1 << 20,)
    assert abs(z.mean()) < 5.0 / math.sqrt(z.size)
    assert abs(z.var() - 1.0) < 5.0 * math.sqrt(2.0 / z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-4
    # the four outputs of a block are not correlated with each other
    blocks = z.reshape(-1, 4)
    c = np.corrcoef(blocks.T)
    assert np.all(np.abs(c - np.eye(4)) < 0.01)


def test_gaussian_noise_box_muller_radius():
    # z_{4g}^2 + z_{4g+1}^2 = -2 ln u_a with u_a from the first Philox word
    n = 4096
    z = o.gaussian_noise(n, seed=7).astype(np.float64).reshape(-1, 4)
    g = np.arange(n // 4, dtype=np.uint64)
    ctr = np.stack([g, np.zeros_like(g), np.zeros_like(g), np.zeros_like(g)])
    x = o.philox4x32_10(ctr, (7, 0))
    r2 = -2.0 * np.log(o.uniform23(x[0]))
    np.testing.assert_allclose(z[:, 0] ** 2 + z[:, 1] ** 2, r2, rtol=1e-5, atol=1e-6)


def test_noise_depends_on_seed_high_word():
    a = o.gaussian_noise(64, seed=5)
    b = o.gaussian_noise(64, seed=5 + (1 << 32))
    assert not np.array_equal(a, b)


# ---------------------------------------------------------------- schedule, window, CFG, Euler
def test_sigma_schedule_closed_forms():
    s = o.sigma_schedule(50, 5.0)
    assert s.dtype == np.float32 and s.shape == (51,)
    assert s[0] == 1.0 and s[-1] == 0.0
    assert np.all(np.diff(s) < 0)
    assert abs(float(s[25]) - 5.0 * 0.5 / (1 + 4 * 0.5)) < 1e-7           # s = 1/2 -> 5/6
    assert abs(float(s[1]) - 4.9 / 4.92) < 1e-7                           # s = 0.98
    lin = o.sigma_schedule(10, 1.0)                                        # shift 1 = no shift
    np.testing.assert_array_equal(lin, (1.0 - np.arange(11) / 10).astype(np.float32))


def test_shift_moves_time_toward_noise():
    # shift > 1 keeps sigma above the unshifted value at every interior step
    s5, s1 = o.sigma_schedule(50, 5.0), o.sigma_schedule(50, 1.0)
    assert np.all(s5[1:-1] > s1[1:-1])


def test_slg_window_matches_pages():
    d = FACTS["defaults"]
    act = [o.slg_active(i, d["steps"], d["slg_start"], d["slg_stop"]) for i in range(d["steps"])]
    assert act[0] is False                                                # first step full CFG
    assert all(act[1:])
    act0 = [o.slg_active(i, 50, 0.0, 1.0) for i in range(50)]
    assert all(act0)                                                      # start at zero
    # a window that closes early
    act_half = [o.slg_active(i, 50, 0.01, 0.5) for i in range(50)]
    assert act_half.index(False, 1) == 26


def test_cfg_euler_closed_forms():
    x = np.float32([0.0, 1.0, -2.0])
    vc = np.float32([2.0, 0.5, 1.0])
    vu = np.float32([1.0, 0.5, 3.0])
    out = o.cfg_euler(x, vc, vu, 3.0, 1.0, 0.5)
    # v = vu + 3 (vc - vu) = [4, 0.5, -3]; dt = -0.5
    np.testing.assert_array_equal(out, np.float32([-2.0, 0.75, -0.5]))
    # cfg = 1 -> conditional velocity; v_c = v_u -> that velocity
    np.testing.assert_array_equal(o.cfg_combine(vc, vu, 1.0), vc)
    np.testing.assert_array_equal(o.cfg_combine(vc, vc, 3.0), vc)
    assert o.cfg_euler(x, vc, vu, 3.0, 1.0, 0.5).dtype == np.float32


def test_constant_velocity_euler_reaches_x0_minus_v():
    sig = o.sigma_schedule(50, 5.0)
    x = np.float32([0.3, -1.0, 2.0])
    v = np.float32([1.0, -0.5, 0.25])
    for i in range(50):
        x = o.cfg_euler(x, v, v, 3.0, sig[i], sig[i + 1])
    np.testing.assert_allclose(x, np.float32([0.3, -1.0, 2.0]) - v, atol=2e-6)


# ---------------------------------------------------------------- request validation, sizes
def test_size_rule():
    r = FACTS["size_rule"]
    assert o.validate_size(1024, 1024) == (True, "")
    assert o.validate_size(2048, 2048)[0]                                 # 4.19 MP
    for h, w in [(1000, 1024), (0, 1024), (-16, 64), (1024, 8)]:
        ok, msg = o.validate_size(h, w)
        assert not ok and msg == r["message"]
    assert not o.validate_size(4112, 512)[0]                              # side > 4096
    assert not o.validate_size(4096, 2048)[0]                             # 8.4 MP
    assert o.validate_size(4096, 1024)[0]                                 # 4.19 MP


def test_image_token_count():
    assert o.image_tokens(1024, 1024) == FACTS["image_tokens_1024"]["value"]
    assert o.image_tokens(2048, 2048) == 16384
    assert o.image_tokens(64, 64) == 16
    assert o.patchify(np.zeros((128, 128, 32))).shape == (4096, 128)


def test_architecture_size_matches_pages():
    a = FACTS["architecture"]
    assert (FULL.layers, FULL.hidden, FULL.heads, FULL.head_dim, FULL.ffn) == (
        a["layers"], a["hidden"], a["heads"], a["head_dim"], a["ffn"])
    assert FULL.heads * FULL.head_dim == FULL.hidden
    D, F, L, C = FULL.hidden, FULL.ffn, FULL.layers, FULL.c_t
    per_layer = 3 * D * D + D * D + 3 * D * F + 6 * D * C + 6 * D + 2 * FULL.head_dim
    glob = C * 256 + C + C * C + C + D * 128 + D + 2 * D * C + 2 * D + 128 * D + 128
    n = L * per_layer + glob
    f = FACTS["dit_params_billion"]
    assert abs(n / 1e9 - f["value"]) / f["value"] < f["rel_tol"]
    g = FACTS["dit_bf16_gb"]
    assert abs(2 * n / 1e9 - g["value"]) / g["value"] < g["rel_tol"]
    q = FACTS["q_projections_gib"]                                        # Wq is D x D
    assert abs(L * D * D * 2 / 2**30 - q["value"]) < q["abs_tol"]


# ---------------------------------------------------------------- patches
def test_patchify_matches_einops_and_roundtrips():
    rng = np.random.default_rng(0)
    lat = rng.standard_normal((8, 12, 32))
    ref = rearrange(lat, "(h p1) (w p2) c -> (h w) (p1 p2 c)", p1=2, p2=2)
    np.testing.assert_array_equal(o.patchify(lat), ref)
    np.testing.assert_array_equal(o.unpatchify(o.patchify(lat), 8, 12), lat)


# ---------------------------------------------------------------- conditioning
def test_timestep_embedding_closed_form():
    e0 = o.timestep_embedding(0.0)
    np.testing.assert_array_equal(e0, np.concatenate([np.ones(128), np.zeros(128)]))
    e = o.timestep_embedding(0.25)
    assert abs(e[0] - math.cos(250.0)) < 1e-12 and abs(e[128] - math.sin(250.0)) < 1e-12
    # last frequency is 1e4^(-127/128)
    f = 10000.0 ** (-127 / 128)
    assert abs(e[127] - math.cos(250.0 * f)) < 1e-12
    np.testing.assert_allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-12)


def test_silu_matches_torch():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(o.silu(x), Fnn.silu(torch.from_numpy(x)).numpy(), rtol=1e-13, atol=1e-15)


def test_conditioning_and_modulation_shapes_and_linearity():
    w = numpy_weights(make_weights(TINY, 3))
    c = o.conditioning(0.5, w)
    assert c.shape == (TINY.c_t,)
    m = o.block_modulation(c, w["mod_w"][0], w["mod_b"][0])
    assert m.shape == (6 * TINY.hidden,)
    # zero modulation weights leave only the bias
    np.testing.assert_array_equal(o.block_modulation(c, np.zeros_like(w["mod_w"][0]), w["mod_b"][0]),
                                  w["mod_b"][0])


def _T(a):
    return torch.from_numpy(np.ascontiguousarray(a))


def test_conditioning_matches_torch_composition():
    """The time MLP (InvokeAI MOSS-Image guide, Transformer formats: time-embedding layers; reading
    R7) as nn.Linear -> SiLU -> nn.Linear on nonzero random weights.  A dropped SiLU, a transposed
    W1 or W2 (W2 is square, so only the values tell) or a missing bias fails here."""
    w = numpy_weights(make_weights(TINY, 21))
    for t in (0.0, 0.37, 0.9):
        emb = _T(o.timestep_embedding(t))
        ref = Fnn.linear(Fnn.silu(Fnn.linear(emb, _T(w["t_w1"]), _T(w["t_b1"]))), _T(w["t_w2"]), _T(w["t_b2"]))
        got = o.conditioning(t, w)
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-15)
    # the same MLP with W2 transposed is a different function on these weights
    wt = dict(w, t_w2=w["t_w2"].T.copy())
    assert np.abs(o.conditioning(0.37, wt) - o.conditioning(0.37, w)).max() > 1e-3


def test_conditioning_closed_form_at_t0():
    """At t = 0 the sinusoid is [1]*128 + [0]*128, so with W2 = I and b2 = 0 the MLP is
    SiLU(sum of W1's first 128 columns + b1), written with scipy's logistic function."""
    from scipy.special import expit
    w = numpy_weights(make_weights(TINY, 22))
    C = TINY.c_t
    w2 = dict(w, t_w2=np.eye(C), t_b2=np.zeros(C))
    h1 = w["t_w1"][:, :128].sum(axis=1) + w["t_b1"]
    np.testing.assert_allclose(o.conditioning(0.0, w2), h1 * expit(h1), rtol=1e-12, atol=1e-15)


def test_block_modulation_matches_torch_composition():
    """W_mod SiLU(c) + b_mod (reading R7) against nn.Linear(SiLU(c)); then the SiLU is located by its
    limits: c -> -inf switches the weights off (only b remains), c -> +inf passes c through."""
    w = numpy_weights(make_weights(TINY, 23))
    c = o.conditioning(0.61, w)
    for l in range(TINY.layers):
        ref = Fnn.linear(Fnn.silu(_T(c)), _T(w["mod_w"][l]), _T(w["mod_b"][l])).numpy()
        np.testing.assert_allclose(o.block_modulation(c, w["mod_w"][l], w["mod_b"][l]), ref, rtol=1e-12, atol=1e-15)
    W, b = w["mod_w"][0], w["mod_b"][0]
    neg = np.full(TINY.c_t, -60.0)
    np.testing.assert_allclose(o.block_modulation(neg, W, b), b, rtol=0, atol=1e-20)
    pos = np.full(TINY.c_t, 60.0)
    np.testing.assert_allclose(o.block_modulation(pos, W, b), 60.0 * W.sum(axis=1) + b, rtol=1e-12, atol=1e-12)


def test_final_layer_matches_torch_composition():
    """The output layers (InvokeAI guide, Transformer formats; reading R7): [shift_f, scale_f] =
    Linear(SiLU(c)), then LayerNorm(x) (1 + scale_f) + shift_f, then Linear(out_w, out_b)."""
    w = numpy_weights(make_weights(TINY, 24))
    rng = np.random.default_rng(24)
    D = TINY.hidden
    x = rng.standard_normal((16, D)) * 2 + 0.5
    c = o.conditioning(0.44, w)
    sh, sc = Fnn.linear(Fnn.silu(_T(c)), _T(w["final_mod_w"]), _T(w["final_mod_b"])).chunk(2)
    y = Fnn.layer_norm(_T(x), (D,), eps=1e-6) * (1 + sc) + sh
    ref = Fnn.linear(y, _T(w["out_w"]), _T(w["out_b"])).numpy()
    got = o.final_layer(x, c, w)
    assert got.shape == (16, 128)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-13)
    # shift and scale swapped is a different function on these weights
    y_sw = Fnn.layer_norm(_T(x), (D,), eps=1e-6) * (1 + sh) + sc
    ref_sw = Fnn.linear(y_sw, _T(w["out_w"]), _T(w["out_b"])).numpy()
    assert np.abs(got - ref_sw).max() > 1e-3


def test_final_layer_scale_minus_one_leaves_the_shift():
    """With zero modulation weights and bias [shift, -1], the normalised input drops out: every
    row's output is shift . out_w^T + out_b, whatever x is."""
    w = numpy_weights(make_weights(TINY, 25))
    D = TINY.hidden
    rng = np.random.default_rng(25)
    shift = rng.standard_normal(D)
    wz = dict(w, final_mod_w=np.zeros_like(w["final_mod_w"]), final_mod_b=np.concatenate([shift, -np.ones(D)]))
    x = rng.standard_normal((8, D)) * 3
    want = shift @ w["out_w"].T + w["out_b"]
    np.testing.assert_allclose(o.final_layer(x, rng.standard_normal(TINY.c_t), wz), np.broadcast_to(want, (8, 128)),
                               rtol=1e-12, atol=1e-12)


def _torch_forward_skip_all(lat, c, w, gh, gw):
    """Patch embedding -> final layer -> unpatchify with einops and torch.nn.functional."""
    D = w["img_w"].shape[0]
    tok = rearrange(_T(lat), "(h p1) (w p2) c -> (h w) (p1 p2 c)", p1=2, p2=2)
    img = Fnn.linear(tok, _T(w["img_w"]), _T(w["img_b"]))
    sh, sc = Fnn.linear(Fnn.silu(_T(c)), _T(w["final_mod_w"]), _T(w["final_mod_b"])).chunk(2)
    y = Fnn.layer_norm(img, (D,), eps=1e-6) * (1 + sc) + sh
    v = Fnn.linear(y, _T(w["out_w"]), _T(w["out_b"]))
    return rearrange(v, "(h w) (p1 p2 c) -> (h p1) (w p2) c", h=gh, w=gw, p1=2, p2=2).numpy()


def test_patch_embed_line_matches_torch_composition():
    """The image embedding of the forward (2x2 patches of the 32-channel latent, windpaint.ai
    Architecture and specs; reading R10): with every layer skipped, the forward is patch embed ->
    final layer -> unpatchify, here rebuilt from einops and nn.functional on a non-square latent."""
    w = numpy_weights(make_weights(TINY, 26))
    rng = np.random.default_rng(26)
    lat = rng.standard_normal((8, 12, 32)).astype(np.float32)
    txt = rng.standard_normal((2, 5, TINY.hidden))
    v = o.dit_forward(lat, txt, 0.52, [(0, 1), (0, 1)], w, TINY.heads)
    ref = _torch_forward_skip_all(lat.astype(np.float64), o.conditioning(0.52, w), w, 4, 6)
    np.testing.assert_allclose(v[0], ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(v[1], ref, rtol=1e-11, atol=1e-13)


def test_patch_embed_is_local_to_its_patch():
    """With every layer skipped, tokens do not interact: changing the latent inside the 2x2 patch of
    token (r, c) changes the velocity in exactly that patch and nowhere else."""
    w = numpy_weights(make_weights(TINY, 27))
    rng = np.random.default_rng(27)
    lat = rng.standard_normal((8, 12, 32)).astype(np.float32)
    txt = rng.standard_normal((1, 3, TINY.hidden))
    base = o.dit_forward(lat, txt, 0.3, [(0, 1)], w, TINY.heads)[0]
    r, c = 2, 5
    lat2 = lat.copy()
    lat2[2 * r + 1, 2 * c, 7] += 3.0
    moved = np.abs(o.dit_forward(lat2, txt, 0.3, [(0, 1)], w, TINY.heads)[0] - base).max(axis=-1) > 0
    want = np.zeros((8, 12), dtype=bool)
    want[2 * r:2 * r + 2, 2 * c:2 * c + 2] = True
    np.testing.assert_array_equal(moved, want)


def test_forward_matches_torch_composition():
    """The whole forward on both branches (one with layer 1 skipped) rebuilt from the torch block
    composition below, the torch patch embedding and the torch final layer."""
    w = numpy_weights(make_weights(TINY, 28))
    rng = np.random.default_rng(28)
    lat = rng.standard_normal((8, 8, 32)).astype(np.float32)
    txt = rng.standard_normal((2, 6, TINY.hidden))
    t = 0.71
    v = o.dit_forward(lat, txt, t, [(), (1,)], w, TINY.heads)
    c = _T(o.conditioning(t, w))
    ang = o.rope_angles(o.token_positions(4, 4, 6))
    tok = rearrange(_T(lat.astype(np.float64)), "(h p1) (w p2) c -> (h w) (p1 p2 c)", p1=2, p2=2)
    img = Fnn.linear(tok, _T(w["img_w"]), _T(w["img_b"])).numpy()
    for b, skip in enumerate([(), (1,)]):
        x = np.concatenate([img, txt[b]])
        for l in range(TINY.layers):
            if l in skip:
                continue
            mod = Fnn.linear(Fnn.silu(c), _T(w["mod_w"][l]), _T(w["mod_b"][l])).numpy()
            x = _torch_block(x, o.layer_weights(w, l), mod, ang, TINY.heads)
        sh, sc = Fnn.linear(Fnn.silu(c), _T(w["final_mod_w"]), _T(w["final_mod_b"])).chunk(2)
        y = Fnn.layer_norm(_T(x[:16]), (TINY.hidden,), eps=1e-6) * (1 + sc) + sh
        vt = Fnn.linear(y, _T(w["out_w"]), _T(w["out_b"]))
        ref = rearrange(vt, "(h w) (p1 p2 c) -> (h p1) (w p2) c", h=4, w=4, p1=2, p2=2).numpy()
        np.testing.assert_allclose(v[b], ref, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- normalisation
def test_layer_norm_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 96)) * 3 + 1
    ref = Fnn.layer_norm(torch.from_numpy(x), (96,), eps=1e-6).numpy()
    np.testing.assert_allclose(o.layer_norm(x), ref, rtol=1e-12, atol=1e-12)
    shift, scale = rng.standard_normal(96), rng.standard_normal(96)
    np.testing.assert_allclose(o.ln_modulate(x, shift, scale), ref * (1 + scale) + shift, rtol=1e-12, atol=1e-12)
    y = o.ln_modulate(x, np.zeros(96), np.zeros(96))
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(-1), 1, atol=1e-5)
    # scale = -1 removes the normalised input: only the shift is left
    np.testing.assert_allclose(o.ln_modulate(x, shift, -np.ones(96)), np.broadcast_to(shift, x.shape), atol=1e-12)


def test_rms_norm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 7, 128))
    g = 1 + 0.1 * rng.standard_normal(128)
    ref = Fnn.rms_norm(torch.from_numpy(x), (128,), weight=torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(o.rms_norm(x, g), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- RoPE
def test_rope_matches_complex_multiplication():
    rng = np.random.default_rng(3)
    pos = o.token_positions(3, 5, 4)
    ang = o.rope_angles(pos)
    x = rng.standard_normal((2, pos.shape[0], 128))
    xc = torch.view_as_complex(torch.from_numpy(x.copy()).reshape(2, -1, 64, 2))
    rot = torch.polar(torch.ones_like(torch.from_numpy(ang)), torch.from_numpy(ang))
    ref = torch.view_as_real(xc * rot).reshape(2, -1, 128).numpy()
    np.testing.assert_allclose(o.apply_rope(x, ang), ref, rtol=1e-12, atol=1e-12)


def test_rope_axes_and_frequencies():
    pos = np.array([[0, 0, 0], [0, 3, 0], [0, 0, 5], [7, 0, 0]])
    ang = o.rope_angles(pos)
    assert np.all(ang[0] == 0)
    # row axis: pairs 16..39, first frequency 1
    assert np.all(ang[1, :16] == 0) and np.all(ang[1, 40:] == 0) and ang[1, 16] == 3.0
    assert abs(ang[1, 17] - 3.0 * 10000 ** (-2 / 48)) < 1e-12
    # column axis: pairs 40..63
    assert np.all(ang[2, :40] == 0) and ang[2, 40] == 5.0
    # text axis: pairs 0..15, frequency 1e4^(-2i/32)
    assert np.all(ang[3, 16:] == 0) and ang[3, 0] == 7.0
    assert abs(ang[3, 15] - 7.0 * 10000 ** (-30 / 32)) < 1e-12
    # positions: image (r, c) -> (0, r, c); text j -> (j+1, 0, 0)
    p = o.token_positions(2, 3, 2)
    np.testing.assert_array_equal(p, [[0, 0, 0], [0, 0, 1], [0, 0, 2], [0, 1, 0], [0, 1, 1], [0, 1, 2],
                                      [1, 0, 0], [2, 0, 0]])


def test_rope_preserves_norm_and_is_relative():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    p1, p2 = np.array([[2, 5, 7]]), np.array([[9, 1, 4]])
    d = np.array([[3, 11, 6]])
    qa = o.apply_rope(q[None], o.rope_angles(p1))[0]
    ka = o.apply_rope(k[None], o.rope_angles(p2))[0]
    qb = o.apply_rope(q[None], o.rope_angles(p1 + d))[0]
    kb = o.apply_rope(k[None], o.rope_angles(p2 + d))[0]
    assert abs(np.linalg.norm(qa) - np.linalg.norm(q)) < 1e-12
    assert abs(qa @ ka - qb @ kb) < 1e-10


# ---------------------------------------------------------------- attention
def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((3, 40, 128)) for _ in range(3))
    ref = Fnn.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(o.attention(q, k, v), ref, rtol=1e-11, atol=1e-12)


def test_attention_invariants():
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((1, 16, 128)) for _ in range(3))
    perm = rng.permutation(16)
    out = o.attention(q, k, v)
    np.testing.assert_allclose(o.attention(q, k[:, perm], v[:, perm]), out, atol=1e-12)      # keys as a set
    np.testing.assert_allclose(o.attention(q[:, perm], k, v), out[:, perm], atol=1e-12)      # queries equivariant
    np.testing.assert_allclose(o.attention(np.zeros_like(q), k, v)[0], np.broadcast_to(v[0].mean(0), (16, 128)),
                               atol=1e-12)                                                   # uniform weights
    big = k.copy()
    big[0, 3] = 1e3 * q[0, 0]
    assert np.allclose(o.attention(q[:, :1], big, v)[0, 0], v[0, 3])                         # one dominant key


# ---------------------------------------------------------------- block structure
def _tiny_setup(seed=11, n_img_hw=(4, 4), n_txt=16):
    w = numpy_weights(make_weights(TINY, seed))
    gh, gw = n_img_hw
    ang = o.rope_angles(o.token_positions(gh, gw, n_txt))
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((gh * gw + n_txt, TINY.hidden))
    c = o.conditioning(0.5, w)
    mod = o.block_modulation(c, w["mod_w"][0], w["mod_b"][0])
    return w, ang, x, mod


def _torch_block(x, lw, mod, ang, heads):
    """The same block written with torch library primitives: layer_norm, rms_norm,
    scaled_dot_product_attention, complex-multiplication RoPE and silu."""
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    x, mod = T(x), T(mod)
    n, D = x.shape
    sh1, sc1, g1, sh2, sc2, g2 = mod.chunk(6)
    h = Fnn.layer_norm(x, (D,), eps=1e-6) * (1 + sc1) + sh1
    qkv = Fnn.linear(h, T(lw["wqkv"]))
    q, k, v = (t.reshape(n, heads, 128).transpose(0, 1) for t in qkv.chunk(3, dim=1))
    rot = torch.polar(torch.ones_like(T(ang)), T(ang))

    def rope(t):
        return torch.view_as_real(torch.view_as_complex(t.reshape(heads, n, 64, 2).contiguous()) * rot).reshape(heads, n, 128)

    q = rope(Fnn.rms_norm(q, (128,), weight=T(lw["q_gain"]), eps=1e-6))
    k = rope(Fnn.rms_norm(k, (128,), weight=T(lw["k_gain"]), eps=1e-6))
    o_ = Fnn.scaled_dot_product_attention(q, k, v).transpose(0, 1).reshape(n, D)
    x = x + g1 * Fnn.linear(o_, T(lw["wo"]))
    h2 = Fnn.layer_norm(x, (D,), eps=1e-6) * (1 + sc2) + sh2
    x = x + g2 * Fnn.linear(Fnn.silu(Fnn.linear(h2, T(lw["wg"]))) * Fnn.linear(h2, T(lw["wu"])), T(lw["wd"]))
    return x.numpy()


def test_block_matches_library_composition():
    w, ang, x, mod = _tiny_setup()
    lw = o.layer_weights(w, 0)
    y = o.block_forward(x, lw, mod, ang, TINY.heads)
    ref = _torch_block(x, lw, mod, ang, TINY.heads)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)
    assert np.abs(y - x).max() > 1e-3            # the block does change the stream


def test_block_gates_zero_is_identity():
    w, ang, x, mod = _tiny_setup()
    D = TINY.hidden
    m = mod.copy()
    m[2 * D:3 * D] = 0.0
    m[5 * D:6 * D] = 0.0
    np.testing.assert_array_equal(o.block_forward(x, o.layer_weights(w, 0), m, ang, TINY.heads), x)


def test_block_branches_are_separable():
    # gate2 = 0 leaves only the attention branch: the update is gate1 * (attn_out Wo^T)
    w, ang, x, mod = _tiny_setup()
    D = TINY.hidden
    lw = o.layer_weights(w, 0)
    m = mod.copy()
    m[5 * D:] = 0.0
    y = o.block_forward(x, lw, m, ang, TINY.heads)
    lw0 = dict(lw, wo=np.zeros_like(lw["wo"]))
    np.testing.assert_array_equal(o.block_forward(x, lw0, m, ang, TINY.heads), x)
    # the attention update is linear in Wo
    lw2 = dict(lw, wo=2 * lw["wo"])
    np.testing.assert_allclose(o.block_forward(x, lw2, m, ang, TINY.heads) - x, 2 * (y - x), rtol=1e-12, atol=1e-14)


def test_ffn_is_swiglu():
    # with Wu = 0 the FFN contributes nothing; the gate path is SiLU, not GELU/ReLU
    w, ang, x, mod = _tiny_setup()
    D = TINY.hidden
    lw = o.layer_weights(w, 0)
    m = mod.copy()
    m[2 * D:3 * D] = 0.0           # attention branch off
    lw0 = dict(lw, wu=np.zeros_like(lw["wu"]))
    np.testing.assert_array_equal(o.block_forward(x, lw0, m, ang, TINY.heads), x)


# ---------------------------------------------------------------- forward and sampler
def test_forward_skip_is_identity_on_the_stream():
    w = numpy_weights(make_weights(TINY, 12))
    rng = np.random.default_rng(12)
    lat = rng.standard_normal((8, 8, 32)).astype(np.float32)
    txt = rng.standard_normal((2, 16, TINY.hidden))
    v = o.dit_forward(lat, txt, 0.3, [(), (1,)], w, TINY.heads)
    # branch 1 with layer 1 skipped == one block then the final layer, composed by hand
    ang = o.rope_angles(o.token_positions(4, 4, 16))
    c = o.conditioning(0.3, w)
    x = np.concatenate([o.patchify(lat.astype(np.float64)) @ w["img_w"].T + w["img_b"], txt[1]])
    x = o.block_forward(x, o.layer_weights(w, 0), o.block_modulation(c, w["mod_w"][0], w["mod_b"][0]), ang, TINY.heads)
    ref1 = o.unpatchify(o.final_layer(x[:16], c, w), 8, 8)
    np.testing.assert_array_equal(v[1], ref1)
    # skipping every layer: the image velocity no longer sees the text
    v_all = o.dit_forward(lat, txt, 0.3, [(0, 1), (0, 1)], w, TINY.heads)
    np.testing.assert_array_equal(v_all[0], v_all[1])
    assert not np.allclose(v[0], v[1])


def test_forward_output_shape_and_branch_independence():
    w = numpy_weights(make_weights(TINY, 13))
    rng = np.random.default_rng(13)
    lat = rng.standard_normal((8, 8, 32)).astype(np.float32)
    txt = rng.standard_normal((2, 16, TINY.hidden))
    v = o.dit_forward(lat, txt, 0.7, [(), ()], w, TINY.heads)
    assert v.shape == (2, 8, 8, 32)
    v0 = o.dit_forward(lat, txt[:1], 0.7, [()], w, TINY.heads)
    np.testing.assert_array_equal(v[0], v0[0])


def _constant_velocity_weights(vel):
    w = numpy_weights(make_weights(TINY, 14))
    for k in w:
        w[k] = np.zeros_like(w[k])
    w["q_gain"][:] = 1.0
    w["k_gain"][:] = 1.0
    w["out_b"] = vel.copy()
    return w


def test_sampler_constant_velocity():
    vel = np.linspace(-1, 1, 128)
    w = _constant_velocity_weights(vel)
    txt = np.zeros((16, TINY.hidden))
    x0 = o.gaussian_noise(8 * 8 * 32, 0).reshape(8, 8, 32)
    out = o.sample(w, TINY.heads, 64, 64, txt, txt, steps=4, cfg=3.0, shift=5.0, seed=0,
                   uncond_skip_layers=(1,))
    v_lat = o.unpatchify(np.broadcast_to(vel, (16, 128)), 8, 8)
    np.testing.assert_allclose(out, x0 - v_lat, atol=2e-6)


def test_sampler_cfg1_runs_no_negative_pass():
    vel = np.linspace(-1, 1, 128)
    w = _constant_velocity_weights(vel)
    txt = np.zeros((16, TINY.hidden))
    bad = np.full((16, TINY.hidden), np.nan)
    out = o.sample(w, TINY.heads, 64, 64, txt, bad, steps=3, cfg=1.0, seed=1)
    assert np.all(np.isfinite(out))
    with pytest.raises(ValueError):
        o.sample(w, TINY.heads, 60, 64, txt, txt, steps=1)


def test_psnr():
    ref = np.array([0.0, 1.0, 2.0, 3.0])
    assert o.psnr(ref, ref) == float("inf")
    assert abs(o.psnr(ref, ref + 0.03) - 10 * math.log10(9 / 0.0009)) < 1e-9


def test_block_rows_equals_full_block():
    w, ang, x, mod = _tiny_setup()
    lw = o.layer_weights(w, 0)
    full = o.block_forward(x, lw, mod, ang, TINY.heads)
    rows = [0, 5, 17, 31]
    np.testing.assert_allclose(o.block_forward_rows(x, lw, mod, ang, rows, TINY.heads), full[rows],
                               rtol=1e-12, atol=1e-12)


def test_sampler_branches_with_different_text_lengths():
    """Each branch uses its own prompt length: the sampler with a short negative prompt equals
    the guided Euler update of two separate single-branch forwards."""
    w = numpy_weights(make_weights(TINY, 15))
    rng = np.random.default_rng(15)
    tc = rng.standard_normal((16, TINY.hidden))
    tu = rng.standard_normal((5, TINY.hidden))
    x0 = rng.standard_normal((8, 8, 32)).astype(np.float32)
    out = o.sample(w, TINY.heads, 64, 64, tc, tu, steps=2, cfg=3.0, uncond_skip_layers=(1,), x0=x0)
    sig = o.sigma_schedule(2, 5.0)
    x = x0
    for i in range(2):
        su = (1,) if o.slg_active(i, 2, 0.01, 1.0) else ()
        vc = o.dit_forward(x, tc[None], float(sig[i]), [()], w, TINY.heads)[0].astype(np.float32)
        vu = o.dit_forward(x, tu[None], float(sig[i]), [su], w, TINY.heads)[0].astype(np.float32)
        x = o.cfg_euler(x, vc, vu, 3.0, sig[i], sig[i + 1])
    np.testing.assert_array_equal(out, x)
    # padding the short prompt with zero tokens changes the result (no padding semantics)
    tu_pad = np.concatenate([tu, np.zeros((11, TINY.hidden))])
    out_pad = o.sample(w, TINY.heads, 64, 64, tc, tu_pad, steps=2, cfg=3.0, uncond_skip_layers=(1,), x0=x0)
    assert not np.allclose(out, out_pad)
