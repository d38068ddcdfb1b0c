"""Pins of the oracle's text path: projection of the encoder's final-layer states and the
text-only refiner blocks (windpaint.ai MOSS-Image specs, Architecture and specs; readings R22,
R23).  Each pin goes through torch library primitives or an invariant, not the oracle itself."""
import os
import sys

import numpy as np
import torch
import torch.nn.functional as Fnn

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle.moss_oracle as o  # noqa: E402
from synth import TINY, make_encoder_states, make_text_weights, numpy_weights  # noqa: E402
from tests.test_oracle_pins import _torch_block  # noqa: E402

ENC = 512  # encoder width of the tiny text path


def _setup(seed=41, n=12):
    tw = numpy_weights(make_text_weights(TINY, seed, enc_dim=ENC))
    e = make_encoder_states(n, seed + 1, enc_dim=ENC).double().numpy()
    return tw, e


def test_projection_is_a_linear_layer_with_bias():
    tw, e = _setup()
    ref = Fnn.linear(torch.from_numpy(e), torch.from_numpy(tw["proj_w"]), torch.from_numpy(tw["proj_b"])).numpy()
    np.testing.assert_allclose(o.text_projection(e, tw["proj_w"], tw["proj_b"]), ref, rtol=1e-12, atol=1e-12)


def test_text_positions_do_not_depend_on_the_image_grid():
    """Text token j sits at (j+1, 0, 0) in the joint sequence and in the text-only one."""
    np.testing.assert_array_equal(o.token_positions(0, 0, 7), o.token_positions(3, 5, 7)[15:])
    assert o.token_positions(0, 0, 3).tolist() == [[1, 0, 0], [2, 0, 0], [3, 0, 0]]


def test_refiner_matches_torch_composition():
    tw, e = _setup()
    D = TINY.hidden
    x = Fnn.linear(torch.from_numpy(e), torch.from_numpy(tw["proj_w"]), torch.from_numpy(tw["proj_b"])).numpy()
    mod = np.concatenate([np.zeros(2 * D), np.ones(D), np.zeros(2 * D), np.ones(D)])
    ang = o.rope_angles(o.token_positions(0, 0, e.shape[0]))
    for l in range(tw["wqkv"].shape[0]):
        x = _torch_block(x, o.layer_weights(tw, l), mod, ang, TINY.heads)
    y = o.text_refine(e, tw, TINY.heads)
    np.testing.assert_allclose(y, x, rtol=1e-10, atol=1e-12)
    assert np.abs(y - o.text_projection(e, tw["proj_w"], tw["proj_b"])).max() > 1e-3


def test_refiner_with_zero_output_projections_is_the_projection():
    tw, e = _setup()
    tw["wo"] = np.zeros_like(tw["wo"])
    tw["wd"] = np.zeros_like(tw["wd"])
    np.testing.assert_array_equal(o.text_refine(e, tw, TINY.heads), o.text_projection(e, tw["proj_w"], tw["proj_b"]))


def test_refiner_of_zero_states_is_zero():
    """LayerNorm of a zero row is zero (eps > 0), so every block adds nothing."""
    tw, e = _setup()
    tw["proj_w"] = np.zeros_like(tw["proj_w"])
    tw["proj_b"] = np.zeros_like(tw["proj_b"])
    np.testing.assert_array_equal(o.text_refine(e, tw, TINY.heads), np.zeros((e.shape[0], TINY.hidden)))


def test_refiner_rows_mix_only_through_attention():
    """One token alone: attention over itself returns its own value vector, so the block reduces to
    per-row maps; the first row of a 1-token and of a longer prompt differ (tokens see each other)."""
    tw, e = _setup(n=5)
    one = o.text_refine(e[:1], tw, TINY.heads)
    many = o.text_refine(e, tw, TINY.heads)
    assert one.shape == (1, TINY.hidden)
    assert not np.allclose(one[0], many[0])
