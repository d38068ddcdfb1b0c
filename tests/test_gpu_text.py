"""GPU parity of the text path (moss_text_refine): projection of the encoder's final-layer
states and the text-only refiner blocks, against the oracle's text_refine (windpaint.ai MOSS-Image
specs, Architecture and specs; readings R22, R23).  Tolerance: the joint blocks' per-block bound
(relative L2 <= 1e-2); the projection alone (BF16 inputs, FP32 accumulation and output) <= 1e-5."""
import numpy as np
import pytest
import torch

import diffusion_transformer_text_block_b200 as moss
import oracle.moss_oracle as o
from synth import TINY, make_encoder_states, make_text_weights, make_weights, numpy_weights
from tests.gpu_common import WIDE1, assert_no_device_error, rel_l2

pytestmark = pytest.mark.gpu


def _model(shape, seed, enc_dim, blocks, max_tokens):
    w = {k: v.cuda() for k, v in make_weights(shape, seed, layers=1).items()}
    model = moss.Model(shape, w, max_tokens=max_tokens, max_batch=2, max_latent_hw=64, max_steps=1)
    tw = make_text_weights(shape, seed + 1, enc_dim=enc_dim, blocks=blocks)
    model.set_text_weights({k: v.cuda() for k, v in tw.items()})
    return model, numpy_weights(tw)


@pytest.mark.parametrize("n_txt", [1, 5, 16, 77, 128])
def test_text_refine_tiny_matches_oracle(n_txt):
    model, twn = _model(TINY, 51, 512, 2, max_tokens=128)
    enc = make_encoder_states(n_txt, 53, enc_dim=512)
    out = model.text_refine(enc.cuda())
    torch.cuda.synchronize()
    ref = o.text_refine(enc.double().numpy(), twn, TINY.heads)
    proj = o.text_projection(enc.double().numpy(), twn["proj_w"], twn["proj_b"])
    assert rel_l2(out.cpu().numpy(), ref) <= 1e-2
    assert rel_l2(out.cpu().numpy() - proj, ref - proj) <= 1e-2         # the blocks' update itself
    model.close()
    assert_no_device_error()


def test_text_projection_only_is_tight():
    model, twn = _model(TINY, 55, 512, 0, max_tokens=64)
    enc = make_encoder_states(40, 56, enc_dim=512)
    out = model.text_refine(enc.cuda())
    torch.cuda.synchronize()
    ref = o.text_projection(enc.double().numpy(), twn["proj_w"], twn["proj_b"])
    assert rel_l2(out.cpu().numpy(), ref) <= 1e-5
    model.close()
    assert_no_device_error()


def test_text_refine_full_width_512_tokens():
    """The full text path: encoder width 4096, hidden 3072, 24 heads, FFN 8192, two blocks, the
    benchmark's 512-token prompt."""
    model, twn = _model(WIDE1, 57, 4096, 2, max_tokens=4096)
    enc = make_encoder_states(512, 58, enc_dim=4096)
    out = model.text_refine(enc.cuda())
    torch.cuda.synchronize()
    ref = o.text_refine(enc.double().numpy(), twn, WIDE1.heads)
    assert rel_l2(out.cpu().numpy(), ref) <= 1e-2
    model.close()
    assert_no_device_error()


def test_text_refine_then_image_forward_rebuilds_rope():
    """The refiner replaces the model's cached RoPE table; the next image forward must rebuild it:
    forward before and after a refine call agree bitwise."""
    model, _ = _model(TINY, 61, 512, 2, max_tokens=64)
    from synth import make_latent, make_text
    lat = make_latent(8, 8, 62, device="cuda")
    txt = make_text(2, 16, TINY.hidden, 63, device="cuda")
    a = model.forward(lat, txt, 64, 64, 0.4).clone()
    model.text_refine(make_encoder_states(9, 64, enc_dim=512).cuda())
    b = model.forward(lat, txt, 64, 64, 0.4).clone()
    assert torch.equal(a, b)
    model.close()
    assert_no_device_error()
