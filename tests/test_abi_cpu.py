"""The C-ABI library without a GPU: it loads, exports every declared symbol, and its
host-only logic (size rule, schedule, skip window, argument checks) agrees with the
oracle and the pages.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import diffusion_transformer_text_block_b200 as moss
from oracle import moss_oracle as o


def _declared_functions():
    src = open(moss.HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moss_[a-z0-9_]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = moss.lib()
    names = _declared_functions()
    assert "moss_dit_block_forward" in names and "moss_sample" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.moss_abi_version() == moss.ABI_VERSION


def test_binding_covers_header():
    assert set(_declared_functions()) == set(moss._SIGS)


def test_validate_matches_oracle_and_pages():
    for h, w in [(1024, 1024), (2048, 2048), (1000, 1024), (0, 64), (4112, 512), (4096, 2048), (4096, 1024),
                 (16, 16), (64, 48)]:
        ok, msg = o.validate_size(h, w)
        rc = moss.lib().moss_validate(h, w)
        assert (rc == 0) == ok
        if not ok:
            assert moss.lib().moss_last_error().decode() == msg


def test_sigma_schedule_matches_oracle():
    for steps, shift in [(50, 5.0), (4, 5.0), (10, 1.0), (7, 3.0)]:
        np.testing.assert_array_equal(np.float32(moss.sigma_schedule(steps, shift)), o.sigma_schedule(steps, shift))
    with pytest.raises(moss.MossError):
        moss.sigma_schedule(0, 5.0)


def test_slg_window_matches_oracle():
    for steps, a, b in [(50, 0.01, 1.0), (50, 0.0, 1.0), (4, 0.01, 1.0), (50, 0.2, 0.6)]:
        for i in range(steps):
            assert moss.slg_active(i, steps, a, b) == o.slg_active(i, steps, a, b)


def test_config_defaults_are_the_full_model():
    c = moss.Config()
    moss.lib().moss_config_init(ctypes.byref(c), ctypes.sizeof(moss.Config))
    assert (c.layers, c.hidden, c.heads, c.head_dim, c.ffn, c.cond_dim) == (42, 3072, 24, 128, 8192, 256)
    assert c.max_batch == 2 and c.max_tokens == 4096 + 512 and c.max_latent_hw == 128 * 128


def _create(cfg_edit=None, size=None):
    c = moss.Config()
    moss.lib().moss_config_init(ctypes.byref(c), ctypes.sizeof(moss.Config))
    if cfg_edit:
        cfg_edit(c)
    if size is not None:
        c.struct_size = size
    w = moss.Weights()
    moss.lib().moss_weights_init(ctypes.byref(w), ctypes.sizeof(moss.Weights))
    h = ctypes.c_void_p()
    return moss.lib().moss_model_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)), h


def test_model_create_rejects_bad_arguments_on_the_host():
    rc, h = _create(size=12)
    assert rc == 5 and not h.value                                         # ABI mismatch
    rc, _ = _create(lambda c: setattr(c, "head_dim", 64))
    assert rc == 6                                                          # unsupported
    rc, _ = _create(lambda c: setattr(c, "hidden", 3000))
    assert rc == 1
    rc, _ = _create(lambda c: setattr(c, "ffn", 100))
    assert rc == 1
    rc, _ = _create()                                                       # NULL weight pointers
    assert rc == 1 and "NULL" in moss.lib().moss_last_error().decode()


def test_elementwise_entry_points_check_arguments_without_launching():
    lib = moss.lib()
    before = lib.moss_launch_count(0)
    assert lib.moss_cfg_euler_step(None, None, None, 0, 3.0, 1.0, 0.9, None) == 0      # empty: nothing to do
    assert lib.moss_cfg_euler_step(None, None, None, -1, 3.0, 1.0, 0.9, None) == 1
    assert lib.moss_cfg_euler_step(None, None, None, 8, 3.0, 1.0, 0.9, None) == 1
    assert lib.moss_cfg_euler_step(ctypes.c_void_p(8), ctypes.c_void_p(16), ctypes.c_void_p(32), 8, 3.0, 1.0, 0.9,
                                   None) == 1                                            # misaligned
    assert lib.moss_init_noise(None, 16, 42, None) == 1
    assert lib.moss_op_gemm_bf16(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 8, 48, 64, None) == 1
    assert lib.moss_dit_forward(None, 2, None, None, 0, 64, 64, 0.5, None, 0, None, None) == 1
    assert lib.moss_slg_active(50, 50, 0.0, 1.0) == -1
    a16, b16 = ctypes.c_void_p(4096), ctypes.c_void_p(8192)
    assert lib.moss_op_attention(None, b16, 1, 128, 1, None) == 1
    assert lib.moss_op_attention(ctypes.c_void_p(4100), b16, 1, 128, 1, None) == 1          # misaligned
    assert lib.moss_op_attention(a16, b16, 1, 0, 1, None) == 1
    # the attention failure-path self-test: the step must be a key step of the sequence
    assert lib.moss_selftest_attention_timeout(a16, b16, 1, 256, 1, -1, None) == 1
    assert lib.moss_selftest_attention_timeout(a16, b16, 1, 256, 1, 2, None) == 1          # 2 key steps
    assert lib.moss_selftest_attention_timeout(None, b16, 1, 256, 1, 0, None) == 1
    # the host-buffer step: bad schedule arguments, a NULL model and NULL buffers are refused first
    hx = (ctypes.c_float * 32)()
    assert lib.moss_denoise_step_host(None, hx, hx, 1, hx, 1, 64, 64, 0, 0, 3.0, 5.0, None, 0, 0.01, 1.0, None) == 1
    assert lib.moss_denoise_step_host(None, hx, hx, 1, hx, 1, 64, 64, 4, 4, 3.0, 5.0, None, 0, 0.01, 1.0, None) == 1
    assert lib.moss_denoise_step_host(None, hx, hx, 1, hx, 1, 64, 64, 0, 4, 3.0, 5.0, None, 0, 0.01, 1.0, None) == 1
    assert "model" in lib.moss_last_error().decode()
    assert lib.moss_launch_count(0) == before


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(8)
    with pytest.raises(moss.MossError):
        moss.cfg_euler_step(x, x, x, 3.0, 1.0, 0.9)


def test_sample_options_defaults_and_checks_without_launching():
    lib = moss.lib()
    opt = moss.SampleOptions()
    lib.moss_sample_options_init(ctypes.byref(opt), ctypes.sizeof(moss.SampleOptions))
    assert opt.struct_size == ctypes.sizeof(moss.SampleOptions)
    assert opt.cfg_truncation == 1.0 and opt.step_cache_threshold == 0.0
    assert not opt.cached_out and not opt.change_out
    before = lib.moss_launch_count(0)

    def call(o):
        return lib.moss_sample_ex(None, 4, 3.0, 5.0, 42, None, 0, 0.01, 1.0, None, 0, None, 0, 64, 64,
                                  ctypes.byref(o), None, None)

    bad = moss.SampleOptions()
    lib.moss_sample_options_init(ctypes.byref(bad), 12)
    assert call(bad) == 5                                                    # struct_size mismatch
    for field, value in (("cfg_truncation", 1.5), ("cfg_truncation", -0.1), ("cfg_truncation", float("nan")),
                         ("step_cache_threshold", -1.0), ("step_cache_threshold", float("nan"))):
        o = moss.SampleOptions()
        lib.moss_sample_options_init(ctypes.byref(o), ctypes.sizeof(moss.SampleOptions))
        setattr(o, field, value)
        assert call(o) == 1, (field, value)
    ok = moss.SampleOptions()
    lib.moss_sample_options_init(ctypes.byref(ok), ctypes.sizeof(moss.SampleOptions))
    assert call(ok) == 1 and "model" in lib.moss_last_error().decode()   # NULL model
    assert lib.moss_launch_count(0) == before


def test_text_path_entry_points_check_arguments_without_launching():
    lib = moss.lib()
    tw = moss.TextWeights()
    lib.moss_text_weights_init(ctypes.byref(tw), ctypes.sizeof(moss.TextWeights))
    assert tw.struct_size == ctypes.sizeof(moss.TextWeights) and tw.enc_dim == 4096 and tw.blocks == 2
    assert not tw.proj_w and not tw.wqkv
    before = lib.moss_launch_count(0)
    assert lib.moss_text_refiner_set(None, ctypes.byref(tw)) == 1
    assert lib.moss_text_refine(None, ctypes.c_void_p(16), 4, ctypes.c_void_p(16), None) == 1
    assert "no text path" in lib.moss_last_error().decode()
    assert lib.moss_launch_count(0) == before
