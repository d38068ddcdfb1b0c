"""Pins of the oracle's lossy accelerators (CFG truncation, first-block step cache).

MossInfer integration guide, What works (Lossy accelerators) and Per-image settings: CFG
truncation drops the negative branch from step X*steps on (X = 1 is off); the step cache reuses
blocks 1..L-1 of the last full call while block 0's output changed by less than a threshold.
Each test pins the accelerated sampler to the plain sampler (pinned in test_oracle_pins.py) or
to an invariant that a dropped term, a wrong comparison or a stale reference would break.
"""
import math
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle.moss_oracle as o  # noqa: E402
from synth import TINY, make_weights, numpy_weights  # noqa: E402


def _setup(seed=21, n_u=16):
    w = numpy_weights(make_weights(TINY, seed))
    rng = np.random.default_rng(seed)
    tc = rng.standard_normal((16, TINY.hidden))
    tu = rng.standard_normal((n_u, TINY.hidden))
    x0 = rng.standard_normal((8, 8, 32)).astype(np.float32)
    return w, tc, tu, x0


def _run(w, tc, tu, x0, **kw):
    args = dict(steps=4, cfg=3.0, shift=5.0, uncond_skip_layers=(1,), x0=x0)
    args.update(kw)
    return o.sample_accelerated(w, TINY.heads, 64, 64, tc, tu, **args)


def test_accelerators_off_is_the_plain_sampler():
    w, tc, tu, x0 = _setup()
    x, cached, change = _run(w, tc, tu, x0)
    ref = o.sample(w, TINY.heads, 64, 64, tc, tu, steps=4, cfg=3.0, uncond_skip_layers=(1,), x0=x0)
    np.testing.assert_array_equal(x, ref)
    assert cached == [False] * 4 and all(math.isnan(c) for c in change)


def test_cfg_truncation_zero_is_the_conditional_sampler():
    w, tc, tu, x0 = _setup()
    x, _, _ = _run(w, tc, tu, x0, cfg_truncation=0.0)
    ref = o.sample(w, TINY.heads, 64, 64, tc, tu, steps=4, cfg=1.0, x0=x0)
    np.testing.assert_array_equal(x, ref)


def test_cfg_truncation_starts_at_step_x_times_steps():
    """'From step X*steps on', inclusive: with 4 steps, X = 0.5 and X = 0.26 both drop the
    negative branch at steps 2 and 3 (2 >= 2.0, 2 >= 1.04 > 1), X = 0.24 already at step 1."""
    assert [o.cfg_truncated(i, 4, 0.5) for i in range(4)] == [False, False, True, True]
    assert [o.cfg_truncated(i, 4, 0.26) for i in range(4)] == [False, False, True, True]
    assert [o.cfg_truncated(i, 4, 0.24) for i in range(4)] == [False, True, True, True]
    assert not any(o.cfg_truncated(i, 50, 1.0) for i in range(50))
    w, tc, tu, x0 = _setup()
    a, _, _ = _run(w, tc, tu, x0, cfg_truncation=0.5)
    b, _, _ = _run(w, tc, tu, x0, cfg_truncation=0.26)
    c, _, _ = _run(w, tc, tu, x0, cfg_truncation=0.24)
    full, _, _ = _run(w, tc, tu, x0)
    np.testing.assert_array_equal(a, b)
    assert not np.allclose(a, c) and not np.allclose(a, full)


def test_cfg_truncation_negative_prompt_unused_after_the_switch():
    """With every step truncated the negative prompt is never read (NaN stays out)."""
    w, tc, tu, x0 = _setup()
    bad = np.full_like(tu, np.nan)
    x, _, _ = _run(w, tc, bad, x0, cfg_truncation=0.0)
    assert np.all(np.isfinite(x))


def test_step_cache_threshold_zero_never_reuses():
    w, tc, tu, x0 = _setup()
    x, cached, change = _run(w, tc, tu, x0, step_cache_threshold=0.0)
    ref = o.sample(w, TINY.heads, 64, 64, tc, tu, steps=4, cfg=3.0, uncond_skip_layers=(1,), x0=x0)
    np.testing.assert_array_equal(x, ref)
    assert not any(cached)


def test_relative_change_definition():
    a = [np.array([[1.0, -2.0]]), np.array([[3.0]])]
    b = [np.array([[1.5, -2.0]]), np.array([[2.0]])]
    # (0.5 + 0 + 1) / (1.5 + 2 + 2)
    assert abs(o.relative_change(a, b) - 1.5 / 5.5) < 1e-15
    assert o.relative_change(b, b) == 0.0


def _static_weights(seed=22, zero_out=True, zero_later_gates=False):
    """Modulation independent of t (mod_w = 0); optionally zero velocity (so x never moves)
    and/or blocks 1..L-1 made identities (their gates zero)."""
    w = numpy_weights(make_weights(TINY, seed))
    D = TINY.hidden
    w["mod_w"] = np.zeros_like(w["mod_w"])
    if zero_out:
        w["out_w"] = np.zeros_like(w["out_w"])
        w["out_b"] = np.zeros_like(w["out_b"])
    if zero_later_gates:
        for l in range(1, w["mod_b"].shape[0]):
            w["mod_b"][l][2 * D:3 * D] = 0.0
            w["mod_b"][l][5 * D:6 * D] = 0.0
    return w


def test_step_cache_reuses_every_step_when_nothing_changes():
    """v = 0 and t-independent modulation: x and block 0's output never change, so every step
    after the first reuses the cache (change exactly 0) and x stays the initial latent."""
    w = _static_weights()
    _, tc, tu, x0 = _setup()
    x, cached, change = _run(w, tc, tu, x0, step_cache_threshold=1e-9)
    assert cached == [False, True, True, True]
    assert math.isnan(change[0]) and change[1:] == [0.0, 0.0, 0.0]
    np.testing.assert_array_equal(x, x0)


def test_step_cache_reuse_is_exact_when_later_blocks_are_identities():
    """Blocks 1..L-1 with zero gates add nothing, so the cached residual is 0 and a reused step
    equals a full one: any threshold gives the plain sampler's result."""
    w = _static_weights(zero_out=False, zero_later_gates=True)
    _, tc, tu, x0 = _setup()
    x, cached, change = _run(w, tc, tu, x0, step_cache_threshold=1e9)
    assert cached == [False, True, True, True]
    assert all(c > 0 for c in change[1:])
    ref = o.sample(w, TINY.heads, 64, 64, tc, tu, steps=4, cfg=3.0, uncond_skip_layers=(1,), x0=x0)
    np.testing.assert_allclose(x, ref, rtol=0, atol=1e-6)


def test_step_cache_reference_is_the_last_full_call():
    """Replayed decisions: a reused step leaves the reference where it was (the change at the
    next step is measured against the older full call), a full step moves it."""
    w, tc, tu, x0 = _setup()
    _, c1, ch1 = _run(w, tc, tu, x0, decisions=[False, True, True, False])
    _, c2, ch2 = _run(w, tc, tu, x0, decisions=[False, False, True, False])
    assert c1 == [False, True, True, False] and c2 == [False, False, True, False]
    # step 1 compares with step 0's output in both runs
    assert ch1[1] == ch2[1]
    # step 2: run 1 still compares with step 0, run 2 with step 1, which is closer in t
    assert ch1[2] != ch2[2]


def test_step_cache_full_call_after_branch_count_changes():
    """CFG truncation changes the number of branches: the first truncated step cannot reuse a
    two-branch reference and runs in full."""
    w = _static_weights()
    _, tc, tu, x0 = _setup()
    _, cached, change = _run(w, tc, tu, x0, step_cache_threshold=1e-9, cfg_truncation=0.5)
    assert cached == [False, True, False, True]
    assert math.isnan(change[2])


# Three-pass SLG (reading R24; the pages name the option and the extra skipped conditional
# pass but give no formula, so these pins check the reading's arithmetic and its invariants,
# not the pages).
def test_slg_combine_closed_forms():
    rng = np.random.default_rng(3)
    vc, vu, vcs = (rng.standard_normal(64).astype(np.float32) for _ in range(3))
    np.testing.assert_array_equal(o.slg_combine(vc, vu, vcs, 3.0, 0.0), o.cfg_combine(vc, vu, 3.0))
    np.testing.assert_array_equal(o.slg_combine(vc, vu, vc, 3.0, 2.5), o.cfg_combine(vc, vu, 3.0))
    np.testing.assert_allclose(o.slg_combine(vc, vu, vcs, 1.0, 2.0), vc + 2.0 * (vc - vcs), rtol=1e-6, atol=1e-6)


def test_three_pass_off_and_outside_window_are_two_pass():
    w, tc, tu, x0 = _setup()
    ref, _, _ = _run(w, tc, tu, x0)
    a, _, _ = _run(w, tc, tu, x0, slg_scale=0.0)
    b, _, _ = _run(w, tc, tu, x0, slg_scale=2.0, slg_start=2.0, slg_stop=3.0)  # window never active
    np.testing.assert_array_equal(a, ref)
    # outside the window the uncond branch does not skip either: compare with a two-pass run
    # that has the same (inactive) window
    ref2, _, _ = _run(w, tc, tu, x0, slg_start=2.0, slg_stop=3.0)
    np.testing.assert_array_equal(b, ref2)


def test_three_pass_is_cfg_plus_scaled_skip_difference():
    """Inside the window: v = CFG(v_c, v_u) + s (v_c - v_cs) with v_cs the conditional forward
    skipping the SLG layers, composed here from the pinned single-branch forward."""
    w, tc, tu, x0 = _setup()
    out, _, _ = _run(w, tc, tu, x0, slg_scale=2.0, steps=2)
    sig = o.sigma_schedule(2, 5.0)
    x = x0
    for i in range(2):
        su = (1,) if o.slg_active(i, 2, 0.01, 1.0) else ()
        vc = o.dit_forward(x, tc[None], float(sig[i]), [()], w, TINY.heads)[0].astype(np.float32)
        vu = o.dit_forward(x, tu[None], float(sig[i]), [su], w, TINY.heads)[0].astype(np.float32)
        if su:
            vcs = o.dit_forward(x, tc[None], float(sig[i]), [su], w, TINY.heads)[0].astype(np.float32)
            v = o.slg_combine(vc, vu, vcs, 3.0, 2.0)
        else:
            v = o.cfg_combine(vc, vu, 3.0)
        x = o.euler_update(x, v, sig[i], sig[i + 1])
    np.testing.assert_array_equal(out, x)


def test_three_pass_with_identity_skip_layer_is_two_pass():
    """When the skipped layer adds nothing (its gates are zero), v_cs = v_c and the third pass
    changes nothing."""
    w, tc, tu, x0 = _setup()
    D = TINY.hidden
    w["mod_w"][1] = 0.0
    w["mod_b"][1][2 * D:3 * D] = 0.0
    w["mod_b"][1][5 * D:6 * D] = 0.0
    a, _, _ = _run(w, tc, tu, x0, slg_scale=2.0)
    b, _, _ = _run(w, tc, tu, x0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-6)
