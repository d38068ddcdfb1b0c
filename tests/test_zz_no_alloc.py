"""The allocation-free modulation entry point against the regular one.

moss_modulation_noalloc serves callers that must not allocate device memory; its scratch
is a fixed array inside the library.  Two calls in a row (with different timesteps, so the
second reuses the scratch the first left behind) must match moss_op_modulation within the
modulation tolerance of the kernel tests (relative L2 <= 1e-5).  This file is collected
last so that a failure here comes after every other test has run.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_text_block_b200 as moss
from synth import TINY
from tests.gpu_common import assert_no_device_error, make_model, rel_l2

pytestmark = pytest.mark.gpu


def test_modulation_noalloc_matches_regular_entry_point():
    model, wg, _ = make_model(TINY, 91, max_tokens=32)
    calls = [[0.25, 0.9, 1.0], [0.5]]
    for ts in calls:
        got = moss.modulation_noalloc(TINY, wg, ts)
        torch.cuda.synchronize()
        for i, t in enumerate(ts):
            ref = model.modulation(t)
            torch.cuda.synchronize()
            assert rel_l2(got[i].cpu().numpy(), ref.cpu().numpy()) <= 1e-5
    model.close()
    assert_no_device_error()


def test_modulation_noalloc_rejects_sizes_beyond_the_scratch():
    _, wg, _ = make_model(TINY, 92, max_tokens=32)
    with pytest.raises(moss.MossError, match="MOSS_NOALLOC_MAX_TIMESTEPS"):
        moss.modulation_noalloc(TINY, wg, [0.5] * (moss.NOALLOC_MAX_TIMESTEPS + 1),
                                out=torch.empty(65, 2 * 6 * 256 + 512, device="cuda"))
