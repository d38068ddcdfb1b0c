"""The device-side failure path: every wait of the library's kernels on an mbarrier gives up after
a bounded time (2 s), records a code in the device error word and lets the kernel return, so the
context stays usable.  The self-test kernel waits on a barrier phase that nothing completes; no
fault, trap or endless loop is involved."""
import time

import pytest
import torch
import torch.nn.functional as F

import diffusion_transformer_text_block_b200 as moss

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_survives():
    assert moss.device_status(clear=True) == 0
    t0 = time.time()
    moss.selftest_wait_timeout()
    status = moss.device_status()            # synchronises
    elapsed = time.time() - t0
    assert status == 0x301
    assert 1.0 < elapsed < 30.0
    assert moss.device_status(clear=True) == 0x301
    assert moss.device_status() == 0
    # kernels still run and still compute: one attention call against torch's
    B, N, H = 1, 300, 2
    g = torch.Generator(device="cuda").manual_seed(3)
    qkv = torch.randn(B, N, 3 * H * 128, generator=g, device="cuda").to(torch.bfloat16)
    o = moss.op_attention(qkv, H)
    q, k, v = qkv.view(B, N, 3, H, 128).permute(2, 0, 3, 1, 4).float()
    ref = F.scaled_dot_product_attention(q, k, v).permute(0, 2, 1, 3).reshape(B, N, H * 128)
    err = ((o.float() - ref).norm() / ref.norm()).item()
    assert err < 1e-2
    assert moss.device_status(clear=True) == 0


def test_attention_wait_gives_up_and_every_warp_finishes():
    """One CTA of the attention kernel never receives a V tile: its bounded waits give up, the
    named-barrier handoffs still complete (their arrivals are unconditional), the launch ends,
    and the next launches are correct."""
    B, N, H = 1, 1024, 2
    g = torch.Generator(device="cuda").manual_seed(4)
    qkv = torch.randn(B, N, 3 * H * 128, generator=g, device="cuda").to(torch.bfloat16)
    q, k, v = qkv.view(B, N, 3, H, 128).permute(2, 0, 3, 1, 4).float()
    ref = F.scaled_dot_product_attention(q, k, v).permute(0, 2, 1, 3).reshape(B, N, H * 128)

    def rel(o):
        return ((o.float() - ref).norm() / ref.norm()).item()

    assert moss.device_status(clear=True) == 0
    assert rel(moss.op_attention(qkv, H)) < 1e-2
    t0 = time.time()
    moss.selftest_attention_timeout(qkv, H, 3)
    status = moss.device_status(clear=True)  # synchronises
    elapsed = time.time() - t0
    assert status in (0x201, 0x202)
    assert 1.0 < elapsed < 60.0
    for _ in range(2):
        assert rel(moss.op_attention(qkv, H)) < 1e-2
        assert moss.device_status(clear=True) == 0


def test_attention_wait_gives_up_in_a_grid_larger_than_the_gpu():
    """192 CTAs, more than one wave: the CTA that loses a V tile gives up while the other CTAs,
    and the later wave on the SMs they free, complete; the launch ends, the error word holds the
    code, and later launches are correct."""
    B, N, H = 2, 1024, 24
    g = torch.Generator(device="cuda").manual_seed(5)
    qkv = torch.randn(B, N, 3 * H * 128, generator=g, device="cuda").to(torch.bfloat16)
    q, k, v = qkv.view(B, N, 3, H, 128).permute(2, 0, 3, 1, 4).float()
    ref = F.scaled_dot_product_attention(q, k, v).permute(0, 2, 1, 3).reshape(B, N, H * 128)

    def rel(o):
        return ((o.float() - ref).norm() / ref.norm()).item()

    assert moss.device_status(clear=True) == 0
    assert rel(moss.op_attention(qkv, H)) < 1e-2
    t0 = time.time()
    moss.selftest_attention_timeout(qkv, H, 3)
    status = moss.device_status(clear=True)  # synchronises
    elapsed = time.time() - t0
    assert status in (0x201, 0x202)
    assert 1.0 < elapsed < 60.0
    for _ in range(2):
        assert rel(moss.op_attention(qkv, H)) < 1e-2
        assert moss.device_status(clear=True) == 0
