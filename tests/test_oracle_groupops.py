"""Pins of the oracle's DBuffer group operations beyond scale/zero (CPU).

DBuffer fuses identical operations such as add, scale and zero across the
tensors of a bucket (paper Sec. 5, gist.science 'Technische samenvatting'
2C).  Gradient accumulation (add) and global-norm clipping are pinned here
against library routines: torch's bf16 conversion, numpy's float64 norm and
torch.nn.utils.clip_grad_norm_.
"""
import numpy as np
import pytest
import torch

import oracle


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("scale", [1.0, 0.25, 1 / 64, 0.3])
def test_accumulate_matches_torch(scale):
    rng = np.random.default_rng(0)
    dst = bf16_bits(rng.normal(0, 1e-3, 20000))
    src = bf16_bits(rng.normal(0, 1e-3, 20000))
    want = (torch.from_numpy(bits_to_f32(dst)) + torch.from_numpy(bits_to_f32(src)) * np.float32(scale)).to(torch.bfloat16)
    got = dst.copy()
    oracle.accumulate(src, got, scale)
    assert np.array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def test_accumulate_twice_equals_sum_for_exact_values():
    # small integers: every sum is exact in bf16, so two adds give 1+2+3
    dst = bf16_bits(np.full(100, 1.0))
    oracle.accumulate(bf16_bits(np.full(100, 2.0)), dst, 1.0)
    oracle.accumulate(bf16_bits(np.full(100, 3.0)), dst, 1.0)
    assert np.all(bits_to_f32(dst) == 6.0)


@pytest.mark.parametrize("scale", [1.0, 0.125, 0.3])
def test_grad_norm_matches_numpy(scale):
    rng = np.random.default_rng(1)
    g = bf16_bits(rng.normal(0, 1e-3, 300001))
    x = (bits_to_f32(g) * np.float32(scale)).astype(np.float64)
    assert oracle.grad_norm(g, scale) == pytest.approx(np.linalg.norm(x), rel=1e-12)


def test_grad_norm_closed_form():
    # n = 4096 equal values c: norm = |c| * 64 exactly
    g = bf16_bits(np.full(4096, -0.375))
    assert oracle.grad_norm(g, 1.0) == 0.375 * 64
    assert oracle.grad_norm(np.zeros(10, np.uint16), 1.0) == 0.0


@pytest.mark.parametrize("max_norm", [0.01, 0.5, 10.0])
def test_clipped_scale_matches_torch_clip_grad_norm(max_norm):
    max_norm = float(np.float32(max_norm))      # the C-ABI takes max_norm as float
    rng = np.random.default_rng(2)
    grad = torch.tensor(rng.normal(0, 0.01, 5000), dtype=torch.float64)
    p = torch.zeros(5000, dtype=torch.float64, requires_grad=True)
    p.grad = grad.clone()
    total = float(torch.nn.utils.clip_grad_norm_([p], max_norm))
    coef = oracle.clip_coef(total, max_norm)
    assert torch.equal(p.grad, grad * coef)      # torch scaled every gradient by our coefficient
    assert oracle.clipped_scale(total, 1.0, max_norm) == np.float32(coef)
    assert oracle.clipped_scale(total, 0.125, max_norm) == np.float32(0.125 * coef)
