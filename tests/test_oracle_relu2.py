"""Pins for the oracle's squared-ReLU activation and its derivative (CPU only).

h = relu(y)^2 and dY1 = dh * 2 relu(y), each one binary32 operation then a
round-to-nearest-even cast to bf16, checked against torch's CPU float32
arithmetic and bf16 cast (an independent library); relu(y) is +0 for y <= 0.
"""
import numpy as np
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import workloads


def _inputs(seed, n=200000):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal(n).astype(np.float32) * np.float32(3)
    y[:6] = [0.0, -0.0, 1e-30, -1e-30, 3e19, -5.0]
    return workloads.bf16_bits(y)


def test_relu2_fwd_matches_torch():
    y = _inputs(0)
    yt = workloads.bits_to_torch_bf16(y).float()
    r = torch.where(yt > 0, yt, torch.zeros_like(yt))
    ref = (r * r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.relu2_fwd(y), ref)


def test_relu2_bwd_matches_torch():
    y = _inputs(1)
    dh = workloads.bf16_bits(np.random.default_rng(2).standard_normal(y.size).astype(np.float32) * 1e-3)
    yt = workloads.bits_to_torch_bf16(y).float()
    dht = workloads.bits_to_torch_bf16(dh).float()
    g = 2.0 * torch.where(yt > 0, yt, torch.zeros_like(yt))
    ref = (dht * g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.relu2_bwd(dh, y), ref)


def test_relu2_zero_sign():
    y = workloads.bf16_bits(np.array([-0.0, -1.0], np.float32))
    assert list(oracle.relu2_fwd(y)) == [0, 0]
    # relu(-0) is +0, so the derivative factor is +0 and the product takes dh's sign
    dh = workloads.bf16_bits(np.array([-2.0, 2.0], np.float32))
    assert list(oracle.relu2_bwd(dh, y)) == [0x8000, 0]
