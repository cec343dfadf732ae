"""MXFP4 quantiser (nvfp4_quantize_mx, both orientations) vs the CPU oracle, bit for bit:
E2M1 codes, E8M0 scales in the atom order (four 32-blocks per atom word) and
their zero padding."""
import numpy as np
import pytest
import torch

import layout
import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import first_mismatch, to_dev

pytestmark = pytest.mark.gpu

SHAPES = [(1, 32), (7, 96), (200, 288), (256, 256), (300, 1056), (130, 4096)]


def check_mx(x, colwise=False):
    q = B.nvfp4_quantize_mx(to_dev(x), orientation=B.NVFP4_COLWISE if colwise else B.NVFP4_ROWWISE)
    torch.cuda.synchronize()
    oc, osc = oracle.quantize_mx(x, colwise=colwise)
    rows, k = (x.shape[1], x.shape[0]) if colwise else x.shape
    mm = first_mismatch(q.codes.cpu().numpy(), oc)
    assert mm is None, "codes differ: %s" % (mm,)
    buf = q.scales.cpu().numpy()[:B.nvfp4_mx_scales_bytes(rows, k)]
    # the MX atom order is the NVFP4 one of a tensor with half as many columns (32 vs 16 per block)
    plain = layout.atoms_to_plain(buf, rows, k // 2)
    mm = first_mismatch(plain, osc)
    assert mm is None, "scales differ: %s" % (mm,)
    assert not buf[layout.padding_mask(rows, k // 2)].any(), "scale padding not zero"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mx_small_ragged(dtype, cuda_lib):
    rng = np.random.default_rng(41 + (dtype == "bf16"))
    for shape in SHAPES:
        x = (rng.standard_normal(shape) * np.exp(rng.standard_normal((shape[0], 1)) * 3)).astype(np.float32)
        x = W.with_outliers(rng, x, max(1, x.size // 500), 60.0)
        check_mx(W.bf16_bits(x) if dtype == "bf16" else x)


def test_mx_special_inputs(cuda_lib):
    shape = (64, 128)
    idx = np.arange(64 * 128).reshape(shape)
    cases = {
        "zeros": np.zeros(shape, np.float32),
        "neg_zero": -np.zeros(shape, np.float32),
        "powers_of_two": np.ldexp(1.0, (idx % 60) - 30).astype(np.float32),
        "subnormal": (np.random.default_rng(1).standard_normal(shape) * 1e-40).astype(np.float32),
        "tiny": (np.random.default_rng(2).standard_normal(shape) * 1e-37).astype(np.float32),
        "huge": (np.random.default_rng(3).standard_normal(shape) * 1e37).astype(np.float32),
        "saturating": np.where(idx % 32 == 0, 7.9, 0.3).astype(np.float32),
        "ties": np.where(idx % 32 == 0, 6.0, 0.25 * (idx % 5)).astype(np.float32),
    }
    for name, x in cases.items():
        check_mx(x)
        check_mx(W.bf16_bits(x))


def test_mx_full_size(cuda_lib):
    rng = np.random.default_rng(5)
    check_mx(W.bf16_bits(rng.standard_normal((8192, 5120)).astype(np.float32)))


COL_SHAPES = [(32, 8), (96, 200), (224, 136), (256, 256), (544, 1032), (4096, 130 * 8)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mx_colwise_small_ragged(dtype, cuda_lib):
    rng = np.random.default_rng(61 + (dtype == "bf16"))
    for shape in COL_SHAPES:
        if dtype == "f32" and shape[1] % 4:
            continue
        x = (rng.standard_normal(shape) * np.exp(rng.standard_normal((1, shape[1])) * 3)).astype(np.float32)
        x = W.with_outliers(rng, x, max(1, x.size // 500), 60.0)
        check_mx(W.bf16_bits(x) if dtype == "bf16" else x, colwise=True)


def test_mx_colwise_special_and_full_size(cuda_lib):
    shape = (128, 64)
    idx = np.arange(128 * 64).reshape(shape)
    for x in (np.zeros(shape, np.float32), np.ldexp(1.0, (idx % 60) - 30).astype(np.float32),
              (np.random.default_rng(3).standard_normal(shape) * 1e37).astype(np.float32),
              np.where(idx // 64 % 32 == 0, 7.9, 0.3).astype(np.float32)):
        check_mx(x, colwise=True)
        check_mx(W.bf16_bits(x), colwise=True)
    rng = np.random.default_rng(6)
    check_mx(W.bf16_bits(rng.standard_normal((8192, 5120)).astype(np.float32)), colwise=True)
