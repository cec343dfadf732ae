"""Dual-orientation quantiser (nvfp4_quantize_dual) vs the CPU oracle: the
rowwise output must equal the oracle's rowwise RTN quantisation and the
colwise output the oracle's colwise quantisation (RTN or SR, with or without
the Hadamard transform), bit for bit, and at full size both must equal the two
single-orientation GPU calls byte for byte."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import compare_quantize, f32_bits, first_mismatch, to_dev
import layout

pytestmark = pytest.mark.gpu

COL_MODES = [(False, False), (True, False), (False, True), (True, True)]  # (sr, rht) of the colwise output
SHAPES = [(16, 16), (48, 208), (208, 272), (272, 400), (528, 272), (256, 512)]  # R % 16 == 0 and C % 16 == 0


def gpu_dual(x, sr, rht, seed, amax_row=None, amax_col=None):
    xd = to_dev(x)
    t = lambda v: torch.tensor([v], dtype=torch.float32, device="cuda") if v is not None else None  # noqa: E731
    row, col = B.nvfp4_quantize_dual(xd, col_rounding=B.NVFP4_SR if sr else B.NVFP4_RTN, col_rht=rht, seed=seed,
                                     amax_row_in=t(amax_row), amax_col_in=t(amax_col))
    torch.cuda.synchronize()
    return row, col


def check_dual(x, sr, rht, seed, amax_row=None, amax_col=None):
    row, col = gpu_dual(x, sr, rht, seed, amax_row, amax_col)
    compare_quantize(row, x, False, False, False, seed, amax_row)
    compare_quantize(col, x, True, sr, rht, seed, amax_col)


@pytest.mark.parametrize("mode", COL_MODES, ids=lambda m: "sr%d-rht%d" % m)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dual_small_ragged(mode, dtype, cuda_lib):
    sr, rht = mode
    rng = np.random.default_rng(31 + 2 * sr + rht + 8 * (dtype == "bf16"))
    for shape in SHAPES:
        x = rng.standard_normal(shape).astype(np.float32) * np.float32(rng.uniform(1e-3, 10))
        x = W.with_outliers(rng, x, max(1, x.size // 500), 60.0)
        if dtype == "bf16":
            x = W.bf16_bits(x)
        check_dual(x, sr, rht, seed=int(rng.integers(1 << 62)))


@pytest.mark.parametrize("mode", COL_MODES, ids=lambda m: "sr%d-rht%d" % m)
def test_dual_special_inputs(mode, cuda_lib):
    sr, rht = mode
    shape = (64, 64)
    cases = {
        "zeros": np.zeros(shape, np.float32),
        "equal": np.full(shape, 0.37, np.float32),
        "single_outlier": np.where(np.arange(64 * 64).reshape(shape) == 777, 1e4, 1e-3).astype(np.float32),
        "tiny_amax": (np.random.default_rng(2).standard_normal(shape) * 1e-30).astype(np.float32),
        "huge": (np.random.default_rng(3).standard_normal(shape) * 1e37).astype(np.float32),
    }
    for name, x in cases.items():
        check_dual(x, sr, rht, seed=99)
        check_dual(W.bf16_bits(x), sr, rht, seed=99)


def test_dual_amax_supplied(cuda_lib):
    rng = np.random.default_rng(5)
    x = W.bf16_bits(rng.standard_normal((256, 320)).astype(np.float32))
    for rht in (False, True):
        check_dual(x, True, rht, 7, amax_row=3.5)
        check_dual(x, True, rht, 7, amax_col=2688.0)
        check_dual(x, True, rht, 7, amax_row=1e-3, amax_col=6.0)


def test_dual_empty(cuda_lib):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    row, col = B.nvfp4_quantize_dual(x, col_rht=True)
    torch.cuda.synchronize()
    assert row.tensor_scale.item() == 1.0 and col.tensor_scale.item() == 1.0


def _bytes(q):
    return (q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.tensor_scale.cpu().numpy())


@pytest.mark.parametrize("name,sr,rht", [("dY1", True, True), ("h", False, True), ("W2", False, False)])
def test_dual_equals_single_calls_full_size(name, sr, rht, cuda_lib):
    """MLP step operands at full size: the dual call's two outputs equal the two
    single-orientation calls (themselves bit-exact against the oracle) byte for byte,
    and sampled rows of both match the oracle."""
    rng = np.random.default_rng(9)
    shapes = {"dY1": (8192, 20480), "h": (8192, 20480), "W2": (5120, 20480)}
    x = torch.from_numpy(W.bf16_bits(rng.standard_normal(shapes[name]).astype(np.float32) * 0.02)).view(
        torch.bfloat16).cuda()
    rnd = B.NVFP4_SR if sr else B.NVFP4_RTN
    row, col = B.nvfp4_quantize_dual(x, col_rounding=rnd, col_rht=rht, seed=1234)
    r1 = B.nvfp4_quantize(x, orientation=B.NVFP4_ROWWISE, seed=1234)
    c1 = B.nvfp4_quantize(x, orientation=B.NVFP4_COLWISE, rounding=rnd, rht=rht, seed=1234)
    torch.cuda.synchronize()
    for a, b, what in ((row, r1, "rowwise"), (col, c1, "colwise")):
        for u, v, part in zip(_bytes(a), _bytes(b), ("codes", "scales", "tensor scale")):
            mm = first_mismatch(u, v)
            assert mm is None, "%s %s differ: %s" % (what, part, mm)
    # sampled oracle rows of the colwise output (the transformed, stochastically rounded one)
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    am = oracle.amax(xb, colwise=True, rht=rht, seed=1234)
    assert f32_bits(col.tensor_scale.cpu().numpy()[0]) == f32_bits(oracle.tensor_scale(am))
    rows = np.array([0, 1, 777, xb.shape[1] - 1])
    oc, osc = oracle.quantize_rows(xb, rows, am, colwise=True, sr=sr, rht=rht, seed=1234)
    mm = first_mismatch(col.codes[rows].cpu().numpy(), oc)
    assert mm is None, "codes differ: %s" % (mm,)
    plain = col.scales.cpu().numpy()[layout.atom_offsets(xb.shape[1], xb.shape[0])[rows]]
    mm = first_mismatch(plain, osc)
    assert mm is None, "scales differ: %s" % (mm,)
