"""GPU quantiser vs the CPU oracle, bit for bit (codes, E4M3 scales and their
padding, FP32 tensor scale), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import check_quantize, gpu_quantize, f32_bits, first_mismatch, to_dev
import layout

pytestmark = pytest.mark.gpu

MODES = [(False, False, False), (False, True, False),            # rowwise RTN / SR
         (True, False, False), (True, True, False),               # colwise RTN / SR
         (True, False, True), (True, True, True)]                 # colwise + RHT, RTN / SR


def _bf16(rng, shape, scale=1.0):
    return W.bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(scale))


ROW_SHAPES = [(1, 16), (7, 48), (200, 272), (256, 256), (300, 1040)]
COL_SHAPES = [(16, 8), (48, 200), (208, 272), (272, 392), (528, 264)]


@pytest.mark.parametrize("mode", MODES, ids=lambda m: "cw%d-sr%d-rht%d" % m)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_small_ragged_shapes(mode, dtype, cuda_lib):
    colwise, sr, rht = mode
    rng = np.random.default_rng(17 + 4 * mode[0] + 2 * mode[1] + mode[2] + 8 * (dtype == "bf16"))
    for shape in (COL_SHAPES if colwise else ROW_SHAPES):
        x = rng.standard_normal(shape).astype(np.float32) * np.float32(rng.uniform(1e-3, 10))
        x = W.with_outliers(rng, x, max(1, x.size // 500), 60.0)
        if dtype == "bf16":
            x = W.bf16_bits(x)
        check_quantize(x, colwise, sr, rht, seed=int(rng.integers(1 << 62)))


def test_tiny_workload(cuda_lib):
    w = W.tiny()
    for name in ("X", "W"):
        check_quantize(w[name])


@pytest.mark.parametrize("mode", MODES, ids=lambda m: "cw%d-sr%d-rht%d" % m)
def test_special_inputs(mode, cuda_lib):
    colwise, sr, rht = mode
    shape = (64, 64)
    cases = {
        "zeros": np.zeros(shape, np.float32),
        "equal": np.full(shape, 0.37, np.float32),
        "single_outlier": np.where(np.arange(64 * 64).reshape(shape) == 777, 1e4, 1e-3).astype(np.float32),
        "subnormal": (np.random.default_rng(1).standard_normal(shape) * 1e-39).astype(np.float32),
        "tiny_amax": (np.random.default_rng(2).standard_normal(shape) * 1e-30).astype(np.float32),
        "huge": (np.random.default_rng(3).standard_normal(shape) * 1e37).astype(np.float32),
        "neg_zero": -np.zeros(shape, np.float32),
    }
    for name, x in cases.items():
        check_quantize(x, colwise, sr, rht, seed=99)
        check_quantize(W.bf16_bits(x), colwise, sr, rht, seed=99)


@pytest.mark.parametrize("colwise", [False, True])
def test_amax_supplied(colwise, cuda_lib):
    rng = np.random.default_rng(4)
    x = _bf16(rng, (256, 320))
    for amax in (2688.0, 3.5, 1e-3):
        check_quantize(x, colwise=colwise, sr=True, amax_in=amax)


@pytest.mark.parametrize("mode", [m for m in MODES if m[1]], ids=lambda m: "cw%d-sr%d-rht%d" % m)
def test_amax_supplied_overflow(mode, cuda_lib):
    """A supplied amax far below the data's: every block scale saturates at 448, the element
    scale 1/(448 s_t) stays finite (~1e10) and v / scale overflows to +-inf for most elements,
    which must encode as +-6 like any |v / scale| >= 6 (the saturation rule of the E2M1 encoding)."""
    colwise, sr, rht = mode
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((64, 96)) * 1e36).astype(np.float32)
    for v in (x, W.bf16_bits(x)):
        check_quantize(v, colwise, sr, rht, seed=5, amax_in=6e-10)


def test_e2m1_conversion_sweep(cuda_lib):
    """Every element is rounded at exactly its own value: blocks [6, v1..v15] with a
    supplied amax of 2688 give s_t = 1 and block scale 1, so r = v.  The v sweep covers
    a strided set of all binary32 values in [0, 6], every tie point, and signs."""
    lo = np.float32(0.0).view(np.uint32)
    hi = np.float32(6.0).view(np.uint32)
    vals = np.arange(lo, hi, 613, dtype=np.uint32).view(np.float32)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([ties, np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(9))])
    vals = np.concatenate([vals, near, -vals, -near, [0.0, -0.0, 6.0, -6.0]]).astype(np.float32)
    vals = np.concatenate([vals, np.zeros((-vals.size) % (15 * 64), np.float32)])
    blocks = vals.reshape(-1, 15)
    x = np.concatenate([np.full((blocks.shape[0], 1), 6.0, np.float32), blocks], axis=1).reshape(-1, 1024)
    check_quantize(x, amax_in=2688.0)
    check_quantize(x, sr=True, amax_in=2688.0)


def test_e4m3_conversion_sweep(cuda_lib):
    """Block amax values swept over a dense strided set of binary32 values so the
    E4M3 encoder sees every binade, the subnormal range, every tie and saturation."""
    lo = np.float32(2.0 ** -14).view(np.uint32)
    hi = np.float32(6.0 * 600).view(np.uint32)
    amaxes = np.arange(lo, hi, 1009, dtype=np.uint32).view(np.float32)
    amaxes = amaxes[: (amaxes.size // 64) * 64]
    x = np.zeros((amaxes.size, 16), np.float32)
    x[:, 3] = amaxes
    x[:, 7] = -amaxes * np.float32(0.3)
    check_quantize(x.reshape(-1, 1024), amax_in=2688.0)


# ---------------------------------------------------------------- full sizes
def _sampled_check(x, colwise, sr, rht, seed, n_rows=48):
    q = gpu_quantize(x, colwise, sr, rht, seed)
    am = oracle.amax(x, colwise=colwise, rht=rht, seed=seed)
    ts = oracle.tensor_scale(am)
    assert f32_bits(q.tensor_scale.cpu().numpy()[0]) == f32_bits(ts)
    rows_total = x.shape[1] if colwise else x.shape[0]
    k = x.shape[0] if colwise else x.shape[1]
    rng = np.random.default_rng(seed % 1000)
    rows = np.unique(np.concatenate([[0, rows_total - 1], rng.integers(0, rows_total, n_rows)]))
    oc, osc = oracle.quantize_rows(x, rows, am, colwise=colwise, sr=sr, rht=rht, seed=seed)
    gc = q.codes[rows].cpu().numpy()
    mm = first_mismatch(gc, oc)
    assert mm is None, "codes differ: %s" % (mm,)
    buf = q.scales.cpu().numpy()
    plain = buf[layout.atom_offsets(rows_total, k)[rows]]
    mm = first_mismatch(plain, osc)
    assert mm is None, "scales differ: %s" % (mm,)


@pytest.fixture(scope="module")
def qsweep_inputs():
    return W.qsweep()


@pytest.mark.parametrize("mode", MODES, ids=lambda m: "cw%d-sr%d-rht%d" % m)
def test_qsweep_full_size(mode, qsweep_inputs, cuda_lib):
    w = qsweep_inputs
    colwise, sr, rht = mode
    for name in ("A", "B"):
        _sampled_check(w[name], colwise, sr, rht, seed=1234)


def test_wgrad_operands_full_size(cuda_lib):
    w = W.wgrad()
    _sampled_check(w["dY"], True, True, True, seed=1234, n_rows=24)
    _sampled_check(w["X"], True, False, True, seed=1234, n_rows=24)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rht", [False, True], ids=["plain", "rht"])
def test_amax_matches_oracle(dtype, rht, cuda_lib):
    """nvfp4_amax: the tensor amax (after the 16-row RHT when asked) bit-exact against the
    oracle's, on ragged shapes and at a full weight shape; the quantisations it feeds give the
    same codes as their own amax pass (aisight.pl, sections "Architektura NVFP4 kontra
    ograniczenia mikroskalowania" and "Technologie stabilizujace proces treningowy")."""
    B = cuda_lib
    rng = np.random.default_rng(17)
    for R, C in [(16, 16), (48, 272), (528, 64), (1024, 1040)]:
        x = W.normal(rng, (R, C), 0.5)
        xb = W.bf16_bits(x) if dtype == "bf16" else x.astype(np.float32)
        got = B.nvfp4_amax(to_dev(xb), rht=rht, seed=1234)
        want = oracle.amax(xb, colwise=rht, rht=rht, seed=1234)
        assert f32_bits(got.cpu().numpy()[0]) == f32_bits(np.float32(want)), (R, C)
    x = to_dev(W.bf16_bits(W.normal(rng, (5120, 2048), 0.02)))
    ws = B.workspace(B.nvfp4_quantize_workspace_size(), x.device)
    a = B.nvfp4_amax(x, ws=ws)
    for orient in (B.NVFP4_ROWWISE, B.NVFP4_COLWISE):
        q0 = B.nvfp4_quantize(x, orientation=orient, ws=ws)
        q1 = B.nvfp4_quantize(x, orientation=orient, amax_in=a, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(q0.codes, q1.codes) and torch.equal(q0.scales, q1.scales)
        assert torch.equal(q0.tensor_scale, q1.tensor_scale)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_amax_dual_matches_oracle(dtype, cuda_lib):
    """nvfp4_amax_dual: both amaxes from one read, each bit-exact against the oracle's (the same
    passages as nvfp4_amax)."""
    B = cuda_lib
    rng = np.random.default_rng(19)
    for R, C in [(16, 16), (48, 272), (528, 64), (1024, 1040)]:
        x = W.normal(rng, (R, C), 0.5)
        xb = W.bf16_bits(x) if dtype == "bf16" else x.astype(np.float32)
        a, b = B.nvfp4_amax_dual(to_dev(xb), seed=99)
        assert f32_bits(a.cpu().numpy()[0]) == f32_bits(oracle.amax(xb)), (R, C)
        assert f32_bits(b.cpu().numpy()[0]) == f32_bits(oracle.amax(xb, colwise=True, rht=True, seed=99)), (R, C)
