"""Pins for the oracle's NVFP4 quantiser (CPU only).

Format facts from aisight.pl, section "Architektura NVFP4 kontra ograniczenia
mikroskalowania": blocks of 16 elements, an E4M3 block scale, an extra FP32
per-tensor scale.  Storage ratio from aibuzzwire.news (Thinking Machines
"End-to-End 4-Bit Training"), section "Drei Formate, ein Trainingslauf":
NVFP4 stores values with about 3.6x fewer bits than BF16.  Stochastic
rounding must remove systematic bias (aisight.pl, section "Technologie
stabilizujace proces treningowy"; aibuzzwire.news, section "Unterschiedliche
Phasen, unterschiedliche Regeln").
"""
import os

import numpy as np
import pytest

import oracle
from nvfp4_bit_precision_quantize_b200 import workloads

from test_oracle_formats import E2M1_MAGS, e4m3_literal_values

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_block_of_16_locality():
    """Changing one element changes only its own 16-element block."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    c0, s0, _, _ = oracle.quantize(x, amax_in=20.0)
    y = x.copy()
    y[2, 37] = 9.5  # block 2 of row 2 (elements 32..47)
    c1, s1, _, _ = oracle.quantize(y, amax_in=20.0)
    diff_s = np.argwhere(s0 != s1)
    assert diff_s.tolist() == [[2, 2]]
    dc = np.argwhere(c0 != c1)  # code bytes: 8 per block
    assert all(r == 2 and 16 <= b < 24 for r, b in dc)
    assert s0.shape == (4, 64 // 16)


def test_block_scale_and_codes_bruteforce():
    """1x16 tensors: the scale is the E4M3 value nearest amax_b/6/s_t and each code
    the E2M1 value nearest v/(sb*s_t), both found by scanning every code."""
    rng = np.random.default_rng(1)
    e4 = e4m3_literal_values()
    for trial in range(300):
        mag = 10.0 ** rng.uniform(-6, 3)
        v = (rng.standard_normal(16) * mag).astype(np.float32)
        if trial % 7 == 0:
            v[rng.integers(16)] *= np.float32(40)
        amax_in = np.float32(np.abs(v).max() * 10.0 ** rng.uniform(0, 3)) if trial % 3 else None
        codes, scales, st, amax = oracle.quantize(v[None, :], amax_in=amax_in)
        s_t = np.float32(amax) / np.float32(2688.0) if amax > 0 else np.float32(1.0)
        assert st == s_t
        t = (np.float32(np.abs(v).max()) / np.float32(6.0)) / s_t
        d = np.abs(np.minimum(np.float64(t), 448.0) - e4)
        cands = np.flatnonzero(d == d.min())
        sb = cands[0] if len(cands) == 1 else cands[cands % 2 == 0][0]
        assert scales[0, 0] == sb
        dec = np.float32(e4[sb]) * s_t
        if sb == 0:
            assert np.all(codes == 0)
            continue
        inv = np.float32(1.0) / dec
        r = v * inv
        q = np.stack([codes[0] & 0xF, codes[0] >> 4], axis=-1).reshape(-1)
        for j in range(16):
            a = min(abs(float(r[j])), 6.0)
            dd = np.abs(a - E2M1_MAGS)
            cc = np.flatnonzero(dd == dd.min())
            mc = cc[0] if len(cc) == 1 else cc[cc % 2 == 0][0]
            assert q[j] & 7 == mc
            assert (q[j] >> 3) == int(np.signbit(r[j]))


def test_tensor_scale_bounds_and_top_block():
    rng = np.random.default_rng(2)
    for trial in range(20):
        x = (rng.standard_t(3, size=(32, 128)) * 10.0 ** rng.uniform(-4, 2)).astype(np.float32)
        codes, scales, st, amax = oracle.quantize(x)
        assert amax == np.abs(x).max()
        assert st == np.float32(amax) / np.float32(2688.0)
        deq = oracle.dequantize(codes, scales, st)
        assert np.abs(deq).max() <= amax * (1 + 2 ** -4) * (1 + 1e-6)
        # the block holding the tensor amax gets the largest E4M3 scale, 448
        r, c = np.unravel_index(np.abs(x).argmax(), x.shape)
        assert scales[r, c // 16] == 0x7E


def test_all_zero_tensor():
    codes, scales, st, amax = oracle.quantize(np.zeros((16, 32), np.float32))
    assert amax == 0 and st == 1.0
    assert not codes.any() and not scales.any()


def test_storage_ratio_vs_bf16():
    x = np.ones((128, 256), np.float32)
    codes, scales, _, _ = oracle.quantize(x)
    bytes_per_elem = (codes.nbytes + scales.nbytes) / x.size
    assert bytes_per_elem == 0.5625  # 4 bits + one 8-bit scale per 16 elements
    assert abs(16 / (8 * bytes_per_elem) - 3.6) < 0.05


def _exact_r_blocks(r, n_blocks):
    """Blocks [6, r, r, ...]: with amax_in = 2688 the tensor scale is 1, the block
    scale E4M3(1) = 1, so every element is rounded at exactly its own value."""
    x = np.full((n_blocks, 16), r, np.float32)
    x[:, 0] = 6.0
    return x.reshape(1, -1)


@pytest.mark.parametrize("r", [0.3, 2.7, 4.5, 3.2])
def test_sr_unbiased_over_1e6_draws(r):
    nb = 66667
    x = _exact_r_blocks(r, nb)
    codes, scales, st, _ = oracle.quantize(x, sr=True, seed=1234, amax_in=2688.0)
    assert st == 1.0 and np.all(scales == 0x38)
    deq = oracle.dequantize(codes, scales, st).reshape(nb, 16)[:, 1:].ravel()
    step = 0.5 if r < 2 else (1.0 if r < 4 else 2.0)
    lo = step * np.floor(np.float32(r) / step)
    f = (np.float64(np.float32(r)) - lo) / step
    assert set(np.unique(deq)) <= {lo, lo + step}
    sigma = step * np.sqrt(f * (1 - f) / deq.size)
    assert deq.size > 10 ** 6
    assert abs(deq.mean() - np.float32(r)) < 5 * sigma
    # round-to-nearest on the same input is biased by far more than 5 sigma
    c2, s2, _, _ = oracle.quantize(x, sr=False, amax_in=2688.0)
    rtn = oracle.dequantize(c2, s2, 1.0).reshape(nb, 16)[:, 1:].ravel()
    assert abs(rtn.mean() - np.float32(r)) > 50 * sigma


def test_sr_colwise_equals_rowwise_of_transpose():
    """The SR draw is keyed on the element's index in the output view, so the
    transposed quantisation of x equals the plain quantisation of x^T."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 48)).astype(np.float32)
    a = oracle.quantize(x, colwise=True, sr=True, seed=77)
    b = oracle.quantize(np.ascontiguousarray(x.T), colwise=False, sr=True, seed=77)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    c = oracle.quantize(x, colwise=True, sr=True, seed=78)
    assert not np.array_equal(a[0], c[0])


def test_rht_quantize_is_quantize_of_transformed_input():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 40)).astype(np.float32)
    d = oracle.rht_signs(1234)
    xt = np.empty_like(x)
    for c in range(x.shape[1]):
        for g in range(0, x.shape[0], 16):
            xt[g:g + 16, c] = oracle.rht16(x[g:g + 16, c], d)
    a = oracle.quantize(x, colwise=True, rht=True, seed=1234)
    b = oracle.quantize(xt, colwise=True, rht=False)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    with pytest.raises(ValueError):
        oracle.quantize(x, colwise=False, rht=True)


def test_bf16_input_widening():
    rng = np.random.default_rng(5)
    x32 = rng.standard_normal((16, 64)).astype(np.float32)
    bits = workloads.bf16_bits(x32)
    widened = (bits.astype(np.uint32) << 16).view(np.float32)
    a = oracle.quantize(bits)
    b = oracle.quantize(widened)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_quantized_product_tracks_exact_product():
    """NVFP4 X.W^T stays close to the exact product; a wrong tensor scale does not."""
    w = workloads.tiny()
    X, W = w["X"], w["W"]
    qx = oracle.quantize(X)
    qw = oracle.quantize(W)
    ref, _ = oracle.gemm(qx[:3], qw[:3])
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    rel = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    assert rel < 0.15
    bad, _ = oracle.gemm((qx[0], qx[1], qx[2] * 2), qw[:3])
    assert np.linalg.norm(bad - exact) / np.linalg.norm(exact) > 0.5


def test_golden_toy_example():
    """tests/golden/toy_rounding.txt holds the pages' worked rounding example."""
    vals = {}
    with open(os.path.join(GOLDEN, "toy_rounding.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = line.split("=")
                vals[k.strip()] = float(v)
    q = oracle.e2m1_rtn(vals["input"])
    assert oracle.e2m1_value(q) == vals["rounded"]
    assert abs(abs(np.float32(vals["input"]) - oracle.e2m1_value(q)) - vals["error"]) < 1e-6
