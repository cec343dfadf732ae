"""Pin for oracle.quantize_rows, the checker of the full-size GPU parity tests.

quantize_rows re-quantises only selected output rows of a tensor, given its
amax, so that tensors too large for the whole-tensor oracle can still be
checked row by row.  Its rows must be byte-identical to the same rows of the
whole-tensor oracle.quantize, which the other oracle pins tie to the format of
aisight.pl, section "Architektura NVFP4 kontra ograniczenia mikroskalowania"
(blocks of 16, E4M3 block scale, FP32 tensor scale) and to the Hadamard
transform and stochastic rounding of section "Technologie stabilizujace proces
treningowy".  A row-offset slip, a dropped transform, a wrong SR element index
or a mishandled amax in quantize_rows fails here, on the CPU.
"""
import numpy as np
import pytest

import oracle
from nvfp4_bit_precision_quantize_b200 import workloads as W

MODES = [  # (colwise, sr, rht)
    (False, False, False),
    (False, True, False),
    (True, False, False),
    (True, True, False),
    (True, False, True),
    (True, True, True),
]
SHAPES = [(16, 16), (48, 80), (96, 272), (144, 64), (272, 48), (32, 40)]  # ragged against 128 / 64


def _rows_to_check(rng, n):
    picks = {0, n - 1, n // 2}
    picks.update(int(i) for i in rng.integers(0, n, size=min(n, 6)))
    return np.array(sorted(picks), dtype=np.int64)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("mode", MODES)
def test_quantize_rows_equals_whole_tensor(mode, bf16):
    colwise, sr, rht = mode
    rng = np.random.default_rng(17 + 3 * MODES.index(mode) + int(bf16))
    for R, Cc in SHAPES:
        if (colwise and Cc % (8 if bf16 else 4)) or (not colwise and Cc % 16):
            continue
        x = W.normal(rng, (R, Cc)) * np.float32(10.0 ** rng.uniform(-3, 2))
        x[rng.integers(R), rng.integers(Cc)] *= np.float32(60.0)  # one outlier block
        if bf16:
            x = W.bf16_bits(x)
        codes, scales, _, amax = oracle.quantize(x, colwise=colwise, sr=sr, rht=rht, seed=4321)
        rows = _rows_to_check(rng, codes.shape[0])
        c_rows, s_rows = oracle.quantize_rows(x, rows, amax, colwise=colwise, sr=sr, rht=rht, seed=4321)
        np.testing.assert_array_equal(c_rows, codes[rows], err_msg="codes %s %dx%d" % (mode, R, Cc))
        np.testing.assert_array_equal(s_rows, scales[rows], err_msg="scales %s %dx%d" % (mode, R, Cc))


@pytest.mark.parametrize("mode", [(False, False, False), (True, True, True)])
def test_quantize_rows_with_supplied_amax(mode):
    """With an amax larger than the tensor's own (a producer-supplied value), the
    rows still match the whole-tensor oracle given the same amax_in."""
    colwise, sr, rht = mode
    rng = np.random.default_rng(5)
    x = W.bf16_bits(W.normal(rng, (64, 96)))
    amax_in = np.float32(37.5)
    codes, scales, ts, am = oracle.quantize(x, colwise=colwise, sr=sr, rht=rht, seed=99, amax_in=amax_in)
    assert am == amax_in and ts == np.float32(amax_in) / np.float32(2688.0)
    rows = np.arange(codes.shape[0], dtype=np.int64)[::-3]
    c_rows, s_rows = oracle.quantize_rows(x, rows, amax_in, colwise=colwise, sr=sr, rht=rht, seed=99)
    np.testing.assert_array_equal(c_rows, codes[rows])
    np.testing.assert_array_equal(s_rows, scales[rows])


def test_quantize_rows_seed_and_row_sensitivity():
    """Different seeds change SR rows; rows passed out of order come back in that order."""
    rng = np.random.default_rng(6)
    x = W.normal(rng, (32, 64))
    amax = oracle.amax(x, colwise=True, rht=True, seed=1)
    a, _ = oracle.quantize_rows(x, np.array([3, 1]), amax, colwise=True, sr=True, rht=True, seed=1)
    b, _ = oracle.quantize_rows(x, np.array([1, 3]), amax, colwise=True, sr=True, rht=True, seed=1)
    np.testing.assert_array_equal(a[::-1], b)
    c, _ = oracle.quantize_rows(x, np.array([1, 3]), amax, colwise=True, sr=True, rht=True, seed=2)
    assert not np.array_equal(b, c)
