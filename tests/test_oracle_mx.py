"""Pins of the oracle's MXFP4 functions (blocks of 32, E8M0 power-of-two
scale, no tensor scale) against facts fixed by the format definition and by
the round-to-nearest-even rule: E8M0 values, the shared exponent on binade
boundaries, an exact round trip of every E2M1 code at many exponents,
saturation, and the RTN error bound.  CPU only."""
import math

import numpy as np
import pytest

import oracle

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e8m0_values():
    assert oracle.e8m0_value(127) == 1.0
    assert oracle.e8m0_value(0) == 2.0 ** -127
    assert oracle.e8m0_value(254) == 2.0 ** 127
    assert oracle.e8m0_value(130) == 8.0
    assert math.isnan(oracle.e8m0_value(255))


@pytest.mark.parametrize("amax,x", [
    (6.0, 0), (4.0, 0), (7.999, 0), (8.0, 1), (3.999, -1), (2.0, -1), (1.0, -2), (0.75, -3),
    (2.0 ** 100 * 1.5, 98), (2.0 ** 127 * 1.9, 125), (2.0 ** -120, -122), (2.0 ** -125, -127),
    (2.0 ** -126, -127), (1e-45, -127), (0.0, -127)])
def test_shared_exponent_on_binade_boundaries(amax, x):
    # X = floor(log2 amax) - 2, clamped to [-127, 127]; the amax values are exact float32
    assert np.float32(amax) == amax or amax in (7.999, 3.999, 0.75, 1e-45)
    assert oracle.mx_scale(np.float32(amax)) == x + 127


def _pack(codes_row):
    c = np.asarray(codes_row, np.uint8)
    return c[0::2] | (c[1::2] << 4)


@pytest.mark.parametrize("x", [-127, -100, -9, -2, 0, 1, 5, 40, 120, 125])
def test_every_code_round_trips(x):
    """A block whose largest magnitude is 6 * 2^X (so its shared exponent is X) and
    whose other elements are E2M1 values times 2^X quantises to exactly those codes."""
    rng = np.random.default_rng(x + 200)
    rows = []
    want_codes = []
    for _ in range(8):
        codes = rng.integers(0, 16, 32)
        codes[rng.integers(0, 32)] = 7 | (8 if rng.random() < 0.5 else 0)  # +-6 sets the exponent
        vals = [(-1.0 if c & 8 else 1.0) * E2M1[c & 7] * 2.0 ** x for c in codes]
        rows.append(vals)
        want_codes.append(codes)
    xs = np.array(rows, np.float32)
    assert np.all(xs.astype(np.float64) == np.array(rows))  # exactly representable inputs
    got_codes, got_scales = oracle.quantize_mx(xs)
    assert np.all(got_scales == x + 127)
    for r in range(8):
        assert np.array_equal(got_codes[r], _pack(want_codes[r]))
    assert np.array_equal(oracle.dequantize_mx(got_codes, got_scales), np.array(rows))


def test_saturation_and_packing_order():
    v = np.zeros((1, 32), np.float32)
    v[0, 0], v[0, 1], v[0, 2], v[0, 3] = 7.5, -7.9, 0.25, 0.26   # amax 7.9 -> X = 0
    codes, scales = oracle.quantize_mx(v)
    assert scales[0, 0] == 127
    assert codes[0, 0] == (0x7 | (0xF << 4))            # 7.5 -> +6, -7.9 -> -6
    assert codes[0, 1] == (0x0 | (0x1 << 4))            # 0.25 ties to even (0), 0.26 -> 0.5


def test_zero_block_and_bf16_input():
    z = np.zeros((2, 64), np.uint16)
    codes, scales = oracle.quantize_mx(z)
    assert not codes.any() and not scales.any()
    with pytest.raises(ValueError):
        oracle.quantize_mx(np.zeros((2, 48), np.float32))   # C % 32 != 0


def test_rtn_error_bound():
    """|v - deq| <= half the E2M1 spacing of v's scaled binade (times 2^X), unless
    |v| 2^-X >= 6 (saturation, |deq| = 6 2^X)."""
    rng = np.random.default_rng(3)
    xs = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)) * 4)).astype(np.float32)
    codes, scales = oracle.quantize_mx(xs)
    deq = oracle.dequantize_mx(codes, scales)
    scale = np.repeat(2.0 ** (scales.astype(np.float64) - 127), 32, axis=1)
    a = np.abs(xs.astype(np.float64)) / scale
    spacing = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    err = np.abs(xs - deq) / scale
    sat = a >= 6
    assert np.all(err[~sat] <= spacing[~sat] / 2 + 1e-12)
    assert np.all(np.abs(deq[sat]) / scale[sat] == 6.0)
    # the shared exponent keeps every scaled magnitude below 8: at most one binade saturates
    assert np.all(a < 8.0)


def test_nvfp4_error_below_mxfp4():
    """The pages' comparison: NVFP4 (16-element blocks, E4M3 scales, FP32 tensor scale)
    keeps less quantisation error than MXFP4 (32-element blocks, power-of-two scales)
    on the same data.  Relative RMS error on normal and heavy-tailed synthetic tensors."""
    rng = np.random.default_rng(11)
    cases = {"normal": rng.standard_normal((256, 1024)).astype(np.float32),
             "heavy_rows": (rng.standard_normal((256, 1024)) * np.abs(rng.standard_t(2, (256, 1)))).astype(
                 np.float32)}
    for name, x in cases.items():
        c, s, ts, _ = oracle.quantize(x)
        e_nv = np.linalg.norm(oracle.dequantize(c, s, ts) - x) / np.linalg.norm(x)
        cm, sm = oracle.quantize_mx(x)
        e_mx = np.linalg.norm(oracle.dequantize_mx(cm, sm) - x) / np.linalg.norm(x)
        assert e_nv < e_mx, (name, e_nv, e_mx)


def test_colwise_is_rowwise_of_the_transpose():
    """Colwise MXFP4 of x (blocks down the rows, transposed output) is, by definition of
    the orientation, the rowwise MXFP4 of x^T."""
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((96, 40)) * np.exp(rng.standard_normal((96, 1)))).astype(np.float32)
    c1, s1 = oracle.quantize_mx(x, colwise=True)
    c2, s2 = oracle.quantize_mx(np.ascontiguousarray(x.T))
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    with pytest.raises(ValueError):
        oracle.quantize_mx(np.zeros((48, 64), np.float32), colwise=True)   # R % 32 != 0


# ---------------------------------------------------------------- MXFP4 GEMM
def _pack_rows(codes):
    codes = np.asarray(codes, np.uint8)
    return codes[:, 0::2] | (codes[:, 1::2] << 4)


def test_gemm_mx_closed_form():
    """Every element of a row holds one code c and every block the row's exponent x:
    C[m, n] = K * e2m1(c_m) * e2m1(c_n) * 2^(x_m + x_n) exactly."""
    rng = np.random.default_rng(31)
    M, N, K = 5, 7, 96
    ca, cb = rng.integers(0, 16, M), rng.integers(0, 16, N)
    xa, xb = rng.integers(-20, 21, M), rng.integers(-20, 21, N)
    a = (_pack_rows(np.repeat(ca[:, None], K, 1)), np.repeat((xa + 127)[:, None], K // 32, 1).astype(np.uint8))
    b = (_pack_rows(np.repeat(cb[:, None], K, 1)), np.repeat((xb + 127)[:, None], K // 32, 1).astype(np.uint8))
    ref, ab = oracle.gemm_mx(a, b)
    val = lambda c: (-1.0 if c & 8 else 1.0) * E2M1[c & 7]  # noqa: E731
    want = np.array([[K * val(ca[m]) * val(cb[n]) * 2.0 ** (xa[m] + xb[n]) for n in range(N)] for m in range(M)])
    assert np.array_equal(ref, want)
    assert np.array_equal(ab, np.abs(want))


def test_gemm_mx_one_hot_indexing():
    """One nonzero per row at a known k, each 32-block with its own exponent: the product
    is nonzero only where the positions meet, with both blocks' scales -- this pins
    the nibble order and the block index k // 32."""
    rng = np.random.default_rng(32)
    K, R = 128, 12
    pos_a, pos_b = rng.integers(0, K, R), rng.integers(0, K, R)
    pos_b[:4] = pos_a[:4]
    ea, eb = rng.integers(100, 150, (R, K // 32)), rng.integers(100, 150, (R, K // 32))
    codes_a, codes_b = np.zeros((R, K), np.uint8), np.zeros((R, K), np.uint8)
    codes_a[np.arange(R), pos_a] = 5   # 3.0
    codes_b[np.arange(R), pos_b] = 11  # -1.5
    ref, _ = oracle.gemm_mx((_pack_rows(codes_a), ea.astype(np.uint8)), (_pack_rows(codes_b), eb.astype(np.uint8)))
    for m in range(R):
        for n in range(R):
            k = pos_a[m]
            want = 3.0 * -1.5 * 2.0 ** (int(ea[m, k // 32]) - 127 + int(eb[n, k // 32]) - 127) if k == pos_b[n] else 0.0
            assert ref[m, n] == want, (m, n)


def _e4m3_code_of(v):
    return next(c for c in range(127) if oracle.e4m3_value(c) == v)


def test_gemm_mx_equals_nvfp4_gemm_on_shared_scales():
    """An MXFP4 tensor whose block exponents are also E4M3 values is the NVFP4 tensor
    with that scale on both 16-halves of each 32-block and tensor scale 1: the two
    oracles' FP64 GEMMs (independent scale decoders and block sizes) agree exactly."""
    rng = np.random.default_rng(33)
    M, N, K = 9, 11, 160
    def operand(rows):
        codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
        x = rng.integers(-9, 9, (rows, K // 32))                  # 2^x is an E4M3 value for x in [-9, 8]
        e8 = (x + 127).astype(np.uint8)
        e4 = np.array([[_e4m3_code_of(2.0 ** int(v)) for v in row] for row in x], np.uint8)
        return (codes, e8), (codes, np.repeat(e4, 2, axis=1), np.float32(1.0))
    (amx, anv), (bmx, bnv) = operand(M), operand(N)
    ref_mx, ab_mx = oracle.gemm_mx(amx, bmx)
    ref_nv, ab_nv = oracle.gemm(anv, bnv)
    assert np.array_equal(ref_mx, ref_nv)
    assert np.array_equal(ab_mx, ab_nv)


def test_gemm_mx_of_quantised_operands_tracks_the_product():
    """gemm_mx(quantize_mx(X), quantize_mx(W)) approximates X W^T, and less closely
    than the NVFP4 path on the same data (the pages' point about finer scaling)."""
    rng = np.random.default_rng(34)
    X = rng.standard_normal((64, 512)).astype(np.float32)
    W = rng.standard_normal((48, 512)).astype(np.float32)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    ref_mx, _ = oracle.gemm_mx(oracle.quantize_mx(X), oracle.quantize_mx(W))
    ref_nv, _ = oracle.gemm(oracle.quantize(X)[:3], oracle.quantize(W)[:3])
    err_mx = np.linalg.norm(ref_mx - exact) / np.linalg.norm(exact)
    err_nv = np.linalg.norm(ref_nv - exact) / np.linalg.norm(exact)
    assert err_mx < 0.25 and err_nv < err_mx, (err_mx, err_nv)


def test_gemm_mx_rejects_mismatched_operands():
    c, s = np.zeros((4, 16), np.uint8), np.zeros((4, 1), np.uint8)
    with pytest.raises(ValueError):
        oracle.gemm_mx((c, s), (np.zeros((4, 32), np.uint8), np.zeros((4, 2), np.uint8)))
    with pytest.raises(ValueError):
        oracle.gemm_mx((c, np.zeros((4, 2), np.uint8)), (c, s))
