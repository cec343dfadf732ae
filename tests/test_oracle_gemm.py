"""Pins for the oracle's block-scaled NVFP4 GEMM in binary64 (CPU only).

With unit scales every product is a multiple of 0.25 and every partial sum is
exact in binary64, so the oracle must equal numpy's matmul of the decoded
values exactly.  With random scales it must agree with numpy to rounding.
The operand values are decoded here from the literal E2M1 / E4M3 definitions,
not from the oracle.
"""
import numpy as np

import oracle

from test_oracle_formats import E2M1_MAGS, e4m3_literal_values

E2M1_SIGNED = np.concatenate([E2M1_MAGS, -E2M1_MAGS])


def decode(codes, scales, ts):
    e4 = np.concatenate([e4m3_literal_values(), [np.nan]])
    q = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    return E2M1_SIGNED[q] * np.repeat(e4[scales], 16, axis=1) * float(ts)


def random_operand(rng, rows, K, unit=False):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    if unit:
        scales = np.full((rows, K // 16), 0x38, np.uint8)  # E4M3 1.0
        ts = np.float32(1.0)
    else:
        scales = rng.integers(0, 0x7F, size=(rows, K // 16), dtype=np.uint8)
        ts = np.float32(rng.uniform(1e-3, 1e-1))
    return codes, scales, ts


def test_unit_scales_exact():
    rng = np.random.default_rng(0)
    a = random_operand(rng, 37, 256, unit=True)
    b = random_operand(rng, 29, 256, unit=True)
    ref, ab = oracle.gemm(a, b)
    A, B = decode(*a), decode(*b)
    assert np.array_equal(ref, A @ B.T)
    assert np.array_equal(ab, np.abs(A) @ np.abs(B).T)


def test_random_scales_close_to_numpy():
    rng = np.random.default_rng(1)
    a = random_operand(rng, 20, 512)
    b = random_operand(rng, 24, 512)
    ref, ab = oracle.gemm(a, b)
    A, B = decode(*a), decode(*b)
    expect = A @ B.T
    assert np.all(np.abs(ref - expect) <= 1e-13 * (np.abs(A) @ np.abs(B).T))
    assert np.all(ab >= np.abs(ref))


def test_orientation_and_sampling():
    rng = np.random.default_rng(2)
    a = random_operand(rng, 16, 128)
    b = random_operand(rng, 40, 128)
    ref, ab = oracle.gemm(a, b)
    refT, _ = oracle.gemm(b, a)
    assert np.array_equal(ref, refT.T)
    ms = rng.integers(0, 16, 50)
    ns = rng.integers(0, 40, 50)
    sref, sab = oracle.gemm_sampled(a, b, ms, ns)
    assert np.array_equal(sref, ref[ms, ns]) and np.array_equal(sab, ab[ms, ns])


def test_dequantize_matches_literal_decode():
    rng = np.random.default_rng(3)
    c, s, ts = random_operand(rng, 8, 64)
    assert np.array_equal(oracle.dequantize(c, s, ts), decode(c, s, ts))
