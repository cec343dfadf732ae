"""The quantisation kernels take the stochastic-rounding decision on the binary32
bit pattern instead of computing frac(|r|/spacing) and comparing it with the
draw (both give reading R7: round the magnitude up iff u < frac, u = rnd16 /
2^16; stochastic rounding of the gradients is named on aisight.pl, section
"Technologie stabilizujace proces treningowy").  This file restates the
kernels' steps in numpy and checks them against the oracle's SR encoder on
every draw at and beside each decision threshold and on a strided sweep of
all binary32 values in (-16, 16); the GPU parity tests check the kernels
themselves.

The steps: for |r| >= 1 the grid spacing is the weight of the first mantissa
bit, so adding 2^22 - 1 - rnd16 * 2^6 to the bit pattern carries into bit 22
exactly when the low 22 mantissa bits exceed rnd16 * 2^6; clearing them rounds.
For |r| < 1 the same is done to 1 + |r| rounded up to binary32, then 1 is
subtracted.  Magnitudes are clamped to 7 first, so every result is a grid
value or 8, and the saturating E2M1 conversion takes 8 to 6.
"""
import numpy as np

import oracle

GRID_CODE = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def below_one(a):
    """The kernels' offset: sat(2^24 - 2^24 a) as one binary32 FMA (the exact value,
    formed in float64 where it is exact for a binary32 a, rounded once)."""
    v = (2.0 ** 24 - 2.0 ** 24 * np.asarray(a, dtype=np.float64)).astype(np.float32)
    return np.clip(v, np.float32(0.0), np.float32(1.0)).astype(np.float32)


def round_bits(t_bits, rnd16):
    """The kernels' rounding step: bits + 2^22 - 1 - 64 rnd16 (mod 2^32), low 22 bits cleared."""
    t_bits = np.asarray(t_bits, dtype=np.uint32)
    rnd16 = np.asarray(rnd16, dtype=np.uint32)
    with np.errstate(over="ignore"):
        return (t_bits + np.uint32(0x3FFFFF) + rnd16 * np.uint32(0xFFFFFFC0)) & np.uint32(0xFFC00000)


def test_offset_and_constant_forms():
    """The offset equals [a < 1] for every binary32 a in [0, 8) on a dense sweep and at 1's
    neighbours; the rounding constant equals the carry (2^16 - 1 - rnd16) * 2^6 + 63 for
    every draw."""
    a = np.arange(0, 0x41000000, 97, dtype=np.uint32).view(np.float32)
    a = np.concatenate([a, np.float32([0.0, np.nextafter(np.float32(1), np.float32(0)), 1.0,
                                       np.nextafter(np.float32(1), np.float32(2)), 7.0])])
    assert np.array_equal(below_one(a), (a < np.float32(1.0)).astype(np.float32))
    rnd = np.arange(65536, dtype=np.uint32)
    carry = (((~rnd) & np.uint32(0xFFFF)) << np.uint32(6)) | np.uint32(63)
    t = np.uint32(0x40E00000)  # 7.0
    with np.errstate(over="ignore"):
        assert np.array_equal(round_bits(np.full(rnd.shape, t), rnd), (t + carry) & np.uint32(0xFFC00000))
    assert np.array_equal(np.uint32(0x3FFFFF) + rnd * np.uint32(0xFFFFFFC0), carry)


def bit_pattern_sr(r, rnd16):
    """Codes from the kernels' bit-pattern SR decision (numpy restatement)."""
    r = np.asarray(r, dtype=np.float32)
    rnd16 = np.asarray(rnd16, dtype=np.uint32)
    a = np.minimum(np.abs(r), np.float32(7.0))
    small = a < np.float32(1.0)
    base = below_one(a)
    # 1 + a rounded up to binary32 (exact in float64: a * 2^23 is an integer-valued double)
    up_sum = (1.0 + np.ceil(a.astype(np.float64) * 2.0 ** 23) / 2.0 ** 23).astype(np.float32)
    t = np.where(small, up_sum, a).astype(np.float32)
    with np.errstate(over="ignore"):
        bits = round_bits(t.view(np.uint32), rnd16)
    mag = bits.view(np.float32) - base
    assert (mag <= np.float32(8.0)).all()
    mag = np.where(mag == np.float32(8.0), np.float32(6.0), mag)  # the conversion's saturation
    codes = np.full(mag.shape, 255, dtype=np.uint8)
    for v, c in GRID_CODE.items():
        codes[mag == np.float32(v)] = c
    assert (codes != 255).all(), "a magnitude off the E2M1 grid"
    sign = (r.view(np.uint32) >> np.uint32(31)).astype(np.uint8) << np.uint8(3)
    return codes | sign


def _check(r, rnd):
    r = np.ascontiguousarray(r, dtype=np.float32)
    rnd = np.ascontiguousarray(rnd, dtype=np.uint32)
    got = bit_pattern_sr(r, rnd)
    want = oracle.e2m1_sr_array(r, rnd)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(r[i]), int(rnd[i]), int(got[i]), int(want[i])) for i in bad[:5]]


def test_every_draw_at_each_threshold():
    rnd = np.arange(65536, dtype=np.uint32)
    for lo, step in [(0.0, 0.5), (0.5, 0.5), (1.0, 0.5), (1.5, 0.5), (2.0, 1.0), (3.0, 1.0), (4.0, 2.0)]:
        thr = (lo + step * rnd.astype(np.float64) / 65536.0).astype(np.float32)  # exact
        cands = [thr, np.nextafter(thr, np.float32(0)), np.nextafter(thr, np.float32(100)),
                 np.nextafter(np.nextafter(thr, np.float32(100)), np.float32(100)),
                 (lo + step * (rnd.astype(np.float64) + 0.5) / 65536.0).astype(np.float32)]
        for c in cands:
            _check(c, rnd)
            _check(-c, rnd)


def test_strided_sweep_of_all_binary32_below_16():
    lim = int(np.float32(16.0).view(np.uint32))
    bits = np.arange(0, lim + 1, 89, dtype=np.uint32)      # every 89th pattern, all binades
    r = bits.view(np.float32)
    rng = np.random.default_rng(5)
    for rnd in [np.zeros_like(bits), np.full_like(bits, 0xFFFF), rng.integers(0, 65536, bits.size, dtype=np.uint32)]:
        _check(r, rnd)
        _check(-r, rnd)


def test_large_and_special_magnitudes():
    rng = np.random.default_rng(6)
    e = rng.integers(130, 255, 200000, dtype=np.uint32)
    m = rng.integers(0, 1 << 23, 200000, dtype=np.uint32)
    bits = (e << np.uint32(23)) | m
    bits[:3] = [0x7F7FFFFF, 0x40C00000, 0x40BFFFFF]          # FLT_MAX, 6, just below 6
    r = bits.view(np.float32)
    rnd = rng.integers(0, 65536, r.size, dtype=np.uint32)
    rnd[:3] = 0
    _check(r, rnd)
    _check(-r, rnd)
    sub = np.arange(1, 200001, dtype=np.uint32).view(np.float32)  # subnormals
    _check(sub, np.zeros(sub.size, dtype=np.uint32))
    _check(sub, np.full(sub.size, 0xFFFF, dtype=np.uint32))
    _check(np.array([0.0, -0.0], dtype=np.float32), np.array([0, 0], dtype=np.uint32))
