"""Pins for the oracle's element and scale formats (CPU only).

E2M1 and E4M3 encoders are checked against brute-force nearest-value scans
over every code (decoded here from the literal value sets), and the E4M3
decode/encode against torch's float8_e4m3fn casts (an independent library).
The toy rounding example is the one on aibuzzwire.news, Thinking Machines
"End-to-End 4-Bit Training", section "Warum weniger Bits ein schnelleres
Training bedeuten": a grid holding only 3 and 4 rounds 3.2 to 3, error 0.2.
"""
import numpy as np
import pytest
import torch

import oracle

# The E2M1 value set, written out: +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}; codes 0..7 positive, 8..15 negative.
E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_literal_values():
    """Every finite positive E4M3 ('fn') value from the definition: subnormals m*2^-9,
    normals 2^(E-7)*(1+m/8) for E=1..15 except (15,7) which is NaN."""
    vals = []
    for code in range(0x7F):
        E, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if E == 0 else 2.0 ** (E - 7) * (1 + m / 8))
    return np.array(vals)


def nearest_code(values, grid, code_of_index):
    """Brute force: index of the nearest grid value to each input; ties -> even code."""
    v = np.asarray(values, np.float64)[:, None]
    d = np.abs(v - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    codes = np.array(code_of_index)
    out = np.empty(v.shape[0], np.int64)
    for i in range(v.shape[0]):
        c = codes[cand[i]]
        out[i] = c[0] if len(c) == 1 else c[(c & 1) == 0][0]
    return out


def test_e2m1_decode_table():
    for code in range(16):
        expect = E2M1_MAGS[code & 7] * (-1.0 if code & 8 else 1.0)
        got = oracle.e2m1_value(code)
        assert got == expect and np.signbit(got) == bool(code & 8)


def test_e2m1_rtn_bruteforce():
    grid = np.arange(-8, 8, 1 / 64, dtype=np.float32)
    ties = (E2M1_MAGS[1:] + E2M1_MAGS[:-1]) / 2
    near = np.concatenate([ties, np.nextafter(ties.astype(np.float32), np.float32(0)),
                           np.nextafter(ties.astype(np.float32), np.float32(10))])
    rng = np.random.default_rng(0)
    vals = np.concatenate([grid, near, -near, rng.uniform(-9, 9, 20000).astype(np.float32),
                           np.array([6.0, 7.0, 1e30, 5.999999], np.float32)]).astype(np.float32)
    got = oracle.e2m1_rtn_array(vals)
    mags = np.minimum(np.abs(vals.astype(np.float64)), 6.0)  # satfinite: beyond 6 -> 6
    idx = nearest_code(mags, E2M1_MAGS, list(range(8)))
    expect = idx | np.where(np.signbit(vals), 8, 0)
    assert np.array_equal(got.astype(np.int64), expect)


def test_e2m1_named_ties():
    for r, v in [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0),
                 (5.0, 4.0), (6.5, 6.0), (100.0, 6.0)]:
        assert oracle.e2m1_value(oracle.e2m1_rtn(r)) == v
        assert oracle.e2m1_value(oracle.e2m1_rtn(-r)) == -v
    assert oracle.e2m1_rtn(-0.1) == 0x8  # negative zero keeps its sign
    assert oracle.e2m1_rtn(0.0) == 0x0


def test_toy_rounding_example():
    """3.2 on a grid holding only 3 and 4: RTN gives 3 with error 0.2."""
    q = oracle.e2m1_rtn(3.2)
    assert oracle.e2m1_value(q) == 3.0
    assert abs(np.float32(3.2) - oracle.e2m1_value(q) - 0.2) < 1e-6
    # SR never leaves {3, 4} and is biased by at most 2^-16 for each draw level
    ups = [oracle.e2m1_value(oracle.e2m1_sr(3.2, u)) for u in range(0, 65536, 97)]
    assert set(ups) == {3.0, 4.0}


def test_e2m1_sr_neighbours_and_exact():
    rng = np.random.default_rng(1)
    r = rng.uniform(-7, 7, 50000).astype(np.float32)
    u = rng.integers(0, 65536, r.size).astype(np.uint32)
    got = np.array([oracle.e2m1_value(c) for c in oracle.e2m1_sr_array(r, u)])
    a = np.minimum(np.abs(r.astype(np.float64)), 6.0)
    lower = np.array([E2M1_MAGS[E2M1_MAGS <= x].max() for x in a])
    upper = np.array([E2M1_MAGS[E2M1_MAGS >= x].min() for x in a])
    assert np.all((np.abs(got) == lower) | (np.abs(got) == upper))
    assert np.all(np.signbit(got) == np.signbit(r))
    # representable values never move, whatever the draw
    for v in E2M1_MAGS:
        for uu in (0, 1, 32768, 65535):
            assert oracle.e2m1_value(oracle.e2m1_sr(v, uu)) == v


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~finite)
    assert np.array_equal(got[finite], ref[finite])
    assert oracle.e4m3_value(0x7E) == 448.0


def _e4m3_sweep_values():
    vals = e4m3_literal_values()
    mids = (vals[1:] + vals[:-1]) / 2  # every tie point
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)  # ties are exact in fp32
    rng = np.random.default_rng(2)
    # every 97th binary32 bit pattern between 2^-12 and 512
    lo = np.array([2.0 ** -12], np.float32).view(np.uint32)[0]
    hi = np.array([512.0], np.float32).view(np.uint32)[0]
    strided = np.arange(lo, hi, 97, dtype=np.uint32).view(np.float32)
    extra = np.concatenate([mids32, np.nextafter(mids32, np.float32(0)), np.nextafter(mids32, np.float32(1e9)),
                            vals.astype(np.float32), rng.uniform(0, 500, 100000).astype(np.float32),
                            np.array([0.0, 1e-30, 2.0 ** -10, 448.0, 463.99, 464.0, 1e6], np.float32)])
    return np.concatenate([strided, extra]).astype(np.float32)


def test_e4m3_rn_bruteforce():
    t = _e4m3_sweep_values()
    got = oracle.e4m3_rn_array(t).astype(np.int64)
    grid = e4m3_literal_values()
    clamped = np.minimum(t.astype(np.float64), 448.0)  # satfinite
    expect = np.empty_like(got)
    chunk = 1 << 16
    for s in range(0, t.size, chunk):
        v = clamped[s:s + chunk, None]
        d = np.abs(v - grid[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        first = cand.argmax(axis=1)
        two = cand.sum(axis=1) == 2
        # tie: the two candidates are adjacent codes; pick the even one
        pick = np.where(two & (first % 2 == 1), first + 1, first)
        expect[s:s + chunk] = pick
    assert np.array_equal(got, expect)


def test_e4m3_rn_matches_torch_cast_in_range():
    t = _e4m3_sweep_values()
    t = t[t <= 448.0]
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    got = oracle.e4m3_rn_array(t).astype(np.int64)
    assert np.array_equal(got, ref)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    f = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        (rng.integers(0, 2 ** 32, 100000, dtype=np.uint64).astype(np.uint32)
                         & np.uint32(0x7F7FFFFF)).view(np.float32),
                        np.array([0x3F808000, 0x3F818000, 0x3F80FFFF], np.uint32).view(np.float32)])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_f32(x) for x in f[:5000]] +
                   [oracle.bf16_from_f32(x) for x in f[-3:]], np.uint16)
    assert np.array_equal(got, np.concatenate([ref[:5000], ref[-3:]]))
