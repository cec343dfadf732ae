"""Pins for the oracle's Philox4x32-10 and 16-point random Hadamard transform.

Philox4x32-10 (Salmon et al., SC'11) is checked against torch's independent
header-only engine (ATen/core/PhiloxRNGEngine.h), compiled here with g++.
The Hadamard transform ("losowe transformaty Hadamarda" on the weight
gradients: aisight.pl, section "Technologie stabilizujace proces treningowy")
is checked against closed forms: H H^T = 16 I, columns (-1)^popcount(i&j),
the transform's orthonormality and its self-inverse property.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch.utils.cpp_extension as cpp

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def torch_philox(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("philox") / "philox_torch_ref")
    inc = [f"-I{p}" for p in cpp.include_paths()]
    subprocess.check_call(["g++", "-O1", "-std=c++17", *inc,
                           os.path.join(HERE, "helpers", "philox_torch_ref.cpp"), "-o", exe])

    def run(rows):
        text = "\n".join(" ".join(str(int(v)) for v in r) for r in rows) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        return np.array([[int(v) for v in line.split()] for line in out.strip().splitlines()],
                        dtype=np.uint64)
    return run


def test_philox_matches_torch_engine(torch_philox):
    rng = np.random.default_rng(7)
    rows = [[0, 0, 0, 0, 0, 0], [2 ** 32 - 1] * 6, [1234, 0, 0, 0, 1, 0], [1234, 0, 5, 0, 0, 0]]
    rows += rng.integers(0, 2 ** 32, size=(400, 6), dtype=np.uint64).tolist()
    ref = torch_philox(rows)
    got = np.array([oracle.philox4x32_10(r[2:], r[:2]) for r in rows], dtype=np.uint64)
    assert np.array_equal(got, ref)


def test_rht_signs_come_from_philox_word():
    seed = 1234
    w = oracle.philox4x32_10([0, 0, 1, 0], [seed & 0xFFFFFFFF, seed >> 32])[0]
    d = oracle.rht_signs(seed)
    for j in range(16):
        assert d[j] == (-1.0 if (int(w) >> j) & 1 else 1.0)
    assert set(np.unique(d)) <= {-1.0, 1.0}


def hadamard_from_oracle():
    return np.stack([oracle.fwht16(np.eye(16, dtype=np.float32)[j]) for j in range(16)], axis=1)


def test_hadamard_closed_form_and_orthogonality():
    H = hadamard_from_oracle().astype(np.float64)
    closed = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(16)] for i in range(16)])
    assert np.array_equal(H, closed)
    assert np.array_equal(H @ H.T, 16 * np.eye(16))


def test_rht_is_orthonormal_and_self_inverse():
    rng = np.random.default_rng(11)
    d = oracle.rht_signs(1234)
    for _ in range(200):
        v = rng.standard_normal(16).astype(np.float32)
        y = oracle.rht16(v, d)
        # norm preserved (orthonormal transform), up to fp32 rounding
        assert abs(np.linalg.norm(y.astype(np.float64)) - np.linalg.norm(v.astype(np.float64))) \
            <= 1e-5 * np.linalg.norm(v)
        # Q^T y = D (H/4) y recovers v
        back = (oracle.fwht16(y) * np.float32(0.25)) * d
        assert np.allclose(back, v, rtol=0, atol=4e-7 * max(1.0, np.abs(v).max()))
    # exact on small integers: the butterfly adds exactly
    v = np.arange(16, dtype=np.float32) - 7
    assert np.array_equal(oracle.rht16(v, np.ones(16, np.float32)),
                          (hadamard_from_oracle() @ v / 4).astype(np.float32))


def test_rht_preserves_wgrad_product():
    """(Q dY)^T (Q X) = dY^T X when Q is applied to every 16-row block of both."""
    rng = np.random.default_rng(12)
    d = oracle.rht_signs(99)
    T, n, m = 64, 5, 3
    dY = rng.standard_normal((T, n)).astype(np.float32)
    X = rng.standard_normal((T, m)).astype(np.float32)

    def q(A):
        out = np.empty_like(A)
        for c in range(A.shape[1]):
            for g in range(0, A.shape[0], 16):
                out[g:g + 16, c] = oracle.rht16(A[g:g + 16, c], d)
        return out
    lhs = q(dY).astype(np.float64).T @ q(X).astype(np.float64)
    rhs = dY.astype(np.float64).T @ X.astype(np.float64)
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-5 * np.abs(rhs).max())
    # a transform without the sign diagonal or scaling would not preserve it
    assert not np.allclose(q(dY).astype(np.float64).T @ X.astype(np.float64), rhs, atol=1e-3)
