"""The GEMMs with the squared ReLU in their epilogue (nvfp4_gemm_relu2_fwd/bwd)
against the unfused calls and the oracle.

The MLP block of the 12B model runs up-projection -> relu^2 -> down-projection
in NVFP4 (hyper.ai, "NVIDIA revolutioniert KI-Praetrainingsgeschwindigkeit mit
4-Bit-Genauigkeit"; format: aisight.pl, section "Architektura NVFP4 kontra
ograniczenia mikroskalowania").  The fused epilogue must store exactly what
nvfp4_gemm + nvfp4_relu2_* store (bit for bit), the GEMM part within the
oracle's 1e-4 * sum|a_k b_k|, the activation bit-exact against the oracle's
relu^2 on the stored y, and both amax values (max |out| and max |RHT(out)|,
the transform of the Wgrad operands: same page, section "Technologie
stabilizujace proces treningowy") exactly as the oracle computes them."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B

from gpu_helpers import f32_bits, random_operand, upload

pytestmark = pytest.mark.gpu


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


SHAPES = [(256, 256, 256), (512, 768, 1024), (768, 512, 320)]


def operands(M, N, K, seed):
    rng = np.random.default_rng(seed)
    return random_operand(rng, M, K), random_operand(rng, N, K)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "%dx%dx%d" % s)
def test_relu2_fwd_epilogue(shape, cuda_lib):
    M, N, K = shape
    a, b = operands(M, N, K, M + N + K)
    A, Bt = upload(*a), upload(*b)
    y, h, am, amr = B.nvfp4_gemm_relu2_fwd(A, Bt, seed=77)
    y_ref = B.nvfp4_gemm(A, Bt, out_dtype=torch.bfloat16)
    y32 = B.nvfp4_gemm(A, Bt, out_dtype=torch.float32)
    h_ref, am_ref, amr_ref = B.nvfp4_relu2_fwd_amax_rht(y_ref, seed=77)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y), bits(y_ref))
    assert np.array_equal(bits(h), bits(h_ref))
    assert f32_bits(am[0].item()) == f32_bits(am_ref[0].item())
    assert f32_bits(amr[0].item()) == f32_bits(amr_ref[0].item())
    # against the oracle: the GEMM, then relu^2 and both amaxes of the stored values
    ref, ab = oracle.gemm(a, b)
    err = np.abs(y32.cpu().numpy().astype(np.float64) - ref)
    assert (err <= 1e-4 * ab).all()
    yb, hb = bits(y), bits(h)
    assert np.array_equal(hb, oracle.relu2_fwd(yb.ravel()).reshape(M, N))
    assert f32_bits(am[0].item()) == f32_bits(oracle.amax(hb))
    assert f32_bits(amr[0].item()) == f32_bits(oracle.amax(hb, colwise=True, rht=True, seed=77))


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "%dx%dx%d" % s)
def test_relu2_bwd_epilogue(shape, cuda_lib):
    M, N, K = shape
    a, b = operands(M, N, K, 3 * M + N + K)
    A, Bt = upload(*a), upload(*b)
    rng = np.random.default_rng(9)
    y_fwd = torch.from_numpy((rng.standard_normal((M, N)) * 2).astype(np.float32)).cuda().to(torch.bfloat16)
    dy, am, amr = B.nvfp4_gemm_relu2_bwd(A, Bt, y_fwd, seed=5)
    dh = B.nvfp4_gemm(A, Bt, out_dtype=torch.bfloat16)
    dy_ref, am_ref, amr_ref = B.nvfp4_relu2_bwd_amax_rht(dh, y_fwd, seed=5)
    torch.cuda.synchronize()
    assert np.array_equal(bits(dy), bits(dy_ref))
    assert f32_bits(am[0].item()) == f32_bits(am_ref[0].item())
    assert f32_bits(amr[0].item()) == f32_bits(amr_ref[0].item())
    db = bits(dy)
    assert np.array_equal(db, oracle.relu2_bwd(bits(dh).ravel(), bits(y_fwd).ravel()).reshape(M, N))
    assert f32_bits(am[0].item()) == f32_bits(oracle.amax(db))
    assert f32_bits(amr[0].item()) == f32_bits(oracle.amax(db, colwise=True, rht=True, seed=5))


def test_relu2_epilogue_full_size(cuda_lib):
    """The up-projection and the down-projection's Dgrad at the MLP's shapes."""
    M, N, K = 8192, 20480, 5120
    a, b = operands(M, N, K, 11)
    A, Bt = upload(*a), upload(*b)
    y, h, am, amr = B.nvfp4_gemm_relu2_fwd(A, Bt, seed=1234)
    h_ref, am_ref, amr_ref = B.nvfp4_relu2_fwd_amax_rht(y, seed=1234)
    dy, bm, bmr = B.nvfp4_gemm_relu2_bwd(A, Bt, y, seed=1234)
    dh = B.nvfp4_gemm(A, Bt, out_dtype=torch.bfloat16)
    assert torch.equal(dh, y)
    dy_ref, bm_ref, bmr_ref = B.nvfp4_relu2_bwd_amax_rht(dh, y, seed=1234)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), h_ref.view(torch.int16))
    assert torch.equal(dy.view(torch.int16), dy_ref.view(torch.int16))
    for x, r in ((am, am_ref), (amr, amr_ref), (bm, bm_ref), (bmr, bmr_ref)):
        assert f32_bits(x[0].item()) == f32_bits(r[0].item())


def test_relu2_epilogue_rejects_ragged(cuda_lib):
    a, b = operands(200, 256, 256, 1)
    with pytest.raises(B.NVFP4Error) as e:
        B.nvfp4_gemm_relu2_fwd(upload(*a), upload(*b))
    assert e.value.status == B.NVFP4_ERR_SHAPE
