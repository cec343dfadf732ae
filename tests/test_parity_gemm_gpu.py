"""GPU block-scaled NVFP4 GEMM vs the oracle's FP64 dot products, per element
|gpu - ref| <= 1e-4 * sum|a_k b_k|, through the C ABI.  Operands come from the
oracle's quantiser or are random NVFP4 tensors generated on the host; the same
operand bytes go to both sides."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import assert_gemm_close, random_operand, upload

pytestmark = pytest.mark.gpu


def run_gemm(a, b, out_dtype=torch.float32):
    A, Bt = upload(*a), upload(*b)
    ws = B.workspace(256)
    out = B.nvfp4_gemm(A, Bt, out_dtype=out_dtype, ws=ws)
    B.nvfp4_check(ws)
    return out


SHAPES = [(256, 256, 256), (128, 256, 64), (1, 8, 64), (200, 392, 320), (384, 640, 1024), (520, 264, 2112),
          (1000, 1000, 1024), (300, 520, 640), (264, 392, 704)]  # K % 256 = 0, 64, 128, 192: every stage length


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "%dx%dx%d" % s)
def test_random_operands(shape, cuda_lib):
    M, N, K = shape
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    a, b = random_operand(rng, M, K), random_operand(rng, N, K)
    got = run_gemm(a, b).cpu().numpy()
    ref, ab = oracle.gemm(a, b)
    assert_gemm_close(got, ref, ab, "f32 out")
    got16 = run_gemm(a, b, torch.bfloat16)
    assert torch.equal(got16.cpu(), torch.from_numpy(got).to(torch.bfloat16)), "bf16 out != RN(f32 out)"


def test_unit_scales_exact(cuda_lib):
    """Unit scales: every partial sum is a small multiple of 0.25, exact in FP32."""
    rng = np.random.default_rng(5)
    a, b = random_operand(rng, 256, 4096, unit=True), random_operand(rng, 512, 4096, unit=True)
    got = run_gemm(a, b).cpu().numpy().astype(np.float64)
    ref, _ = oracle.gemm(a, b)
    assert np.array_equal(got, ref)


def test_quantized_tiny_workload(cuda_lib):
    """The tiny workload end to end: oracle-quantised X, W (RTN), GPU GEMM, FP32 out."""
    w = W.tiny()
    qx = oracle.quantize(w["X"])
    qw = oracle.quantize(w["W"])
    a, b = qx[:3], qw[:3]
    got = run_gemm(a, b).cpu().numpy()
    ref, ab = oracle.gemm(a, b)
    assert_gemm_close(got, ref, ab, "tiny")


def test_k_zero_and_empty(cuda_lib):
    e = B.NVFP4Tensor(codes=torch.zeros(1, dtype=torch.uint8, device="cuda"),
                      scales=torch.zeros(16, dtype=torch.uint8, device="cuda"),
                      tensor_scale=torch.ones(1, device="cuda"), rows=64, k=0)
    out = torch.full((64, 64), 7.0, device="cuda")
    B.nvfp4_gemm(e, e, out=out)
    torch.cuda.synchronize()
    assert not out.any()


@pytest.mark.parametrize("shape", [(8192, 20480, 5120), (20480, 5120, 16384)], ids=["fprop", "wgrad"])
def test_full_size_sampled(shape, cuda_lib):
    M, N, K = shape
    rng = np.random.default_rng(11)
    a, b = random_operand(rng, M, K), random_operand(rng, N, K)
    got = run_gemm(a, b)
    ms = np.concatenate([[0, M - 1, 0, M - 1], rng.integers(0, M, 1500)])
    ns = np.concatenate([[0, N - 1, N - 1, 0], rng.integers(0, N, 1500)])
    g = got[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()].cpu().numpy()
    ref, ab = oracle.gemm_sampled(a, b, ms, ns)
    assert_gemm_close(g, ref, ab, "sampled")
