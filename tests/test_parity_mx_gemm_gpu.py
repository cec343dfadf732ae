"""MXFP4 GEMM (nvfp4_gemm_mx, tcgen05 kind::mxf4 with E8M0 block scales) against
the oracle's FP64 dot products, per element |gpu - ref| <= 1e-4 * sum|a_k b_k|.

MXFP4 is the format the pages compare NVFP4 with (aisight.pl, section
"Architektura NVFP4 kontra ograniczenia mikroskalowania": blocks of 32 with
power-of-two scales, no tensor scale).  Operands are random MXFP4 tensors made
on the host, or the GPU quantiser's own output (itself bit-exact against the
oracle); the same operand bytes go to both sides."""
import numpy as np
import pytest
import torch

import layout
import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def random_mx(rng, rows, K, unit=False):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    if unit:
        return codes, np.full((rows, K // 32), 127, np.uint8)
    return codes, rng.integers(118, 136, size=(rows, K // 32), dtype=np.uint8)


def upload_mx(codes, scales):
    rows, k = codes.shape[0], codes.shape[1] * 2
    buf = np.zeros(max(B.nvfp4_mx_scales_bytes(rows, k), 16), np.uint8)
    buf[layout.atom_offsets(rows, k // 2)] = scales  # four 32-blocks per atom word
    return B.NVFP4Tensor(codes=torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
                         scales=torch.from_numpy(buf).cuda(), tensor_scale=None, rows=rows, k=k)


def run(a, b, out_dtype=torch.float32):
    ws = B.workspace(256)
    out = B.nvfp4_gemm_mx(upload_mx(*a), upload_mx(*b), out_dtype=out_dtype, ws=ws)
    B.nvfp4_check(ws)
    return out


def test_mx_gemm_256_cube(cuda_lib):
    rng = np.random.default_rng(1)
    a, b = random_mx(rng, 256, 256), random_mx(rng, 256, 256)
    ref, ab = oracle.gemm_mx(a, b)
    assert_gemm_close(run(a, b).cpu().numpy(), ref, ab, "256^3")


SHAPES = [(1, 8, 64), (128, 256, 64), (200, 392, 320), (384, 640, 1024), (520, 264, 2112), (1000, 1000, 1088),
          (300, 520, 640), (264, 392, 704)]  # K % 256 = 0, 64, 128, 192: every stage length


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "%dx%dx%d" % s)
def test_mx_gemm_ragged(shape, cuda_lib):
    M, N, K = shape
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    a, b = random_mx(rng, M, K), random_mx(rng, N, K)
    ref, ab = oracle.gemm_mx(a, b)
    got = run(a, b).cpu().numpy()
    assert_gemm_close(got, ref, ab, "f32 out")
    got16 = run(a, b, torch.bfloat16)
    assert torch.equal(got16.cpu(), torch.from_numpy(got).to(torch.bfloat16)), "bf16 out != RN(f32 out)"


def test_mx_gemm_unit_scales_exact(cuda_lib):
    """Scale 2^0 everywhere: every partial sum is a small multiple of 0.25, exact in FP32."""
    rng = np.random.default_rng(2)
    a, b = random_mx(rng, 256, 4096, unit=True), random_mx(rng, 384, 4096, unit=True)
    ref, _ = oracle.gemm_mx(a, b)
    assert np.array_equal(run(a, b).cpu().numpy().astype(np.float64), ref)


def test_mx_gemm_scale_per_32_block(cuda_lib):
    """One nonzero scale per operand row, moved across the 32-blocks of K: the
    product picks the matching block pair only (catches a wrong scale byte)."""
    K = 512
    rng = np.random.default_rng(3)
    for blk in range(K // 32):
        a = (rng.integers(0, 256, size=(128, K // 2), dtype=np.uint8), np.zeros((128, K // 32), np.uint8))
        b = (rng.integers(0, 256, size=(256, K // 2), dtype=np.uint8), np.zeros((256, K // 32), np.uint8))
        a[1][:, blk] = 127 + (blk % 3)
        b[1][:, blk] = 126
        ref, ab = oracle.gemm_mx(a, b)
        assert_gemm_close(run(a, b).cpu().numpy(), ref, ab, "block %d" % blk)


def test_mx_gemm_on_quantised_operands(cuda_lib):
    """GPU-quantised MXFP4 operands (rowwise), as in an MXFP4 Fprop."""
    rng = np.random.default_rng(4)
    X = W.bf16_bits(W.normal(rng, (512, 1024)))
    Wt = W.bf16_bits(W.normal(rng, (640, 1024), 0.02))
    qx, qw = B.nvfp4_quantize_mx(to_dev(X)), B.nvfp4_quantize_mx(to_dev(Wt))
    Y = B.nvfp4_gemm_mx(qx, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, ab = oracle.gemm_mx(oracle.quantize_mx(X), oracle.quantize_mx(Wt))
    assert_gemm_close(Y.cpu().numpy(), ref, ab, "quantised")


def test_mx_gemm_full_size_sampled(cuda_lib):
    M, N, K = 8192, 20480, 5120
    rng = np.random.default_rng(5)
    a, b = random_mx(rng, M, K), random_mx(rng, N, K)
    got = run(a, b)
    mr = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 40)]))
    nr = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 40)]))
    ref, ab = oracle.gemm_mx((a[0][mr], a[1][mr]), (b[0][nr], b[1][nr]))
    g = got[torch.from_numpy(mr).cuda()][:, torch.from_numpy(nr).cuda()].cpu().numpy()
    assert_gemm_close(g, ref, ab, "full size")
