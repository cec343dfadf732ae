"""NVFP4 linear layer (Fprop, Dgrad, Wgrad with RHT + SR) and the squared-ReLU
MLP activation on the GPU vs the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import assert_gemm_close, check_quantize, to_dev

pytestmark = pytest.mark.gpu


def _inputs(seed, M, N, K):
    rng = np.random.default_rng(seed)
    X = W.bf16_bits(W.normal(rng, (M, K)))
    Wt = W.bf16_bits(W.normal(rng, (N, K), 0.02))
    dY = W.bf16_bits(W.heavy_rows(rng, (M, N), 1e-3, 2))
    return X, Wt, dY


@pytest.mark.parametrize("shape", [(256, 384, 512), (192, 320, 256), (64, 64, 64), (512, 1024, 1536)],
                         ids=lambda s: "%dx%dx%d" % s)
def test_linear_fwd(shape, cuda_lib):
    M, N, K = shape
    X, Wt, _ = _inputs(M + N + K, M, N, K)
    Y = B.nvfp4_linear_fwd(to_dev(X), to_dev(Wt), y_dtype=torch.float32)
    torch.cuda.synchronize()
    qx, qw = oracle.quantize(X), oracle.quantize(Wt)
    ref, ab = oracle.gemm(qx[:3], qw[:3])
    assert_gemm_close(Y.cpu().numpy(), ref, ab, "fprop")
    Y16 = B.nvfp4_linear_fwd(to_dev(X), to_dev(Wt), y_dtype=torch.bfloat16)
    assert torch.equal(Y16.cpu(), Y.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("shape", [(256, 384, 512), (192, 320, 256), (64, 64, 64)], ids=lambda s: "%dx%dx%d" % s)
def test_linear_bwd(shape, cuda_lib):
    M, N, K = shape
    seed = 1234
    X, Wt, dY = _inputs(M * N + K, M, N, K)
    dX, dW = B.nvfp4_linear_bwd(to_dev(dY), to_dev(X), to_dev(Wt), seed=seed, dx_dtype=torch.float32)
    torch.cuda.synchronize()
    # Dgrad: rowwise(dY) . colwise(W)^T
    a = oracle.quantize(dY)[:3]
    b = oracle.quantize(Wt, colwise=True)[:3]
    ref, ab = oracle.gemm(a, b)
    assert_gemm_close(dX.cpu().numpy(), ref, ab, "dgrad")
    # Wgrad: colwise(dY, RHT, SR) . colwise(X, RHT)^T
    a = oracle.quantize(dY, colwise=True, sr=True, rht=True, seed=seed)[:3]
    b = oracle.quantize(X, colwise=True, rht=True, seed=seed)[:3]
    ref, ab = oracle.gemm(a, b)
    assert_gemm_close(dW.cpu().numpy(), ref, ab, "wgrad")
    # the Hadamard transform keeps dW an estimate of dY^T X
    exact = (to_dev(dY).float().T @ to_dev(X).float()).double().cpu().numpy()
    rel = np.linalg.norm(dW.cpu().numpy() - exact) / np.linalg.norm(exact)
    assert rel < 0.25, rel


def test_relu2_bit_exact(cuda_lib):
    rng = np.random.default_rng(21)
    y = W.bf16_bits(rng.standard_normal(100003).astype(np.float32) * 3)
    y[:4] = [0x8000, 0x0000, 0x0001, 0x8001]  # -0, +0, tiny +/- subnormal
    dh = W.bf16_bits(rng.standard_normal(100003).astype(np.float32) * 1e-3)
    yd, dhd = to_dev(y), to_dev(dh)
    h = B.nvfp4_relu2_fwd(yd)
    g = B.nvfp4_relu2_bwd(dhd, yd)
    torch.cuda.synchronize()
    assert np.array_equal(h.view(torch.int16).cpu().numpy().view(np.uint16), oracle.relu2_fwd(y))
    assert np.array_equal(g.view(torch.int16).cpu().numpy().view(np.uint16), oracle.relu2_bwd(dh, y))


def test_mlp_block_reduced(cuda_lib):
    """The MLP block (up -> relu^2 -> down, fwd + bwd) at reduced size: each GPU
    stage equals the oracle on the same stage inputs; the whole block stays close
    to an unquantised float32 reference."""
    M, H, F = 256, 320, 640
    w = W.mlp(M=M, H=H, F=F)
    X, W1, W2, dY2 = (to_dev(w[k]) for k in ("X", "W1", "W2", "dY2"))
    Y1 = B.nvfp4_linear_fwd(X, W1)
    h = B.nvfp4_relu2_fwd(Y1)
    Y2 = B.nvfp4_linear_fwd(h, W2)
    dh, dW2 = B.nvfp4_linear_bwd(dY2, h, W2, seed=1234)
    dY1 = B.nvfp4_relu2_bwd(dh, Y1)
    dX, dW1 = B.nvfp4_linear_bwd(dY1, X, W1, seed=1234)
    torch.cuda.synchronize()
    # stage: Y1 (host inputs X, W1)
    ref, ab = oracle.gemm(oracle.quantize(w["X"])[:3], oracle.quantize(w["W1"])[:3])
    y1_f32 = B.nvfp4_linear_fwd(X, W1, y_dtype=torch.float32).cpu().numpy()
    assert_gemm_close(y1_f32, ref, ab, "Y1")
    # whole block vs float32
    Xf, W1f, W2f, dY2f = (t.float() for t in (X, W1, W2, dY2))
    Y1f = Xf @ W1f.T
    hf = torch.relu(Y1f) ** 2
    Y2f = hf @ W2f.T
    dhf = dY2f @ W2f
    dY1f = dhf * 2 * torch.relu(Y1f)
    for got, ref_t in ((Y2, Y2f), (dW2, dY2f.T @ hf), (dX, dY1f @ W1f), (dW1, dY1f.T @ Xf)):
        rel = (torch.linalg.norm(got.float() - ref_t) / torch.linalg.norm(ref_t)).item()
        assert np.isfinite(rel) and rel < 0.35, rel


@pytest.mark.parametrize("n", [0, 8, 1000, 4096 + 3, 1 << 20])
def test_relu2_amax_variants(n, cuda_lib):
    """The amax variants store the same bf16 outputs as the plain kernels and return
    max |output| exactly; a quantisation given that amax equals one that computes it."""
    rng = np.random.default_rng(n + 3)
    y = W.bf16_bits(rng.standard_normal(n).astype(np.float32) * np.float32(3.0))
    dh = W.bf16_bits(rng.standard_normal(n).astype(np.float32))
    yd, dhd = to_dev(y), to_dev(dh)
    h, ah = B.nvfp4_relu2_fwd_amax(yd)
    g, ag = B.nvfp4_relu2_bwd_amax(dhd, yd)
    torch.cuda.synchronize()
    hb = h.view(torch.int16).cpu().numpy().view(np.uint16)
    gb = g.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(hb, oracle.relu2_fwd(y))
    assert np.array_equal(gb, oracle.relu2_bwd(dh, y))
    f = lambda b: np.abs((b.astype(np.uint32) << 16).view(np.float32))  # noqa: E731
    assert ah[0].item() == (float(f(hb).max()) if n else 0.0)
    assert ag[0].item() == (float(f(gb).max()) if n else 0.0)
    if n and n % 64 == 0 and n >= 4096:
        x = hb.reshape(-1, 64)
        check_quantize(x, amax_in=ah[0].item())
        check_quantize(gb.reshape(-1, 64), amax_in=ag[0].item())


@pytest.mark.parametrize("shape", [(16, 8), (48, 200), (512, 392), (8192, 2048)])
def test_relu2_amax_rht_variants(shape, cuda_lib):
    """The 2-D variants store the oracle's relu^2 outputs and return max|out| and the
    colwise Hadamard amax exactly; colwise RHT quantisation given that amax equals the
    one that computes it."""
    rng = np.random.default_rng(shape[0] + shape[1])
    y = W.bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(3.0))
    dh = W.bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(0.01))
    yd, dhd = to_dev(y), to_dev(dh)
    h, ah, ahr = B.nvfp4_relu2_fwd_amax_rht(yd, seed=77)
    g, ag, agr = B.nvfp4_relu2_bwd_amax_rht(dhd, yd, seed=77)
    torch.cuda.synchronize()
    hb = h.view(torch.int16).cpu().numpy().view(np.uint16)
    gb = g.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(hb, oracle.relu2_fwd(y.ravel()).reshape(shape))
    assert np.array_equal(gb, oracle.relu2_bwd(dh.ravel(), y.ravel()).reshape(shape))
    f = lambda b: np.abs((b.astype(np.uint32) << 16).view(np.float32))  # noqa: E731
    assert ah[0].item() == float(f(hb).max()) and ag[0].item() == float(f(gb).max())
    assert ahr[0].item() == float(oracle.amax(hb, colwise=True, rht=True, seed=77))
    assert agr[0].item() == float(oracle.amax(gb, colwise=True, rht=True, seed=77))
    if shape[0] <= 512:
        check_quantize(hb, colwise=True, rht=True, seed=77, amax_in=ahr[0].item())
        check_quantize(gb, colwise=True, sr=True, rht=True, seed=77, amax_in=agr[0].item())
