"""Host-only checks of the Python binding's argument checks: a tensor the C ABI
cannot validate itself (host memory, a strided view, a mismatched dtype or
shape) raises in Python before any library call.  No GPU is needed: every case
fails before a kernel could be launched."""
import pytest
import torch

from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import build


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return B.load()


bf16, f32 = torch.bfloat16, torch.float32


def test_host_tensors_are_refused():
    x = torch.zeros((64, 64), dtype=bf16)
    with pytest.raises(ValueError, match="CUDA"):
        B.nvfp4_quantize(x)
    with pytest.raises(ValueError, match="CUDA"):
        B.nvfp4_quantize_mx(x)
    with pytest.raises(ValueError, match="CUDA"):
        B.nvfp4_quantize_dual(x)
    with pytest.raises(ValueError, match="CUDA"):
        B.nvfp4_linear_fwd(x, x)
    with pytest.raises(ValueError, match="CUDA"):
        B.nvfp4_relu2_fwd(x)
    q = B.NVFP4Tensor(codes=torch.zeros((64, 32), dtype=torch.uint8), scales=torch.zeros(512, dtype=torch.uint8),
                      tensor_scale=torch.ones(1), rows=64, k=64)
    with pytest.raises(ValueError, match="CUDA"):
        B.nvfp4_gemm(q, q, out=torch.empty((64, 64), dtype=f32))


def test_rows_must_be_contiguous():
    x = torch.zeros((64, 128), dtype=bf16)
    with pytest.raises(ValueError, match="stride"):
        B.nvfp4_quantize(x.t())
    with pytest.raises(ValueError, match="2-D"):
        B.nvfp4_quantize(torch.zeros(64, dtype=bf16))
    with pytest.raises(TypeError):
        B.nvfp4_quantize(torch.zeros((64, 64), dtype=torch.float16))


def test_linear_operands_must_agree():
    X = torch.zeros((64, 128), dtype=bf16)
    with pytest.raises(TypeError, match="dtype"):
        B.nvfp4_linear_fwd(X, torch.zeros((64, 128), dtype=f32))
    with pytest.raises(ValueError, match="shape"):
        B.nvfp4_linear_fwd(X, torch.zeros((64, 64), dtype=bf16))
    with pytest.raises(ValueError, match="contiguous"):
        B.nvfp4_linear_fwd(torch.zeros((64, 256), dtype=bf16)[:, :128], torch.zeros((64, 128), dtype=bf16))
    W = torch.zeros((32, 128), dtype=bf16)
    with pytest.raises(ValueError, match="dY: shape"):
        B.nvfp4_linear_bwd(torch.zeros((64, 64), dtype=bf16), X, W)
    with pytest.raises(TypeError, match="dY: dtype"):
        B.nvfp4_linear_bwd(torch.zeros((64, 32), dtype=f32), X, W)
    with pytest.raises(TypeError, match="dW: dtype"):
        B.nvfp4_linear_bwd(torch.zeros((64, 32), dtype=bf16), X, W, dW=torch.zeros((32, 128), dtype=bf16))
    with pytest.raises(ValueError, match="out: shape"):
        B.nvfp4_linear_fwd_noalloc(X, W, out=torch.zeros((64, 64), dtype=bf16))


def test_relu2_takes_bf16_of_one_shape():
    y = torch.zeros((32, 64), dtype=bf16)
    with pytest.raises(TypeError, match="dtype"):
        B.nvfp4_relu2_fwd(y.float())
    with pytest.raises(ValueError, match="dh: shape"):
        B.nvfp4_relu2_bwd(torch.zeros((32, 32), dtype=bf16), y)
    with pytest.raises(ValueError, match="out: shape"):
        B.nvfp4_relu2_fwd_amax(y, out=torch.zeros((64, 32), dtype=bf16))
    with pytest.raises(ValueError, match="float32"):
        B.nvfp4_relu2_fwd_amax_rht(y, amax_out=torch.zeros(1, dtype=torch.float64))
