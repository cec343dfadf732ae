"""nvfp4_linear_fwd_noalloc against nvfp4_linear_fwd.

The no-alloc variant is for callers that cannot allocate device memory: code
inside a framework that owns every byte of device memory through its own pool,
or a latency-critical loop that cannot afford the synchronisation of
cudaMalloc/cudaFree.  Its scratch is a fixed buffer inside the library instead
of a caller workspace.  This file is named so that pytest collects it last: a
run that stops at the first failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B
from nvfp4_bit_precision_quantize_b200 import workloads as W

from gpu_helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def _case(seed, M, N, K):
    rng = np.random.default_rng(seed)
    return W.bf16_bits(W.normal(rng, (M, K))), W.bf16_bits(W.normal(rng, (N, K), 0.02))


def test_noalloc_matches_linear_fwd_on_two_calls(cuda_lib):
    """Two calls in a row (different shapes, so stale scratch would show): the
    variant's output agrees with nvfp4_linear_fwd's within the GEMM tolerance
    |a - b| <= 1e-4 * sum|a_k b_k| used by every GEMM parity test."""
    for call, (M, N, K) in enumerate([(256, 384, 512), (192, 320, 1024)]):
        X, Wt = _case(100 + call, M, N, K)
        Xd, Wd = to_dev(X), to_dev(Wt)
        expect = B.nvfp4_linear_fwd(Xd, Wd, y_dtype=torch.float32)
        got = B.nvfp4_linear_fwd_noalloc(Xd, Wd, y_dtype=torch.float32)
        got16 = B.nvfp4_linear_fwd_noalloc(Xd, Wd, y_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        _, abs_sum = oracle.gemm(oracle.quantize(X)[:3], oracle.quantize(Wt)[:3])
        assert_gemm_close(got.cpu().numpy(), expect.cpu().numpy().astype(np.float64), abs_sum,
                          "no-alloc call %d" % call)
        assert torch.equal(got16.cpu(), got.cpu().to(torch.bfloat16))


def test_noalloc_refuses_problems_beyond_its_buffer(cuda_lib):
    X = torch.zeros((8192, 5120), dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros((8192, 5120), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((8192, 8192), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.NVFP4Error) as err:
        B.nvfp4_linear_fwd_noalloc(X, Wt, out=Y)
    assert err.value.status == B.NVFP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((Y == 3.0).all())  # nothing ran
