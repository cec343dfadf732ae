"""Failure detection on the GPU without a fault: a bounded device-side wait
that nothing satisfies must end by itself, report NVFP4_ERR_DEVICE_TIMEOUT
through the workspace status word, and leave the CUDA context usable."""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, random_operand, upload


@pytest.mark.gpu
def test_device_timeout_reported_and_context_survives(cuda_lib):
    B = cuda_lib
    dev = torch.device("cuda", 0)
    ws = B.workspace(256, dev)
    B.nvfp4_check(ws)  # fresh status word
    t0 = time.perf_counter()
    B.nvfp4_selftest_wait_timeout(ws, 20_000_000)  # 20 ms limit
    with pytest.raises(B.NVFP4Error) as err:
        B.nvfp4_check(ws)
    elapsed = time.perf_counter() - t0
    assert err.value.status == B.NVFP4_ERR_DEVICE_TIMEOUT
    assert 0.015 < elapsed < 5.0
    B.nvfp4_check(ws)  # the check cleared the status word

    # the same context still runs real work: a small block-scaled GEMM against the oracle
    rng = np.random.default_rng(11)
    M, N, K = 256, 256, 256
    a = random_operand(rng, M, K)
    b = random_operand(rng, N, K)
    out = torch.empty((M, N), dtype=torch.float32, device=dev)
    B.nvfp4_gemm(upload(*a), upload(*b), out=out, ws=ws)
    B.nvfp4_check(ws)
    ref, absref = oracle.gemm(a, b)
    assert_gemm_close(out.cpu().numpy(), ref, absref, "gemm after a device timeout")
