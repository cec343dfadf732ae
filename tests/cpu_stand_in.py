"""A CPU stand-in for the binding, computing with the oracle (test-only).

It offers the calls mlp.MlpStep makes, with the binding's names and argument
conventions, on CPU torch tensors, so that the step's exact call sequence can
run in CPU tests (the data-parallel gloo test).  Quantised tensors keep their
scales in plain [rows x k/16] order: only this stand-in reads them.  Every call
is appended to `calls`, for order checks.
"""
from dataclasses import dataclass

import numpy as np
import torch

import oracle

NVFP4_ROWWISE, NVFP4_COLWISE = 0, 1
NVFP4_RTN, NVFP4_SR = 0, 1

calls = []


@dataclass
class Tensor:
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor
    rows: int
    k: int


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16)


def workspace(nbytes, device=None):
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8)


def nvfp4_quantize_dual_workspace_size():
    return 256


def nvfp4_last_launch_count():
    return 0


def empty_nvfp4(rows, k, device=None):
    return Tensor(torch.zeros((rows, k // 2), dtype=torch.uint8), torch.zeros((rows, k // 16), dtype=torch.uint8),
                  torch.zeros(1), rows, k)


def _store(out, q):
    codes, scales, ts, _ = q
    out.codes.copy_(torch.from_numpy(codes))
    out.scales.copy_(torch.from_numpy(scales))
    out.tensor_scale.fill_(float(ts))


def nvfp4_quantize(x, orientation=NVFP4_ROWWISE, rounding=NVFP4_RTN, rht=False, seed=1234, amax_in=None, out=None,
                   ws=None):
    calls.append("quantize")
    am = None if amax_in is None else float(amax_in[0])
    _store(out, oracle.quantize(_bits(x), colwise=orientation == NVFP4_COLWISE, sr=rounding == NVFP4_SR, rht=rht,
                                seed=seed, amax_in=am))
    return out


def nvfp4_amax(x, rht=False, seed=1234, out=None, ws=None):
    calls.append("amax")
    out.fill_(float(oracle.amax(_bits(x), colwise=bool(rht), rht=bool(rht), seed=seed)))
    return out


def nvfp4_amax_dual(x, seed=1234, out=None, out_rht=None, ws=None):
    calls.append("amax_dual")
    b = _bits(x)
    out.fill_(float(oracle.amax(b)))
    out_rht.fill_(float(oracle.amax(b, colwise=True, rht=True, seed=seed)))
    return out, out_rht


def nvfp4_quantize_dual(x, col_rounding=NVFP4_RTN, col_rht=False, seed=1234, out_row=None, out_col=None, ws=None):
    calls.append("quantize_dual")
    b = _bits(x)
    _store(out_row, oracle.quantize(b, seed=seed))
    _store(out_col, oracle.quantize(b, colwise=True, sr=col_rounding == NVFP4_SR, rht=col_rht, seed=seed))
    return out_row, out_col


def nvfp4_gemm(A, B, out=None, ws=None):
    calls.append("gemm")
    ref, _ = oracle.gemm((A.codes.numpy(), A.scales.numpy(), A.tensor_scale.item()),
                         (B.codes.numpy(), B.scales.numpy(), B.tensor_scale.item()))
    out.copy_(torch.from_numpy(ref).to(out.dtype))
    return out


def _relu2_amax(out_bits, seed, out, amax_out, amax_rht_out):
    out.copy_(_bf16(out_bits.reshape(out.shape)))
    amax_out.fill_(float(oracle.amax(out_bits.reshape(out.shape))))
    amax_rht_out.fill_(float(oracle.amax(out_bits.reshape(out.shape), colwise=True, rht=True, seed=seed)))


def nvfp4_relu2_fwd_amax_rht(y, seed=1234, out=None, amax_out=None, amax_rht_out=None, ws=None):
    calls.append("relu2_fwd")
    _relu2_amax(oracle.relu2_fwd(_bits(y).ravel()), seed, out, amax_out, amax_rht_out)


def nvfp4_relu2_bwd_amax_rht(dh, y, seed=1234, out=None, amax_out=None, amax_rht_out=None, ws=None):
    calls.append("relu2_bwd")
    _relu2_amax(oracle.relu2_bwd(_bits(dh).ravel(), _bits(y).ravel()), seed, out, amax_out, amax_rht_out)


def nvfp4_gemm_relu2_fwd(A, B, seed=1234, y=None, h=None, amax_out=None, amax_rht_out=None, ws=None):
    calls.append("gemm_relu2_fwd")
    ref, _ = oracle.gemm((A.codes.numpy(), A.scales.numpy(), A.tensor_scale.item()),
                         (B.codes.numpy(), B.scales.numpy(), B.tensor_scale.item()))
    y.copy_(torch.from_numpy(ref).to(torch.bfloat16))
    _relu2_amax(oracle.relu2_fwd(_bits(y).ravel()), seed, h, amax_out, amax_rht_out)
    return y, h, amax_out, amax_rht_out


def nvfp4_gemm_relu2_bwd(A, B, y, seed=1234, out=None, amax_out=None, amax_rht_out=None, ws=None):
    calls.append("gemm_relu2_bwd")
    ref, _ = oracle.gemm((A.codes.numpy(), A.scales.numpy(), A.tensor_scale.item()),
                         (B.codes.numpy(), B.scales.numpy(), B.tensor_scale.item()))
    dh = _bits(torch.from_numpy(ref).to(torch.bfloat16))
    _relu2_amax(oracle.relu2_bwd(dh.ravel(), _bits(y).ravel()), seed, out, amax_out, amax_rht_out)
    return out, amax_out, amax_rht_out
