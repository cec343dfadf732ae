"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
(via the binding) and the oracle on the same host data, then compare."""
import numpy as np
import torch

import layout
import oracle
from nvfp4_bit_precision_quantize_b200 import binding as B


def to_dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def f32_bits(v):
    return np.float32(v).view(np.uint32)


def gpu_quantize(x, colwise=False, sr=False, rht=False, seed=1234, amax_in=None):
    xd = to_dev(x)
    a = torch.tensor([amax_in], dtype=torch.float32, device="cuda") if amax_in is not None else None
    q = B.nvfp4_quantize(xd, orientation=B.NVFP4_COLWISE if colwise else B.NVFP4_ROWWISE,
                         rounding=B.NVFP4_SR if sr else B.NVFP4_RTN, rht=rht, seed=seed, amax_in=a)
    torch.cuda.synchronize()
    return q


def first_mismatch(a, b):
    idx = np.argwhere(a != b)
    return None if idx.size == 0 else (tuple(idx[0]), a[tuple(idx[0])], b[tuple(idx[0])], len(idx))


def check_quantize(x, colwise=False, sr=False, rht=False, seed=1234, amax_in=None):
    """Bit-exact comparison of codes, scales (and their zero padding) and tensor scale."""
    q = gpu_quantize(x, colwise, sr, rht, seed, amax_in)
    return compare_quantize(q, x, colwise, sr, rht, seed, amax_in)


def compare_quantize(q, x, colwise=False, sr=False, rht=False, seed=1234, amax_in=None):
    """Bit-exact comparison of a GPU NVFP4 tensor q with the oracle's quantisation of x."""
    oc, osc, ots, _ = oracle.quantize(x, colwise=colwise, sr=sr, rht=rht, seed=seed, amax_in=amax_in)
    rows, k = oc.shape[0], oc.shape[1] * 2
    gts = q.tensor_scale.cpu().numpy()[0]
    assert f32_bits(gts) == f32_bits(ots), (gts, ots)
    gc = q.codes.cpu().numpy()
    assert gc.shape == oc.shape
    mm = first_mismatch(gc, oc)
    assert mm is None, "codes differ: %s" % (mm,)
    buf = q.scales.cpu().numpy()
    plain = layout.atoms_to_plain(buf, rows, k)
    mm = first_mismatch(plain, osc)
    assert mm is None, "scales differ: %s" % (mm,)
    pad = layout.padding_mask(rows, k)
    assert not buf[pad].any(), "scale padding not zero"
    return q


def upload(codes, scales_plain, ts):
    rows, k = codes.shape[0], codes.shape[1] * 2
    return B.NVFP4Tensor(codes=torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
                         scales=torch.from_numpy(layout.plain_to_atoms(scales_plain, rows, k)).cuda(),
                         tensor_scale=torch.tensor([ts], dtype=torch.float32, device="cuda"), rows=rows, k=k)


def random_operand(rng, rows, K, lo=0x18, hi=0x58, unit=False):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    if unit:
        return codes, np.full((rows, K // 16), 0x38, np.uint8), np.float32(1.0)
    scales = rng.integers(lo, hi, size=(rows, K // 16), dtype=np.uint8)
    return codes, scales, np.float32(rng.uniform(0.25, 4.0))


def assert_gemm_close(gpu, ref, absref, what=""):
    err = np.abs(gpu.astype(np.float64) - ref)
    bound = 1e-4 * absref
    bad = err > bound
    assert not bad.any(), "%s: %d elements out of tolerance, worst err/bound %.3g at %s" % (
        what, int(bad.sum()), float((err / np.maximum(bound, 1e-300)).max()), tuple(np.argwhere(bad)[0]))
