"""The bounds-checked debug build (libnvfp4_checked.so, -DNVFP4_BOUNDS_CHECK) on
the GPU.  A child process loads it (NVFP4_CHECKED=1) and runs every kernel
family on ragged shapes -- tails in each tiled dimension -- then reads the
bounds record: no guarded index may have fallen outside its buffer, and the
outputs must equal, bit for bit, those of the product library run here on the
same inputs (the checks only guard accesses, they never change a result).  The
planted failure of nvfp4_selftest_bounds must be reported with its site.
The format and modes exercised: aisight.pl, sections "Architektura NVFP4
kontra ograniczenia mikroskalowania" and "Technologie stabilizujace proces
treningowy"."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def exercise(B, dev):
    """Run the library's calls on ragged inputs; host copies of every output."""
    g = torch.Generator().manual_seed(5)

    def bf(r, c, std=1.0):
        return (torch.randn(r, c, generator=g) * std).to(torch.bfloat16).to(dev)

    out = {}

    def keep(name, q):
        out[name + ".codes"] = q.codes.cpu()
        out[name + ".scales"] = q.scales.cpu()
        if q.tensor_scale is not None:
            out[name + ".ts"] = q.tensor_scale.cpu()

    ws = B.workspace(B.nvfp4_quantize_dual_workspace_size(), dev)
    x = bf(528, 272)  # R % 32 == 16; C neither a multiple of 64 nor of 256
    for dt, t in (("bf16", x), ("f32", x.float())):
        for orient in (B.NVFP4_ROWWISE, B.NVFP4_COLWISE):
            for sr in (False, True):
                for rht in ((False, True) if orient == B.NVFP4_COLWISE else (False,)):
                    q = B.nvfp4_quantize(t, orientation=orient, rounding=B.NVFP4_SR if sr else B.NVFP4_RTN, rht=rht,
                                         seed=1234, ws=ws)
                    keep("q.%s.%d%d%d" % (dt, orient, sr, rht), q)
    r, c = B.nvfp4_quantize_dual(x, col_rounding=B.NVFP4_SR, col_rht=True, seed=1234, ws=ws)
    keep("dual.r", r)
    keep("dual.c", c)
    xm = bf(544, 288)  # MXFP4: C % 32 == 0 (rowwise), R % 32 == 0 (colwise), neither a multiple of 128
    keep("mx.r", B.nvfp4_quantize_mx(xm))
    keep("mx.c", B.nvfp4_quantize_mx(xm, orientation=B.NVFP4_COLWISE))
    a = B.nvfp4_quantize(bf(300, 320), ws=ws)
    b = B.nvfp4_quantize(bf(200, 320, 0.02), ws=ws)
    out["gemm.f32"] = B.nvfp4_gemm(a, b, out_dtype=torch.float32, ws=ws).cpu()
    out["gemm.bf16"] = B.nvfp4_gemm(a, b, out_dtype=torch.bfloat16, ws=ws).cpu()
    am = B.nvfp4_quantize_mx(bf(300, 384))
    bm = B.nvfp4_quantize_mx(bf(200, 384, 0.02))
    out["gemm_mx"] = B.nvfp4_gemm_mx(am, bm, out_dtype=torch.float32, ws=ws).cpu()
    a2 = B.nvfp4_quantize(bf(256, 320), ws=ws)
    b2 = B.nvfp4_quantize(bf(512, 320, 0.02), ws=ws)
    y, h, m0, m1 = B.nvfp4_gemm_relu2_fwd(a2, b2, seed=1234, ws=ws)
    out.update({"relu2_fwd.y": y.cpu(), "relu2_fwd.h": h.cpu(), "relu2_fwd.m0": m0.cpu(), "relu2_fwd.m1": m1.cpu()})
    dy, n0, n1 = B.nvfp4_gemm_relu2_bwd(a2, b2, y, seed=1234, ws=ws)
    out.update({"relu2_bwd.dy": dy.cpu(), "relu2_bwd.m0": n0.cpu(), "relu2_bwd.m1": n1.cpu()})
    v = bf(37, 9)  # 333 elements: a tail after the 8-element vectors
    out["relu2"] = B.nvfp4_relu2_fwd(v).cpu()
    out["drelu2"] = B.nvfp4_relu2_bwd(bf(37, 9), v).cpu()
    hv, k0, k1 = B.nvfp4_relu2_fwd_amax_rht(bf(48, 40), seed=1234, ws=ws)
    out.update({"relu2_rht.h": hv.cpu(), "relu2_rht.m0": k0.cpu(), "relu2_rht.m1": k1.cpu()})
    X, W = bf(320, 192), bf(192, 192, 0.02)
    out["linear_fwd"] = B.nvfp4_linear_fwd(X, W, y_dtype=torch.float32).cpu()
    dX, dW = B.nvfp4_linear_bwd(bf(320, 192, 1e-3), X, W, seed=1234, dx_dtype=torch.float32)
    out["linear_bwd.dX"] = dX.cpu()
    out["linear_bwd.dW"] = dW.cpu()
    torch.cuda.synchronize()
    B.nvfp4_check(ws)
    return out


def child(path):
    """Runs under NVFP4_CHECKED=1: the checked library's outputs and bounds records."""
    from nvfp4_bit_precision_quantize_b200 import binding as B
    from nvfp4_bit_precision_quantize_b200 import build
    build.build(checked=True)
    assert B.LIB_PATH.endswith("libnvfp4_checked.so")
    dev = torch.device("cuda", 0)
    checked, site, st = B.nvfp4_bounds_status()
    assert checked and site == 0 and st == B.NVFP4_OK
    out = exercise(B, dev)
    checked, site, st = B.nvfp4_bounds_status()
    out["bounds.after_exercise"] = torch.tensor([site, st])
    buf = torch.zeros(17, dtype=torch.uint8, device=dev)
    B.nvfp4_selftest_bounds(buf)
    checked, site2, st2 = B.nvfp4_bounds_status()
    out["bounds.selftest"] = torch.tensor([site2, st2])
    out["bounds.selftest_buf"] = buf.cpu()
    _, site3, st3 = B.nvfp4_bounds_status()  # the read cleared the record
    out["bounds.cleared"] = torch.tensor([site3, st3])
    torch.save(out, path)


def test_checked_build_clean_and_identical(cuda_lib, tmp_path):
    B = cuda_lib
    path = str(tmp_path / "checked.pt")
    env = dict(os.environ, NVFP4_CHECKED="1")
    code = "import sys; sys.path[:0] = [%r, %r]; import test_bounds_checked_gpu as t; t.child(%r)" % (HERE, ROOT, path)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    got = torch.load(path)
    assert got["bounds.after_exercise"].tolist() == [0, B.NVFP4_OK], "a guarded index fell outside its buffer: %s" % (
        got["bounds.after_exercise"].tolist())
    site, st = got["bounds.selftest"].tolist()
    assert st == B.NVFP4_ERR_DEVICE_BOUNDS and site // 100000 == 4 and site % 100000 > 0
    assert got["bounds.selftest_buf"].tolist() == [1] + [0] * 16  # the passing write happened, the failing one not
    assert got["bounds.cleared"].tolist() == [0, B.NVFP4_OK]
    ref = exercise(B, torch.device("cuda", 0))
    assert B.nvfp4_bounds_status()[0] is False
    for k, v in ref.items():
        w = got[k]
        assert w.dtype == v.dtype and w.shape == v.shape, k
        assert torch.equal(w.view(torch.uint8) if w.dtype != torch.uint8 else w,
                           v.view(torch.uint8) if v.dtype != torch.uint8 else v), k
