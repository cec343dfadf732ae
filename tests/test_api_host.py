"""Host-only checks of the C ABI (no GPU): the library loads, exports every
function include/nvfp4.h declares, sizes match the documented layout, and
invalid arguments are rejected before anything is launched."""
import ctypes as C
import os
import re
import subprocess
import sys
import textwrap

import pytest

from nvfp4_bit_precision_quantize_b200 import binding, build
import layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_function(lib):
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTS)


def test_checked_build_exports_and_reports(lib):
    """The bounds-checked debug build exports the same functions; the product build
    records nothing and refuses the bounds self-test."""
    path = build.build(checked=True)
    L = C.CDLL(path)
    for n in declared_functions():
        assert hasattr(L, n), n
    checked, site = C.c_int(-1), C.c_int(-1)
    f = lib.nvfp4_bounds_status
    f.argtypes = [C.POINTER(C.c_int), C.POINTER(C.c_int)]
    assert f(C.byref(checked), C.byref(site)) == binding.NVFP4_OK and (checked.value, site.value) == (0, 0)
    assert f(None, C.byref(site)) == binding.NVFP4_ERR_INVALID_ARG
    lib.nvfp4_selftest_bounds.argtypes = [C.c_void_p, C.c_int64, C.c_void_p]
    assert lib.nvfp4_selftest_bounds(C.c_void_p(0x20000), 16, None) == binding.NVFP4_ERR_INVALID_ARG
    g = L.nvfp4_bounds_status
    g.argtypes = [C.POINTER(C.c_int), C.POINTER(C.c_int)]
    st = g(C.byref(checked), C.byref(site))
    assert checked.value == 1
    assert st in (binding.NVFP4_OK, binding.NVFP4_ERR_CUDA)  # NVFP4_ERR_CUDA where no GPU is present
    L.nvfp4_selftest_bounds.argtypes = [C.c_void_p, C.c_int64, C.c_void_p]
    assert L.nvfp4_selftest_bounds(None, 16, None) == binding.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_selftest_bounds(C.c_void_p(0x20000), 0, None) == binding.NVFP4_ERR_INVALID_ARG


def test_sizes(lib):
    assert lib.nvfp4_codes_bytes(256, 256) == 256 * 128
    for rows, k in [(1, 16), (128, 64), (129, 64), (200, 272), (8192, 5120), (0, 64), (64, 0)]:
        assert lib.nvfp4_scales_bytes(rows, k) == layout.scales_bytes(rows, k)
    assert lib.nvfp4_quantize_workspace_size() >= 256 + 4 * 1024
    assert lib.nvfp4_linear_workspace_size(8192, 20480, 5120) > 0.5625 * 8192 * 20480 * 2
    # forward footprint: the rowwise X [M x K] and W [N x K] operands, plus the fixed header
    for M, N, K in [(8192, 20480, 5120), (256, 4096, 64), (128, 128, 128)]:
        fwd = lib.nvfp4_linear_fwd_workspace_size(M, N, K)
        ops = sum(lib.nvfp4_codes_bytes(r, K) + lib.nvfp4_scales_bytes(r, K) for r in (M, N))
        assert ops <= fwd <= ops + 16384
        assert fwd <= lib.nvfp4_linear_workspace_size(M, N, K)
    assert lib.nvfp4_linear_fwd_workspace_size(-1, 1, 64) == 0


def test_status_strings(lib):
    for s in range(8):
        assert len(binding.status_string(s)) > 0


def _tensor(rows, k, codes=0x1000, scales=0x2000, ts=0x3000):
    return binding.CTensor(codes, scales, ts, rows, k)


def _q(lib, x=0x10000, dtype=1, R=64, Cc=64, ld=64, ori=0, rnd=0, rht=0, out=None, ws=0x20000,
       wsb=1 << 20, amax=None):
    out = out if out is not None else _tensor(R if ori == 0 else Cc, Cc if ori == 0 else R)
    return lib.nvfp4_quantize(C.c_void_p(x), dtype, R, Cc, ld, ori, rnd, rht, 1234, amax, C.byref(out),
                              C.c_void_p(ws), wsb, None)


def test_quantize_rejections(lib):
    E = binding
    assert lib.nvfp4_quantize(C.c_void_p(0x10000), 1, 64, 64, 64, 0, 0, 0, 1, None, None, None, 0, None) \
        == E.NVFP4_ERR_INVALID_ARG
    assert _q(lib, x=0) == E.NVFP4_ERR_INVALID_ARG
    assert _q(lib, dtype=7) == E.NVFP4_ERR_INVALID_ARG
    assert _q(lib, ori=2) == E.NVFP4_ERR_INVALID_ARG
    assert _q(lib, rnd=3) == E.NVFP4_ERR_INVALID_ARG
    assert _q(lib, rht=1, ori=0) == E.NVFP4_ERR_INVALID_ARG          # RHT only colwise
    assert _q(lib, Cc=40, ld=40) == E.NVFP4_ERR_SHAPE                # rowwise C % 16
    assert _q(lib, R=40, ori=1, out=_tensor(64, 40)) == E.NVFP4_ERR_SHAPE  # colwise R % 16
    assert _q(lib, ld=32) == E.NVFP4_ERR_SHAPE                       # ld < C
    assert _q(lib, out=_tensor(64, 32)) == E.NVFP4_ERR_SHAPE         # output shape mismatch
    assert _q(lib, R=-1) == E.NVFP4_ERR_SHAPE
    assert _q(lib, x=0x10008) == E.NVFP4_ERR_ALIGNMENT
    assert _q(lib, ld=72, Cc=64) == E.NVFP4_ERR_SHAPE or _q(lib, ld=68, Cc=64) == E.NVFP4_ERR_ALIGNMENT
    assert _q(lib, ld=68, Cc=64) == E.NVFP4_ERR_ALIGNMENT            # 136-byte rows
    assert _q(lib, out=_tensor(64, 64, codes=0x1004)) == E.NVFP4_ERR_ALIGNMENT
    assert _q(lib, ws=0) == E.NVFP4_ERR_WORKSPACE
    assert _q(lib, wsb=100) == E.NVFP4_ERR_WORKSPACE
    big = 65535 * 256 + 16                                            # colwise grid rows run out
    assert _q(lib, R=big, ld=64, ori=1, out=_tensor(64, big)) == E.NVFP4_ERR_SHAPE
    assert _q(lib, R=(1 << 31) + 16, Cc=64, out=_tensor((1 << 31) + 16, 64)) == E.NVFP4_ERR_SHAPE


def test_gemm_rejections(lib):
    E = binding
    a, b = _tensor(128, 256), _tensor(256, 256)

    def g(A=a, B=b, Cp=0x40000, dt=1, ldc=256, ws=0x50000, wsb=256):
        return lib.nvfp4_gemm(C.byref(A), C.byref(B), C.c_void_p(Cp), dt, ldc, C.c_void_p(ws), wsb, None)
    assert lib.nvfp4_gemm(None, C.byref(b), C.c_void_p(0x40000), 1, 256, C.c_void_p(0x50000), 256, None) \
        == E.NVFP4_ERR_INVALID_ARG
    assert g(B=_tensor(256, 128)) == E.NVFP4_ERR_SHAPE                # K mismatch
    assert g(A=_tensor(128, 96), B=_tensor(256, 96)) == E.NVFP4_ERR_SHAPE  # K % 64
    assert g(ldc=128) == E.NVFP4_ERR_SHAPE
    assert g(Cp=0) == E.NVFP4_ERR_INVALID_ARG
    assert g(Cp=0x40002) == E.NVFP4_ERR_ALIGNMENT
    assert g(ldc=260) == E.NVFP4_ERR_ALIGNMENT                        # 520-byte bf16 rows
    assert g(dt=5) == E.NVFP4_ERR_INVALID_ARG
    assert g(ws=0) == E.NVFP4_ERR_WORKSPACE
    assert g(A=_tensor(0, 256)) == E.NVFP4_OK                         # empty: nothing to do


def test_gemm_mx_rejections(lib):
    E = binding
    A, Bt = _tensor(256, 256), _tensor(256, 256)
    Bt.tensor_scale = None                                             # MXFP4 tensors carry no tensor scale
    p = C.c_void_p
    g = lambda A=A, Bt=Bt, Cp=0x40000, dt=0, ldc=256, ws=0x50000: lib.nvfp4_gemm_mx(  # noqa: E731
        C.byref(A), C.byref(Bt), p(Cp), dt, ldc, p(ws) if ws else None, 256, None)
    assert g(A=_tensor(256, 96)) == E.NVFP4_ERR_SHAPE                 # K mismatch
    assert g(A=_tensor(256, 96), Bt=_tensor(256, 96)) == E.NVFP4_ERR_SHAPE  # K % 64
    assert g(Cp=0) == E.NVFP4_ERR_INVALID_ARG
    assert g(Cp=0x40004) == E.NVFP4_ERR_ALIGNMENT
    assert g(ws=0) == E.NVFP4_ERR_WORKSPACE
    assert g(dt=3) == E.NVFP4_ERR_INVALID_ARG
    assert g(A=_tensor(0, 256)) == E.NVFP4_OK


def test_linear_rejections(lib):
    E = binding
    ws = lib.nvfp4_linear_workspace_size(128, 128, 128)
    p = C.c_void_p
    assert lib.nvfp4_linear_fwd(p(0x1000), p(0x2000), p(0x3000), 128, 128, 96, 1, 1, p(0x4000), ws, None) \
        == E.NVFP4_ERR_SHAPE
    wsf = lib.nvfp4_linear_fwd_workspace_size(128, 128, 128)
    assert wsf < ws                                                   # the forward pass needs 2 of the 4 operands
    assert lib.nvfp4_linear_fwd(p(0x1000), p(0x2000), p(0x3000), 128, 128, 128, 1, 1, p(0x4000), wsf - 1,
                                None) == E.NVFP4_ERR_WORKSPACE
    assert lib.nvfp4_linear_fwd(None, p(0x2000), p(0x3000), 128, 128, 128, 1, 1, p(0x4000), ws, None) \
        == E.NVFP4_ERR_INVALID_ARG
    assert lib.nvfp4_linear_bwd(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), 100, 128, 128, 1, 1,
                                1, p(0x6000), ws, None) == E.NVFP4_ERR_SHAPE
    big = 65535 * 256 + 64                                            # colwise dY / X: R = M too large
    wsb = lib.nvfp4_linear_workspace_size(big, 128, 128)
    assert lib.nvfp4_linear_bwd(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), big, 128, 128, 1, 1,
                                1, p(0x6000), wsb, None) == E.NVFP4_ERR_SHAPE
    assert lib.nvfp4_relu2_fwd(p(0x1001), p(0x2000), 16, None) == E.NVFP4_ERR_ALIGNMENT
    assert lib.nvfp4_relu2_bwd(None, p(0x2000), p(0x3000), 16, None) == E.NVFP4_ERR_INVALID_ARG


def test_selftest_rejections(lib):
    ws = C.c_void_p(0x20000)
    assert lib.nvfp4_selftest_wait_timeout(None, 256, 1000, None) == binding.NVFP4_ERR_WORKSPACE
    assert lib.nvfp4_selftest_wait_timeout(ws, 255, 1000, None) == binding.NVFP4_ERR_WORKSPACE
    assert lib.nvfp4_selftest_wait_timeout(C.c_void_p(0x20008), 256, 1000, None) == binding.NVFP4_ERR_ALIGNMENT
    assert lib.nvfp4_selftest_wait_timeout(ws, 256, 0, None) == binding.NVFP4_ERR_INVALID_ARG
    assert lib.nvfp4_selftest_wait_timeout(ws, 256, 3_000_000_000, None) == binding.NVFP4_ERR_INVALID_ARG


def test_amax_rejections(lib):
    f = lib.nvfp4_amax
    f.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64, C.c_int, C.c_uint64, C.c_void_p, C.c_void_p,
                  C.c_size_t, C.c_void_p]
    E, bf = binding, binding.NVFP4_DTYPE_BF16
    x, out, ws = C.c_void_p(0x10000), C.c_void_p(0x30000), C.c_void_p(0x40000)
    wsb = lib.nvfp4_quantize_workspace_size()
    assert f(x, bf, 64, 64, 64, 0, 1, None, ws, wsb, None) == E.NVFP4_ERR_INVALID_ARG        # no output
    assert f(x, 7, 64, 64, 64, 0, 1, out, ws, wsb, None) == E.NVFP4_ERR_INVALID_ARG          # dtype
    assert f(x, bf, 64, 64, 64, 2, 1, out, ws, wsb, None) == E.NVFP4_ERR_INVALID_ARG         # rht flag
    assert f(x, bf, 64, 64, 64, 0, 1, C.c_void_p(0x30002), ws, wsb, None) == E.NVFP4_ERR_ALIGNMENT
    assert f(x, bf, -1, 64, 64, 0, 1, out, ws, wsb, None) == E.NVFP4_ERR_SHAPE
    assert f(x, bf, 64, 64, 64, 0, 1, out, None, wsb, None) == E.NVFP4_ERR_WORKSPACE
    assert f(x, bf, 64, 64, 64, 0, 1, out, ws, wsb - 1, None) == E.NVFP4_ERR_WORKSPACE
    assert f(None, bf, 64, 64, 64, 0, 1, out, ws, wsb, None) == E.NVFP4_ERR_INVALID_ARG      # no input
    assert f(x, bf, 64, 60, 64, 0, 1, out, ws, wsb, None) == E.NVFP4_ERR_SHAPE               # C * 2 % 16
    assert f(x, bf, 40, 64, 64, 1, 1, out, ws, wsb, None) == E.NVFP4_ERR_SHAPE               # rht: R % 16
    assert f(x, bf, 64, 64, 32, 0, 1, out, ws, wsb, None) == E.NVFP4_ERR_SHAPE               # ld < C
    assert f(C.c_void_p(0x10008), bf, 64, 64, 64, 0, 1, out, ws, wsb, None) == E.NVFP4_ERR_ALIGNMENT


def test_amax_dual_rejections(lib):
    f = lib.nvfp4_amax_dual
    f.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64, C.c_uint64, C.c_void_p, C.c_void_p,
                  C.c_void_p, C.c_size_t, C.c_void_p]
    E, bf = binding, binding.NVFP4_DTYPE_BF16
    x, o1, o2, ws = C.c_void_p(0x10000), C.c_void_p(0x30000), C.c_void_p(0x30010), C.c_void_p(0x40000)
    wsb = lib.nvfp4_quantize_dual_workspace_size()
    assert f(x, bf, 64, 64, 64, 1, None, o2, ws, wsb, None) == E.NVFP4_ERR_INVALID_ARG
    assert f(x, bf, 64, 64, 64, 1, o1, None, ws, wsb, None) == E.NVFP4_ERR_INVALID_ARG
    assert f(x, bf, 64, 64, 64, 1, o1, C.c_void_p(0x30011), ws, wsb, None) == E.NVFP4_ERR_ALIGNMENT
    assert f(x, bf, 64, 64, 64, 1, o1, o2, ws, lib.nvfp4_quantize_workspace_size(), None) == E.NVFP4_ERR_WORKSPACE
    assert f(x, bf, 40, 64, 64, 1, o1, o2, ws, wsb, None) == E.NVFP4_ERR_SHAPE               # R % 16
    assert f(x, bf, 64, 60, 64, 1, o1, o2, ws, wsb, None) == E.NVFP4_ERR_SHAPE               # C * 2 % 16
    assert f(C.c_void_p(0x10008), bf, 64, 64, 64, 1, o1, o2, ws, wsb, None) == E.NVFP4_ERR_ALIGNMENT


def test_mma_rate_probe_rejections(lib):
    ws, cyc, pairs = C.c_void_p(0x20000), C.c_void_p(0x40000), C.c_int(0)
    f = lib.nvfp4_selftest_mma_rate
    f.argtypes = [C.c_int, C.c_int64, C.c_void_p, C.c_int64, C.POINTER(C.c_int), C.c_void_p, C.c_size_t, C.c_void_p]
    E = binding
    assert f(0, 10, None, 74, C.byref(pairs), ws, 256, None) == E.NVFP4_ERR_INVALID_ARG      # no output buffer
    assert f(0, 10, cyc, 74, None, ws, 256, None) == E.NVFP4_ERR_INVALID_ARG                 # no pair count
    assert f(2, 10, cyc, 74, C.byref(pairs), ws, 256, None) == E.NVFP4_ERR_INVALID_ARG       # mx not 0/1
    assert f(0, 0, cyc, 74, C.byref(pairs), ws, 256, None) == E.NVFP4_ERR_INVALID_ARG        # iters < 1
    assert f(1, 1000001, cyc, 74, C.byref(pairs), ws, 256, None) == E.NVFP4_ERR_INVALID_ARG  # iters too many
    assert f(0, 10, cyc, 74, C.byref(pairs), None, 256, None) == E.NVFP4_ERR_WORKSPACE
    assert f(0, 10, cyc, 74, C.byref(pairs), ws, 255, None) == E.NVFP4_ERR_WORKSPACE
    assert f(0, 10, cyc, 74, C.byref(pairs), C.c_void_p(0x20008), 256, None) == E.NVFP4_ERR_ALIGNMENT
    assert f(0, 10, C.c_void_p(0x40004), 74, C.byref(pairs), ws, 256, None) == E.NVFP4_ERR_ALIGNMENT


def test_quantize_dual_rejections(lib):
    ws = C.c_void_p(0x20000)
    row, col = _tensor(64, 64), _tensor(64, 64)

    def dual(x=0x10000, dtype=1, R=64, Cc=64, ld=64, rnd=0, rht=0, r=None, c=None, w=ws, wsb=1 << 20, ar=None,
             ac=None):
        return lib.nvfp4_quantize_dual(C.c_void_p(x), dtype, R, Cc, ld, rnd, rht, 7, ar, ac,
                                       C.byref(r if r is not None else row), C.byref(c if c is not None else col),
                                       w, wsb, None)
    assert lib.nvfp4_quantize_dual_workspace_size() >= 256 + 2 * 4 * 1024
    assert dual(rnd=2) == binding.NVFP4_ERR_INVALID_ARG
    assert dual(rht=2) == binding.NVFP4_ERR_INVALID_ARG
    assert dual(R=60, r=_tensor(60, 64), c=_tensor(64, 60)) == binding.NVFP4_ERR_SHAPE        # colwise needs R % 16
    assert dual(Cc=72, ld=72, r=_tensor(64, 72), c=_tensor(72, 64)) == binding.NVFP4_ERR_SHAPE  # rowwise needs C % 16
    assert dual(c=_tensor(32, 64)) == binding.NVFP4_ERR_SHAPE
    assert dual(wsb=4352) == binding.NVFP4_ERR_WORKSPACE              # single-orientation size is not enough
    assert dual(w=None) == binding.NVFP4_ERR_WORKSPACE
    assert dual(x=0x10008) == binding.NVFP4_ERR_ALIGNMENT


def test_relu2_amax_rejections(lib):
    ws, a = C.c_void_p(0x20000), C.c_void_p(0x30000)
    y, h = C.c_void_p(0x10000), C.c_void_p(0x40000)
    assert lib.nvfp4_relu2_fwd_amax(y, h, -1, a, ws, 1 << 20, None) == binding.NVFP4_ERR_SHAPE
    assert lib.nvfp4_relu2_fwd_amax(y, h, 64, None, ws, 1 << 20, None) == binding.NVFP4_ERR_INVALID_ARG
    assert lib.nvfp4_relu2_fwd_amax(y, h, 64, C.c_void_p(0x30004), ws, 1 << 20, None) == binding.NVFP4_ERR_ALIGNMENT
    assert lib.nvfp4_relu2_fwd_amax(y, h, 64, a, ws, 100, None) == binding.NVFP4_ERR_WORKSPACE
    assert lib.nvfp4_relu2_bwd_amax(y, y, h, 64, a, None, 1 << 20, None) == binding.NVFP4_ERR_WORKSPACE
    assert lib.nvfp4_relu2_bwd_amax(None, y, h, 64, a, ws, 1 << 20, None) == binding.NVFP4_ERR_INVALID_ARG


def test_quantize_mx_rejections(lib):
    assert lib.nvfp4_mx_scales_bytes(1, 32) == 128 * 4
    assert lib.nvfp4_mx_scales_bytes(129, 160) == 256 * 8
    out = _tensor(64, 64)
    q = lambda x=0x10000, dtype=1, R=64, Cc=64, ld=64, ori=0, o=out: lib.nvfp4_quantize_mx(  # noqa: E731
        C.c_void_p(x), dtype, R, Cc, ld, ori, C.byref(o), None)
    assert q(dtype=5) == binding.NVFP4_ERR_INVALID_ARG
    assert q(ori=2) == binding.NVFP4_ERR_INVALID_ARG
    assert q(o=_tensor(64, 48), Cc=48, ld=48) == binding.NVFP4_ERR_SHAPE       # rowwise C % 32 != 0
    assert q(ori=1, R=48, o=_tensor(64, 48)) == binding.NVFP4_ERR_SHAPE       # colwise R % 32 != 0
    assert q(ori=1, Cc=68, ld=72, o=_tensor(68, 64)) == binding.NVFP4_ERR_SHAPE  # colwise C * 2 % 16 != 0
    assert q(o=_tensor(32, 64)) == binding.NVFP4_ERR_SHAPE                     # out shape
    assert q(ori=1, R=96, o=_tensor(96, 64)) == binding.NVFP4_ERR_SHAPE       # colwise out is [C x R]
    assert q(ld=60) == binding.NVFP4_ERR_SHAPE
    assert q(x=0x10008) == binding.NVFP4_ERR_ALIGNMENT
    big = 65535 * 256 + 32
    assert q(ori=1, R=big, o=_tensor(64, big)) == binding.NVFP4_ERR_SHAPE      # colwise R limit
    assert lib.nvfp4_quantize_mx(C.c_void_p(0x10000), 1, 64, 64, 64, 0, None, None) == binding.NVFP4_ERR_INVALID_ARG


def test_relu2_amax_rht_rejections(lib):
    ws, a, b = C.c_void_p(0x20000), C.c_void_p(0x30000), C.c_void_p(0x30010)
    y, h = C.c_void_p(0x10000), C.c_void_p(0x40000)
    f = lib.nvfp4_relu2_fwd_amax_rht
    assert f(y, h, 24, 64, 1, a, b, ws, 1 << 20, None) == binding.NVFP4_ERR_SHAPE       # R % 16
    assert f(y, h, 32, 60, 1, a, b, ws, 1 << 20, None) == binding.NVFP4_ERR_SHAPE       # C % 8
    assert f(y, h, 32, 64, 1, a, None, ws, 1 << 20, None) == binding.NVFP4_ERR_INVALID_ARG
    assert f(y, h, 32, 64, 1, a, b, ws, 4352, None) == binding.NVFP4_ERR_WORKSPACE       # needs two partial sets
    assert lib.nvfp4_relu2_bwd_amax_rht(None, y, h, 32, 64, 1, a, b, ws, 1 << 20, None) == \
        binding.NVFP4_ERR_INVALID_ARG


def test_nvtx_ranges_switch_on(lib):
    """NVFP4_NVTX=1 wraps every call in an NVTX range; with no profiler attached
    the calls still return their status (here: a rejected flag combination)."""
    code = textwrap.dedent("""
        import ctypes as C, sys
        sys.path.insert(0, %r)
        from nvfp4_bit_precision_quantize_b200 import binding
        lib = binding.load()
        out = binding.CTensor(0x1000, 0x2000, 0x3000, 64, 64)
        for _ in range(3):
            st = lib.nvfp4_quantize(C.c_void_p(0x10000), 1, 64, 64, 64, 0, 0, 1, 1, None, C.byref(out),
                                    C.c_void_p(0x20000), 1 << 20, None)
        print(st)
    """ % ROOT)
    env = dict(os.environ, NVFP4_NVTX="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert int(r.stdout.strip().splitlines()[-1]) == binding.NVFP4_ERR_INVALID_ARG
