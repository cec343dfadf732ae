"""CPU oracle for the NVFP4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product path (the CUDA library and its binding) never uses
it; the two share no code.  The arithmetic lives in nvfp4_oracle.c (plain C,
IEEE binary32 / binary64); this module only marshals numpy arrays.

Parity pins: see the header of nvfp4_oracle.c and tests/test_oracle_*.py.
"""
import ctypes as C

import numpy as np

from .build import build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = C.CDLL(path)
        u8p, u16p, u32p = C.POINTER(C.c_uint8), C.POINTER(C.c_uint16), C.POINTER(C.c_uint32)
        f32p, f64p, i64p = C.POINTER(C.c_float), C.POINTER(C.c_double), C.POINTER(C.c_int64)
        L.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        L.oracle_e2m1_value.argtypes = [C.c_uint]
        L.oracle_e2m1_value.restype = C.c_double
        L.oracle_e4m3_value.argtypes = [C.c_uint]
        L.oracle_e4m3_value.restype = C.c_double
        L.oracle_e2m1_rtn.argtypes = [C.c_float]
        L.oracle_e2m1_rtn.restype = C.c_uint
        L.oracle_e2m1_sr.argtypes = [C.c_float, C.c_uint32]
        L.oracle_e2m1_sr.restype = C.c_uint
        L.oracle_e4m3_rn_satfinite.argtypes = [C.c_float]
        L.oracle_e4m3_rn_satfinite.restype = C.c_uint
        L.oracle_rht_signs.argtypes = [C.c_uint64, f32p]
        L.oracle_fwht16.argtypes = [f32p]
        L.oracle_rht16.argtypes = [f32p, f32p]
        L.oracle_tensor_scale.argtypes = [C.c_float]
        L.oracle_tensor_scale.restype = C.c_float
        L.oracle_block_scale.argtypes = [C.c_float, C.c_float]
        L.oracle_block_scale.restype = C.c_uint
        L.oracle_quantize.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64,
                                      C.c_int, C.c_int, C.c_int, C.c_uint64, f32p,
                                      u8p, u8p, f32p, f32p]
        L.oracle_quantize.restype = C.c_int
        L.oracle_dot.argtypes = [u8p, u8p, C.c_float, u8p, u8p, C.c_float,
                                 C.c_int64, C.c_int64, C.c_int64, f64p, f64p]
        L.oracle_gemm.argtypes = [u8p, u8p, C.c_float, u8p, u8p, C.c_float,
                                  C.c_int64, C.c_int64, C.c_int64, f64p, f64p]
        L.oracle_gemm_sampled.argtypes = [u8p, u8p, C.c_float, u8p, u8p, C.c_float,
                                          C.c_int64, i64p, i64p, C.c_int64, f64p, f64p]
        L.oracle_bf16_from_f32.argtypes = [C.c_float]
        L.oracle_bf16_from_f32.restype = C.c_uint16
        L.oracle_relu2_fwd.argtypes = [u16p, C.c_int64, u16p]
        L.oracle_relu2_bwd.argtypes = [u16p, u16p, C.c_int64, u16p]
        L.oracle_amax.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64, C.c_int,
                                  C.c_int, C.c_uint64]
        L.oracle_amax.restype = C.c_float
        L.oracle_e8m0_value.argtypes = [C.c_uint]
        L.oracle_e8m0_value.restype = C.c_double
        L.oracle_mx_scale.argtypes = [C.c_float]
        L.oracle_mx_scale.restype = C.c_uint
        L.oracle_quantize_mx.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64, C.c_int, u8p, u8p]
        L.oracle_quantize_mx.restype = C.c_int
        L.oracle_gemm_mx.argtypes = [u8p, u8p, u8p, u8p, C.c_int64, C.c_int64, C.c_int64, f64p, f64p]
        L.oracle_quantize_rows.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64,
                                           C.c_int, C.c_int, C.c_int, C.c_uint64, C.c_float,
                                           i64p, C.c_int64, u8p, u8p]
        L.oracle_quantize_rows.restype = C.c_int
        L.oracle_e2m1_rtn_array.argtypes = [f32p, C.c_int64, u8p]
        L.oracle_e2m1_sr_array.argtypes = [f32p, u32p, C.c_int64, u8p]
        L.oracle_e4m3_rn_array.argtypes = [f32p, C.c_int64, u8p]
        _lib = L
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(C.POINTER(ct))


def philox4x32_10(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(_p(c, C.c_uint32), _p(k, C.c_uint32), _p(out, C.c_uint32))
    return out


def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code):
    return lib().oracle_e4m3_value(int(code))


def e2m1_rtn(r):
    return lib().oracle_e2m1_rtn(float(np.float32(r)))


def e2m1_sr(r, rnd16):
    return lib().oracle_e2m1_sr(float(np.float32(r)), int(rnd16))


def e4m3_rn(t):
    return lib().oracle_e4m3_rn_satfinite(float(np.float32(t)))


def e2m1_rtn_array(r):
    a = np.ascontiguousarray(r, dtype=np.float32)
    out = np.zeros(a.shape, np.uint8)
    lib().oracle_e2m1_rtn_array(_p(a, C.c_float), a.size, _p(out, C.c_uint8))
    return out


def e2m1_sr_array(r, rnd16):
    a = np.ascontiguousarray(r, dtype=np.float32)
    u = np.ascontiguousarray(rnd16, dtype=np.uint32)
    out = np.zeros(a.shape, np.uint8)
    lib().oracle_e2m1_sr_array(_p(a, C.c_float), _p(u, C.c_uint32), a.size, _p(out, C.c_uint8))
    return out


def e4m3_rn_array(t):
    a = np.ascontiguousarray(t, dtype=np.float32)
    out = np.zeros(a.shape, np.uint8)
    lib().oracle_e4m3_rn_array(_p(a, C.c_float), a.size, _p(out, C.c_uint8))
    return out


def tensor_scale(amax):
    return np.float32(lib().oracle_tensor_scale(float(np.float32(amax))))


def block_scale(amax_b, s_t):
    return lib().oracle_block_scale(float(np.float32(amax_b)), float(np.float32(s_t)))


def rht_signs(seed):
    d = np.zeros(16, np.float32)
    lib().oracle_rht_signs(C.c_uint64(seed), _p(d, C.c_float))
    return d


def fwht16(v):
    a = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().oracle_fwht16(_p(a, C.c_float))
    return a


def rht16(v, d):
    a = np.ascontiguousarray(v, dtype=np.float32).copy()
    dd = np.ascontiguousarray(d, dtype=np.float32)
    lib().oracle_rht16(_p(a, C.c_float), _p(dd, C.c_float))
    return a


def quantize(x, colwise=False, sr=False, rht=False, seed=1234, amax_in=None):
    """Quantise a 2-D array to NVFP4.

    x: float32 array, or uint16 array of bf16 bit patterns ([R x C], row-major).
    Returns (codes [rows' x K/2] uint8, scales [rows' x K/16] uint8 (plain
    row-major order), tensor_scale float32, amax float32).
    """
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        bf16 = 1
    elif x.dtype == np.float32:
        bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    R, Cc = x.shape
    rows, K = (Cc, R) if colwise else (R, Cc)
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    am = np.zeros(1, np.float32)
    ain = None
    if amax_in is not None:
        ain_arr = np.array([amax_in], np.float32)
        ain = _p(ain_arr, C.c_float)
    rc = lib().oracle_quantize(x.ctypes.data_as(C.c_void_p), bf16, R, Cc, Cc, int(colwise), int(sr),
                               int(rht), C.c_uint64(seed), ain, _p(codes, C.c_uint8),
                               _p(scales, C.c_uint8), _p(ts, C.c_float), _p(am, C.c_float))
    if rc != 0:
        raise ValueError("oracle_quantize rejected the arguments")
    return codes, scales, ts[0], am[0]


def _in(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, 1
    if x.dtype == np.float32:
        return x, 0
    raise TypeError("x must be float32 or uint16 (bf16 bits)")


def amax(x, colwise=False, rht=False, seed=1234):
    """Tensor amax of the (optionally transformed) output view."""
    x, bf16 = _in(x)
    R, Cc = x.shape
    return np.float32(lib().oracle_amax(x.ctypes.data_as(C.c_void_p), bf16, R, Cc, Cc, int(colwise),
                                        int(rht), C.c_uint64(seed)))


def quantize_rows(x, rows, amax_value, colwise=False, sr=False, rht=False, seed=1234):
    """Codes and plain scales of selected output rows of the quantised tensor."""
    x, bf16 = _in(x)
    R, Cc = x.shape
    K = R if colwise else Cc
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    codes = np.zeros((rows.size, K // 2), np.uint8)
    scales = np.zeros((rows.size, K // 16), np.uint8)
    rc = lib().oracle_quantize_rows(x.ctypes.data_as(C.c_void_p), bf16, R, Cc, Cc, int(colwise), int(sr),
                                    int(rht), C.c_uint64(seed), float(amax_value), _p(rows, C.c_int64),
                                    rows.size, _p(codes, C.c_uint8), _p(scales, C.c_uint8))
    if rc != 0:
        raise ValueError("oracle_quantize_rows rejected the arguments")
    return codes, scales


def dequantize(codes, scales, tensor_scale):
    """Dequantised values (float64 [rows x K]) of an NVFP4 tensor: e2m1 * e4m3 * s_t."""
    e2m1 = np.array([e2m1_value(c) for c in range(16)])
    e4m3 = np.array([e4m3_value(c) for c in range(256)])
    lo = codes & 0xF
    hi = codes >> 4
    q = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    sc = np.repeat(scales, 16, axis=1)
    return e2m1[q] * e4m3[sc] * float(tensor_scale)


def gemm(a, b):
    """Full FP64 GEMM of two NVFP4 tensors a, b = (codes, scales, ts).

    Returns (ref [M x N], abs [M x N]) with ref = A.B^T, abs = sum |a_k b_k|."""
    ac, asc, ats = a[0], a[1], a[2]
    bc, bsc, bts = b[0], b[1], b[2]
    M, N = ac.shape[0], bc.shape[0]
    K = ac.shape[1] * 2
    ref = np.zeros((M, N), np.float64)
    ab = np.zeros((M, N), np.float64)
    ac, asc, bc, bsc = (np.ascontiguousarray(t) for t in (ac, asc, bc, bsc))
    lib().oracle_gemm(_p(ac, C.c_uint8), _p(asc, C.c_uint8), float(ats), _p(bc, C.c_uint8),
                      _p(bsc, C.c_uint8), float(bts), M, N, K, _p(ref, C.c_double),
                      _p(ab, C.c_double))
    return ref, ab


def gemm_sampled(a, b, ms, ns):
    """FP64 reference for selected outputs (ms[i], ns[i])."""
    ac, asc, ats = (np.ascontiguousarray(a[0]), np.ascontiguousarray(a[1]), a[2])
    bc, bsc, bts = (np.ascontiguousarray(b[0]), np.ascontiguousarray(b[1]), b[2])
    K = ac.shape[1] * 2
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    ref = np.zeros(len(ms), np.float64)
    ab = np.zeros(len(ms), np.float64)
    lib().oracle_gemm_sampled(_p(ac, C.c_uint8), _p(asc, C.c_uint8), float(ats),
                              _p(bc, C.c_uint8), _p(bsc, C.c_uint8), float(bts), K,
                              _p(ms, C.c_int64), _p(ns, C.c_int64), len(ms),
                              _p(ref, C.c_double), _p(ab, C.c_double))
    return ref, ab


def bf16_from_f32(f):
    return lib().oracle_bf16_from_f32(float(np.float32(f)))


def relu2_fwd(y_bits):
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    h = np.zeros_like(y)
    lib().oracle_relu2_fwd(_p(y, C.c_uint16), y.size, _p(h, C.c_uint16))
    return h


def relu2_bwd(dh_bits, y_bits):
    dh = np.ascontiguousarray(dh_bits, dtype=np.uint16)
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    out = np.zeros_like(y)
    lib().oracle_relu2_bwd(_p(dh, C.c_uint16), _p(y, C.c_uint16), y.size, _p(out, C.c_uint16))
    return out


def e8m0_value(code):
    return lib().oracle_e8m0_value(int(code))


def mx_scale(amax_b):
    return lib().oracle_mx_scale(float(amax_b))


def quantize_mx(x, colwise=False):
    """MXFP4 quantisation of a 2-D array (float32, or uint16 bf16 bits); rowwise needs
    C % 32 == 0, colwise (transposed output) R % 32 == 0.

    Returns (codes [rows' x K/2] uint8, scales [rows' x K/32] uint8 E8M0 codes, plain row-major)."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        bf16 = 1
    elif x.dtype == np.float32:
        bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bf16 bits)")
    R, Cc = x.shape
    rows, K = (Cc, R) if colwise else (R, Cc)
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    if lib().oracle_quantize_mx(x.ctypes.data_as(C.c_void_p), bf16, R, Cc, Cc, int(colwise), _p(codes, C.c_uint8),
                                _p(scales, C.c_uint8)) != 0:
        raise ValueError("oracle_quantize_mx rejected the arguments")
    return codes, scales


def gemm_mx(a, b):
    """FP64 GEMM of two MXFP4 tensors a, b = (codes [rows x K/2], scales [rows x K/32]).

    Returns (ref [M x N], abs [M x N]) with ref = A.B^T, abs = sum |a_k b_k|."""
    ac, asc = (np.ascontiguousarray(t, dtype=np.uint8) for t in a[:2])
    bc, bsc = (np.ascontiguousarray(t, dtype=np.uint8) for t in b[:2])
    M, N, K = ac.shape[0], bc.shape[0], ac.shape[1] * 2
    if bc.shape[1] * 2 != K or K % 32 or asc.shape != (M, K // 32) or bsc.shape != (N, K // 32):
        raise ValueError("MXFP4 operands: codes [rows x K/2], scales [rows x K/32], one K (a multiple of 32)")
    ref = np.zeros((M, N), np.float64)
    ab = np.zeros((M, N), np.float64)
    lib().oracle_gemm_mx(_p(ac, C.c_uint8), _p(asc, C.c_uint8), _p(bc, C.c_uint8), _p(bsc, C.c_uint8), M, N, K,
                         _p(ref, C.c_double), _p(ab, C.c_double))
    return ref, ab


def dequantize_mx(codes, scales):
    """Binary64 values of an MXFP4 tensor (plain scales)."""
    R = codes.shape[0]
    vals = np.array([lib().oracle_e2m1_value(c) for c in range(16)])
    lo, hi = codes & 0xF, codes >> 4
    q = np.empty((R, codes.shape[1] * 2))
    q[:, 0::2], q[:, 1::2] = vals[lo], vals[hi]
    sc = np.array([lib().oracle_e8m0_value(int(c)) for c in range(256)])[scales]
    return q * np.repeat(sc, 32, axis=1)
