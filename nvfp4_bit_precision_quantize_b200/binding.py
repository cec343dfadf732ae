"""Thin ctypes binding of libnvfp4.so (include/nvfp4.h).

Argument marshalling only: torch supplies device memory and the current CUDA
stream; every computation runs in the library's CUDA kernels.  There is no
CPU fallback: if the library is missing or the device is not a B200 the calls
raise.  Function names follow the C ABI.
"""
import ctypes as C
import os
from dataclasses import dataclass

import torch

# NVFP4_CHECKED=1 selects the bounds-checked debug build (build.build(checked=True)).
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libnvfp4_checked.so" if os.environ.get("NVFP4_CHECKED") == "1" else "libnvfp4.so")

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_ALIGNMENT = 2
NVFP4_ERR_SHAPE = 3
NVFP4_ERR_WORKSPACE = 4
NVFP4_ERR_UNSUPPORTED_DEVICE = 5
NVFP4_ERR_CUDA = 6
NVFP4_ERR_DEVICE_TIMEOUT = 7
NVFP4_ERR_DEVICE_BOUNDS = 8

NVFP4_DTYPE_F32 = 0
NVFP4_DTYPE_BF16 = 1
NVFP4_ROWWISE = 0
NVFP4_COLWISE = 1
NVFP4_RTN = 0
NVFP4_SR = 1

# Functions declared in include/nvfp4.h (checked by the tests against the header).
EXPORTS = ("nvfp4_codes_bytes", "nvfp4_scales_bytes", "nvfp4_quantize_workspace_size", "nvfp4_quantize",
           "nvfp4_gemm", "nvfp4_linear_workspace_size", "nvfp4_linear_fwd", "nvfp4_linear_bwd",
           "nvfp4_relu2_fwd", "nvfp4_relu2_bwd", "nvfp4_check", "nvfp4_last_launch_count",
           "nvfp4_status_string", "nvfp4_linear_fwd_noalloc", "nvfp4_selftest_wait_timeout",
           "nvfp4_quantize_dual_workspace_size", "nvfp4_quantize_dual", "nvfp4_relu2_fwd_amax",
           "nvfp4_relu2_bwd_amax", "nvfp4_mx_scales_bytes", "nvfp4_quantize_mx",
           "nvfp4_relu2_fwd_amax_rht", "nvfp4_relu2_bwd_amax_rht", "nvfp4_linear_fwd_workspace_size",
           "nvfp4_gemm_mx", "nvfp4_gemm_relu2_fwd", "nvfp4_gemm_relu2_bwd", "nvfp4_selftest_mma_rate",
           "nvfp4_bounds_status", "nvfp4_selftest_bounds", "nvfp4_amax",
           "nvfp4_amax_dual")


class CTensor(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("tensor_scale", C.c_void_p),
                ("rows", C.c_int64), ("k", C.c_int64)]


class NVFP4Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


_lib = None


def load():
    """Load libnvfp4.so (built in-tree by nvfp4_bit_precision_quantize_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libnvfp4.so is not built; run `python -m nvfp4_bit_precision_quantize_b200.build`")
    L = C.CDLL(LIB_PATH)
    vp, i64, sz, i32, u64 = C.c_void_p, C.c_int64, C.c_size_t, C.c_int, C.c_uint64
    tp = C.POINTER(CTensor)
    sig = {
        "nvfp4_codes_bytes": (sz, [i64, i64]),
        "nvfp4_scales_bytes": (sz, [i64, i64]),
        "nvfp4_quantize_workspace_size": (sz, []),
        "nvfp4_quantize": (i32, [vp, i32, i64, i64, i64, i32, i32, i32, u64, vp, tp, vp, sz, vp]),
        "nvfp4_gemm": (i32, [tp, tp, vp, i32, i64, vp, sz, vp]),
        "nvfp4_gemm_mx": (i32, [tp, tp, vp, i32, i64, vp, sz, vp]),
        "nvfp4_gemm_relu2_fwd": (i32, [tp, tp, vp, vp, u64, vp, vp, vp, sz, vp]),
        "nvfp4_gemm_relu2_bwd": (i32, [tp, tp, vp, vp, u64, vp, vp, vp, sz, vp]),
        "nvfp4_linear_workspace_size": (sz, [i64, i64, i64]),
        "nvfp4_linear_fwd_workspace_size": (sz, [i64, i64, i64]),
        "nvfp4_linear_fwd": (i32, [vp, vp, vp, i64, i64, i64, i32, i32, vp, sz, vp]),
        "nvfp4_linear_bwd": (i32, [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, u64, vp, sz, vp]),
        "nvfp4_relu2_fwd": (i32, [vp, vp, i64, vp]),
        "nvfp4_relu2_bwd": (i32, [vp, vp, vp, i64, vp]),
        "nvfp4_check": (i32, [vp, vp]),
        "nvfp4_last_launch_count": (i32, []),
        "nvfp4_status_string": (C.c_char_p, [i32]),
        "nvfp4_linear_fwd_noalloc": (i32, [vp, vp, vp, i64, i64, i64, i32, i32, vp]),
        "nvfp4_selftest_wait_timeout": (i32, [vp, sz, u64, vp]),
        "nvfp4_selftest_mma_rate": (i32, [i32, i64, vp, i64, C.POINTER(C.c_int), vp, sz, vp]),
        "nvfp4_bounds_status": (i32, [C.POINTER(C.c_int), C.POINTER(C.c_int)]),
        "nvfp4_amax": (i32, [vp, i32, i64, i64, i64, i32, u64, vp, vp, sz, vp]),
        "nvfp4_amax_dual": (i32, [vp, i32, i64, i64, i64, u64, vp, vp, vp, sz, vp]),
        "nvfp4_selftest_bounds": (i32, [vp, i64, vp]),
        "nvfp4_quantize_dual_workspace_size": (sz, []),
        "nvfp4_quantize_dual": (i32, [vp, i32, i64, i64, i64, i32, i32, u64, vp, vp, tp, tp, vp, sz, vp]),
        "nvfp4_relu2_fwd_amax": (i32, [vp, vp, i64, vp, vp, sz, vp]),
        "nvfp4_relu2_bwd_amax": (i32, [vp, vp, vp, i64, vp, vp, sz, vp]),
        "nvfp4_mx_scales_bytes": (sz, [i64, i64]),
        "nvfp4_quantize_mx": (i32, [vp, i32, i64, i64, i64, i32, tp, vp]),
        "nvfp4_relu2_fwd_amax_rht": (i32, [vp, vp, i64, i64, u64, vp, vp, vp, sz, vp]),
        "nvfp4_relu2_bwd_amax_rht": (i32, [vp, vp, vp, i64, i64, u64, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return _lib


def status_string(status):
    return load().nvfp4_status_string(int(status)).decode()


def _ok(status, where):
    if status != NVFP4_OK:
        raise NVFP4Error(status, where)


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t == torch.bfloat16:
        return NVFP4_DTYPE_BF16
    if t == torch.float32:
        return NVFP4_DTYPE_F32
    raise TypeError("only float32 and bfloat16 are supported, got %s" % t)


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else None


# ----------------------------------------------------------------- argument checks
# The C ABI sees raw pointers and sizes only.  What it cannot check -- that a
# buffer is device memory of the current device, dense where the call assumes
# it, of the dtype passed and large enough -- is checked here before the call,
# so that a wrong tensor raises instead of reaching a kernel.

def _on_device(*tensors):
    ts = [t for t in tensors if t is not None]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensor on %s: the library takes CUDA tensors" % t.device)
    if ts:
        dev = torch.cuda.current_device()
        for t in ts:
            if t.device.index != dev:
                raise ValueError("tensor on %s: the library runs on the current device, cuda:%d" % (t.device, dev))


def _dense(name, t, shape=None, dtype=None):
    """t is contiguous, with the given shape and dtype."""
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s: dtype %s, expected %s" % (name, t.dtype, dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s: shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _rows(name, t):
    """A 2-D tensor whose rows are contiguous (any row stride)."""
    if t.dim() != 2:
        raise ValueError("%s must be 2-D, got %d-D" % (name, t.dim()))
    if t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError("%s: elements of a row must be contiguous (stride(1) == 1)" % name)
    _dtype_code(t.dtype)


def _nbytes(t):
    return t.numel() * t.element_size()


def _scalar_out(name, t):
    if t is not None and (t.dtype != torch.float32 or t.numel() < 1):
        raise ValueError("%s must be a float32 tensor with at least one element" % name)


def _workspace(ws):
    if ws is not None and not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")
    return _nbytes(ws) if ws is not None else 0


def _quantised(name, q, scales_bytes, tensor_scale=True):
    """The buffers of an NVFP4 / MXFP4 tensor are device memory and large enough."""
    _on_device(q.codes, q.scales, *([q.tensor_scale] if tensor_scale else []))
    for part, t in (("codes", q.codes), ("scales", q.scales)):
        if not t.is_contiguous():
            raise ValueError("%s.%s must be contiguous" % (name, part))
    if _nbytes(q.codes) < q.rows * (q.k // 2):
        raise ValueError("%s.codes: %d bytes, need %d" % (name, _nbytes(q.codes), q.rows * (q.k // 2)))
    if _nbytes(q.scales) < scales_bytes:
        raise ValueError("%s.scales: %d bytes, need %d" % (name, _nbytes(q.scales), scales_bytes))
    if tensor_scale:
        _scalar_out(name + ".tensor_scale", q.tensor_scale)


@dataclass
class NVFP4Tensor:
    """Device NVFP4 tensor [rows x k]: codes (uint8 [rows, k/2]), scales (uint8,
    scale-atom layout), tensor_scale (float32 [1])."""
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor
    rows: int
    k: int

    def c(self):
        ts = self.tensor_scale.data_ptr() if self.tensor_scale is not None else None  # MXFP4 has none
        return CTensor(self.codes.data_ptr(), self.scales.data_ptr(), ts, self.rows, self.k)


def nvfp4_codes_bytes(rows, k):
    return load().nvfp4_codes_bytes(rows, k)


def nvfp4_scales_bytes(rows, k):
    return load().nvfp4_scales_bytes(rows, k)


def nvfp4_quantize_workspace_size():
    return load().nvfp4_quantize_workspace_size()


def nvfp4_linear_workspace_size(M, N, K):
    return load().nvfp4_linear_workspace_size(M, N, K)


def nvfp4_linear_fwd_workspace_size(M, N, K):
    return load().nvfp4_linear_fwd_workspace_size(M, N, K)


def workspace(nbytes, device=None):
    """A zeroed workspace (its status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def empty_nvfp4(rows, k, device=None):
    device = device or "cuda"
    return NVFP4Tensor(
        codes=torch.empty((rows, k // 2), dtype=torch.uint8, device=device),
        scales=torch.empty(max(nvfp4_scales_bytes(rows, k), 16), dtype=torch.uint8, device=device),
        tensor_scale=torch.empty(1, dtype=torch.float32, device=device), rows=rows, k=k)


def nvfp4_quantize(x, orientation=NVFP4_ROWWISE, rounding=NVFP4_RTN, rht=False, seed=1234, amax_in=None,
                   out=None, ws=None, stream=None):
    """Quantise a 2-D float32/bfloat16 CUDA tensor to NVFP4 (see include/nvfp4.h)."""
    _rows("x", x)
    R, Cc = x.shape
    rows, k = (Cc, R) if orientation == NVFP4_COLWISE else (R, Cc)
    out = out or empty_nvfp4(rows, k, x.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_workspace_size(), x.device)
    _on_device(x, amax_in, ws)
    _scalar_out("amax_in", amax_in)
    _quantised("out", out, nvfp4_scales_bytes(out.rows, out.k))
    ct = out.c()
    st = load().nvfp4_quantize(_ptr(x), _dtype_code(x.dtype), R, Cc, x.stride(0), orientation, rounding,
                               int(bool(rht)), seed, _ptr(amax_in), C.byref(ct), _ptr(ws), _workspace(ws),
                               _stream(stream))
    _ok(st, "nvfp4_quantize")
    return out


def nvfp4_amax(x, rht=False, seed=1234, out=None, ws=None, stream=None):
    """max |x| of a 2-D float32/bfloat16 CUDA tensor (with rht, of the 16-row Hadamard transform of
    its columns) into a one-float device tensor, as nvfp4_quantize's amax pass computes it."""
    _rows("x", x)
    R, Cc = x.shape
    out = _amax_buffer(out, x.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_workspace_size(), x.device)
    _on_device(x, out, ws)
    _ok(load().nvfp4_amax(_ptr(x), _dtype_code(x.dtype), R, Cc, x.stride(0), int(bool(rht)), seed, _ptr(out),
                          _ptr(ws), _workspace(ws), _stream(stream)), "nvfp4_amax")
    return out


def nvfp4_amax_dual(x, seed=1234, out=None, out_rht=None, ws=None, stream=None):
    """max |x| and max |RHT(x)| (16-row transform down the columns) of a 2-D float32/bfloat16 CUDA
    tensor from one read; returns the two one-float device tensors."""
    _rows("x", x)
    R, Cc = x.shape
    out = _amax_buffer(out, x.device)
    out_rht = _amax_buffer(out_rht, x.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_dual_workspace_size(), x.device)
    _on_device(x, out, out_rht, ws)
    _ok(load().nvfp4_amax_dual(_ptr(x), _dtype_code(x.dtype), R, Cc, x.stride(0), seed, _ptr(out), _ptr(out_rht),
                               _ptr(ws), _workspace(ws), _stream(stream)), "nvfp4_amax_dual")
    return out, out_rht


def nvfp4_mx_scales_bytes(rows, k):
    return load().nvfp4_mx_scales_bytes(rows, k)


def nvfp4_quantize_mx(x, orientation=NVFP4_ROWWISE, out=None, stream=None):
    """MXFP4 quantisation of a 2-D float32/bfloat16 CUDA tensor (rowwise: C % 32 == 0;
    colwise, transposed output: R % 32 == 0)."""
    _rows("x", x)
    R, Cc = x.shape
    rows, k = (Cc, R) if orientation == NVFP4_COLWISE else (R, Cc)
    out = out or NVFP4Tensor(codes=torch.empty((rows, k // 2), dtype=torch.uint8, device=x.device),
                             scales=torch.empty(max(nvfp4_mx_scales_bytes(rows, k), 16), dtype=torch.uint8,
                                                device=x.device),
                             tensor_scale=None, rows=rows, k=k)
    _on_device(x)
    _quantised("out", out, nvfp4_mx_scales_bytes(out.rows, out.k), tensor_scale=False)
    ct = out.c()
    _ok(load().nvfp4_quantize_mx(_ptr(x), _dtype_code(x.dtype), R, Cc, x.stride(0), orientation, C.byref(ct),
                                 _stream(stream)), "nvfp4_quantize_mx")
    return out


def nvfp4_quantize_dual_workspace_size():
    return load().nvfp4_quantize_dual_workspace_size()


def nvfp4_quantize_dual(x, col_rounding=NVFP4_RTN, col_rht=False, seed=1234, amax_row_in=None, amax_col_in=None,
                        out_row=None, out_col=None, ws=None, stream=None):
    """Rowwise (RTN) and colwise NVFP4 of one 2-D tensor from one read; returns (row, col)."""
    _rows("x", x)
    R, Cc = x.shape
    out_row = out_row or empty_nvfp4(R, Cc, x.device)
    out_col = out_col or empty_nvfp4(Cc, R, x.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_dual_workspace_size(), x.device)
    _on_device(x, amax_row_in, amax_col_in, ws)
    _scalar_out("amax_row_in", amax_row_in)
    _scalar_out("amax_col_in", amax_col_in)
    _quantised("out_row", out_row, nvfp4_scales_bytes(out_row.rows, out_row.k))
    _quantised("out_col", out_col, nvfp4_scales_bytes(out_col.rows, out_col.k))
    cr, cc = out_row.c(), out_col.c()
    st = load().nvfp4_quantize_dual(_ptr(x), _dtype_code(x.dtype), R, Cc, x.stride(0), col_rounding,
                                    int(bool(col_rht)), seed, _ptr(amax_row_in), _ptr(amax_col_in), C.byref(cr),
                                    C.byref(cc), _ptr(ws), _workspace(ws), _stream(stream))
    _ok(st, "nvfp4_quantize_dual")
    return out_row, out_col


def nvfp4_gemm(A, B, out_dtype=torch.bfloat16, out=None, ws=None, stream=None):
    """C = (A . B^T) * sA * sB for NVFP4 tensors A [M x K], B [N x K]."""
    M, N = A.rows, B.rows
    out = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=A.codes.device)
    ws = ws if ws is not None else workspace(256, A.codes.device)
    _quantised("A", A, nvfp4_scales_bytes(A.rows, A.k))
    _quantised("B", B, nvfp4_scales_bytes(B.rows, B.k))
    _rows("out", out)
    if out.shape[0] < M or out.shape[1] < N:
        raise ValueError("out: shape %s, need at least (%d, %d)" % (tuple(out.shape), M, N))
    _on_device(out, ws)
    ca, cb = A.c(), B.c()
    st = load().nvfp4_gemm(C.byref(ca), C.byref(cb), _ptr(out), _dtype_code(out.dtype), out.stride(0), _ptr(ws),
                           _workspace(ws), _stream(stream))
    _ok(st, "nvfp4_gemm")
    return out


def nvfp4_gemm_mx(A, B, out_dtype=torch.bfloat16, out=None, ws=None, stream=None):
    """C = A . B^T for MXFP4 tensors A [M x K], B [N x K] (from nvfp4_quantize_mx)."""
    M, N = A.rows, B.rows
    out = out if out is not None else torch.empty((M, N), dtype=out_dtype, device=A.codes.device)
    ws = ws if ws is not None else workspace(256, A.codes.device)
    _quantised("A", A, nvfp4_mx_scales_bytes(A.rows, A.k), tensor_scale=False)
    _quantised("B", B, nvfp4_mx_scales_bytes(B.rows, B.k), tensor_scale=False)
    _rows("out", out)
    if out.shape[0] < M or out.shape[1] < N:
        raise ValueError("out: shape %s, need at least (%d, %d)" % (tuple(out.shape), M, N))
    _on_device(out, ws)
    ca, cb = A.c(), B.c()
    st = load().nvfp4_gemm_mx(C.byref(ca), C.byref(cb), _ptr(out), _dtype_code(out.dtype), out.stride(0), _ptr(ws),
                              _workspace(ws), _stream(stream))
    _ok(st, "nvfp4_gemm_mx")
    return out


def _gemm_relu2(name, A, B, y, out, seed, amax_out, amax_rht_out, ws, stream):
    M, N = A.rows, B.rows
    dev = A.codes.device
    out = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    amax_out = _amax_buffer(amax_out, dev)
    amax_rht_out = _amax_buffer(amax_rht_out, dev)
    ws = ws if ws is not None else workspace(nvfp4_quantize_dual_workspace_size(), dev)
    _quantised("A", A, nvfp4_scales_bytes(A.rows, A.k))
    _quantised("B", B, nvfp4_scales_bytes(B.rows, B.k))
    for nm, t in (("y", y), ("out", out)):
        _dense(nm, t, shape=(M, N), dtype=torch.bfloat16)
    _on_device(y, out, amax_out, amax_rht_out, ws)
    ca, cb = A.c(), B.c()
    st = getattr(load(), name)(C.byref(ca), C.byref(cb), _ptr(y), _ptr(out), seed, _ptr(amax_out),
                               _ptr(amax_rht_out), _ptr(ws), _workspace(ws), _stream(stream))
    _ok(st, name)
    return out, amax_out, amax_rht_out


def nvfp4_gemm_relu2_fwd(A, B, seed=1234, y=None, h=None, amax_out=None, amax_rht_out=None, ws=None, stream=None):
    """y = bf16(A . B^T sA sB) and h = relu(y)^2 (bf16), with max|h| and max|RHT(h)|.
    Returns (y, h, amax, amax_rht)."""
    y = y if y is not None else torch.empty((A.rows, B.rows), dtype=torch.bfloat16, device=A.codes.device)
    h, a0, a1 = _gemm_relu2("nvfp4_gemm_relu2_fwd", A, B, y, h, seed, amax_out, amax_rht_out, ws, stream)
    return y, h, a0, a1


def nvfp4_gemm_relu2_bwd(A, B, y, seed=1234, out=None, amax_out=None, amax_rht_out=None, ws=None, stream=None):
    """dY = bf16(bf16(A . B^T sA sB) * 2 relu(y)) for the forward's y, with max|dY| and
    max|RHT(dY)|.  Returns (dY, amax, amax_rht)."""
    return _gemm_relu2("nvfp4_gemm_relu2_bwd", A, B, y, out, seed, amax_out, amax_rht_out, ws, stream)


def _linear_operands(X, W):
    """X [M x K] and W [N x K], contiguous, one dtype; returns (M, N, K)."""
    _rows("X", X)
    _rows("W", W)
    M, K = X.shape
    N = W.shape[0]
    _dense("X", X)
    _dense("W", W, shape=(N, K), dtype=X.dtype)
    return M, N, K


def nvfp4_linear_fwd(X, W, y_dtype=torch.bfloat16, out=None, ws=None, stream=None):
    M, N, K = _linear_operands(X, W)
    out = out if out is not None else torch.empty((M, N), dtype=y_dtype, device=X.device)
    ws = ws if ws is not None else workspace(nvfp4_linear_fwd_workspace_size(M, N, K), X.device)
    _dense("out", out, shape=(M, N))
    _on_device(X, W, out, ws)
    st = load().nvfp4_linear_fwd(_ptr(X), _ptr(W), _ptr(out), M, N, K, _dtype_code(X.dtype),
                                 _dtype_code(out.dtype), _ptr(ws), _workspace(ws), _stream(stream))
    _ok(st, "nvfp4_linear_fwd")
    return out


def nvfp4_linear_bwd(dY, X, W, seed=1234, dx_dtype=torch.bfloat16, dX=None, dW=None, ws=None, stream=None):
    M, N, K = _linear_operands(X, W)
    _dense("dY", dY, shape=(M, N), dtype=X.dtype)
    dX = dX if dX is not None else torch.empty((M, K), dtype=dx_dtype, device=X.device)
    dW = dW if dW is not None else torch.empty((N, K), dtype=torch.float32, device=X.device)
    ws = ws if ws is not None else workspace(nvfp4_linear_workspace_size(M, N, K), X.device)
    _dense("dX", dX, shape=(M, K))
    _dense("dW", dW, shape=(N, K), dtype=torch.float32)
    _on_device(dY, X, W, dX, dW, ws)
    st = load().nvfp4_linear_bwd(_ptr(dY), _ptr(X), _ptr(W), _ptr(dX), _ptr(dW), M, N, K, _dtype_code(X.dtype),
                                 _dtype_code(dX.dtype), seed, _ptr(ws), _workspace(ws), _stream(stream))
    _ok(st, "nvfp4_linear_bwd")
    return dX, dW


def nvfp4_linear_fwd_noalloc(X, W, y_dtype=torch.bfloat16, out=None, stream=None):
    """nvfp4_linear_fwd without a workspace: the library's fixed scratch buffer is
    used instead (see include/nvfp4.h).  Only `out` may be allocated here, and only
    when the caller passes none."""
    M, N, K = _linear_operands(X, W)
    out = out if out is not None else torch.empty((M, N), dtype=y_dtype, device=X.device)
    _dense("out", out, shape=(M, N))
    _on_device(X, W, out)
    st = load().nvfp4_linear_fwd_noalloc(_ptr(X), _ptr(W), _ptr(out), M, N, K, _dtype_code(X.dtype),
                                         _dtype_code(out.dtype), _stream(stream))
    _ok(st, "nvfp4_linear_fwd_noalloc")
    return out


def _bf16_like(name, t, ref):
    _dense(name, t, shape=tuple(ref.shape), dtype=torch.bfloat16)


def nvfp4_relu2_fwd(y, out=None, stream=None):
    _dense("y", y, dtype=torch.bfloat16)
    out = out if out is not None else torch.empty_like(y)
    _bf16_like("out", out, y)
    _on_device(y, out)
    _ok(load().nvfp4_relu2_fwd(_ptr(y), _ptr(out), y.numel(), _stream(stream)), "nvfp4_relu2_fwd")
    return out


def nvfp4_relu2_bwd(dh, y, out=None, stream=None):
    _dense("y", y, dtype=torch.bfloat16)
    _bf16_like("dh", dh, y)
    out = out if out is not None else torch.empty_like(y)
    _bf16_like("out", out, y)
    _on_device(dh, y, out)
    _ok(load().nvfp4_relu2_bwd(_ptr(dh), _ptr(y), _ptr(out), y.numel(), _stream(stream)), "nvfp4_relu2_bwd")
    return out


def _amax_buffer(t, device):
    t = t if t is not None else torch.empty(4, dtype=torch.float32, device=device)
    _scalar_out("amax output", t)
    return t


def nvfp4_relu2_fwd_amax(y, out=None, amax_out=None, ws=None, stream=None):
    """relu(y)^2 and max |output| (a 1-element float32 CUDA tensor); returns (out, amax_out)."""
    _dense("y", y, dtype=torch.bfloat16)
    out = out if out is not None else torch.empty_like(y)
    _bf16_like("out", out, y)
    amax_out = _amax_buffer(amax_out, y.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_workspace_size(), y.device)
    _on_device(y, out, amax_out, ws)
    _ok(load().nvfp4_relu2_fwd_amax(_ptr(y), _ptr(out), y.numel(), _ptr(amax_out), _ptr(ws), _workspace(ws),
                                    _stream(stream)), "nvfp4_relu2_fwd_amax")
    return out, amax_out


def nvfp4_relu2_bwd_amax(dh, y, out=None, amax_out=None, ws=None, stream=None):
    """dh * 2 relu(y) and max |output|; returns (out, amax_out)."""
    _dense("y", y, dtype=torch.bfloat16)
    _bf16_like("dh", dh, y)
    out = out if out is not None else torch.empty_like(y)
    _bf16_like("out", out, y)
    amax_out = _amax_buffer(amax_out, y.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_workspace_size(), y.device)
    _on_device(dh, y, out, amax_out, ws)
    _ok(load().nvfp4_relu2_bwd_amax(_ptr(dh), _ptr(y), _ptr(out), y.numel(), _ptr(amax_out), _ptr(ws),
                                    _workspace(ws), _stream(stream)), "nvfp4_relu2_bwd_amax")
    return out, amax_out


def nvfp4_relu2_fwd_amax_rht(y, seed=1234, out=None, amax_out=None, amax_rht_out=None, ws=None, stream=None):
    """relu(y)^2 of a 2-D bf16 tensor plus max|out| and max|RHT(out)|; returns (out, amax, amax_rht)."""
    _rows("y", y)
    _dense("y", y, dtype=torch.bfloat16)
    R, Cc = y.shape
    out = out if out is not None else torch.empty_like(y)
    _bf16_like("out", out, y)
    amax_out = _amax_buffer(amax_out, y.device)
    amax_rht_out = _amax_buffer(amax_rht_out, y.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_dual_workspace_size(), y.device)
    _on_device(y, out, amax_out, amax_rht_out, ws)
    _ok(load().nvfp4_relu2_fwd_amax_rht(_ptr(y), _ptr(out), R, Cc, seed, _ptr(amax_out), _ptr(amax_rht_out),
                                        _ptr(ws), _workspace(ws), _stream(stream)), "nvfp4_relu2_fwd_amax_rht")
    return out, amax_out, amax_rht_out


def nvfp4_relu2_bwd_amax_rht(dh, y, seed=1234, out=None, amax_out=None, amax_rht_out=None, ws=None, stream=None):
    """dh * 2 relu(y) of 2-D bf16 tensors plus max|out| and max|RHT(out)|; returns (out, amax, amax_rht)."""
    _rows("y", y)
    _dense("y", y, dtype=torch.bfloat16)
    _bf16_like("dh", dh, y)
    R, Cc = y.shape
    out = out if out is not None else torch.empty_like(y)
    _bf16_like("out", out, y)
    amax_out = _amax_buffer(amax_out, y.device)
    amax_rht_out = _amax_buffer(amax_rht_out, y.device)
    ws = ws if ws is not None else workspace(nvfp4_quantize_dual_workspace_size(), y.device)
    _on_device(dh, y, out, amax_out, amax_rht_out, ws)
    _ok(load().nvfp4_relu2_bwd_amax_rht(_ptr(dh), _ptr(y), _ptr(out), R, Cc, seed, _ptr(amax_out),
                                        _ptr(amax_rht_out), _ptr(ws), _workspace(ws), _stream(stream)),
        "nvfp4_relu2_bwd_amax_rht")
    return out, amax_out, amax_rht_out


def nvfp4_check(ws, stream=None):
    """Synchronise and read/clear the workspace status word; raises on a device error."""
    _on_device(ws)
    _ok(load().nvfp4_check(_ptr(ws), _stream(stream)), "nvfp4_check")


def nvfp4_selftest_wait_timeout(ws, limit_ns, stream=None):
    """Launch the device-timeout self-test (its status is read by nvfp4_check)."""
    _on_device(ws)
    _ok(load().nvfp4_selftest_wait_timeout(_ptr(ws), _workspace(ws), int(limit_ns), _stream(stream)),
        "nvfp4_selftest_wait_timeout")


def nvfp4_selftest_mma_rate(cycles, ws, iters, mx=False, stream=None):
    """Launch the tensor-pipe rate probe; `cycles` is an int64 device tensor with at
    least SMs/2 entries.  Returns the number of CTA pairs that ran (cycles[:pairs]
    hold their cycle counts once the stream reaches the launch)."""
    _on_device(cycles, ws)
    if cycles.dtype != torch.int64 or not cycles.is_contiguous():
        raise ValueError("cycles must be a contiguous int64 tensor")
    pairs = C.c_int(0)
    _ok(load().nvfp4_selftest_mma_rate(1 if mx else 0, int(iters), _ptr(cycles), cycles.numel(), C.byref(pairs),
                                       _ptr(ws), _workspace(ws), _stream(stream)), "nvfp4_selftest_mma_rate")
    return pairs.value


def nvfp4_bounds_status():
    """(checked_build, site, status) from the bounds-checked build's records (read and
    cleared); in the product build (False, 0, NVFP4_OK)."""
    checked, site = C.c_int(0), C.c_int(0)
    st = load().nvfp4_bounds_status(C.byref(checked), C.byref(site))
    if st not in (NVFP4_OK, NVFP4_ERR_DEVICE_BOUNDS):
        raise NVFP4Error(st, "nvfp4_bounds_status")
    return bool(checked.value), site.value, st


def nvfp4_selftest_bounds(buf, stream=None):
    """Checked build only: one passing and one failing index check on a uint8 device
    tensor of n + 1 bytes (n = buf.numel() - 1)."""
    _on_device(buf)
    if buf.dtype != torch.uint8 or buf.numel() < 2:
        raise ValueError("buf must be a uint8 tensor of at least 2 bytes")
    _ok(load().nvfp4_selftest_bounds(_ptr(buf), buf.numel() - 1, _stream(stream)), "nvfp4_selftest_bounds")


def nvfp4_last_launch_count():
    return load().nvfp4_last_launch_count()
