// api.cu -- the C ABI (include/nvfp4.h): argument checks, workspace layout and
// the kernel sequences of the linear layer.  Nothing here allocates memory.
#include <algorithm>
#include <cstdint>
#include <cstdlib>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"
#include "nvfp4.h"

namespace nvfp4 {

namespace {
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {};
int g_cc_ok[kMaxDevices] = {};  // 0 unknown, 1 sm_100, 2 other
}  // namespace

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (!g_sms[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_sms[dev] = n > 0 ? n : 148;
    }
    return g_sms[dev];
}

}  // namespace nvfp4

namespace {

using namespace nvfp4;

thread_local int g_last_launches = 0;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
size_t esize(nvfp4_dtype d) { return d == NVFP4_DTYPE_BF16 ? 2 : 4; }
bool valid_dtype(int d) { return d == NVFP4_DTYPE_F32 || d == NVFP4_DTYPE_BF16; }

nvfp4_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    if (!g_cc_ok[dev]) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        g_cc_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return g_cc_ok[dev] == 1 ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED_DEVICE;
}

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Host-side checks of nvfp4_quantize; launches nothing.
nvfp4_status validate_quantize(const void *x, int dtype, int64_t R, int64_t C, int64_t ld, int orientation,
                               int rounding, int rht, const float *amax_in, const nvfp4_tensor *out,
                               const void *ws, size_t ws_bytes) {
    if (!out || !out->tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || (orientation != NVFP4_ROWWISE && orientation != NVFP4_COLWISE) ||
        (rounding != NVFP4_RTN && rounding != NVFP4_SR) || (rht != 0 && rht != 1))
        return NVFP4_ERR_INVALID_ARG;
    if (rht && orientation != NVFP4_COLWISE) return NVFP4_ERR_INVALID_ARG;
    if (R < 0 || C < 0) return NVFP4_ERR_SHAPE;
    const bool colwise = orientation == NVFP4_COLWISE;
    const int64_t rows = colwise ? C : R, k = colwise ? R : C;
    if (out->rows != rows || out->k != k) return NVFP4_ERR_SHAPE;
    if (R == 0 || C == 0) return NVFP4_OK;
    const size_t es = esize((nvfp4_dtype)dtype);
    if (!x || !out->codes || !out->scales) return NVFP4_ERR_INVALID_ARG;
    if (ld < C) return NVFP4_ERR_SHAPE;
    if (!colwise && C % 16 != 0) return NVFP4_ERR_SHAPE;
    if (colwise && (R % 16 != 0 || (C * (int64_t)es) % 16 != 0)) return NVFP4_ERR_SHAPE;
    if (R > (1LL << 31) || C > (1LL << 31) || (colwise && R > kMaxColwiseRows)) return NVFP4_ERR_SHAPE;
    if (!aligned16(x) || (ld * (int64_t)es) % 16 != 0 || !aligned16(out->codes) || !aligned16(out->scales))
        return NVFP4_ERR_ALIGNMENT;
    if (!amax_in) {
        if (!ws || ws_bytes < kQuantizeWorkspace) return NVFP4_ERR_WORKSPACE;
        if (!aligned16(ws)) return NVFP4_ERR_ALIGNMENT;
    }
    return NVFP4_OK;
}

nvfp4_status validate_gemm(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *C, int c_dtype, int64_t ldc,
                           const void *ws, size_t ws_bytes) {
    if (!A || !B || !valid_dtype(c_dtype)) return NVFP4_ERR_INVALID_ARG;
    if (A->rows < 0 || B->rows < 0 || A->k < 0 || A->k != B->k) return NVFP4_ERR_SHAPE;
    const int64_t M = A->rows, N = B->rows, K = A->k;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!C) return NVFP4_ERR_INVALID_ARG;
    if (ldc < N) return NVFP4_ERR_SHAPE;
    if (K % 64 != 0 || M >= (1LL << 31) || N >= (1LL << 31) || K >= (1LL << 31)) return NVFP4_ERR_SHAPE;
    const size_t es = esize((nvfp4_dtype)c_dtype);
    if (!aligned16(C) || (ldc * (int64_t)es) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
    if (K > 0) {
        if (!A->codes || !A->scales || !A->tensor_scale || !B->codes || !B->scales || !B->tensor_scale)
            return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(A->codes) || !aligned16(B->codes) || !aligned16(A->scales) || !aligned16(B->scales))
            return NVFP4_ERR_ALIGNMENT;
        if (!ws || ws_bytes < kStatusBytes) return NVFP4_ERR_WORKSPACE;
        if (!aligned16(ws)) return NVFP4_ERR_ALIGNMENT;
    }
    return NVFP4_OK;
}

// Carves NVFP4 operand buffers out of a linear-layer workspace (after the
// status word and the amax partials).
struct Carver {
    uint8_t *base;
    size_t off;
    nvfp4_tensor take(int64_t rows, int64_t k, float *ts) {
        nvfp4_tensor t;
        t.rows = rows;
        t.k = k;
        t.codes = base ? base + off : nullptr;
        off = round256(off + nvfp4_codes_bytes(rows, k));
        t.scales = base ? base + off : nullptr;
        off = round256(off + nvfp4_scales_bytes(rows, k));
        t.tensor_scale = ts;
        return t;
    }
};
constexpr size_t kScalarsOff = kDualWorkspace;                // 4 tensor scales (after two amax partial sets)
constexpr size_t kBuffersOff = kDualWorkspace + 256;

size_t fwd_bytes(int64_t M, int64_t N, int64_t K) {
    Carver c{nullptr, kBuffersOff};
    c.take(M, K, nullptr);
    c.take(N, K, nullptr);
    return c.off;
}
size_t bwd_bytes(int64_t M, int64_t N, int64_t K) {
    Carver c{nullptr, kBuffersOff};
    c.take(M, N, nullptr);
    c.take(K, N, nullptr);
    c.take(N, M, nullptr);
    c.take(K, M, nullptr);
    return c.off;
}

// NVTX ranges around the C-ABI calls, for timeline profilers: off unless the
// process starts with NVFP4_NVTX=1 in its environment (read once).  Without a
// profiler attached the NVTX calls do nothing.
bool nvtx_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("NVFP4_NVTX");
        return e != nullptr && e[0] == '1' && e[1] == '\0';
    }();
    return on;
}

struct Call {  // per-call launch accounting and the optional NVTX range
    int launches = 0;
    const bool ranged;
    explicit Call(const char *name) : ranged(nvtx_enabled()) {
        if (ranged) nvtxRangePushA(name);
    }
    ~Call() {
        if (ranged) nvtxRangePop();
    }
    Call(const Call &) = delete;
    Call &operator=(const Call &) = delete;
    nvfp4_status done(nvfp4_status st) {
        if (st == NVFP4_OK) g_last_launches = launches;
        return st;
    }
};

nvfp4_status quantize_impl(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, int orientation,
                           int rounding, int rht, uint64_t seed, const float *amax_in, const nvfp4_tensor *out,
                           void *ws, cudaStream_t stream, int *launches) {
    QuantizeArgs a;
    a.x = x;
    a.bf16 = dtype == NVFP4_DTYPE_BF16;
    a.R = R;
    a.C = C;
    a.ld = ld;
    a.colwise = orientation == NVFP4_COLWISE;
    a.sr = rounding == NVFP4_SR;
    a.rht = rht != 0;
    a.seed = seed;
    a.amax_in = amax_in;
    a.codes = out->codes;
    a.scales = out->scales;
    a.tensor_scale = out->tensor_scale;
    a.partials = ws ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kStatusBytes) : nullptr;
    a.status = static_cast<int *>(ws);
    return from_cuda(launch_quantize(a, stream, launches));
}

nvfp4_status gemm_impl(const nvfp4_tensor *A, const nvfp4_tensor *B, void *C, nvfp4_dtype c_dtype, int64_t ldc,
                       void *ws, cudaStream_t stream, int *launches, bool mx = false) {
    GemmArgs g;
    g.a_codes = A->codes;
    g.a_scales = A->scales;
    g.a_ts = A->tensor_scale;
    g.b_codes = B->codes;
    g.b_scales = B->scales;
    g.b_ts = B->tensor_scale;
    g.M = A->rows;
    g.N = B->rows;
    g.K = A->k;
    g.C = C;
    g.c_bf16 = c_dtype == NVFP4_DTYPE_BF16;
    g.ldc = ldc;
    g.status = static_cast<int *>(ws);
    g.mx = mx;
    return from_cuda(launch_gemm(g, stream, launches));
}

nvfp4_status dual_impl(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, int col_rounding,
                       int col_rht, uint64_t seed, const float *amax_row_in, const float *amax_col_in,
                       const nvfp4_tensor *out_row, const nvfp4_tensor *out_col, void *ws, cudaStream_t stream,
                       int *launches) {
    DualQuantizeArgs a;
    a.x = x;
    a.bf16 = dtype == NVFP4_DTYPE_BF16;
    a.R = R;
    a.C = C;
    a.ld = ld;
    a.col_sr = col_rounding == NVFP4_SR;
    a.col_rht = col_rht != 0;
    a.seed = seed;
    a.amax_row_in = amax_row_in;
    a.amax_col_in = amax_col_in;
    a.row_codes = out_row->codes;
    a.row_scales = out_row->scales;
    a.row_tensor_scale = out_row->tensor_scale;
    a.col_codes = out_col->codes;
    a.col_scales = out_col->scales;
    a.col_tensor_scale = out_col->tensor_scale;
    a.row_partials = ws ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kStatusBytes) : nullptr;
    a.col_partials = a.row_partials ? a.row_partials + kMaxPartials : nullptr;
    return from_cuda(launch_quantize_dual(a, stream, launches));
}

}  // namespace

namespace nvfp4 {

size_t linear_fwd_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 0) return 0;
    return fwd_bytes(M, N, K);
}

// Every host-side check nvfp4_linear_fwd makes before it launches anything,
// device check included; M or N == 0 passes (nothing to do).
nvfp4_status linear_fwd_validate(const void *X, const void *W, const void *Y, int64_t M, int64_t N, int64_t K,
                                 nvfp4_dtype dtype, nvfp4_dtype y_dtype, const void *workspace, size_t ws_bytes) {
    if (!valid_dtype(dtype) || !valid_dtype(y_dtype)) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || K % 64 != 0) return NVFP4_ERR_SHAPE;
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!X || !W || !Y) return NVFP4_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < fwd_bytes(M, N, K)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    uint8_t *ws = static_cast<uint8_t *>(const_cast<void *>(workspace));
    float *ts = reinterpret_cast<float *>(ws + kScalarsOff);
    Carver cv{ws, kBuffersOff};
    const nvfp4_tensor xq = cv.take(M, K, ts + 0), wq = cv.take(N, K, ts + 1);
    nvfp4_status st;
    if ((st = validate_quantize(X, dtype, M, K, K, NVFP4_ROWWISE, NVFP4_RTN, 0, nullptr, &xq, ws, ws_bytes)) ||
        (st = validate_quantize(W, dtype, N, K, K, NVFP4_ROWWISE, NVFP4_RTN, 0, nullptr, &wq, ws, ws_bytes)) ||
        (st = validate_gemm(&xq, &wq, Y, y_dtype, N, ws, ws_bytes)))
        return st;
    return check_device();
}

}  // namespace nvfp4

extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t k) {
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)rows * (size_t)(k / 2);
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t k) {
    if (rows <= 0 || k <= 0) return 0;
    const size_t rows_pad = (size_t)((rows + 127) / 128) * 128;
    const size_t kb_pad = (size_t)((k + 63) / 64) * 4;
    return rows_pad * kb_pad;
}

size_t nvfp4_quantize_workspace_size(void) { return kQuantizeWorkspace; }

size_t nvfp4_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 0) return 0;
    return std::max(fwd_bytes(M, N, K), bwd_bytes(M, N, K));
}

size_t nvfp4_linear_fwd_workspace_size(int64_t M, int64_t N, int64_t K) {
    return nvfp4::linear_fwd_workspace_bytes(M, N, K);
}

nvfp4_status nvfp4_quantize(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, int orientation,
                            int rounding, int rht, uint64_t seed, const float *amax_in, const nvfp4_tensor *out,
                            void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    nvfp4_status st =
        validate_quantize(x, dtype, R, C, ld, orientation, rounding, rht, amax_in, out, workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if ((st = check_device()) != NVFP4_OK) return st;
    st = quantize_impl(x, dtype, R, C, ld, orientation, rounding, rht, seed, amax_in, out, workspace, stream,
                       &call.launches);
    return call.done(st);
}

nvfp4_status nvfp4_amax(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, int rht, uint64_t seed,
                        float *amax_out, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    if (!amax_out || !valid_dtype(dtype) || (rht != 0 && rht != 1)) return NVFP4_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(amax_out) % 4 != 0) return NVFP4_ERR_ALIGNMENT;
    if (R < 0 || C < 0 || R > (1LL << 31) || C > (1LL << 31)) return NVFP4_ERR_SHAPE;
    if (!workspace || ws_bytes < kQuantizeWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    const size_t es = esize(dtype);
    if (R > 0 && C > 0) {
        if (!x) return NVFP4_ERR_INVALID_ARG;
        if (ld < C || (C * (int64_t)es) % 16 != 0 || (rht && R % 16 != 0)) return NVFP4_ERR_SHAPE;
        if (!aligned16(x) || (ld * (int64_t)es) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
    }
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    return call.done(from_cuda(launch_amax(x, dtype == NVFP4_DTYPE_BF16, R, C, ld, rht != 0, seed, partials, amax_out,
                                           stream, &call.launches)));
}

nvfp4_status nvfp4_amax_dual(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, uint64_t seed,
                             float *amax_out, float *amax_rht_out, void *workspace, size_t ws_bytes,
                             cudaStream_t stream) {
    Call call(__func__);
    if (!amax_out || !amax_rht_out || !valid_dtype(dtype)) return NVFP4_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(amax_out) % 4 != 0 || reinterpret_cast<uintptr_t>(amax_rht_out) % 4 != 0)
        return NVFP4_ERR_ALIGNMENT;
    if (R < 0 || C < 0 || R > (1LL << 31) || C > (1LL << 31)) return NVFP4_ERR_SHAPE;
    if (!workspace || ws_bytes < kDualWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    const size_t es = esize(dtype);
    if (R > 0 && C > 0) {
        if (!x) return NVFP4_ERR_INVALID_ARG;
        if (ld < C || (C * (int64_t)es) % 16 != 0 || R % 16 != 0) return NVFP4_ERR_SHAPE;
        if (!aligned16(x) || (ld * (int64_t)es) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
    }
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    return call.done(from_cuda(launch_amax_dual(x, dtype == NVFP4_DTYPE_BF16, R, C, ld, seed, partials, amax_out,
                                                amax_rht_out, stream, &call.launches)));
}

size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t k) {
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)((k + 127) / 128) * 4;
}

nvfp4_status nvfp4_quantize_mx(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, int orientation,
                               const nvfp4_tensor *out, cudaStream_t stream) {
    Call call(__func__);
    if (!out || !valid_dtype(dtype) || (orientation != NVFP4_ROWWISE && orientation != NVFP4_COLWISE))
        return NVFP4_ERR_INVALID_ARG;
    const bool colwise = orientation == NVFP4_COLWISE;
    if (R < 0 || C < 0 || out->rows != (colwise ? C : R) || out->k != (colwise ? R : C)) return NVFP4_ERR_SHAPE;
    if (R == 0 || C == 0) return call.done(NVFP4_OK);
    if (!x || !out->codes || !out->scales) return NVFP4_ERR_INVALID_ARG;
    const size_t es = esize(dtype);
    if (ld < C || R > (1LL << 31) || C > (1LL << 31)) return NVFP4_ERR_SHAPE;
    if (!colwise && C % 32 != 0) return NVFP4_ERR_SHAPE;
    if (colwise && (R % 32 != 0 || (C * (int64_t)es) % 16 != 0 || R > kMaxColwiseRows)) return NVFP4_ERR_SHAPE;
    if (!aligned16(x) || (ld * (int64_t)es) % 16 != 0 || !aligned16(out->codes) || !aligned16(out->scales))
        return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    return call.done(from_cuda(launch_quantize_mx(x, dtype == NVFP4_DTYPE_BF16, R, C, ld, colwise, out->codes,
                                                  out->scales, stream, &call.launches)));
}

size_t nvfp4_quantize_dual_workspace_size(void) { return kDualWorkspace; }

nvfp4_status nvfp4_quantize_dual(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld,
                                 int col_rounding, int col_rht, uint64_t seed, const float *amax_row_in,
                                 const float *amax_col_in, const nvfp4_tensor *out_row,
                                 const nvfp4_tensor *out_col, void *workspace, size_t ws_bytes,
                                 cudaStream_t stream) {
    Call call(__func__);
    // each orientation's own checks; the dual workspace holds both amax partial sets
    nvfp4_status st = validate_quantize(x, dtype, R, C, ld, NVFP4_ROWWISE, NVFP4_RTN, 0, amax_row_in, out_row,
                                        workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    st = validate_quantize(x, dtype, R, C, ld, NVFP4_COLWISE, col_rounding, col_rht, amax_col_in, out_col,
                           workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if (R > 0 && C > 0 && !(amax_row_in && amax_col_in) && (!workspace || ws_bytes < kDualWorkspace))
        return NVFP4_ERR_WORKSPACE;
    if ((st = check_device()) != NVFP4_OK) return st;
    return call.done(dual_impl(x, dtype, R, C, ld, col_rounding, col_rht, seed, amax_row_in, amax_col_in, out_row,
                               out_col, workspace, stream, &call.launches));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *B, void *C, nvfp4_dtype c_dtype, int64_t ldc,
                        void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    nvfp4_status st = validate_gemm(A, B, C, c_dtype, ldc, workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if (A->rows == 0 || B->rows == 0) return call.done(NVFP4_OK);  // nothing to launch
    if ((st = check_device()) != NVFP4_OK) return st;
    return call.done(gemm_impl(A, B, C, c_dtype, ldc, workspace, stream, &call.launches));
}

nvfp4_status nvfp4_gemm_mx(const nvfp4_tensor *A, const nvfp4_tensor *B, void *C, nvfp4_dtype c_dtype, int64_t ldc,
                           void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    if (!A || !B) return NVFP4_ERR_INVALID_ARG;
    // the same checks as nvfp4_gemm, without the tensor scales (MXFP4 has none)
    nvfp4_tensor a = *A, b = *B;
    static float placeholder;
    a.tensor_scale = b.tensor_scale = &placeholder;
    nvfp4_status st = validate_gemm(&a, &b, C, c_dtype, ldc, workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if (A->rows == 0 || B->rows == 0) return call.done(NVFP4_OK);
    if ((st = check_device()) != NVFP4_OK) return st;
    a.tensor_scale = b.tensor_scale = nullptr;
    return call.done(gemm_impl(&a, &b, C, c_dtype, ldc, workspace, stream, &call.launches, true));
}

namespace {
nvfp4_status gemm_relu2_impl(const char *name, int epi, const nvfp4_tensor *A, const nvfp4_tensor *B, void *C,
                             void *aux, uint64_t seed, float *amax_out, float *amax_rht_out, void *workspace,
                             size_t ws_bytes, cudaStream_t stream) {
    Call call(name);
    nvfp4_status st = validate_gemm(A, B, C, NVFP4_DTYPE_BF16, B ? B->rows : 0, workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    const int64_t M = A->rows, N = B->rows;
    if (M == 0 || N == 0 || A->k == 0 || M % 256 != 0 || N % 256 != 0) return NVFP4_ERR_SHAPE;
    if (!aux || !amax_out || !amax_rht_out) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(aux) || !aligned16(amax_out) || !aligned16(amax_rht_out)) return NVFP4_ERR_ALIGNMENT;
    if (ws_bytes < kDualWorkspace) return NVFP4_ERR_WORKSPACE;
    if ((st = check_device()) != NVFP4_OK) return st;
    GemmArgs g;
    g.a_codes = A->codes;
    g.a_scales = A->scales;
    g.a_ts = A->tensor_scale;
    g.b_codes = B->codes;
    g.b_scales = B->scales;
    g.b_ts = B->tensor_scale;
    g.M = M;
    g.N = N;
    g.K = A->k;
    g.C = C;
    g.c_bf16 = true;
    g.ldc = N;
    g.status = static_cast<int *>(workspace);
    g.epi = epi;
    g.aux = aux;
    g.seed = seed;
    g.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    g.amax_out = amax_out;
    g.amax_rht_out = amax_rht_out;
    return call.done(from_cuda(launch_gemm(g, stream, &call.launches)));
}
}  // namespace

nvfp4_status nvfp4_gemm_relu2_fwd(const nvfp4_tensor *A, const nvfp4_tensor *B, void *Y, void *H, uint64_t seed,
                                  float *amax_out, float *amax_rht_out, void *workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
    return gemm_relu2_impl(__func__, GEMM_EPI_RELU2_FWD, A, B, Y, H, seed, amax_out, amax_rht_out, workspace,
                           ws_bytes, stream);
}

nvfp4_status nvfp4_gemm_relu2_bwd(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *Y, void *dY,
                                  uint64_t seed, float *amax_out, float *amax_rht_out, void *workspace,
                                  size_t ws_bytes, cudaStream_t stream) {
    return gemm_relu2_impl(__func__, GEMM_EPI_RELU2_BWD, A, B, dY, const_cast<void *>(Y), seed, amax_out,
                           amax_rht_out, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_linear_fwd(const void *X, const void *W, void *Y, int64_t M, int64_t N, int64_t K,
                              nvfp4_dtype dtype, nvfp4_dtype y_dtype, void *workspace, size_t ws_bytes,
                              cudaStream_t stream) {
    Call call(__func__);
    nvfp4_status st = nvfp4::linear_fwd_validate(X, W, Y, M, N, K, dtype, y_dtype, workspace, ws_bytes);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return call.done(NVFP4_OK);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *ts = reinterpret_cast<float *>(ws + kScalarsOff);
    Carver cv{ws, kBuffersOff};
    const nvfp4_tensor xq = cv.take(M, K, ts + 0), wq = cv.take(N, K, ts + 1);
    if ((st = quantize_impl(X, dtype, M, K, K, NVFP4_ROWWISE, NVFP4_RTN, 0, 0, nullptr, &xq, ws, stream,
                            &call.launches)) ||
        (st = quantize_impl(W, dtype, N, K, K, NVFP4_ROWWISE, NVFP4_RTN, 0, 0, nullptr, &wq, ws, stream,
                            &call.launches)) ||
        (st = gemm_impl(&xq, &wq, Y, y_dtype, N, ws, stream, &call.launches)))
        return st;
    return call.done(NVFP4_OK);
}

nvfp4_status nvfp4_linear_bwd(const void *dY, const void *X, const void *W, void *dX, float *dW, int64_t M,
                              int64_t N, int64_t K, nvfp4_dtype dtype, nvfp4_dtype dx_dtype, uint64_t seed,
                              void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    if (!valid_dtype(dtype) || !valid_dtype(dx_dtype)) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || M % 64 != 0 || N % 64 != 0 || K % 64 != 0) return NVFP4_ERR_SHAPE;
    if (M == 0 || N == 0 || K == 0) return NVFP4_ERR_SHAPE;
    if (!dY || !X || !W || !dX || !dW) return NVFP4_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < nvfp4_linear_workspace_size(M, N, K)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *ts = reinterpret_cast<float *>(ws + kScalarsOff);
    Carver cv{ws, kBuffersOff};
    const nvfp4_tensor dy_r = cv.take(M, N, ts + 0);  // Dgrad A: rowwise(dY)         [M x N]
    const nvfp4_tensor w_c = cv.take(K, N, ts + 1);   // Dgrad B: colwise(W)          [K x N]
    const nvfp4_tensor dy_c = cv.take(N, M, ts + 2);  // Wgrad A: colwise(dY) RHT+SR  [N x M]
    const nvfp4_tensor x_c = cv.take(K, M, ts + 3);   // Wgrad B: colwise(X) RHT      [K x M]
    nvfp4_status st;
    if ((st = validate_quantize(dY, dtype, M, N, N, NVFP4_ROWWISE, NVFP4_RTN, 0, nullptr, &dy_r, ws, ws_bytes)) ||
        (st = validate_quantize(W, dtype, N, K, K, NVFP4_COLWISE, NVFP4_RTN, 0, nullptr, &w_c, ws, ws_bytes)) ||
        (st = validate_quantize(dY, dtype, M, N, N, NVFP4_COLWISE, NVFP4_SR, 1, nullptr, &dy_c, ws, ws_bytes)) ||
        (st = validate_quantize(X, dtype, M, K, K, NVFP4_COLWISE, NVFP4_RTN, 1, nullptr, &x_c, ws, ws_bytes)) ||
        (st = validate_gemm(&dy_r, &w_c, dX, dx_dtype, K, ws, ws_bytes)) ||
        (st = validate_gemm(&dy_c, &x_c, dW, NVFP4_DTYPE_F32, K, ws, ws_bytes)))
        return st;
    if ((st = check_device()) != NVFP4_OK) return st;
    // dY's two operands (Dgrad rowwise, Wgrad colwise with RHT + SR) from one read
    if ((st = dual_impl(dY, dtype, M, N, N, NVFP4_SR, 1, seed, nullptr, nullptr, &dy_r, &dy_c, ws, stream,
                        &call.launches)))
        return st;
    // Dgrad: dX = dY . W
    if ((st = quantize_impl(W, dtype, N, K, K, NVFP4_COLWISE, NVFP4_RTN, 0, seed, nullptr, &w_c, ws, stream,
                            &call.launches)) ||
        (st = gemm_impl(&dy_r, &w_c, dX, dx_dtype, K, ws, stream, &call.launches)))
        return st;
    // Wgrad: dW = dY^T . X with the Hadamard transform on both operands, SR on dY
    if ((st = quantize_impl(X, dtype, M, K, K, NVFP4_COLWISE, NVFP4_RTN, 1, seed, nullptr, &x_c, ws, stream,
                            &call.launches)) ||
        (st = gemm_impl(&dy_c, &x_c, dW, NVFP4_DTYPE_F32, K, ws, stream, &call.launches)))
        return st;
    return call.done(NVFP4_OK);
}

nvfp4_status nvfp4_relu2_fwd(const void *y, void *h, int64_t n, cudaStream_t stream) {
    Call call(__func__);
    if (n < 0) return NVFP4_ERR_SHAPE;
    if (n == 0) return call.done(NVFP4_OK);
    if (!y || !h) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(h)) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    return call.done(from_cuda(launch_relu2_fwd(y, h, n, nullptr, nullptr, stream, &call.launches)));
}

nvfp4_status nvfp4_relu2_bwd(const void *dh, const void *y, void *dy, int64_t n, cudaStream_t stream) {
    Call call(__func__);
    if (n < 0) return NVFP4_ERR_SHAPE;
    if (n == 0) return call.done(NVFP4_OK);
    if (!dh || !y || !dy) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(dh) || !aligned16(y) || !aligned16(dy)) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    return call.done(from_cuda(launch_relu2_bwd(dh, y, dy, n, nullptr, nullptr, stream, &call.launches)));
}

nvfp4_status nvfp4_relu2_fwd_amax(const void *y, void *h, int64_t n, float *amax_out, void *workspace,
                                  size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    if (n < 0) return NVFP4_ERR_SHAPE;
    if (!amax_out || (n > 0 && (!y || !h))) return NVFP4_ERR_INVALID_ARG;
    if ((n > 0 && (!aligned16(y) || !aligned16(h))) || !aligned16(amax_out)) return NVFP4_ERR_ALIGNMENT;
    if (!workspace || ws_bytes < kQuantizeWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    return call.done(from_cuda(launch_relu2_fwd(y, h, n, amax_out, partials, stream, &call.launches)));
}

nvfp4_status nvfp4_relu2_bwd_amax(const void *dh, const void *y, void *dy, int64_t n, float *amax_out,
                                  void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    if (n < 0) return NVFP4_ERR_SHAPE;
    if (!amax_out || (n > 0 && (!dh || !y || !dy))) return NVFP4_ERR_INVALID_ARG;
    if ((n > 0 && (!aligned16(dh) || !aligned16(y) || !aligned16(dy))) || !aligned16(amax_out))
        return NVFP4_ERR_ALIGNMENT;
    if (!workspace || ws_bytes < kQuantizeWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    return call.done(from_cuda(launch_relu2_bwd(dh, y, dy, n, amax_out, partials, stream, &call.launches)));
}

namespace {
nvfp4_status relu2_amax_rht_impl(const void *dh, const void *y, void *out, int64_t R, int64_t C, uint64_t seed,
                                 float *amax_out, float *amax_rht_out, void *workspace, size_t ws_bytes,
                                 cudaStream_t stream) {
    Call call(__func__);
    if (R < 0 || C < 0 || R % 16 != 0 || C % 8 != 0) return NVFP4_ERR_SHAPE;
    if (!amax_out || !amax_rht_out || !y || !out) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out) || (dh && !aligned16(dh)) || !aligned16(amax_out) ||
        !aligned16(amax_rht_out))
        return NVFP4_ERR_ALIGNMENT;
    if (!workspace || ws_bytes < kDualWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    return call.done(from_cuda(launch_relu2_amax_rht(dh, y, out, R, C, seed, amax_out, amax_rht_out, partials,
                                                     stream, &call.launches)));
}
}  // namespace

nvfp4_status nvfp4_relu2_fwd_amax_rht(const void *y, void *h, int64_t R, int64_t C, uint64_t seed, float *amax_out,
                                      float *amax_rht_out, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    return relu2_amax_rht_impl(nullptr, y, h, R, C, seed, amax_out, amax_rht_out, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_relu2_bwd_amax_rht(const void *dh, const void *y, void *dy, int64_t R, int64_t C, uint64_t seed,
                                      float *amax_out, float *amax_rht_out, void *workspace, size_t ws_bytes,
                                      cudaStream_t stream) {
    if (!dh) return NVFP4_ERR_INVALID_ARG;
    return relu2_amax_rht_impl(dh, y, dy, R, C, seed, amax_out, amax_rht_out, workspace, ws_bytes, stream);
}

nvfp4_status nvfp4_check(void *workspace, cudaStream_t stream) {
    if (!workspace) return NVFP4_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    int status = 0;
    if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (status != 0) {
        if (cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return NVFP4_ERR_CUDA;
        return status == NVFP4_ERR_DEVICE_TIMEOUT ? NVFP4_ERR_DEVICE_TIMEOUT : NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

nvfp4_status nvfp4_selftest_wait_timeout(void *workspace, size_t ws_bytes, uint64_t limit_ns, cudaStream_t stream) {
    Call call(__func__);
    if (!workspace || ws_bytes < kStatusBytes) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    if (limit_ns == 0 || limit_ns > 2000000000ull) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    return call.done(from_cuda(launch_wait_timeout(static_cast<int *>(workspace), limit_ns, stream, &call.launches)));
}

nvfp4_status nvfp4_selftest_mma_rate(int mx, int64_t iters, uint64_t *cycles, int64_t cycles_len, int *pairs_out,
                                     void *workspace, size_t ws_bytes, cudaStream_t stream) {
    Call call(__func__);
    if (!cycles || !pairs_out || (mx != 0 && mx != 1) || iters < 1 || iters > 1000000) return NVFP4_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < kStatusBytes) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(workspace) || reinterpret_cast<uintptr_t>(cycles) % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    if (cycles_len < num_sms() / 2) return NVFP4_ERR_INVALID_ARG;
    return call.done(from_cuda(launch_mma_rate(mx == 1, iters, cycles, cycles_len, pairs_out,
                                               static_cast<int *>(workspace), stream, &call.launches)));
}

#ifdef NVFP4_BOUNDS_CHECK
constexpr int kCheckedBuild = 1;
#else
constexpr int kCheckedBuild = 0;
#endif

nvfp4_status nvfp4_bounds_status(int *checked, int *site) {
    if (!checked || !site) return NVFP4_ERR_INVALID_ARG;
    *checked = kCheckedBuild;
    *site = 0;
    if (!kCheckedBuild) return NVFP4_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) return NVFP4_ERR_CUDA;
    cudaError_t (*readers[4])(int *) = {read_bounds_quantize, read_bounds_elementwise, read_bounds_gemm,
                                        read_bounds_selftest};
    for (int f = 0; f < 4; ++f) {  // read (and clear) every record; report the first file's
        int line = 0;
        if (readers[f](&line) != cudaSuccess) return NVFP4_ERR_CUDA;
        if (line && !*site) *site = (f + 1) * 100000 + line;
    }
    return *site ? NVFP4_ERR_DEVICE_BOUNDS : NVFP4_OK;
}

nvfp4_status nvfp4_selftest_bounds(uint8_t *buf, int64_t n, cudaStream_t stream) {
    Call call(__func__);
    if (!kCheckedBuild || !buf || n < 1) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    return call.done(from_cuda(launch_selftest_bounds(buf, n, stream, &call.launches)));
}

int nvfp4_last_launch_count(void) { return g_last_launches; }

const char *nvfp4_status_string(nvfp4_status status) {
    switch (status) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument (null pointer, bad enum or flag combination)";
        case NVFP4_ERR_ALIGNMENT: return "pointer or leading dimension is not 16-byte aligned";
        case NVFP4_ERR_SHAPE: return "unsupported or inconsistent shape";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
        case NVFP4_ERR_UNSUPPORTED_DEVICE: return "current device is not compute capability 10.0 (B200)";
        case NVFP4_ERR_CUDA: return "CUDA runtime error";
        case NVFP4_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
        case NVFP4_ERR_DEVICE_BOUNDS: return "a kernel index fell outside its buffer (bounds-checked build)";
    }
    return "unknown status";
}

}  // extern "C"
