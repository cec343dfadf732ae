/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 linear-layer library.
 *
 * NVFP4 as this library stores it (aisight.pl, "Koniec marnowania mocy.
 * NVIDIA udowadnia, ze 4 bity wystarcza do trenowania gigantow", section
 * "Architektura NVFP4 kontra ograniczenia mikroskalowania": blocks of 16
 * elements instead of 32, an E4M3 block scale instead of a power of two, and
 * an extra FP32 scale for the whole tensor):
 *   - codes : E2M1 values (+-{0,0.5,1,1.5,2,3,4,6}), two per byte, element 2i
 *             in bits 0-3 and element 2i+1 in bits 4-7, row-major
 *             [rows x k/2] bytes ("K-major": k, the GEMM reduction index, is
 *             contiguous);
 *   - scales: one unsigned E4M3 byte per 16 consecutive k of a row, stored in
 *             512-byte atoms of 128 rows x 4 blocks: byte offset of (row r,
 *             block b) = atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + b % 4
 *             with atom = (r / 128) * (KB / 4) + b / 4, KB = 4 * ceil(k / 64).
 *             Rows are padded to 128 and blocks to KB; padding bytes are 0.
 *             This is the order in which the tensor cores read block scales;
 *   - tensor_scale: one FP32 decode scale s_t in device memory.
 * A value decodes as e2m1(code) * e4m3(scale) * s_t.
 *
 * Conventions for every call:
 *   - Pointers to tensors are DEVICE pointers on the current CUDA device; the
 *     caller allocates and owns every buffer (inputs, outputs, workspace).
 *     The library allocates nothing and frees nothing.
 *   - Calls are asynchronous and stream-ordered on `stream` (0 = legacy
 *     default stream); none synchronises the host.
 *   - Arguments are checked on the host before anything is launched; a call
 *     that returns an error has launched nothing and written nothing.
 *   - A workspace serves one stream at a time.  Its first 256 bytes hold a
 *     device status word: zero it once after allocation.  Kernels with bounded
 *     device-side waits record NVFP4_ERR_DEVICE_TIMEOUT there instead of
 *     hanging; nvfp4_check() reads and clears it.
 *   - Non-finite inputs are outside the contract (the result is unspecified).
 *   - With NVFP4_NVTX=1 in the environment when the process starts, every
 *     call is wrapped in an NVTX range named after the function, for
 *     timeline profilers; otherwise no NVTX call is made.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NVFP4_ABI_VERSION 1

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

typedef enum nvfp4_status {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum/flag combination */
    NVFP4_ERR_ALIGNMENT = 2,          /* pointer or leading dimension breaks the 16-byte rule   */
    NVFP4_ERR_SHAPE = 3,              /* sizes the format or the kernels cannot take            */
    NVFP4_ERR_WORKSPACE = 4,          /* workspace missing or smaller than required             */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 5, /* current device is not compute capability 10.0          */
    NVFP4_ERR_CUDA = 6,               /* a CUDA runtime call or launch failed                   */
    NVFP4_ERR_DEVICE_TIMEOUT = 7,     /* a bounded device-side wait expired (see nvfp4_check)   */
    NVFP4_ERR_DEVICE_BOUNDS = 8       /* checked build: a kernel index fell outside its buffer  */
} nvfp4_status;

typedef enum nvfp4_dtype {
    NVFP4_DTYPE_F32 = 0,  /* IEEE binary32 */
    NVFP4_DTYPE_BF16 = 1  /* bfloat16      */
} nvfp4_dtype;

enum { NVFP4_ROWWISE = 0, NVFP4_COLWISE = 1 };
enum { NVFP4_RTN = 0, NVFP4_SR = 1 };

/* An NVFP4 tensor of logical shape [rows x k] (k = reduction dim). */
typedef struct nvfp4_tensor {
    uint8_t *codes;       /* nvfp4_codes_bytes(rows, k) bytes, 16-byte aligned  */
    uint8_t *scales;      /* nvfp4_scales_bytes(rows, k) bytes, 16-byte aligned */
    float *tensor_scale;  /* 1 float                                            */
    int64_t rows;
    int64_t k;
} nvfp4_tensor;

/*
 * nvfp4_amax -- the tensor amax of the FP32 per-tensor scale (aisight.pl,
 * section "Architektura NVFP4 kontra ograniczenia mikroskalowania": one FP32
 * scale per tensor next to the E4M3 block scales): *amax_out = max |x| over the
 * [R x C] tensor x (leading dimension ld elements), or with rht = 1 the max of
 * |y| over y = 1/4 H16 D v, the random Hadamard transform applied down every
 * 16-row group of every column as the colwise quantisation of the Wgrad
 * operands applies it (same page, section "Technologie stabilizujace proces
 * treningowy"; signs D from `seed`).  Exactly the amax nvfp4_quantize computes
 * in its first pass, so handing it on as amax_in gives the same codes; one
 * amax serves both orientations of a tensor without the transform.  An empty
 * tensor gives 0.  amax_out: device memory, one float, caller-owned;
 * workspace: >= nvfp4_quantize_workspace_size() bytes, 16-byte aligned
 * (per-CTA partials).  Requires x 16-byte aligned, ld * element size and
 * C * element size multiples of 16, R % 16 == 0 when rht, R, C <= 2^31.
 * Asynchronous (two launches).  Errors: NVFP4_ERR_INVALID_ARG, NVFP4_ERR_SHAPE,
 * NVFP4_ERR_ALIGNMENT, NVFP4_ERR_WORKSPACE, NVFP4_ERR_UNSUPPORTED_DEVICE,
 * NVFP4_ERR_CUDA.
 */
NVFP4_API nvfp4_status nvfp4_amax(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld, int rht,
                                  uint64_t seed, float *amax_out, void *workspace, size_t ws_bytes,
                                  cudaStream_t stream);

/*
 * nvfp4_amax_dual -- both amaxes of a tensor whose rowwise and colwise-RHT
 * operands are both needed (the Fprop and Wgrad operands of one activation or
 * gradient), from one read: *amax_out = max |x| and *amax_rht_out = max |y|,
 * y = 1/4 H16 D v down every 16-row group of every column, bit for bit what
 * nvfp4_amax gives with rht = 0 and 1 (same passages).  amax_out, amax_rht_out:
 * device memory, one float each; workspace: >= nvfp4_quantize_dual_workspace_size()
 * bytes, 16-byte aligned.  Requires R % 16 == 0 and the rest as nvfp4_amax.
 * Asynchronous (two launches).  Errors as nvfp4_amax.
 */
NVFP4_API nvfp4_status nvfp4_amax_dual(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld,
                                       uint64_t seed, float *amax_out, float *amax_rht_out, void *workspace,
                                       size_t ws_bytes, cudaStream_t stream);

/* Sizes of the two byte buffers of an NVFP4 tensor (k must be a multiple of 16). */
NVFP4_API size_t nvfp4_codes_bytes(int64_t rows, int64_t k);
NVFP4_API size_t nvfp4_scales_bytes(int64_t rows, int64_t k);

/* Workspace bytes needed by nvfp4_quantize (status word + per-CTA amax partials). */
NVFP4_API size_t nvfp4_quantize_workspace_size(void);

/*
 * nvfp4_quantize -- x [R x C] (row-major, leading dimension ld elements) -> out.
 * The step order follows aisight.pl, sections "Architektura NVFP4 ..." and
 * "Technologie stabilizujace proces treningowy":
 *   1. optional 16-point random Hadamard transform y = 1/4 H16 D v of every
 *      16-element block (D = +-1 signs from the seed), colwise only;
 *   2. tensor amax over the (transformed) tensor, unless amax_in supplies it;
 *      s_t = amax / (6 * 448) (1 if that is 0);
 *   3. per 16-block: sb = E4M3_rn_satfinite(amax_b / 6 / s_t);
 *   4. per element: r = v * (1 / (e4m3(sb) * s_t)), then E2M1 by
 *      round-to-nearest-even (rounding = NVFP4_RTN) or stochastic rounding
 *      (NVFP4_SR: up iff u < frac, u a 16-bit Philox4x32-10 draw keyed on
 *      (seed, element index in the output view));
 *   5. store codes, scales (atom layout, padding zeroed) and s_t.
 * orientation = NVFP4_ROWWISE: blocks run along the C columns; out is
 *   [R x C] (out->rows == R, out->k == C).  Requires C % 16 == 0.
 * orientation = NVFP4_COLWISE: blocks run down the R rows and out is the
 *   transpose [C x R] (out->rows == C, out->k == R).  Requires R % 16 == 0
 *   and C a multiple of 8 (bf16) / 4 (f32), and R <= 65535 * 256.
 * R and C are at most 2^31.
 * rht != 0 only with NVFP4_COLWISE.  x must be 16-byte aligned and
 * ld * element size a multiple of 16.  workspace: >= nvfp4_quantize_workspace_size()
 * bytes (may be NULL when amax_in is given).  amax_in: optional device float.
 * R == 0 or C == 0 is allowed: only s_t = 1 is written.
 */
NVFP4_API nvfp4_status nvfp4_quantize(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld,
                            int orientation, int rounding, int rht, uint64_t seed,
                            const float *amax_in, const nvfp4_tensor *out,
                            void *workspace, size_t ws_bytes, cudaStream_t stream);

/* MXFP4, the comparison format of aisight.pl, section "Architektura NVFP4
 * kontra ograniczenia mikroskalowania": blocks of 32 elements along the
 * contiguous dim (rowwise), one E8M0 (power-of-two) scale per block, no
 * per-tensor scale, in either orientation (as for nvfp4_quantize: colwise
 * blocks run down the rows and the output is the transpose).  Scale 2^X with
 * X = floor(log2 amax_b) - 2 (2 is the
 * exponent of E2M1's top binade), clamped to [-127, 127], X = -127 for an
 * all-zero block; each element is E2M1(v * 2^-X), round to nearest even,
 * saturating at +-6 (the OCP Microscaling conversion; the pages name the
 * format only).  One pass over x, no workspace.
 * x: [R x C] dtype, row stride ld elements, 16-byte aligned; rowwise needs
 * C % 32 == 0, colwise R % 32 == 0, R <= 65535 * 256 and C * element size
 * % 16 == 0.  R and C are at most 2^31.
 * out: [rows' x k] = [R x C] (rowwise) or [C x R] (colwise); codes rows'*k/2
 * bytes as for NVFP4 (element 2i in the low nibble); scales
 * nvfp4_mx_scales_bytes(rows', k) bytes of E8M0 codes in the
 * 128x4 atom order of the NVFP4 scales with four 32-blocks per atom word
 * (rows padded to 128, blocks to 4, padding 0); out->tensor_scale unused.
 * Errors: NVFP4_ERR_INVALID_ARG, NVFP4_ERR_SHAPE, NVFP4_ERR_ALIGNMENT,
 * NVFP4_ERR_UNSUPPORTED_DEVICE, NVFP4_ERR_CUDA. */
NVFP4_API size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t k);
NVFP4_API nvfp4_status nvfp4_quantize_mx(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld,
                                         int orientation, const nvfp4_tensor *out, cudaStream_t stream);

/* Both NVFP4 operands of one tensor from one read of it (the layer's
 * backward pass needs dY rowwise for Dgrad and colwise with the Hadamard
 * transform and stochastic rounding for Wgrad; the same holds for every
 * tensor the MLP step quantises in both orientations).  The results are
 * bit-identical to
 *   nvfp4_quantize(x, ..., NVFP4_ROWWISE, NVFP4_RTN, 0, seed, amax_row_in, out_row, ...)
 *   nvfp4_quantize(x, ..., NVFP4_COLWISE, col_rounding, col_rht, seed, amax_col_in, out_col, ...)
 * (format: aisight.pl, section "Architektura NVFP4 kontra ograniczenia
 * mikroskalowania"; Hadamard transform and stochastic rounding on the Wgrad
 * operands: same page, section "Technologie stabilizujace proces
 * treningowy").  x, R, C, ld, dtype, out_row ([R x C]) and out_col ([C x R])
 * follow nvfp4_quantize for their orientation, so both sets of shape and
 * alignment rules apply.  workspace: >= nvfp4_quantize_dual_workspace_size()
 * bytes, 16-byte aligned, zeroed status word, unless both amax_*_in are given.
 * Passes: one amax pass computing max|x| and, with col_rht, max|RHT(x)| in the
 * same read (skipped when both amax values are supplied), then one quantise
 * pass writing both outputs.  Errors as nvfp4_quantize. */
NVFP4_API size_t nvfp4_quantize_dual_workspace_size(void);
NVFP4_API nvfp4_status nvfp4_quantize_dual(const void *x, nvfp4_dtype dtype, int64_t R, int64_t C, int64_t ld,
                                           int col_rounding, int col_rht, uint64_t seed,
                                           const float *amax_row_in, const float *amax_col_in,
                                           const nvfp4_tensor *out_row, const nvfp4_tensor *out_col,
                                           void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * nvfp4_gemm -- C[M x N] = (A . B^T) * sA * sB with A = [M x K], B = [N x K]
 * NVFP4 tensors (the block-scaled GEMM used for Fprop, Dgrad and Wgrad; 4-bit
 * GEMMs on Blackwell tensor cores: nerdman.de, "Nvidia drueckt KI-Training auf
 * 4 Bit runter", section "Was konkret passiert ist").  Products of E2M1 values
 * and E4M3 block scales accumulate in FP32 on the tensor cores; the epilogue
 * multiplies by the two tensor scales and writes c_dtype (f32 or bf16,
 * round-to-nearest-even) row-major with leading dimension ldc elements.
 * Requires A->k == B->k, K % 64 == 0, C 16-byte aligned, ldc * element size a
 * multiple of 16, and M, N, K < 2^31.  M or N == 0: nothing is done.
 * K == 0: C is zero-filled.
 * workspace: >= 256 bytes (status word).
 * Errors: NVFP4_ERR_INVALID_ARG, NVFP4_ERR_SHAPE, NVFP4_ERR_ALIGNMENT,
 * NVFP4_ERR_WORKSPACE, NVFP4_ERR_UNSUPPORTED_DEVICE, NVFP4_ERR_CUDA; a device
 * timeout is recorded in the workspace status word (nvfp4_check).
 */
NVFP4_API nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *B, void *C, nvfp4_dtype c_dtype,
                        int64_t ldc, void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * nvfp4_gemm_mx -- the same GEMM on MXFP4 operands, the comparison format of
 * aisight.pl, section "Architektura NVFP4 kontra ograniczenia
 * mikroskalowania" (32-element blocks, power-of-two E8M0 scales, no tensor
 * scale): C[M x N] = A . B^T with A = [M x K], B = [N x K] as written by
 * nvfp4_quantize_mx (codes as for NVFP4, scales nvfp4_mx_scales_bytes(rows, K)
 * bytes in that layout); tensor_scale is ignored.  Products of E2M1 values
 * and E8M0 block scales accumulate in FP32 on the tensor cores
 * (kind::mxf4.block_scale.block32) and the epilogue writes c_dtype (f32, or
 * bf16 by round-to-nearest-even) with leading dimension ldc elements.
 * Requirements, workspace and errors as nvfp4_gemm.
 */
NVFP4_API nvfp4_status nvfp4_gemm_mx(const nvfp4_tensor *A, const nvfp4_tensor *B, void *C, nvfp4_dtype c_dtype,
                                     int64_t ldc, void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * nvfp4_gemm_relu2_fwd / nvfp4_gemm_relu2_bwd -- the MLP block's GEMMs next to
 * its squared ReLU, with the activation applied in the GEMM's epilogue.  The
 * 12B model's MLP (hyper.ai, "NVIDIA revolutioniert
 * KI-Praetrainingsgeschwindigkeit mit 4-Bit-Genauigkeit") runs up-projection ->
 * relu^2 -> down-projection in NVFP4 (aisight.pl, section "Architektura NVFP4
 * kontra ograniczenia mikroskalowania").  Both take NVFP4 A [M x K] and B [N x K]
 * as nvfp4_gemm and compute y = bf16(A . B^T * sA * sB) (round to nearest
 * even), then:
 *   fwd: Y = y and H = relu(y) * relu(y)      (the up-projection and h)
 *   bwd: dY = y * (2 * relu(Y)), Y the forward's y, y not stored
 *        (the down-projection's Dgrad dh, and dY1 of the up-projection)
 * each product in binary32 then bf16 round-to-nearest-even, bit-identical to
 * nvfp4_gemm followed by nvfp4_relu2_fwd / nvfp4_relu2_bwd.  They also write
 * *amax_out = max |H| (|dY|) and *amax_rht_out = max |RHT(H)| (|RHT(dY)|),
 * the 16-point random Hadamard transform of `seed` down 16-row groups (as
 * nvfp4_relu2_fwd_amax_rht), for the two quantisations of that output.
 * Y, H, dY: contiguous bf16 [M x N], 16-byte aligned, device memory.
 * Requires M and N multiples of 256, K % 64 == 0, K > 0.  workspace: >=
 * nvfp4_quantize_dual_workspace_size() bytes, 16-byte aligned, zeroed status
 * word.  Two launches.  Errors as nvfp4_gemm; NVFP4_ERR_SHAPE for other M, N.
 */
NVFP4_API nvfp4_status nvfp4_gemm_relu2_fwd(const nvfp4_tensor *A, const nvfp4_tensor *B, void *Y, void *H,
                                            uint64_t seed, float *amax_out, float *amax_rht_out, void *workspace,
                                            size_t ws_bytes, cudaStream_t stream);
NVFP4_API nvfp4_status nvfp4_gemm_relu2_bwd(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *Y, void *dY,
                                            uint64_t seed, float *amax_out, float *amax_rht_out, void *workspace,
                                            size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes at these sizes: nvfp4_linear_workspace_size serves both
 * nvfp4_linear_fwd and nvfp4_linear_bwd (the larger of the two footprints);
 * nvfp4_linear_fwd_workspace_size is what nvfp4_linear_fwd alone needs (the
 * status word, amax partials, tensor scales and the two rowwise operands).
 * Both return 0 for negative sizes. */
NVFP4_API size_t nvfp4_linear_workspace_size(int64_t M, int64_t N, int64_t K);
NVFP4_API size_t nvfp4_linear_fwd_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * nvfp4_linear_fwd -- Fprop of Y = X . W^T: X [M x K], W [N x K] (dtype,
 * row-major, contiguous) -> Y [M x N] (y_dtype, contiguous).  The forward
 * GEMM of a layer trained in 4 bits, the step hyper.ai ("NVIDIA
 * revolutioniert KI-Praetrainingsgeschwindigkeit mit 4-Bit-Genauigkeit")
 * credits with the GEMM speed-up, on operands in the format of aisight.pl,
 * section "Architektura NVFP4 kontra ograniczenia mikroskalowania" (blocks of
 * 16, E4M3 block scale, FP32 tensor scale).  The Hadamard transform and
 * stochastic rounding are for the weight gradients only (same page, section
 * "Technologie stabilizujace proces treningowy"), so both operands are
 * quantised rowwise with round-to-nearest-even (nvfp4_quantize, two passes
 * each), then multiplied by nvfp4_gemm.
 * Requires K % 64 == 0; quantised operands live in the workspace
 * (>= nvfp4_linear_fwd_workspace_size(M, N, K) bytes, 16-byte aligned,
 * device memory, caller-owned, zeroed status word).  M or N == 0: nothing is
 * done.  Errors: as nvfp4_quantize and nvfp4_gemm, checked before any launch.
 */
NVFP4_API nvfp4_status nvfp4_linear_fwd(const void *X, const void *W, void *Y, int64_t M, int64_t N, int64_t K,
                              nvfp4_dtype dtype, nvfp4_dtype y_dtype,
                              void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * nvfp4_linear_bwd -- backward of Y = X . W^T, with dY [M x N], X [M x K],
 * W [N x K] (dtype, contiguous):
 *   Dgrad dX [M x K] (dx_dtype) = dY . W :  A = rowwise(dY, RTN), B = colwise(W, RTN)
 *   Wgrad dW [N x K] (f32)      = dY^T . X: A = colwise(dY, RHT, SR), B = colwise(X, RHT, RTN)
 * The random Hadamard transform and stochastic rounding apply to the Wgrad
 * operands only (aisight.pl, section "Technologie stabilizujace proces
 * treningowy"); both Wgrad operands use the same signs, from `seed`, which
 * also keys the SR draws.  dY's two operands come from one read of dY
 * (nvfp4_quantize_dual).  Requires M, N, K > 0 and multiples of 64, and
 * M, N <= 65535 * 256 (the colwise quantisations' limit); workspace as for
 * nvfp4_linear_fwd.  Errors: as nvfp4_quantize and nvfp4_gemm.
 */
NVFP4_API nvfp4_status nvfp4_linear_bwd(const void *dY, const void *X, const void *W, void *dX, float *dW,
                              int64_t M, int64_t N, int64_t K, nvfp4_dtype dtype,
                              nvfp4_dtype dx_dtype, uint64_t seed,
                              void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * nvfp4_linear_fwd_noalloc -- nvfp4_linear_fwd for callers that cannot
 * allocate device memory (for instance code inside a framework that owns all
 * device memory through its own pool, or a latency-critical loop that cannot
 * afford the synchronisation of cudaMalloc/cudaFree).  The pages have no
 * counterpart of this call: it only changes where the scratch lives.
 * Same arguments, checks and result as nvfp4_linear_fwd, without a workspace:
 * the scratch (status word, amax partials, both quantised operands) is one
 * fixed device buffer of NVFP4_NOALLOC_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits.  Calls
 * whose nvfp4_linear_fwd_workspace_size(M, N, K) exceeds it return
 * NVFP4_ERR_WORKSPACE and launch nothing.  The first call on a device looks
 * the buffer's address up (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  The call allocates and
 * frees nothing.  All calls share the one buffer and each call that passes
 * its checks starts by zeroing the status word (a refused call touches
 * neither the buffer nor the stream): calls that overlap on the GPU (other
 * streams, other host threads) race on it and must be serialised by the
 * caller.  A device-side
 * timeout is recorded only in that shared buffer, which no public call reads.
 */
#define NVFP4_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
NVFP4_API nvfp4_status nvfp4_linear_fwd_noalloc(const void *X, const void *W, void *Y, int64_t M, int64_t N,
                                                int64_t K, nvfp4_dtype dtype, nvfp4_dtype y_dtype,
                                                cudaStream_t stream);

/*
 * Squared-ReLU activation of the MLP block and its derivative, bf16 in/out,
 * n elements, contiguous, 16-byte aligned:
 *   h  = relu(y) * relu(y)          (binary32, then bf16 round-to-nearest-even)
 *   dy = dh * (2 * relu(y))         (binary32, then bf16 round-to-nearest-even)
 * with relu(y) = y for y > 0 and +0 otherwise.
 */
NVFP4_API nvfp4_status nvfp4_relu2_fwd(const void *y, void *h, int64_t n, cudaStream_t stream);
NVFP4_API nvfp4_status nvfp4_relu2_bwd(const void *dh, const void *y, void *dy, int64_t n, cudaStream_t stream);

/* The same two kernels, also writing max |output| over the n stored bf16
 * values to *amax_out (device float, 16-byte aligned) -- the amax a
 * following nvfp4_quantize of the output would compute in its first pass, so
 * it can be passed there as amax_in and that pass skipped (the pages'
 * per-tensor FP32 scale, aisight.pl, section "Architektura NVFP4 kontra
 * ograniczenia mikroskalowania", is then derived from it unchanged).
 * workspace: >= nvfp4_quantize_workspace_size() bytes, 16-byte aligned,
 * device memory (per-CTA partials).  Two launches.  n = 0 writes 0. */
NVFP4_API nvfp4_status nvfp4_relu2_fwd_amax(const void *y, void *h, int64_t n, float *amax_out, void *workspace,
                                            size_t ws_bytes, cudaStream_t stream);
NVFP4_API nvfp4_status nvfp4_relu2_bwd_amax(const void *dh, const void *y, void *dy, int64_t n, float *amax_out,
                                            void *workspace, size_t ws_bytes, cudaStream_t stream);

/* The same outputs over a contiguous [R x C] bf16 tensor (R % 16 == 0,
 * C % 8 == 0), writing both amax values the two quantisations of the output
 * need: *amax_out = max |out| (rowwise) and *amax_rht_out = max |RHT(out)|,
 * the 16-point random Hadamard transform with the signs of `seed` applied down
 * each column's 16-row groups -- the amax nvfp4_quantize(out, NVFP4_COLWISE,
 * ..., rht = 1, seed) computes in its first pass (transform on the Wgrad
 * operands: aisight.pl, section "Technologie stabilizujace proces
 * treningowy").  workspace: >= nvfp4_quantize_dual_workspace_size() bytes,
 * 16-byte aligned.  Two launches. */
NVFP4_API nvfp4_status nvfp4_relu2_fwd_amax_rht(const void *y, void *h, int64_t R, int64_t C, uint64_t seed,
                                                float *amax_out, float *amax_rht_out, void *workspace,
                                                size_t ws_bytes, cudaStream_t stream);
NVFP4_API nvfp4_status nvfp4_relu2_bwd_amax_rht(const void *dh, const void *y, void *dy, int64_t R, int64_t C,
                                                uint64_t seed, float *amax_out, float *amax_rht_out,
                                                void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Synchronise `stream`, then read and clear the workspace's device status
 * word: NVFP4_OK, NVFP4_ERR_DEVICE_TIMEOUT, or NVFP4_ERR_CUDA if the stream
 * reports an error. */
NVFP4_API nvfp4_status nvfp4_check(void *workspace, cudaStream_t stream);

/* Self-test of the device-timeout path (no counterpart on the pages): one
 * thread waits on an mbarrier that nothing arrives on, with the same bounded
 * loop the GEMM uses but a limit of limit_ns nanoseconds (1 .. 2e9), then
 * records NVFP4_ERR_DEVICE_TIMEOUT in the workspace status word (workspace:
 * >= 256 bytes, 16-byte aligned, device memory, caller-owned) and returns.
 * Asynchronous; the following nvfp4_check() reports (and clears) the status.
 * Launch errors: NVFP4_ERR_WORKSPACE, NVFP4_ERR_ALIGNMENT,
 * NVFP4_ERR_INVALID_ARG (limit out of range), NVFP4_ERR_UNSUPPORTED_DEVICE. */
NVFP4_API nvfp4_status nvfp4_selftest_wait_timeout(void *workspace, size_t ws_bytes, uint64_t limit_ns,
                                                   cudaStream_t stream);

/* Tensor-pipe rate probe (measurement only; the pages give Blackwell's NVFP4
 * tensor cores as the engine of the method: nerdman.de, section "Was konkret
 * passiert ist").  Every CTA pair the device can hold at once issues `iters`
 * rounds of the GEMM's stage -- four M256 N256 K64 block-scaled MMAs,
 * kind::mxf4nvf4 block16 (mx = 0) or kind::mxf4 block32 (mx = 1), with the
 * GEMM's own descriptors -- on operands resident in shared memory and scales
 * resident in TMEM, and writes the %clock64 cycles from its first MMA to the
 * completion of its last to cycles[pair] (device memory, cycles_len >= the
 * number of pairs; *pairs_out, host memory, receives that number).  FLOPs per
 * pair: iters * 4 * 2 * 256 * 256 * 64.  iters: 1 .. 1000000.  Asynchronous:
 * time it with events on `stream`; a completion not seen within ~2 s records
 * NVFP4_ERR_DEVICE_TIMEOUT in the workspace status word (>= 256 bytes,
 * 16-byte aligned, caller-owned).  Launch errors: NVFP4_ERR_INVALID_ARG (null
 * pointer, mx not 0/1, iters out of range, cycles_len too small),
 * NVFP4_ERR_WORKSPACE, NVFP4_ERR_ALIGNMENT, NVFP4_ERR_UNSUPPORTED_DEVICE. */
NVFP4_API nvfp4_status nvfp4_selftest_mma_rate(int mx, int64_t iters, uint64_t *cycles, int64_t cycles_len,
                                               int *pairs_out, void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Bounds-checked debug build (libnvfp4_checked.so, compiled with
 * -DNVFP4_BOUNDS_CHECK; no counterpart on the pages: it checks the library's
 * own index arithmetic).  There every guarded global access of the kernels
 * first checks the elements it touches against the extent of the buffer as the
 * call's shapes define it; an access that would fall outside is skipped and
 * the source line of the first such check is recorded (nothing traps).
 * nvfp4_bounds_status synchronises the device, reads and clears these records:
 * NVFP4_ERR_DEVICE_BOUNDS with *site = file * 100000 + line (file: 1
 * quantize.cu, 2 elementwise.cu, 3 gemm.cu, 4 selftest.cu) if a check failed
 * since the last call, else NVFP4_OK with *site = 0.  *checked (host memory)
 * is 1 in the checked build, 0 in the product build, which records nothing.
 * Errors: NVFP4_ERR_INVALID_ARG (null pointer), NVFP4_ERR_CUDA. */
NVFP4_API nvfp4_status nvfp4_bounds_status(int *checked, int *site);

/* Self-test of that record (checked build only): one thread makes a check of
 * element 0 of [0, n), which passes and sets buf[0] = 1, and a check of element
 * n, which fails, so buf[n] is not written and the next nvfp4_bounds_status
 * reports it.  buf: device memory of n + 1 bytes (the byte past the checked
 * range exists, so even an unguarded write would stay inside the allocation),
 * caller-owned; 1 <= n.  Asynchronous.  Errors: NVFP4_ERR_INVALID_ARG (null
 * buf, n < 1, or the product build, where it launches nothing),
 * NVFP4_ERR_UNSUPPORTED_DEVICE, NVFP4_ERR_CUDA. */
NVFP4_API nvfp4_status nvfp4_selftest_bounds(uint8_t *buf, int64_t n, cudaStream_t stream);

/* Number of kernel launches the most recent successful call on this host
 * thread issued (launch accounting for benchmarks). */
NVFP4_API int nvfp4_last_launch_count(void);

/* Static description of a status code. */
NVFP4_API const char *nvfp4_status_string(nvfp4_status status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
