// internal.h -- host-side interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4.h"

namespace nvfp4 {

constexpr int kMaxPartials = 1024;          // per-CTA amax partials in a quantize workspace
constexpr size_t kStatusBytes = 256;        // status word region at the start of a workspace
constexpr size_t kQuantizeWorkspace = kStatusBytes + kMaxPartials * sizeof(float);
constexpr size_t kDualWorkspace = kStatusBytes + 2 * kMaxPartials * sizeof(float);
// The colwise kernels tile the input rows 256 per grid row, and a grid has at
// most 65535 rows: the largest R (blocked dim) a colwise quantisation takes.
constexpr int64_t kMaxColwiseRows = 65535LL * 256;

struct QuantizeArgs {
    const void *x;
    bool bf16;
    int64_t R, C, ld;
    bool colwise, sr, rht;
    uint64_t seed;
    const float *amax_in;   // optional
    uint8_t *codes;
    uint8_t *scales;
    float *tensor_scale;
    float *partials;        // kMaxPartials floats (unused when amax_in is set)
    int *status = nullptr;  // workspace status word (device timeouts), or null
};

// Rowwise RTN and colwise (RTN/SR, optional RHT) outputs of one tensor from one read.
struct DualQuantizeArgs {
    const void *x;
    bool bf16;
    int64_t R, C, ld;
    bool col_sr, col_rht;
    uint64_t seed;
    const float *amax_row_in, *amax_col_in;  // optional
    uint8_t *row_codes, *row_scales;
    float *row_tensor_scale;
    uint8_t *col_codes, *col_scales;
    float *col_tensor_scale;
    float *row_partials, *col_partials;      // kMaxPartials floats each
};

struct GemmArgs {
    const uint8_t *a_codes, *a_scales;
    const float *a_ts;
    const uint8_t *b_codes, *b_scales;
    const float *b_ts;
    int64_t M, N, K;
    void *C;
    bool c_bf16;
    int64_t ldc;
    int *status;
    bool mx = false;  // MXFP4 operands (E8M0 scales per 32 k, no tensor scales)
    // Fused squared-ReLU epilogue (bf16 output, M and N multiples of 256, M < 2^31):
    //   GEMM_EPI_RELU2_FWD: C = y = bf16(acc), aux (out) = relu(y)^2
    //   GEMM_EPI_RELU2_BWD: C = bf16(bf16(acc) * 2 relu(aux)), aux (in) = the forward's y
    // with max |relu output| and max |RHT(relu output)| (16-point transform of
    // `seed` down 16-row groups) written to amax_out[0] and amax_out[1] through
    // partials (2 * kMaxPartials floats).
    int epi = 0;
    void *aux = nullptr;
    uint64_t seed = 0;
    float *partials = nullptr;
    float *amax_out = nullptr;
    float *amax_rht_out = nullptr;
};
constexpr int GEMM_EPI_PLAIN = 0, GEMM_EPI_RELU2_FWD = 1, GEMM_EPI_RELU2_BWD = 2;

// Each launcher adds the number of kernels it launched to *launches.
cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_quantize_dual(const DualQuantizeArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_quantize_mx(const void *x, bool bf16, int64_t R, int64_t C, int64_t ld, bool colwise,
                               uint8_t *codes, uint8_t *scales, cudaStream_t s, int *launches);
cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s, int *launches);
// amax_out (optional): max |output| written there; partials: kMaxPartials floats when amax_out is set.
cudaError_t launch_relu2_fwd(const void *y, void *h, int64_t n, float *amax_out, float *partials, cudaStream_t s,
                             int *launches);
cudaError_t launch_relu2_bwd(const void *dh, const void *y, void *dy, int64_t n, float *amax_out, float *partials,
                             cudaStream_t s, int *launches);

// max over per-CTA partials (plain at partials, RHT at partials + kMaxPartials) -> *amax_out, *amax_rht_out
cudaError_t launch_amax_reduce(const float *partials, int count, float *amax_out, cudaStream_t s, int *launches);
// Tensor amax (after the 16-row RHT when rht): per-CTA partials, then one reduce into *amax_out.
cudaError_t launch_amax(const void *x, bool bf16, int64_t R, int64_t C, int64_t ld, bool rht, uint64_t seed,
                        float *partials, float *amax_out, cudaStream_t s, int *launches);
// Both amaxes (plain and after the 16-row RHT) from one read: partials (2 x kMaxPartials), then one reduce.
cudaError_t launch_amax_dual(const void *x, bool bf16, int64_t R, int64_t C, int64_t ld, uint64_t seed,
                             float *partials, float *amax_out, float *amax_rht_out, cudaStream_t s, int *launches);
cudaError_t launch_amax_reduce2(const float *partials, int count, float *amax_out, float *amax_rht_out, cudaStream_t s,
                                int *launches);

// One bounded wait on an mbarrier nothing arrives on; records the timeout status.
cudaError_t launch_wait_timeout(int *status, uint64_t limit_ns, cudaStream_t s, int *launches);
// Bounds-checked build: read and clear each translation unit's record (checked.cuh).
cudaError_t read_bounds_quantize(int *site);
cudaError_t read_bounds_elementwise(int *site);
cudaError_t read_bounds_gemm(int *site);
cudaError_t read_bounds_selftest(int *site);
cudaError_t launch_selftest_bounds(uint8_t *buf, int64_t n, cudaStream_t s, int *launches);
// Tensor-pipe rate probe (gemm.cu): one launch over every co-resident CTA pair.
cudaError_t launch_mma_rate(bool mx, int64_t iters, uint64_t *cycles, int64_t cycles_len, int *pairs_out, int *status,
                            cudaStream_t s, int *launches);

// relu^2 (dh == nullptr) or its derivative over a contiguous [R x C] bf16 tensor (R % 16 == 0,
// C % 8 == 0), also writing max |out| and max |RHT(out)| (transform down 16-row groups);
// partials: 2 * kMaxPartials floats.
cudaError_t launch_relu2_amax_rht(const void *dh, const void *y, void *out, int64_t R, int64_t C, uint64_t seed,
                                  float *amax_out, float *amax_rht_out, float *partials, cudaStream_t s,
                                  int *launches);

int num_sms();  // SM count of the current device (cached)

// Scratch bytes nvfp4_linear_fwd needs (both rowwise operands after the
// status word, amax partials and tensor scales), and every host-side check it
// makes before launching, device check included (M or N == 0 passes).
size_t linear_fwd_workspace_bytes(int64_t M, int64_t N, int64_t K);
nvfp4_status linear_fwd_validate(const void *X, const void *W, const void *Y, int64_t M, int64_t N, int64_t K,
                                 nvfp4_dtype dtype, nvfp4_dtype y_dtype, const void *workspace, size_t ws_bytes);

}  // namespace nvfp4
