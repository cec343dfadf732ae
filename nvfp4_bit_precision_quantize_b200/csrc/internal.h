// internal.h -- host-side interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kMaxPartials = 1024;          // per-CTA amax partials in a quantize workspace
constexpr size_t kStatusBytes = 256;        // status word region at the start of a workspace
constexpr size_t kQuantizeWorkspace = kStatusBytes + kMaxPartials * sizeof(float);

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
};

// Each launcher adds the number of kernels it launched to *launches.
cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_relu2_fwd(const void *y, void *h, int64_t n, cudaStream_t s, int *launches);
cudaError_t launch_relu2_bwd(const void *dh, const void *y, void *dy, int64_t n, cudaStream_t s,
                             int *launches);

int num_sms();  // SM count of the current device (cached)

}  // namespace nvfp4
