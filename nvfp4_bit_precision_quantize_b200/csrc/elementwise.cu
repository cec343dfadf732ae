// elementwise.cu -- squared-ReLU activation of the MLP block and its derivative.
//   h  = relu(y) * relu(y)       dy = dh * (2 * relu(y))
// one binary32 operation each, then bf16 round-to-nearest-even; relu(y) is +0
// for y <= 0.  16-byte vectors (8 bf16) per thread, grid-stride.
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float relu(float y) { return y > 0.0f ? y : 0.0f; }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(hi), "f"(lo));
    return w;
}
__device__ __forceinline__ uint16_t bf16_of(float f) { return (uint16_t)(pack_bf16x2(f, 0.0f) & 0xFFFFu); }

__device__ __forceinline__ uint32_t relu2_pair(uint32_t y) {
    const float a = relu(bf16lo(y)), b = relu(bf16hi(y));
    return pack_bf16x2(__fmul_rn(a, a), __fmul_rn(b, b));
}
__device__ __forceinline__ uint32_t drelu2_pair(uint32_t dh, uint32_t y) {
    const float ga = __fmul_rn(2.0f, relu(bf16lo(y))), gb = __fmul_rn(2.0f, relu(bf16hi(y)));
    return pack_bf16x2(__fmul_rn(bf16lo(dh), ga), __fmul_rn(bf16hi(dh), gb));
}

__global__ void __launch_bounds__(kThreads) relu2_fwd_kernel(const uint16_t *__restrict__ y, uint16_t *__restrict__ h,
                                                             int64_t n) {
    const int64_t nv = n / 8, stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nv; i += stride) {
        const uint4 v = ldg_stream(y + 8 * i);
        reinterpret_cast<uint4 *>(h)[i] = make_uint4(relu2_pair(v.x), relu2_pair(v.y), relu2_pair(v.z), relu2_pair(v.w));
    }
    for (int64_t i = 8 * nv + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
        const float a = relu(__uint_as_float((uint32_t)y[i] << 16));
        h[i] = bf16_of(__fmul_rn(a, a));
    }
}

__global__ void __launch_bounds__(kThreads) relu2_bwd_kernel(const uint16_t *__restrict__ dh,
                                                             const uint16_t *__restrict__ y, uint16_t *__restrict__ dy,
                                                             int64_t n) {
    const int64_t nv = n / 8, stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nv; i += stride) {
        const uint4 g = ldg_stream(dh + 8 * i), v = ldg_stream(y + 8 * i);
        reinterpret_cast<uint4 *>(dy)[i] =
            make_uint4(drelu2_pair(g.x, v.x), drelu2_pair(g.y, v.y), drelu2_pair(g.z, v.z), drelu2_pair(g.w, v.w));
    }
    for (int64_t i = 8 * nv + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
        const float g = __fmul_rn(2.0f, relu(__uint_as_float((uint32_t)y[i] << 16)));
        dy[i] = bf16_of(__fmul_rn(__uint_as_float((uint32_t)dh[i] << 16), g));
    }
}

unsigned grid_for(int64_t n) {
    const int64_t want = (n / 8 + kThreads - 1) / kThreads;
    const int64_t cap = 8LL * num_sms();
    return (unsigned)std::max<int64_t>(1, std::min(want, cap));
}

}  // namespace

cudaError_t launch_relu2_fwd(const void *y, void *h, int64_t n, cudaStream_t s, int *launches) {
    if (n == 0) return cudaSuccess;
    relu2_fwd_kernel<<<grid_for(n), kThreads, 0, s>>>(static_cast<const uint16_t *>(y), static_cast<uint16_t *>(h), n);
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_relu2_bwd(const void *dh, const void *y, void *dy, int64_t n, cudaStream_t s, int *launches) {
    if (n == 0) return cudaSuccess;
    relu2_bwd_kernel<<<grid_for(n), kThreads, 0, s>>>(static_cast<const uint16_t *>(dh),
                                                       static_cast<const uint16_t *>(y), static_cast<uint16_t *>(dy), n);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace nvfp4
