// elementwise.cu -- squared-ReLU activation of the MLP block and its derivative.
//   h  = relu(y) * relu(y)       dy = dh * (2 * relu(y))
// one binary32 operation each, then bf16 round-to-nearest-even; relu(y) is +0
// for y <= 0.  16-byte vectors (8 bf16) per thread, grid-stride.  The AMAX
// variants also return max |output| (of the stored bf16 values), one partial
// per CTA reduced by a second one-CTA kernel, so that the NVFP4 quantisation
// that follows can skip its own amax pass (tensor scale from a supplied amax).
#include "checked.cuh"
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint16_t bf16_of(float f) { return (uint16_t)(pack_bf16x2(f, 0.0f) & 0xFFFFu); }
// Block-wide max written as this CTA's partial.
__device__ __forceinline__ void write_partial(float m, float *partials) {
    __shared__ float s_red[kThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) b = fmaxf(b, s_red[w]);
        if (NVFP4_IN_RANGE(blockIdx.x, 1, kMaxPartials)) partials[blockIdx.x] = b;
    }
}

template <bool AMAX>
__global__ void __launch_bounds__(kThreads) relu2_fwd_kernel(const uint16_t *__restrict__ y, uint16_t *__restrict__ h,
                                                             int64_t n, float *__restrict__ partials) {
    const int64_t nv = n / 8, stride = (int64_t)gridDim.x * kThreads;
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nv; i += stride) {
        if (!NVFP4_IN_RANGE(8 * i, 8, n)) continue;
        const uint4 v = ldg_stream(y + 8 * i);
        const uint4 o = make_uint4(relu2_pair(v.x), relu2_pair(v.y), relu2_pair(v.z), relu2_pair(v.w));
        reinterpret_cast<uint4 *>(h)[i] = o;
        if (AMAX) m = absmax_pair(absmax_pair(absmax_pair(absmax_pair(m, o.x), o.y), o.z), o.w);
    }
    for (int64_t i = 8 * nv + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
        if (!NVFP4_IN_RANGE(i, 1, n)) continue;
        const float a = relu(__uint_as_float((uint32_t)y[i] << 16));
        const uint16_t o = bf16_of(__fmul_rn(a, a));
        h[i] = o;
        if (AMAX) m = fmaxf(m, fabsf(__uint_as_float((uint32_t)o << 16)));
    }
    if (AMAX) write_partial(m, partials);
}

template <bool AMAX>
__global__ void __launch_bounds__(kThreads) relu2_bwd_kernel(const uint16_t *__restrict__ dh,
                                                             const uint16_t *__restrict__ y, uint16_t *__restrict__ dy,
                                                             int64_t n, float *__restrict__ partials) {
    const int64_t nv = n / 8, stride = (int64_t)gridDim.x * kThreads;
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nv; i += stride) {
        if (!NVFP4_IN_RANGE(8 * i, 8, n)) continue;
        const uint4 g = ldg_stream(dh + 8 * i), v = ldg_stream(y + 8 * i);
        const uint4 o =
            make_uint4(drelu2_pair(g.x, v.x), drelu2_pair(g.y, v.y), drelu2_pair(g.z, v.z), drelu2_pair(g.w, v.w));
        reinterpret_cast<uint4 *>(dy)[i] = o;
        if (AMAX) m = absmax_pair(absmax_pair(absmax_pair(absmax_pair(m, o.x), o.y), o.z), o.w);
    }
    for (int64_t i = 8 * nv + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
        if (!NVFP4_IN_RANGE(i, 1, n)) continue;
        const float g = __fmul_rn(2.0f, relu(__uint_as_float((uint32_t)y[i] << 16)));
        const uint16_t o = bf16_of(__fmul_rn(__uint_as_float((uint32_t)dh[i] << 16), g));
        dy[i] = o;
        if (AMAX) m = fmaxf(m, fabsf(__uint_as_float((uint32_t)o << 16)));
    }
    if (AMAX) write_partial(m, partials);
}

// max over the partials -> *out (one CTA)
__global__ void __launch_bounds__(kThreads) amax_reduce_kernel(const float *__restrict__ partials, int count,
                                                               float *__restrict__ out) {
    __shared__ float s_red[kThreads / 32];
    const float m = reduce_partials_max(partials, count, s_red);
    if (threadIdx.x == 0) *out = m;
}

// 2-D variant over a contiguous [R x C] tensor (R % 16 == 0, C % 8 == 0): one
// work unit = a 16-row group x 4 columns (one 8-byte load per row; a warp's
// loads cover 256 contiguous bytes of a row), so each column's 16 consecutive
// outputs sit in one thread and both max |out| and max |RHT(out)| (the 16-point
// transform down the rows, as the colwise quantiser applies it) come from the
// values just stored.
template <bool BWD>
__global__ void __launch_bounds__(kThreads, 2) relu2_amax_rht_kernel(const uint16_t *__restrict__ dh,
                                                                     const uint16_t *__restrict__ y,
                                                                     uint16_t *__restrict__ out, int64_t R, int64_t C,
                                                                     uint64_t seed, float *__restrict__ partials_plain,
                                                                     float *__restrict__ partials_rht) {
    const uint32_t signs = rht_sign_bits(seed);
    const int64_t chunks = C / 4;
    const int64_t total = (R / 16) * chunks;
    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll 1
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < total; u += (int64_t)gridDim.x * kThreads) {
        const int64_t g = u / chunks, cc = u - g * chunks;
        const int64_t base = g * 16 * C + cc * 4;
        if (!NVFP4_IN_RANGE(base, 15 * C + 4, R * C)) continue;  // the unit's 16 rows x 4 columns
        uint2 o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(y + base + i * C));
            if (BWD) {
                const uint2 gr = __ldg(reinterpret_cast<const uint2 *>(dh + base + i * C));
                o[i] = make_uint2(drelu2_pair(gr.x, v.x), drelu2_pair(gr.y, v.y));
            } else {
                o[i] = make_uint2(relu2_pair(v.x), relu2_pair(v.y));
            }
            *reinterpret_cast<uint2 *>(out + base + i * C) = o[i];
            m0 = absmax_pair(absmax_pair(m0, o[i].x), o[i].y);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float t[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t w = (j >> 1) ? o[i].y : o[i].x;
                t[i] = (j & 1) ? bf16hi(w) : bf16lo(w);
            }
            rht16(t, signs);
#pragma unroll
            for (int i = 0; i < 16; ++i) m1 = fmaxf(m1, fabsf(t[i]));
        }
    }
    write_partial(m0, partials_plain);
    __syncthreads();
    write_partial(m1, partials_rht);
}

// max over both partial sets -> *out_plain, *out_rht (one CTA)
__global__ void __launch_bounds__(kThreads) amax_reduce2_kernel(const float *__restrict__ partials_plain,
                                                                const float *__restrict__ partials_rht, int count,
                                                                float *__restrict__ out_plain,
                                                                float *__restrict__ out_rht) {
    __shared__ float s_red[kThreads / 32];
    const float a = reduce_partials_max(partials_plain, count, s_red);
    const float b = reduce_partials_max(partials_rht, count, s_red);
    if (threadIdx.x == 0) {
        *out_plain = a;
        *out_rht = b;
    }
}

unsigned grid_for(int64_t n, int64_t cap_ctas) {
    const int64_t want = (n / 8 + kThreads - 1) / kThreads;
    return (unsigned)std::max<int64_t>(1, std::min(want, cap_ctas));
}

}  // namespace

cudaError_t launch_relu2_fwd(const void *y, void *h, int64_t n, float *amax_out, float *partials, cudaStream_t s,
                             int *launches) {
    const uint16_t *yy = static_cast<const uint16_t *>(y);
    uint16_t *hh = static_cast<uint16_t *>(h);
    if (!amax_out) {
        if (n == 0) return cudaSuccess;
        relu2_fwd_kernel<false><<<grid_for(n, 8LL * num_sms()), kThreads, 0, s>>>(yy, hh, n, nullptr);
        ++*launches;
        return cudaGetLastError();
    }
    const unsigned grid = grid_for(n, std::min<int64_t>(4LL * num_sms(), kMaxPartials));
    relu2_fwd_kernel<true><<<grid, kThreads, 0, s>>>(yy, hh, n, partials);
    amax_reduce_kernel<<<1, kThreads, 0, s>>>(partials, (int)grid, amax_out);
    *launches += 2;
    return cudaGetLastError();
}

cudaError_t launch_relu2_bwd(const void *dh, const void *y, void *dy, int64_t n, float *amax_out, float *partials,
                             cudaStream_t s, int *launches) {
    const uint16_t *gg = static_cast<const uint16_t *>(dh), *yy = static_cast<const uint16_t *>(y);
    uint16_t *dd = static_cast<uint16_t *>(dy);
    if (!amax_out) {
        if (n == 0) return cudaSuccess;
        relu2_bwd_kernel<false><<<grid_for(n, 8LL * num_sms()), kThreads, 0, s>>>(gg, yy, dd, n, nullptr);
        ++*launches;
        return cudaGetLastError();
    }
    const unsigned grid = grid_for(n, std::min<int64_t>(4LL * num_sms(), kMaxPartials));
    relu2_bwd_kernel<true><<<grid, kThreads, 0, s>>>(gg, yy, dd, n, partials);
    amax_reduce_kernel<<<1, kThreads, 0, s>>>(partials, (int)grid, amax_out);
    *launches += 2;
    return cudaGetLastError();
}

}  // namespace nvfp4

namespace nvfp4 {

cudaError_t launch_relu2_amax_rht(const void *dh, const void *y, void *out, int64_t R, int64_t C, uint64_t seed,
                                  float *amax_out, float *amax_rht_out, float *partials, cudaStream_t s,
                                  int *launches) {
    const int64_t units = (R / 16) * (C / 4);
    const unsigned grid = (unsigned)std::max<int64_t>(
        1, std::min<int64_t>((units + kThreads - 1) / kThreads, std::min<int64_t>(4LL * num_sms(), kMaxPartials)));
    const uint16_t *yy = static_cast<const uint16_t *>(y);
    uint16_t *oo = static_cast<uint16_t *>(out);
    if (dh)
        relu2_amax_rht_kernel<true><<<grid, kThreads, 0, s>>>(static_cast<const uint16_t *>(dh), yy, oo, R, C, seed,
                                                              partials, partials + kMaxPartials);
    else
        relu2_amax_rht_kernel<false><<<grid, kThreads, 0, s>>>(nullptr, yy, oo, R, C, seed, partials,
                                                               partials + kMaxPartials);
    amax_reduce2_kernel<<<1, kThreads, 0, s>>>(partials, partials + kMaxPartials, (int)grid, amax_out, amax_rht_out);
    *launches += 2;
    return cudaGetLastError();
}

cudaError_t launch_amax_reduce(const float *partials, int count, float *amax_out, cudaStream_t s, int *launches) {
    amax_reduce_kernel<<<1, kThreads, 0, s>>>(partials, count, amax_out);
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_amax_reduce2(const float *partials, int count, float *amax_out, float *amax_rht_out, cudaStream_t s,
                                int *launches) {
    amax_reduce2_kernel<<<1, kThreads, 0, s>>>(partials, partials + kMaxPartials, count, amax_out, amax_rht_out);
    ++*launches;
    return cudaGetLastError();
}

NVFP4_DEFINE_BOUNDS_READER(read_bounds_elementwise)

}  // namespace nvfp4
