// quantize.cu -- NVFP4 quantisation kernels for sm_100a.
//
// Two passes over the input:
//   pass 1 (amax_*, HBM-bound): tensor amax (after the random Hadamard
//     transform when it is on), written as one partial per CTA -- no atomics,
//     no zeroing;
//   pass 2 (quantize_*): every CTA reduces the partials to the same amax,
//     derives the FP32 tensor scale, and turns its tile into packed E2M1 codes
//     plus E4M3 block scales laid out in the tensor cores' 128x4 scale atoms.
//     HBM-bound in design; with the Hadamard transform and stochastic rounding
//     (Philox per 8 elements) the colwise variant is bound by ALU issue instead.
// Format: aisight.pl, "Koniec marnowania mocy ...", section "Architektura
// NVFP4 kontra ograniczenia mikroskalowania" (block 16, E4M3 block scale, FP32
// tensor scale).  Hadamard transform and stochastic rounding on the Wgrad
// operands: same page, section "Technologie stabilizujace proces treningowy".
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "checked.cuh"
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

#ifdef NVFP4_BOUNDS_CHECK
// Buffer extents for the bounds-checked build (arguments of NVFP4_IN_RANGE only).
__host__ __device__ constexpr int64_t x_extent(int64_t R, int64_t C, int64_t ld) { return (R - 1) * ld + C; }
__host__ __device__ constexpr int64_t nv_scales_extent(int64_t rows, int64_t k) {
    return ((rows + 127) / 128) * 128 * (((k + 63) / 64) * 4);
}
__host__ __device__ constexpr int64_t mx_scales_extent(int64_t rows, int64_t k) {
    return ((rows + 127) / 128) * 128 * (((k + 127) / 128) * 4);
}
#endif

// xor of a 16-byte row chunk with the sign-bit mask of Hadamard input row i
// (bit i of the sign word set: every element of the chunk changes sign).
template <typename T>
__device__ __forceinline__ uint32_t sign_mask(uint32_t signs, int i) {
    return ((signs >> i) & 1u) ? (sizeof(T) == 2 ? 0x80008000u : 0x80000000u) : 0u;
}
__device__ __forceinline__ uint4 xor4(const uint4 &a, uint32_t f) {
    return make_uint4(a.x ^ f, a.y ^ f, a.z ^ f, a.w ^ f);
}

// ---------------------------------------------------------------------------
// Pass 1a: max |x| over an [R x C] tensor (any orientation, no transform).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) amax_kernel(const T *__restrict__ x, int64_t R, int64_t C,
                                                        int64_t ld, float *__restrict__ partials) {
    constexpr int N = Vec<T>::N;
    __shared__ float s_red[kThreads / 32];
    const int64_t chunks_per_row = C / N;
    const int64_t total = R * chunks_per_row;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    float m = 0.0f;
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (ld == C) {
        constexpr int U = 4;  // independent 16-byte loads in flight per thread
        for (; i + (U - 1) * stride < total; i += U * stride) {
            uint4 raw[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                raw[u] = NVFP4_IN_RANGE((i + u * stride) * N, N, R * C) ? ldg_stream(x + (i + u * stride) * N) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float v[N];
                Vec<T>::unpack(raw[u], v);
#pragma unroll
                for (int j = 0; j < N; ++j) m = fmaxf(m, fabsf(v[j]));
            }
        }
        for (; i < total; i += stride) {
            float v[N];
            Vec<T>::unpack(NVFP4_IN_RANGE(i * N, N, R * C) ? ldg_stream(x + i * N) : make_uint4(0u, 0u, 0u, 0u), v);
#pragma unroll
            for (int j = 0; j < N; ++j) m = fmaxf(m, fabsf(v[j]));
        }
    } else {
        for (; i < total; i += stride) {
            const int64_t r = i / chunks_per_row, c = (i - r * chunks_per_row) * N;
            float v[N];
            Vec<T>::unpack(NVFP4_IN_RANGE(r * ld + c, N, x_extent(R, C, ld)) ? ldg_stream(x + r * ld + c) : make_uint4(0u, 0u, 0u, 0u), v);
#pragma unroll
            for (int j = 0; j < N; ++j) m = fmaxf(m, fabsf(v[j]));
        }
    }
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

// ---------------------------------------------------------------------------
// Pass 1b: max |RHT(x)| where the transform runs down 16-row groups of every
// column.  One work unit = one 16-row group x N columns (one 16-byte load per
// row); consecutive threads take consecutive column chunks.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) amax_rht_kernel(const T *__restrict__ x, int64_t R, int64_t C,
                                                            int64_t ld, uint64_t seed,
                                                            float *__restrict__ partials) {
    constexpr int N = Vec<T>::N;
    __shared__ float s_red[kThreads / 32];
    const uint32_t signs = rht_sign_bits(seed);
    const int64_t chunks = C / N;
    const int64_t total = (R / 16) * chunks;
    float m = 0.0f;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * kThreads) {
        const int64_t g = u / chunks, cc = u - g * chunks;
        const T *p = x + (g * 16) * ld + cc * N;
        uint4 raw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            raw[i] = NVFP4_IN_RANGE((g * 16 + i) * ld + cc * N, N, x_extent(R, C, ld)) ? ldg_stream(p + i * ld) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < 16; ++i) raw[i] = xor4(raw[i], sign_mask<T>(signs, i));
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float t[N];
                Vec<T>::unpack(raw[i], t);
                v[i] = t[j];
            }
            fwht16(v);
#pragma unroll
            for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
        }
    }
    m = __fmul_rn(m, 0.25f);  // max |z / 4| = RN(max |z| / 4)
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

// ---------------------------------------------------------------------------
// Pass 1c: both max |x| and max |RHT(x)| (transform down 16-row groups of every
// column) from one read, for the dual quantiser; units as in pass 1b.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) amax_dual_kernel(const T *__restrict__ x, int64_t R, int64_t C,
                                                             int64_t ld, uint64_t seed,
                                                             float *__restrict__ partials_plain,
                                                             float *__restrict__ partials_rht) {
    constexpr int N = Vec<T>::N;
    __shared__ float s_red[2][kThreads / 32];
    const uint32_t signs = rht_sign_bits(seed);
    const int64_t chunks = C / N;
    const int64_t total = (R / 16) * chunks;
    float m0 = 0.0f, m1 = 0.0f;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * kThreads) {
        const int64_t g = u / chunks, cc = u - g * chunks;
        const T *p = x + (g * 16) * ld + cc * N;
        uint4 raw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            raw[i] = NVFP4_IN_RANGE((g * 16 + i) * ld + cc * N, N, x_extent(R, C, ld)) ? ldg_stream(p + i * ld) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < 16; ++i) raw[i] = xor4(raw[i], sign_mask<T>(signs, i));
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float t[N];
                Vec<T>::unpack(raw[i], t);
                v[i] = t[j];
                m0 = fmaxf(m0, fabsf(v[i]));  // the sign flips do not change |v|
            }
            fwht16(v);
#pragma unroll
            for (int i = 0; i < 16; ++i) m1 = fmaxf(m1, fabsf(v[i]));
        }
    }
    m1 = __fmul_rn(m1, 0.25f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, o));
    }
    if ((threadIdx.x & 31) == 0) {
        s_red[0][threadIdx.x >> 5] = m0;
        s_red[1][threadIdx.x >> 5] = m1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float b0 = 0.0f, b1 = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) {
            b0 = fmaxf(b0, s_red[0][w]);
            b1 = fmaxf(b1, s_red[1][w]);
        }
        if (NVFP4_IN_RANGE(blockIdx.x, 1, kMaxPartials)) {
            partials_plain[blockIdx.x] = b0;
            partials_rht[blockIdx.x] = b1;
        }
    }
}

struct QParams {
    const void *x;
    int64_t R, C, ld;
    uint64_t seed;
    const float *amax_in;
    const float *partials;
    int num_partials;
    uint8_t *codes;
    uint8_t *scales;
    float *tensor_scale;
    // dual quantiser only: the rowwise (RTN) output of the same tensor
    const float *row_amax_in;
    const float *row_partials;
    uint8_t *row_codes;
    uint8_t *row_scales;
    float *row_tensor_scale;
    int aligned32;  // x and every row start 32-byte aligned (256-bit loads allowed)
    int *status;    // workspace status word (device timeouts), or null
};

__device__ __forceinline__ float tensor_amax(const QParams &p, float *s_red) {
    return p.amax_in ? *p.amax_in : reduce_partials_max(p.partials, p.num_partials, s_red);
}

// The two Philox blocks that hold the 16-bit SR draws of the 16 consecutive
// output-view indices idx0 .. idx0+15 (idx0 % 16 == 0): counters (idx0 >> 3)
// and (idx0 >> 3) + 1, keyed on the seed.  Draw e of a block is the low (e
// even) or high (e odd) half of word e >> 1.
__device__ __forceinline__ void sr_words16(uint64_t idx0, const PhiloxKeys &k, uint4 &w0, uint4 &w1) {
    const uint64_t c = idx0 >> 3;
    w0 = philox4x32_10(make_uint4((uint32_t)c, (uint32_t)(c >> 32), 0u, 0u), k);
    w1 = philox4x32_10(make_uint4((uint32_t)(c + 1), (uint32_t)((c + 1) >> 32), 0u, 0u), k);
}
__device__ __forceinline__ uint32_t sr_draw(const uint4 &w, int e) {  // e = idx & 7, compile-time after unrolling
    const uint32_t word = (e >> 1) == 0 ? w.x : (e >> 1) == 1 ? w.y : (e >> 1) == 2 ? w.z : w.w;
    return (e & 1) ? sr_rnd_hi(word) : sr_rnd_lo(word);
}

// 16 E2M1 codes of one block (element 0 in the lowest nibble of .x), from the
// block's values as pairs p[k] = (v[2k], v[2k+1]) and its element scale; SR
// draws from w0 (elements 0-7) and w1 (8-15).  A block whose inv is 0 encodes
// +0 everywhere (the products are +-0, and the sign bits are cleared).  The
// products and the SR rounding steps run as pair operations (same bits as
// sr_e2m1_value on each element).
template <bool SR>
__device__ __forceinline__ uint2 encode16_x2(const uint64_t (&p)[8], float inv, const uint4 &w0, const uint4 &w1) {
    const uint64_t inv2 = f2(inv, inv);
    float q[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint64_t r = mul2_rn(p[k], inv2);
        const float r0 = f2lo(r), r1 = f2hi(r);
        if (SR) {
            const float a0 = fminf(fabsf(r0), 7.0f), a1 = fminf(fabsf(r1), 7.0f);
            const uint64_t base = f2(sr_below_one(a0), sr_below_one(a1));
            const uint64_t t = add2_ru(f2(a0, a1), base);
            const uint32_t d0 = sr_draw(k < 4 ? w0 : w1, (2 * k) & 7), d1 = sr_draw(k < 4 ? w0 : w1, (2 * k + 1) & 7);
            const uint64_t up = f2(__uint_as_float(sr_round_bits(__float_as_uint(f2lo(t)), d0)),
                                   __uint_as_float(sr_round_bits(__float_as_uint(f2hi(t)), d1)));
            const uint64_t d = sub2_rn(up, base);
            q[2 * k] = copysignf(f2lo(d), r0);
            q[2 * k + 1] = copysignf(f2hi(d), r1);
        } else {
            q[2 * k] = r0;
            q[2 * k + 1] = r1;
        }
    }
    uint2 c = make_uint2(e2m1x8(q), e2m1x8(q + 8));
    if (inv == 0.0f) {
        c.x &= 0x77777777u;
        c.y &= 0x77777777u;
    }
    return c;
}
template <bool SR>
__device__ __forceinline__ uint2 encode16(const float (&v)[16], float inv, const uint4 &w0, const uint4 &w1) {
    uint64_t p[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) p[k] = f2(v[2 * k], v[2 * k + 1]);
    return encode16_x2<SR>(p, inv, w0, w1);
}

// Loads of one 16-element block row segment: 8 (bf16) or 16 (f32) words.
template <int LW>
__device__ __forceinline__ void load_block(const uint8_t *src, bool a32, uint32_t (&w)[LW]) {
    if (a32) {
#pragma unroll
        for (int h = 0; h < LW / 8; ++h)
            asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                         : "=r"(w[8 * h]), "=r"(w[8 * h + 1]), "=r"(w[8 * h + 2]), "=r"(w[8 * h + 3]), "=r"(w[8 * h + 4]),
                           "=r"(w[8 * h + 5]), "=r"(w[8 * h + 6]), "=r"(w[8 * h + 7])
                         : "l"(src + 32 * h));
    } else {
#pragma unroll
        for (int h = 0; h < LW / 4; ++h)
            asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(w[4 * h]), "=r"(w[4 * h + 1]), "=r"(w[4 * h + 2]), "=r"(w[4 * h + 3])
                         : "l"(src + 16 * h));
    }
}
template <typename T> __device__ __forceinline__ void unpack16(const uint32_t *w, float (&v)[16]);
template <> __device__ __forceinline__ void unpack16<uint16_t>(const uint32_t *w, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = bf16lo(w[i]);
        v[2 * i + 1] = bf16hi(w[i]);
    }
}
template <> __device__ __forceinline__ void unpack16<float>(const uint32_t *w, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(w[i]);
}

// ---------------------------------------------------------------------------
// Pass 2, rowwise: blocks of 16 along the contiguous columns.  Each lane owns
// one whole block of a row (one 32-byte load for bf16, two for f32), so the
// block amax, the scale and the 16 codes (one 8-byte store) need no shuffles;
// a warp covers 512 columns of RPW rows per tile.  Persistent CTAs walk the
// tiles in reverse order (the amax pass swept the tensor front to back, so its
// tail is what L2 still holds) with the next tile's loads in flight.  The four
// scale bytes of a row within a 128x4 atom are one aligned 32-bit word held by
// four neighbouring lanes: two shuffles gather it and one lane stores it.
// Padding rows up to the atoms' 128-row extent and padding blocks up to their
// 4-block width get scale 0 (their loads are zero).
// ---------------------------------------------------------------------------
template <typename T, bool SR>
__global__ void __launch_bounds__(kThreads, 2) quantize_rowwise_kernel(const QParams p) {
    constexpr int LW = 4 * (int)sizeof(T);          // 32-bit words per lane and row
    constexpr int RPW = sizeof(T) == 2 ? 4 : 2;     // rows per warp per tile
    constexpr int TILE_R = RPW * (kThreads / 32);
    constexpr int TILE_B = 32;                      // blocks (of 16 columns) per tile row
    __shared__ float s_inv[128];
    __shared__ float s_red[kThreads / 32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *xb = static_cast<const uint8_t *>(p.x);
    const int64_t K = p.C, KB = K / 16, KB4 = (K + 63) / 64;
    const int64_t tiles_c = (KB + TILE_B - 1) / TILE_B;
    const int64_t tiles_r = ((p.R + 127) / 128) * (128 / TILE_R);
    const int64_t ntiles = tiles_c * tiles_r;
    const bool a32 = p.aligned32 != 0;

    auto load = [&](int64_t t, uint32_t(&buf)[RPW][LW]) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t b = tc * TILE_B + lane;
        const int64_t r0 = tr * TILE_R + warp * RPW;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int64_t r = r0 + i;
            if (b < KB && r < p.R && NVFP4_IN_RANGE(r * p.ld + b * 16, 16, x_extent(p.R, p.C, p.ld))) {
                load_block<LW>(xb + (r * p.ld + b * 16) * (int64_t)sizeof(T), a32, buf[i]);
            } else {
#pragma unroll
                for (int j = 0; j < LW; ++j) buf[i][j] = 0u;
            }
        }
    };

    int64_t t = ntiles - 1 - (int64_t)blockIdx.x;
    uint32_t cur[RPW][LW], nxt[RPW][LW];
    if (t >= 0) load(t, cur);
    const float s_t = tensor_scale_from_amax(tensor_amax(p, s_red));
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.tensor_scale = s_t;
    const ScaleCtx ctx = scale_ctx(s_t);
    scale_table_init(s_inv, nullptr, s_t);
    PhiloxKeys keys;
    if (SR) keys = philox_keys(p.seed);
    __syncthreads();

    for (; t >= 0; t -= gridDim.x) {
        const int64_t tn = t - gridDim.x;
        if (tn >= 0) load(tn, nxt);
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t b = tc * TILE_B + lane, atom = b >> 2;
        const bool col_ok = b < KB;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int64_t r = tr * TILE_R + warp * RPW + i;
            float v[16];
            unpack16<T>(cur[i], v);
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(v[j]));
            const uint32_t sb = block_scale_code(m, ctx);
            const float inv = s_inv[sb];
            uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
            if (SR) sr_words16((uint64_t)r * (uint64_t)K + (uint64_t)b * 16u, keys, w0, w1);
            const uint2 c = encode16<SR>(v, inv, w0, w1);
            if (col_ok && r < p.R && NVFP4_IN_RANGE(r * (K / 2) + b * 8, 8, p.R * (K / 2)))
                *reinterpret_cast<uint2 *>(p.codes + r * (K / 2) + b * 8) = c;
            uint32_t word = sb << (8 * (lane & 3));
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
            if ((lane & 3) == 0 && atom < KB4 &&
                NVFP4_IN_RANGE(((r >> 7) * KB4 + atom) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4, 4,
                               nv_scales_extent(p.R, K)))
                *reinterpret_cast<uint32_t *>(p.scales + ((r >> 7) * KB4 + atom) * 512 + (r & 31) * 16 +
                                              ((r >> 5) & 3) * 4) = word;
        }
#pragma unroll
        for (int i = 0; i < RPW; ++i)
#pragma unroll
            for (int j = 0; j < LW; ++j) cur[i][j] = nxt[i][j];
    }
}

// ---------------------------------------------------------------------------
// Pass 2, colwise, register-fed (f32 input, and the dual pass for both dtypes;
// bf16 single quantisations take quantize_colwise_tma_kernel below): blocks of
// 16 run down the rows; the output is the transpose ([C x R], K = R contiguous).  CTA tile = 256 rows x (32*N) columns; warp w
// owns rows 32w..32w+31 (two 16-row groups) and each lane N adjacent columns,
// so every block (one column x 16 rows) sits in one thread's registers: the
// transform, block amax and encoding need no shuffles.  The Hadamard signs
// are applied to the packed rows (one xor per word) before unpacking; the
// butterfly runs unnormalised and its 1/4 is applied exactly afterwards, or,
// with round-to-nearest and a tensor scale in the fast range, folded into the
// element scale (inv/4, tabulated): RN(RN(z/4) * inv) = RN(z * inv/4) whenever
// z/4 is exact, and where it is not (|z| < 2^-124) both sides give a +-0 code
// with the sign of z.  A lane's 16 code bytes per column (two groups) form one
// 16-byte unit in shared memory (each group writes its 8-byte half as soon as
// it is encoded), placed with an xor swizzle so both the scatter and the
// row-contiguous read-out are free of bank conflicts beyond the 4-wavefront
// minimum.  The DUAL variant also encodes the rowwise (RTN) blocks of the same
// rows from the same registers.
// ---------------------------------------------------------------------------
template <typename T, bool SR, bool RHT, bool DUAL>
__global__ void __launch_bounds__(kThreads, 2) quantize_colwise_kernel(const QParams p) {
    constexpr int N = Vec<T>::N;
    constexpr int W = kThreads / 32;     // warps
    constexpr int TC = 32 * N;           // output rows per tile
    constexpr int TR = 32 * W;           // k (input rows) per tile
    constexpr int P = W;                 // 16-byte code units per output row per tile
    constexpr int AR = TC / 128;         // scale-atom rows per tile
    constexpr int AC = TR / 64;          // scale-atom columns per tile
    __shared__ __align__(16) uint4 s_units[N * P * 32];
    __shared__ __align__(16) uint8_t s_sc[AR * AC * 512];
    __shared__ float s_red[W];
    __shared__ float s_inv[128], s_inv4[RHT ? 128 : 1], s_inv_row[DUAL ? 128 : 1];
    constexpr int LPB = 16 / N;          // dual: lanes per rowwise 16-block
    constexpr int ARR = TR / 128;        // dual: rowwise scale-atom rows per tile
    constexpr int ACR = TC / 64;         // dual: rowwise scale-atom columns per tile
    __shared__ __align__(16) uint8_t s_scr[DUAL ? ARR * ACR * 512 : 16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Tiles run in reverse order: the amax pass swept the rows front to back, so
    // the last row tiles are what L2 still holds when this pass starts.
    const int64_t lin = (int64_t)gridDim.x * gridDim.y - 1 - ((int64_t)blockIdx.y * gridDim.x + blockIdx.x);
    const int64_t bx = lin % gridDim.x, by = lin / gridDim.x;
    const int64_t c = bx * TC + lane * N;
    const int64_t r_warp = by * TR + warp * 32;
    const T *x = static_cast<const T *>(p.x);
    const bool col_ok = c < p.C;
    const int64_t K = p.R;
    const int64_t KB4 = (K + 63) / 64;

    // issue the first group's loads before the amax reduction
    uint4 raw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int64_t r = r_warp + i;
        raw[i] = (col_ok && r < p.R && NVFP4_IN_RANGE(r * p.ld + c, N, x_extent(p.R, p.C, p.ld))) ? ldg_stream(x + r * p.ld + c)
                                                                               : make_uint4(0u, 0u, 0u, 0u);
    }
    const float s_t = tensor_scale_from_amax(tensor_amax(p, s_red));
    float s_t_row = 0.0f;
    if (DUAL)
        s_t_row = tensor_scale_from_amax(p.row_amax_in ? *p.row_amax_in
                                                       : reduce_partials_max(p.row_partials, p.num_partials, s_red));
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        *p.tensor_scale = s_t;
        if (DUAL) *p.row_tensor_scale = s_t_row;
    }
    const ScaleCtx ctx = scale_ctx(s_t);
    scale_table_init(s_inv, RHT ? s_inv4 : nullptr, s_t);
    ScaleCtx ctx_row;
    if (DUAL) {
        ctx_row = scale_ctx(s_t_row);
        scale_table_init(s_inv_row, nullptr, s_t_row);
    }
    const uint32_t signs = RHT ? rht_sign_bits(p.seed) : 0u;
    // Quarter folded into the element scale: round-to-nearest only (a stochastic
    // decision on a value that RN(z/4) would flush to zero can differ).
    const bool fold = RHT && !SR && ctx.fast;
    PhiloxKeys keys;
    if (SR) keys = philox_keys(p.seed);
    __syncthreads();

#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t rg = r_warp + 16 * h;
        if (h == 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int64_t r = rg + i;
                raw[i] = (col_ok && r < p.R && NVFP4_IN_RANGE(r * p.ld + c, N, x_extent(p.R, p.C, p.ld))) ? ldg_stream(x + r * p.ld + c)
                                                                               : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        if (DUAL) {
            // Rowwise RTN encode of the same 16 rows: a lane holds N of a row's 16-block,
            // the partner lane(s) the rest (as in the rowwise quantiser).
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int64_t r = rg + i;
                float v[N];
                Vec<T>::unpack(raw[i], v);
                float m = 0.0f;
#pragma unroll
                for (int j = 0; j < N; ++j) m = fmaxf(m, fabsf(v[j]));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                if (LPB == 4) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                const uint32_t sb = block_scale_code(m, ctx_row);
                const float inv = s_inv_row[sb];
                float q[N];
#pragma unroll
                for (int j = 0; j < N; ++j) q[j] = __fmul_rn(v[j], inv);
                if (col_ok && r < p.R && NVFP4_IN_RANGE(r * (p.C / 2) + c / 2, N / 2, p.R * (p.C / 2))) {
                    uint8_t *dst = p.row_codes + r * (p.C / 2) + c / 2;
                    if (N == 8) *reinterpret_cast<uint32_t *>(dst) = e2m1x8(q) & (inv == 0.0f ? 0x77777777u : ~0u);
                    else *reinterpret_cast<uint16_t *>(dst) =
                             (uint16_t)(e2m1x4(q[0], q[1], q[2], q[3]) & (inv == 0.0f ? 0x7777u : 0xFFFFu));
                }
                if ((lane % LPB) == 0) {
                    const int rl = warp * 32 + 16 * h + i, bl = lane / LPB;
                    s_scr[((rl >> 7) * ACR + (bl >> 2)) * 512 + (rl & 31) * 16 + ((rl >> 5) & 3) * 4 + (bl & 3)] =
                        (uint8_t)sb;
                }
            }
        }
        if (RHT) {  // the sign diagonal, on the packed rows
#pragma unroll
            for (int i = 0; i < 16; ++i) raw[i] = xor4(raw[i], sign_mask<T>(signs, i));
        }
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float t[N];
                Vec<T>::unpack(raw[i], t);
                v[i] = t[j];
            }
            float scale_in;  // the element scale the block's values are multiplied by
            uint32_t sb;
            uint64_t pv[8];  // the block's values as pairs (v[2k], v[2k+1])
            float m = 0.0f;
            if (RHT) {
                fwht16_x2(v, pv);
#pragma unroll
                for (int k = 0; k < 8; ++k) m = fmaxf(m, fmaxf(fabsf(f2lo(pv[k])), fabsf(f2hi(pv[k]))));
                sb = block_scale_code(__fmul_rn(m, 0.25f), ctx);  // max |z/4| = RN(max|z| / 4)
                if (fold) {
                    scale_in = s_inv4[sb];
                } else {
                    const uint64_t quarter = f2(0.25f, 0.25f);
#pragma unroll
                    for (int k = 0; k < 8; ++k) pv[k] = mul2_rn(pv[k], quarter);
                    scale_in = s_inv[sb];
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    pv[k] = f2(v[2 * k], v[2 * k + 1]);
                    m = fmaxf(m, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
                }
                sb = block_scale_code(m, ctx);
                scale_in = s_inv[sb];
            }
            uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
            if (SR) sr_words16((uint64_t)(c + j) * (uint64_t)K + (uint64_t)rg, keys, w0, w1);  // rg % 16 == 0
            const uint2 code = encode16_x2<SR>(pv, scale_in, w0, w1);
            {  // this group's 8 code bytes: half h of the lane's 16-byte unit for column j
                const int qu = j * P + warp;
                reinterpret_cast<uint2 *>(s_units)[(qu * 32 + (lane ^ (qu & 7))) * 2 + h] = code;
            }
            const int cl = lane * N + j, gl = warp * 2 + h;
            s_sc[((cl >> 7) * AC + (gl >> 2)) * 512 + (cl & 31) * 16 + ((cl >> 5) & 3) * 4 + (gl & 3)] = (uint8_t)sb;
        }
    }
    __syncthreads();

    // codes: output row (c0 + cl) gets P units of 16 bytes at k-byte offset r0/2 + 16 p
    const int64_t c0 = bx * TC, r0 = by * TR;
    const bool vec16 = (K % 32) == 0;
    for (int i = threadIdx.x; i < TC * P; i += kThreads) {
        const int cl = i / P, pu = i % P;
        const int l = cl / N, j = cl % N, q = j * P + pu;
        const int64_t orow = c0 + cl;
        const int64_t rem = p.R - (r0 + 32 * pu);
        if (orow < p.C && rem > 0 &&
            NVFP4_IN_RANGE(orow * (K / 2) + (r0 / 2) + 16 * pu, rem >= 32 ? 16 : 8, p.C * (K / 2))) {
            const uint4 u = s_units[q * 32 + (l ^ (q & 7))];
            uint8_t *dst = p.codes + orow * (K / 2) + (r0 / 2) + 16 * pu;
            if (rem >= 32 && vec16) {
                *reinterpret_cast<uint4 *>(dst) = u;
            } else {  // rows only 8-byte aligned (K % 32 == 16), or the K tail
                *reinterpret_cast<uint2 *>(dst) = make_uint2(u.x, u.y);
                if (rem >= 32) *reinterpret_cast<uint2 *>(dst + 8) = make_uint2(u.z, u.w);
            }
        }
    }
    if (DUAL) {  // rowwise scale atoms of the tile: ARR x ACR
        const int64_t rowtiles_r = (p.R + 127) / 128, kb4_r = (p.C + 63) / 64;
        for (int i = threadIdx.x; i < ARR * ACR * 32; i += kThreads) {
            const int atom = i >> 5, ar = atom / ACR, ac = atom % ACR;
            const int64_t grow = by * ARR + ar, gcol = bx * ACR + ac;
            if (grow < rowtiles_r && gcol < kb4_r &&
                NVFP4_IN_RANGE((grow * kb4_r + gcol) * 512 + (i & 31) * 16, 16, nv_scales_extent(p.R, p.C))) {
                uint8_t *dst = p.row_scales + (grow * kb4_r + gcol) * 512 + (i & 31) * 16;
                *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(s_scr + i * 16);
            }
        }
    }
    // scales: AR x AC atoms; each atom row's AC atoms are contiguous in memory
    const int64_t rowtiles = (p.C + 127) / 128;
    for (int i = threadIdx.x; i < AR * AC * 32; i += kThreads) {
        const int atom = i >> 5, ar = atom / AC, ac = atom % AC;
        const int64_t grow = bx * AR + ar, gcol = by * AC + ac;
        if (grow < rowtiles && gcol < KB4 &&
            NVFP4_IN_RANGE((grow * KB4 + gcol) * 512 + (i & 31) * 16, 16, nv_scales_extent(p.C, p.R))) {
            uint8_t *dst = p.scales + (grow * KB4 + gcol) * 512 + (i & 31) * 16;
            *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(s_sc + i * 16);
        }
    }
}

// ---------------------------------------------------------------------------
// Pass 2, colwise, bf16 input fed by TMA.  Each warp works alone on tasks of
// 64 input rows x 128 columns (four 16-row groups; lane l owns columns 4l ..
// 4l+3): 128 output rows x 64 k, i.e. 32 code bytes per output row and exactly
// one 512-byte scale atom.  Lane 0 keeps the next 16-row group in flight with a
// 2-D TMA load (box 128 columns x 16 rows; rows and columns outside the tensor
// arrive as zeros) into the warp's two-stage ring while the warp encodes the
// current group from shared memory, so the loads never wait on the encode.
// Each block is encoded exactly as in quantize_colwise_kernel (same steps, same
// order).  Persistent: the CTA's set-up (tensor scale, element-scale tables,
// Philox keys) happens once, and tasks run in reverse order (the tail of the
// amax sweep is still in L2).  Every wait is bounded; on expiry the warp
// records NVFP4_ERR_DEVICE_TIMEOUT, waits briefly for its loads in flight and
// stops.
// ---------------------------------------------------------------------------
constexpr int kTmaWarps = 4;                        // warps per CTA
constexpr int kTmaCols = 128;                       // columns per task
constexpr int kTmaStageBytes = 16 * kTmaCols * 2;   // one 16-row group: 4 KB
constexpr int kTmaStgBytes = 4 * 4 * 32 * 8;        // a task's codes, [group][column j][lane] x 8 bytes
// Ring depth (groups in flight per warp) and CTAs per SM, measured per mode: round-to-nearest
// is best with 16 warps per SM and two stages (h 8192x20480 with the RHT: 89 us against 93 with
// three stages at 12 warps); stochastic rounding, bound by integer issue, with three stages at
// 12 warps and up to 170 registers (dY 8192x20480: 191.5 us against 200.6).
template <bool SR> __host__ __device__ constexpr int tma_stages() { return SR ? 3 : 2; }
template <bool SR> __host__ __device__ constexpr int tma_ctas() { return SR ? 3 : 4; }
template <bool SR> __host__ __device__ constexpr int tma_warp_bytes() {  // ring, codes, scale atom
    return tma_stages<SR>() * kTmaStageBytes + kTmaStgBytes + 512;
}
template <bool SR> __host__ __device__ constexpr int tma_smem_bytes() {  // + alignment slack
    return kTmaWarps * tma_warp_bytes<SR>() + 128;
}
constexpr uint64_t kTmaWaitNs = 2000000000ull, kTmaDrainNs = 20000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void *ptr) { return (uint32_t)__cvta_generic_to_shared(ptr); }
__device__ __forceinline__ bool q_mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __noinline__ bool q_mbar_wait_slow(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (q_mbar_try(bar, parity)) return true;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > limit_ns) return false;
    }
}
// Warp-uniform bounded wait: false on every lane if any lane gave up.
__device__ __forceinline__ bool q_mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const bool ok = q_mbar_try(bar, parity) || q_mbar_wait_slow(bar, parity, limit_ns);
    return __all_sync(0xFFFFFFFFu, ok);
}
// One 16-row group (box 128 x 16 bf16 = 4 KB) into a ring stage, completing on `bar`.
__device__ __forceinline__ void q_tma_group(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kTmaStageBytes) : "memory");
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

template <bool SR, bool RHT>
__global__ void __launch_bounds__(32 * kTmaWarps, tma_ctas<SR>())
    quantize_colwise_tma_kernel(const __grid_constant__ CUtensorMap map_x, const QParams p) {
    constexpr int kTmaStages = tma_stages<SR>();
    constexpr int kTmaWarpBytes = tma_warp_bytes<SR>();
    extern __shared__ uint8_t q_smem_raw[];
    uint8_t *q_smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(q_smem_raw) + 127) & ~uintptr_t(127));
    __shared__ float s_red[kTmaWarps];
    __shared__ float s_inv[128], s_inv4[RHT ? 128 : 1];
    __shared__ __align__(8) uint64_t s_bar[kTmaStages * kTmaWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *wsm = q_smem + warp * kTmaWarpBytes;
    const uint32_t ring = smem_addr(wsm);
    uint2 *stg = reinterpret_cast<uint2 *>(wsm + kTmaStages * kTmaStageBytes);
    uint8_t *atom = wsm + kTmaStages * kTmaStageBytes + kTmaStgBytes;
    const uint32_t bar = smem_addr(&s_bar[kTmaStages * warp]);
    if (lane == 0) {
        for (int i = 0; i < kTmaStages; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar + 8 * i) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const float s_t = tensor_scale_from_amax(tensor_amax(p, s_red));  // synchronises the CTA
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.tensor_scale = s_t;
    const ScaleCtx ctx = scale_ctx(s_t);
    scale_table_init(s_inv, RHT ? s_inv4 : nullptr, s_t);
    const uint32_t signs = RHT ? rht_sign_bits(p.seed) : 0u;
    const bool fold = RHT && !SR && ctx.fast;  // quarter folded into the element scale (RTN only)
    PhiloxKeys keys;
    if (SR) keys = philox_keys(p.seed);
    __syncthreads();

    const int64_t K = p.R, KB4 = (K + 63) / 64;
    const int64_t strips = (p.C + kTmaCols - 1) / kTmaCols, bands = (p.R + 63) / 64;
    const int64_t ntasks = strips * bands;
    const int64_t gw = (int64_t)blockIdx.x * kTmaWarps + warp, nw = (int64_t)gridDim.x * kTmaWarps;
    const int64_t ngroups = gw < ntasks ? 4 * ((ntasks - 1 - gw) / nw + 1) : 0;
    const bool vec16 = (K % 32) == 0;
    // group q of this warp: task ntasks - 1 - gw - (q / 4) nw (band-major over strips), 16-row group q % 4
    auto issue = [&](int64_t q) {
        const int64_t t = ntasks - 1 - gw - (q >> 2) * nw;
        const int64_t band = t / strips, strip = t - band * strips;
        const uint32_t st = (uint32_t)(q % kTmaStages);
        q_tma_group(ring + st * kTmaStageBytes, &map_x, bar + 8 * st, (int)(strip * kTmaCols),
                    (int)(band * 64 + (q & 3) * 16));
    };
    if (lane == 0)
        for (int64_t i = 0; i < kTmaStages && i < ngroups; ++i) issue(i);
    int64_t q = 0;
    for (; q < ngroups; ++q) {
        const int64_t t = ntasks - 1 - gw - (q >> 2) * nw;
        const int64_t band = t / strips, strip = t - band * strips;
        const int g = (int)(q & 3);
        const uint32_t stage = (uint32_t)(q % kTmaStages);
        if (!q_mbar_wait(bar + 8 * stage, (uint32_t)((q / kTmaStages) & 1), kTmaWaitNs)) break;
        uint2 raw[16];
        const uint32_t src = ring + stage * kTmaStageBytes + (uint32_t)lane * 8u;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(raw[i].x), "=r"(raw[i].y) : "r"(src + 256u * i));
        // every lane's reads of the stage ordered before the async-proxy refill
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && q + kTmaStages < ngroups) issue(q + kTmaStages);
        if (RHT) {  // the sign diagonal, on the packed rows
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                raw[i].x ^= sign_mask<uint16_t>(signs, i);
                raw[i].y ^= sign_mask<uint16_t>(signs, i);
            }
        }
        const int64_t c = strip * kTmaCols + lane * 4;
        const int64_t rg = band * 64 + g * 16;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t w = (j >> 1) ? raw[i].y : raw[i].x;
                v[i] = (j & 1) ? bf16hi(w) : bf16lo(w);
            }
            float scale_in;
            uint32_t sb;
            uint64_t pv[8];
            float m = 0.0f;
            if (RHT) {
                fwht16_x2(v, pv);
#pragma unroll
                for (int k = 0; k < 8; ++k) m = fmaxf(m, fmaxf(fabsf(f2lo(pv[k])), fabsf(f2hi(pv[k]))));
                sb = block_scale_code(__fmul_rn(m, 0.25f), ctx);  // max |z/4| = RN(max|z| / 4)
                if (fold) {
                    scale_in = s_inv4[sb];
                } else {
                    const uint64_t quarter = f2(0.25f, 0.25f);
#pragma unroll
                    for (int k = 0; k < 8; ++k) pv[k] = mul2_rn(pv[k], quarter);
                    scale_in = s_inv[sb];
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    pv[k] = f2(v[2 * k], v[2 * k + 1]);
                    m = fmaxf(m, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
                }
                sb = block_scale_code(m, ctx);
                scale_in = s_inv[sb];
            }
            uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
            if (SR) sr_words16((uint64_t)(c + j) * (uint64_t)K + (uint64_t)rg, keys, w0, w1);  // rg % 16 == 0
            stg[(g * 4 + j) * 32 + lane] = encode16_x2<SR>(pv, scale_in, w0, w1);
            const int orow = lane * 4 + j;  // output row within the strip
            atom[(orow & 31) * 16 + ((orow >> 5) & 3) * 4 + g] = (uint8_t)sb;
        }
        if (g == 3) {  // the task is complete: its 128 code rows and its scale atom
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t orow = c + j;
                const int64_t room = K / 2 - band * 32;  // this band's code bytes in a row: 8, 16, 24 or 32
                if (orow < p.C && NVFP4_IN_RANGE(orow * (K / 2) + band * 32, room < 32 ? room : 32, p.C * (K / 2))) {
                    uint8_t *dst = p.codes + orow * (K / 2) + band * 32;
                    const uint2 a0 = stg[(0 * 4 + j) * 32 + lane], a1 = stg[(1 * 4 + j) * 32 + lane];
                    const uint2 a2 = stg[(2 * 4 + j) * 32 + lane], a3 = stg[(3 * 4 + j) * 32 + lane];
                    if (room >= 32 && vec16) {
                        *reinterpret_cast<uint4 *>(dst) = make_uint4(a0.x, a0.y, a1.x, a1.y);
                        *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(a2.x, a2.y, a3.x, a3.y);
                    } else {  // rows only 8-byte aligned (K % 32 == 16), or the last band
                        *reinterpret_cast<uint2 *>(dst) = a0;
                        if (room >= 16) *reinterpret_cast<uint2 *>(dst + 8) = a1;
                        if (room >= 24) *reinterpret_cast<uint2 *>(dst + 16) = a2;
                        if (room >= 32) *reinterpret_cast<uint2 *>(dst + 24) = a3;
                    }
                }
            }
            if (NVFP4_IN_RANGE((strip * KB4 + band) * 512 + lane * 16, 16, nv_scales_extent(p.C, K)))
                *reinterpret_cast<uint4 *>(p.scales + (strip * KB4 + band) * 512 + lane * 16) =
                    *reinterpret_cast<const uint4 *>(atom + lane * 16);
            __syncwarp();
        }
    }
    if (q < ngroups) {  // a load did not arrive in time: report, then let the loads in flight land
        if (lane == 0 && p.status) atomicExch(p.status, 7);  // NVFP4_ERR_DEVICE_TIMEOUT
        for (int64_t r = q; r < q + kTmaStages && r < ngroups; ++r)
            q_mbar_wait(bar + 8 * (uint32_t)(r % kTmaStages), (uint32_t)((r / kTmaStages) & 1), kTmaDrainNs);
    }
}

// ---------------------------------------------------------------------------
// MXFP4, rowwise, one pass (no tensor scale): blocks of 32 along the columns,
// E8M0 scale 2^X with X = floor(log2 amax_b) - 2 clamped to [-127, 127], each
// element E2M1(v * 2^-X) by round-to-nearest-even.  As in the NVFP4 rowwise
// pass, each lane owns one whole block of a row (64 bytes of bf16, 128 of f32),
// so the block amax, the E8M0 code and the 32 codes (one 16-byte store) need
// no shuffles; a warp covers 1024 columns of RPW rows per tile, persistent CTAs
// walk the tiles in reverse order with the next tile's loads in flight.  Scales
// use the 128x4 atom order with four 32-blocks per atom word, a word held by
// four neighbouring lanes: two shuffles gather it and one lane stores it.
// Padding rows (to the atoms' 128-row extent) and padding blocks (to their
// 4-block width) load zeros and get code 0.
// ---------------------------------------------------------------------------
struct MxParams {
    const void *x;
    int64_t R, C, ld;
    uint8_t *codes;
    uint8_t *scales;
    int aligned32;  // x and every row start 32-byte aligned (256-bit loads allowed)
};

// E8M0 code of a block amax (finite, >= 0): the biased exponent field minus 2
// is floor(log2 amax) - 2 + 127; fields 0..2 (zero, subnormal, tiny) clamp to 0.
__device__ __forceinline__ uint32_t mx_code(float amax) {
    const uint32_t ef = __float_as_uint(amax) >> 23;
    return ef >= 2u ? ef - 2u : 0u;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) quantize_rowwise_mx_kernel(const MxParams p) {
    constexpr int LW = 8 * (int)sizeof(T);          // 32-bit words per lane and row: 16 (bf16), 32 (f32)
    constexpr int RPW = sizeof(T) == 2 ? 2 : 1;     // rows per warp per tile
    constexpr int TILE_R = RPW * (kThreads / 32);
    constexpr int TILE_B = 32;                      // blocks (of 32 columns) per tile row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *xb = static_cast<const uint8_t *>(p.x);
    const int64_t K = p.C, KB = K / 32, KB4 = (K + 127) / 128;
    const int64_t tiles_c = (KB + TILE_B - 1) / TILE_B;
    const int64_t tiles_r = ((p.R + 127) / 128) * (128 / TILE_R);
    const int64_t ntiles = tiles_c * tiles_r;
    const bool a32 = p.aligned32 != 0;

    auto load = [&](int64_t t, uint32_t(&buf)[RPW][LW]) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t b = tc * TILE_B + lane;
        const int64_t r0 = tr * TILE_R + warp * RPW;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int64_t r = r0 + i;
            if (b < KB && r < p.R && NVFP4_IN_RANGE(r * p.ld + b * 32, 32, x_extent(p.R, p.C, p.ld))) {
                load_block<LW>(xb + (r * p.ld + b * 32) * (int64_t)sizeof(T), a32, buf[i]);
            } else {
#pragma unroll
                for (int j = 0; j < LW; ++j) buf[i][j] = 0u;
            }
        }
    };

    int64_t t = ntiles - 1 - (int64_t)blockIdx.x;
    uint32_t cur[RPW][LW], nxt[RPW][LW];
    if (t >= 0) load(t, cur);
    for (; t >= 0; t -= gridDim.x) {
        const int64_t tn = t - gridDim.x;
        if (tn >= 0) load(tn, nxt);
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t b = tc * TILE_B + lane, atom = b >> 2;
        const bool col_ok = b < KB;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int64_t r = tr * TILE_R + warp * RPW + i;
            float v[32];
            float(&v0)[16] = *reinterpret_cast<float(*)[16]>(v);
            float(&v1)[16] = *reinterpret_cast<float(*)[16]>(v + 16);
            unpack16<T>(cur[i], v0);
            unpack16<T>(cur[i] + LW / 2, v1);
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
            const uint32_t code = mx_code(m);
            const float inv = __uint_as_float((254u - code) << 23);  // 2^-X
            float q[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) q[j] = __fmul_rn(v[j], inv);
            if (col_ok && r < p.R && NVFP4_IN_RANGE(r * (K / 2) + b * 16, 16, p.R * (K / 2)))
                *reinterpret_cast<uint4 *>(p.codes + r * (K / 2) + b * 16) =
                    make_uint4(e2m1x8(q), e2m1x8(q + 8), e2m1x8(q + 16), e2m1x8(q + 24));
            uint32_t word = code << (8 * (lane & 3));
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
            if ((lane & 3) == 0 && atom < KB4 &&
                NVFP4_IN_RANGE(((r >> 7) * KB4 + atom) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4, 4,
                               mx_scales_extent(p.R, p.C)))
                *reinterpret_cast<uint32_t *>(p.scales + ((r >> 7) * KB4 + atom) * 512 + (r & 31) * 16 +
                                              ((r >> 5) & 3) * 4) = word;
        }
#pragma unroll
        for (int i = 0; i < RPW; ++i)
#pragma unroll
            for (int j = 0; j < LW; ++j) cur[i][j] = nxt[i][j];
    }
}

// ---------------------------------------------------------------------------
// MXFP4, colwise (blocks of 32 down the rows; output transposed, [C x R]):
// each thread holds one 32-row block of 8 / sizeof(T) adjacent columns (one
// 8-byte load per row), so a column's block is in one thread: amax, E8M0 code
// and the 32 codes (16 bytes, one store into the output row of that column)
// need no shuffles.  The grid spans the scale atoms' padded extent (columns to
// a multiple of 128, rows to a multiple of 128), and threads outside the
// tensor write the zero padding scales.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) quantize_colwise_mx_kernel(const MxParams p) {
    constexpr int CPT = 8 / (int)sizeof(T);  // columns per thread
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t c0 = ((int64_t)blockIdx.x * 32 + lane) * CPT;
    const int64_t r0 = ((int64_t)blockIdx.y * (kThreads / 32) + warp) * 32;
    const int64_t K = p.R;                     // output k (contiguous) = input rows
    const int64_t KB4 = (K + 127) / 128;       // scale atoms per 128-row tile of the output
    const int64_t out_rows_pad = ((p.C + 127) / 128) * 128;
    if (r0 >= KB4 * 128 || c0 >= out_rows_pad) return;
    const bool rows_ok = r0 < p.R;             // R % 32 == 0: a block is all in or all out
    const T *x = static_cast<const T *>(p.x);
    uint2 raw[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
        raw[i] = (rows_ok && c0 < p.C && NVFP4_IN_RANGE((r0 + i) * p.ld + c0, CPT, x_extent(p.R, p.C, p.ld))) ? __ldg(reinterpret_cast<const uint2 *>(x + (r0 + i) * p.ld + c0))
                                       : make_uint2(0u, 0u);
    const int64_t b = r0 / 32;                 // 32-block index along k
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int64_t c = c0 + j;              // output row
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (sizeof(T) == 2) {
                const uint32_t w = (j >> 1) ? raw[i].y : raw[i].x;
                v[i] = (j & 1) ? bf16hi(w) : bf16lo(w);
            } else {
                v[i] = __uint_as_float(j ? raw[i].y : raw[i].x);
            }
        }
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
        const uint32_t code = mx_code(m);      // 0 for padding (all-zero) blocks
        const float inv = __uint_as_float((254u - code) << 23);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], inv);
        if (rows_ok && c < p.C && NVFP4_IN_RANGE(c * (K / 2) + r0 / 2, 16, p.C * (K / 2))) {
            const uint4 u = make_uint4(e2m1x8(v), e2m1x8(v + 8), e2m1x8(v + 16), e2m1x8(v + 24));
            *reinterpret_cast<uint4 *>(p.codes + c * (K / 2) + r0 / 2) = u;
        }
        if (NVFP4_IN_RANGE(((c >> 7) * KB4 + (b >> 2)) * 512 + (c & 31) * 16 + ((c >> 5) & 3) * 4 + (b & 3), 1,
                           mx_scales_extent(p.C, K)))
            p.scales[((c >> 7) * KB4 + (b >> 2)) * 512 + (c & 31) * 16 + ((c >> 5) & 3) * 4 + (b & 3)] = (uint8_t)code;
    }
}

// Empty tensor: only the tensor scale is defined.
__global__ void tensor_scale_only_kernel(const float *amax_in, float *tensor_scale) {
    *tensor_scale = tensor_scale_from_amax(amax_in ? *amax_in : 0.0f);
}

// The driver's tensor-map encoder (looked up once).
PFN_cuTensorMapEncodeTiled_v12000 q_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// bf16 input [R x C] (leading dimension ld) as 16-row x 128-column boxes; outside
// the tensor a box reads zeros.
bool make_colwise_map(CUtensorMap *map, const void *x, int64_t R, int64_t C, int64_t ld) {
    auto fn = q_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)R};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)kTmaCols, 16u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(x), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SR, bool RHT>
cudaError_t launch_colwise_tma(const QParams &p, cudaStream_t s) {
    CUtensorMap map;
    if (!make_colwise_map(&map, p.x, p.R, p.C, p.ld)) return cudaErrorInvalidValue;
    constexpr int kMaxDev = 64;
    static bool attr_set[kMaxDev] = {};  // per instantiation and device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(quantize_colwise_tma_kernel<SR, RHT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tma_smem_bytes<SR>());
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int64_t ntasks = ((p.C + kTmaCols - 1) / kTmaCols) * ((p.R + 63) / 64);
    const unsigned grid =
        (unsigned)std::min<int64_t>((ntasks + kTmaWarps - 1) / kTmaWarps, tma_ctas<SR>() * (int64_t)num_sms());
    quantize_colwise_tma_kernel<SR, RHT><<<grid, 32 * kTmaWarps, tma_smem_bytes<SR>(), s>>>(map, p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t run(const QuantizeArgs &a, cudaStream_t s, int *launches) {
    const T *x = static_cast<const T *>(a.x);
    int num_partials = 0;
    if (!a.amax_in) {
        const int sms = num_sms();
        if (a.rht) {
            const int64_t units = (a.R / 16) * (a.C / Vec<T>::N);
            num_partials = (int)std::min<int64_t>(std::min<int64_t>(4 * sms, kMaxPartials),
                                                  std::max<int64_t>(1, (units + kThreads - 1) / kThreads));
            amax_rht_kernel<T><<<num_partials, kThreads, 0, s>>>(x, a.R, a.C, a.ld, a.seed, a.partials);
        } else {
            const int64_t chunks = a.R * (a.C / Vec<T>::N);
            num_partials = (int)std::min<int64_t>(std::min<int64_t>(4 * sms, kMaxPartials),
                                                  std::max<int64_t>(1, (chunks + kThreads - 1) / kThreads));
            amax_kernel<T><<<num_partials, kThreads, 0, s>>>(x, a.R, a.C, a.ld, a.partials);
        }
        ++*launches;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    QParams p{a.x, a.R, a.C, a.ld, a.seed, a.amax_in, a.partials, num_partials, a.codes, a.scales,
              a.tensor_scale};
    p.aligned32 = (reinterpret_cast<uintptr_t>(a.x) % 32 == 0) && ((a.ld * (int64_t)sizeof(T)) % 32 == 0);
    p.status = a.status;
    constexpr int N = Vec<T>::N;  // columns per lane of the colwise kernels
    if (!a.colwise) {
        constexpr int tile_r = sizeof(T) == 2 ? 32 : 16;  // rows per tile of quantize_rowwise_kernel
        const int64_t tiles = ((a.C / 16 + 31) / 32) * ((a.R + 127) / 128) * (128 / tile_r);
        const unsigned grid = (unsigned)std::min<int64_t>(tiles, 2 * (int64_t)num_sms());
        if (a.sr) quantize_rowwise_kernel<T, true><<<grid, kThreads, 0, s>>>(p);
        else quantize_rowwise_kernel<T, false><<<grid, kThreads, 0, s>>>(p);
    } else if constexpr (sizeof(T) == 2) {  // bf16: the TMA-fed colwise kernel
        cudaError_t e;
        if (a.sr && a.rht) e = launch_colwise_tma<true, true>(p, s);
        else if (a.sr) e = launch_colwise_tma<true, false>(p, s);
        else if (a.rht) e = launch_colwise_tma<false, true>(p, s);
        else e = launch_colwise_tma<false, false>(p, s);
        if (e != cudaSuccess) return e;
    } else {  // f32 input: the register-fed colwise kernel
        dim3 grid((unsigned)((a.C + 32 * N - 1) / (32 * N)), (unsigned)((a.R + 255) / 256));
        if (a.sr && a.rht) quantize_colwise_kernel<T, true, true, false><<<grid, kThreads, 0, s>>>(p);
        else if (a.sr) quantize_colwise_kernel<T, true, false, false><<<grid, kThreads, 0, s>>>(p);
        else if (a.rht) quantize_colwise_kernel<T, false, true, false><<<grid, kThreads, 0, s>>>(p);
        else quantize_colwise_kernel<T, false, false, false><<<grid, kThreads, 0, s>>>(p);
    }
    ++*launches;
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_dual(const DualQuantizeArgs &a, cudaStream_t s, int *launches) {
    const T *x = static_cast<const T *>(a.x);
    constexpr int N = Vec<T>::N;
    int num_partials = 0;
    const float *col_partials = a.col_rht ? a.col_partials : a.row_partials;  // no RHT: one amax serves both
    if (!(a.amax_row_in && a.amax_col_in)) {
        const int sms = num_sms();
        if (a.col_rht) {
            const int64_t units = (a.R / 16) * (a.C / N);
            num_partials = (int)std::min<int64_t>(std::min<int64_t>(4 * sms, kMaxPartials),
                                                  std::max<int64_t>(1, (units + kThreads - 1) / kThreads));
            amax_dual_kernel<T><<<num_partials, kThreads, 0, s>>>(x, a.R, a.C, a.ld, a.seed, a.row_partials,
                                                                  a.col_partials);
        } else {
            const int64_t chunks = a.R * (a.C / N);
            num_partials = (int)std::min<int64_t>(std::min<int64_t>(4 * sms, kMaxPartials),
                                                  std::max<int64_t>(1, (chunks + kThreads - 1) / kThreads));
            amax_kernel<T><<<num_partials, kThreads, 0, s>>>(x, a.R, a.C, a.ld, a.row_partials);
        }
        ++*launches;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    QParams p{a.x, a.R, a.C, a.ld, a.seed, a.amax_col_in, col_partials, num_partials, a.col_codes, a.col_scales,
              a.col_tensor_scale, a.amax_row_in, a.row_partials, a.row_codes, a.row_scales, a.row_tensor_scale};
    dim3 grid((unsigned)((a.C + 32 * N - 1) / (32 * N)), (unsigned)((a.R + 255) / 256));
    if (a.col_sr && a.col_rht) quantize_colwise_kernel<T, true, true, true><<<grid, kThreads, 0, s>>>(p);
    else if (a.col_sr) quantize_colwise_kernel<T, true, false, true><<<grid, kThreads, 0, s>>>(p);
    else if (a.col_rht) quantize_colwise_kernel<T, false, true, true><<<grid, kThreads, 0, s>>>(p);
    else quantize_colwise_kernel<T, false, false, true><<<grid, kThreads, 0, s>>>(p);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace

namespace {
template <typename T>
cudaError_t run_amax(const T *x, int64_t R, int64_t C, int64_t ld, bool rht, uint64_t seed, float *partials,
                     float *amax_out, cudaStream_t s, int *launches) {
    const int sms = num_sms();
    int n;
    if (rht) {
        const int64_t units = (R / 16) * (C / Vec<T>::N);
        n = (int)std::min<int64_t>(std::min<int64_t>(4 * sms, kMaxPartials),
                                   std::max<int64_t>(1, (units + kThreads - 1) / kThreads));
        amax_rht_kernel<T><<<n, kThreads, 0, s>>>(x, R, C, ld, seed, partials);
    } else {
        const int64_t chunks = R * (C / Vec<T>::N);
        n = (int)std::min<int64_t>(std::min<int64_t>(4 * sms, kMaxPartials),
                                   std::max<int64_t>(1, (chunks + kThreads - 1) / kThreads));
        amax_kernel<T><<<n, kThreads, 0, s>>>(x, R, C, ld, partials);
    }
    ++*launches;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_amax_reduce(partials, n, amax_out, s, launches);
}
}  // namespace

namespace {
template <typename T>
cudaError_t run_amax_dual(const T *x, int64_t R, int64_t C, int64_t ld, uint64_t seed, float *partials,
                          float *amax_out, float *amax_rht_out, cudaStream_t s, int *launches) {
    const int64_t units = (R / 16) * (C / Vec<T>::N);
    const int n = (int)std::min<int64_t>(std::min<int64_t>(4 * num_sms(), kMaxPartials),
                                         std::max<int64_t>(1, (units + kThreads - 1) / kThreads));
    amax_dual_kernel<T><<<n, kThreads, 0, s>>>(x, R, C, ld, seed, partials, partials + kMaxPartials);
    ++*launches;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_amax_reduce2(partials, n, amax_out, amax_rht_out, s, launches);
}
}  // namespace

cudaError_t launch_amax_dual(const void *x, bool bf16, int64_t R, int64_t C, int64_t ld, uint64_t seed,
                             float *partials, float *amax_out, float *amax_rht_out, cudaStream_t s, int *launches) {
    if (R == 0 || C == 0) {
        cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), s);
        return e != cudaSuccess ? e : cudaMemsetAsync(amax_rht_out, 0, sizeof(float), s);
    }
    return bf16 ? run_amax_dual(static_cast<const uint16_t *>(x), R, C, ld, seed, partials, amax_out, amax_rht_out,
                                s, launches)
                : run_amax_dual(static_cast<const float *>(x), R, C, ld, seed, partials, amax_out, amax_rht_out, s,
                                launches);
}

cudaError_t launch_amax(const void *x, bool bf16, int64_t R, int64_t C, int64_t ld, bool rht, uint64_t seed,
                        float *partials, float *amax_out, cudaStream_t s, int *launches) {
    if (R == 0 || C == 0) return cudaMemsetAsync(amax_out, 0, sizeof(float), s);
    return bf16 ? run_amax(static_cast<const uint16_t *>(x), R, C, ld, rht, seed, partials, amax_out, s, launches)
                : run_amax(static_cast<const float *>(x), R, C, ld, rht, seed, partials, amax_out, s, launches);
}

cudaError_t launch_quantize_dual(const DualQuantizeArgs &a, cudaStream_t s, int *launches) {
    if (a.R == 0 || a.C == 0) {
        tensor_scale_only_kernel<<<1, 1, 0, s>>>(a.amax_row_in, a.row_tensor_scale);
        tensor_scale_only_kernel<<<1, 1, 0, s>>>(a.amax_col_in, a.col_tensor_scale);
        *launches += 2;
        return cudaGetLastError();
    }
    return a.bf16 ? run_dual<uint16_t>(a, s, launches) : run_dual<float>(a, s, launches);
}

cudaError_t launch_quantize_mx(const void *x, bool bf16, int64_t R, int64_t C, int64_t ld, bool colwise,
                               uint8_t *codes, uint8_t *scales, cudaStream_t s, int *launches) {
    if (R == 0 || C == 0) return cudaSuccess;
    MxParams p{x, R, C, ld, codes, scales, 0};
    const size_t es = bf16 ? 2 : 4;
    p.aligned32 = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && ((ld * (int64_t)es) % 32 == 0);
    if (colwise) {
        const int cpt = bf16 ? 4 : 2;
        const int64_t cols_pad = ((C + 127) / 128) * 128, rows_pad = ((R + 127) / 128) * 128;
        dim3 grid((unsigned)((cols_pad + 32 * cpt - 1) / (32 * cpt)), (unsigned)((rows_pad + 255) / 256));
        if (bf16) quantize_colwise_mx_kernel<uint16_t><<<grid, kThreads, 0, s>>>(p);
        else quantize_colwise_mx_kernel<float><<<grid, kThreads, 0, s>>>(p);
        ++*launches;
        return cudaGetLastError();
    }
    const int64_t tile_r = bf16 ? 16 : 8;  // rows per tile of quantize_rowwise_mx_kernel
    const int64_t tiles = ((C / 32 + 31) / 32) * ((R + 127) / 128) * (128 / tile_r);
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, 2 * (int64_t)num_sms());
    if (bf16) quantize_rowwise_mx_kernel<uint16_t><<<grid, kThreads, 0, s>>>(p);
    else quantize_rowwise_mx_kernel<float><<<grid, kThreads, 0, s>>>(p);
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s, int *launches) {
    if (a.R == 0 || a.C == 0) {
        tensor_scale_only_kernel<<<1, 1, 0, s>>>(a.amax_in, a.tensor_scale);
        ++*launches;
        return cudaGetLastError();
    }
    return a.bf16 ? run<uint16_t>(a, s, launches) : run<float>(a, s, launches);
}

NVFP4_DEFINE_BOUNDS_READER(read_bounds_quantize)

}  // namespace nvfp4
