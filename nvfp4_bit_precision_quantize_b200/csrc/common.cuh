// common.cuh -- device helpers shared by the NVFP4 kernels (sm_100a only).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace nvfp4 {

// ---------------------------------------------------------------------------
// Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw, SC'11):
// ten rounds of (mulhilo, xor with the other counter half and the round key);
// the 2x32-bit key advances by the Weyl constants between rounds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// 16 sign bits of the Hadamard diagonal: word 0 of the block at counter (0,0,1,0).
__device__ __forceinline__ uint32_t rht_sign_bits(uint64_t seed) {
    return philox4x32_10(make_uint4(0u, 0u, 1u, 0u), (uint32_t)seed, (uint32_t)(seed >> 32)).x & 0xFFFFu;
}

// ---------------------------------------------------------------------------
// bf16 / f32 unpacking
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <typename T> struct Vec;  // 16-byte vector of T, unpacked to floats
template <> struct Vec<uint16_t> {  // bf16 bit patterns
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4 &r, float *v) {
        v[0] = bf16lo(r.x); v[1] = bf16hi(r.x); v[2] = bf16lo(r.y); v[3] = bf16hi(r.y);
        v[4] = bf16lo(r.z); v[5] = bf16hi(r.z); v[6] = bf16lo(r.w); v[7] = bf16hi(r.w);
    }
};
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4 &r, float *v) {
        v[0] = __uint_as_float(r.x); v[1] = __uint_as_float(r.y);
        v[2] = __uint_as_float(r.z); v[3] = __uint_as_float(r.w);
    }
};

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// ---------------------------------------------------------------------------
// Format conversions (hardware cvt, round-to-nearest-even, satfinite)
// ---------------------------------------------------------------------------
// E4M3 code of t >= 0 (values above 448 saturate to 448 = 0x7E).
__device__ __forceinline__ uint32_t e4m3_code(float t) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(t));
    return out & 0xFFu;
}

// Exact value of an unsigned E4M3 code (0x7F never occurs here).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// Four E2M1 codes from four floats (element 0 in the lowest nibble) -> 16 bits.
__device__ __forceinline__ uint32_t e2m1x4(float a, float b, float c, float d) {
    uint16_t out;
    asm("{\n\t.reg .b8 lo, hi;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 hi, %4, %3;\n\t"
        "mov.b16 %0, {lo, hi};\n\t}"
        : "=h"(out) : "f"(a), "f"(b), "f"(c), "f"(d));
    return out;
}

// Eight E2M1 codes (element 0 in bits 0-3) -> 32 bits.
__device__ __forceinline__ uint32_t e2m1x8(const float *v) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// Stochastic rounding of r onto the E2M1 grid with a 16-bit draw: the
// magnitude rounds up to the next grid point iff u < frac, u = rnd16 / 2^16,
// frac the position of |r| between its two neighbouring grid points.
// Decided on the binary32 bit pattern.  For |r| >= 1 the grid spacing is the
// weight of the first mantissa bit, so frac * 2^22 is the low 22 mantissa bits
// L, and L > rnd16 * 2^6 exactly when L + (2^22 - 1 - rnd16 * 2^6) carries
// into bit 22; adding that constant and clearing the low 22 bits rounds.
// For |r| < 1 (spacing 0.5) the same step runs on 1 + |r|, which puts the
// 0.5-grid on the first mantissa bit; the sum is rounded UP to binary32, which
// keeps the comparison with the 2^-17-spaced threshold exact (a threshold t on
// the binary32 grid has x > t iff roundup(x) > t), and 1 is subtracted again
// (exact).  Values at or above 6 land on 6 or above and are clamped to 6.
// Returns the exact E2M1 value (sign of r kept), to be encoded by e2m1x*.
__device__ __forceinline__ float sr_e2m1_value(float r, uint32_t rnd16) {
    const float a = fabsf(r);
    const float base = a < 1.0f ? 1.0f : 0.0f;
    const float t = __fadd_ru(a, base);
    const uint32_t carry_in = ((~rnd16 & 0xFFFFu) << 6) | 63u;
    const float up = __uint_as_float((__float_as_uint(t) + carry_in) & 0xFFC00000u);
    const float mag = fminf(__fsub_rn(up, base), 6.0f);
    return copysignf(mag, r);
}

// ---------------------------------------------------------------------------
// Per-block scale computation shared by the quantisers:
//   sb = E4M3(amax_b / 6 / s_t), dec = e4m3(sb) * s_t, inv = 1 / dec.
// ---------------------------------------------------------------------------
struct BlockScale {
    uint32_t sb;
    float inv;
    bool zero;  // every code of the block is +0
};

__device__ __forceinline__ BlockScale block_scale(float amax_b, float s_t) {
    BlockScale s;
    float t = __fdiv_rn(amax_b, 6.0f);
    t = __fdiv_rn(t, s_t);
    s.sb = e4m3_code(t);
    const float dec = __fmul_rn(e4m3_value(s.sb), s_t);
    s.inv = __fdiv_rn(1.0f, dec);
    s.zero = (s.sb == 0u) || (dec == 0.0f) || !isfinite(s.inv);
    return s;
}

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
    float s = __fdiv_rn(amax, 2688.0f);
    if (amax == 0.0f || s == 0.0f) s = 1.0f;
    return s;
}

// Byte offset of (row r, 16-block b) in the scale-atom layout (KB4 = KB / 4 atoms per row-tile).
__device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t b, int64_t KB4) {
    return ((r >> 7) * KB4 + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

// ---------------------------------------------------------------------------
// 16-point random Hadamard transform in registers: sign flips (xor of the sign
// bit), the fixed-order butterfly over strides 1, 2, 4, 8, then a 1/4 scale.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void rht16(float *v, uint32_t signs) {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((signs >> j) & 1u) << 31));
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            const float a = v[i], b = v[i + h];
            v[i] = __fadd_rn(a, b);
            v[i + h] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(v[j], 0.25f);
}

// ---------------------------------------------------------------------------
// Block-wide max of the per-CTA amax partials written by the amax kernels.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float reduce_partials_max(const float *partials, int count, float *smem32) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < count; i += blockDim.x) m = fmaxf(m, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) smem32[warp] = m;
    __syncthreads();
    m = 0.0f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, smem32[i]);
    __syncthreads();
    return m;
}

}  // namespace nvfp4
