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

// The same generator with its ten round keys computed once (the key schedule
// depends only on the seed), and each 32x32 -> 64-bit product taken whole.
struct PhiloxKeys {
    uint32_t k0[10], k1[10];
};
__device__ __forceinline__ PhiloxKeys philox_keys(uint64_t seed) {
    PhiloxKeys k;
    uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        k.k0[round] = a;
        k.k1[round] = b;
        a += 0x9E3779B9u;
        b += 0xBB67AE85u;
    }
    return k;
}
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys &k) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x, p1 = (uint64_t)0xCD9E8D57u * c.z;
        c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k.k0[round], (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k.k1[round],
                       (uint32_t)p0);
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {  // round to nearest even
    uint32_t w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(hi), "f"(lo));
    return w;
}

// Squared ReLU of the MLP block and its derivative on bf16 pairs: one binary32
// operation each, then bf16 round-to-nearest-even; relu(y) = +0 for y <= 0.
//   h = relu(y) * relu(y)        dy = dh * (2 * relu(y))
__device__ __forceinline__ float relu(float y) { return y > 0.0f ? y : 0.0f; }
__device__ __forceinline__ uint32_t relu2_pair(uint32_t y) {
    const float a = relu(bf16lo(y)), b = relu(bf16hi(y));
    return pack_bf16x2(__fmul_rn(a, a), __fmul_rn(b, b));
}
__device__ __forceinline__ uint32_t drelu2_pair(uint32_t dh, uint32_t y) {
    const float ga = __fmul_rn(2.0f, relu(bf16lo(y))), gb = __fmul_rn(2.0f, relu(bf16hi(y)));
    return pack_bf16x2(__fmul_rn(bf16lo(dh), ga), __fmul_rn(bf16hi(dh), gb));
}
__device__ __forceinline__ float absmax_pair(float m, uint32_t w) {
    return fmaxf(m, fmaxf(fabsf(bf16lo(w)), fabsf(bf16hi(w))));
}

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
// (exact).  Magnitudes are first clamped to 7: everything from 6 up lands on 6
// or 8, which the saturating E2M1 conversion turns into 6.
// The constant is (2^16 - 1 - rnd16) * 2^6 + 63 = 2^22 - 1 - 64 rnd16, applied as
// an integer multiply-add.  The "+1 below 1" offset is sat(2^24 - 2^24 a): for a
// < 1 (a <= 1 - 2^-24) the exact value 2^24 (1 - a) is at least 1, for a >= 1 it
// is at most 0, so one saturating FMA gives exactly 1 or 0.
// Returns the E2M1 value (or 8 for 6), sign of r kept, for e2m1x*.
__device__ __forceinline__ float sr_below_one(float a) {  // 1.0f if a < 1, else 0.0f (a finite, >= 0)
    return __saturatef(__fmaf_rn(-a, 16777216.0f, 16777216.0f));
}
__device__ __forceinline__ uint32_t sr_round_bits(uint32_t t_bits, uint32_t rnd16) {
    return (t_bits + 0x3FFFFFu + rnd16 * 0xFFFFFFC0u) & 0xFFC00000u;  // + (2^22 - 1 - 64 rnd16), mod 2^32
}
__device__ __forceinline__ float sr_e2m1_value(float r, uint32_t rnd16) {
    const float a = fminf(fabsf(r), 7.0f);
    const float base = sr_below_one(a);
    const float t = __fadd_ru(a, base);
    const float up = __uint_as_float(sr_round_bits(__float_as_uint(t), rnd16));
    return copysignf(__fsub_rn(up, base), r);
}
// the low / high 16-bit draw of a Philox output word
__device__ __forceinline__ uint32_t sr_rnd_lo(uint32_t w) { return w & 0xFFFFu; }
__device__ __forceinline__ uint32_t sr_rnd_hi(uint32_t w) { return w >> 16; }

// ---------------------------------------------------------------------------
// Per-block scale:  sb = E4M3(RN(RN(amax_b / 6) / s_t)),  dec = e4m3(sb) * s_t,
// inv = RN(1 / dec); a block with sb = 0 (or dec = 0, or inv not finite) has
// every code +0.
//
// The two divisions use Markstein's correction step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Develop. 34(1), 1990): with rb = RN(1/b),
// q0 = RN(a * rb), the residual r = a - q0 * b is exact in one FMA and
// RN(q0 + r * rb) is the correctly rounded a / b, provided nothing underflows
// or overflows.  For b = 6 this holds for every finite a >= 2^-125 (checked on
// the CPU against IEEE division for every binary32 value).  For b = s_t it
// holds whenever s_t lies in [2^-80, 2^100] and the quotient in
// [2^-12, 2^10]; outside that window the code is decided anyway: quotients
// below 2^-11 give sb = 0 whether or not they are correctly rounded, and a
// numerator clamped to s_t * 2^10 gives 1024, which saturates to 448 like
// every true quotient above it.  Tensor scales outside [2^-80, 2^100] (a
// uniform condition) take IEEE divisions instead.
// inv only depends on sb, so each CTA tabulates it once (scale_table_init)
// with an IEEE division per code.
// ---------------------------------------------------------------------------
struct ScaleCtx {
    float s_t;     // tensor scale
    float rcp_st;  // RN(1 / s_t)
    float st_hi;   // s_t * 2^10 (numerator clamp)
    bool fast;     // s_t in [2^-80, 2^100]
};

__device__ __forceinline__ ScaleCtx scale_ctx(float s_t) {
    ScaleCtx c;
    c.s_t = s_t;
    c.fast = s_t >= 0x1p-80f && s_t <= 0x1p+100f;
    c.rcp_st = c.fast ? __fdiv_rn(1.0f, s_t) : 0.0f;
    c.st_hi = s_t * 1024.0f;
    return c;
}

__device__ __forceinline__ float div_markstein(float a, float b, float rb) {
    const float q0 = __fmul_rn(a, rb);
    const float r = __fmaf_rn(-q0, b, a);
    return __fmaf_rn(r, rb, q0);
}

// E4M3 code of t >= 0 (values above 448 saturate to 448 = 0x7E).
__device__ __forceinline__ uint32_t e4m3_code(float t) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(t));
    return out & 0xFFu;
}

__device__ __forceinline__ uint32_t block_scale_code(float amax_b, const ScaleCtx &c) {
    float t2;
    if (c.fast) {
        const float t = fminf(div_markstein(amax_b, 6.0f, 0x1.555556p-3f), c.st_hi);  // RN(1/6)
        t2 = div_markstein(t, c.s_t, c.rcp_st);
    } else {
        t2 = __fdiv_rn(__fdiv_rn(amax_b, 6.0f), c.s_t);
    }
    return e4m3_code(t2);
}

// Exact value of an unsigned E4M3 code (0x7F never occurs here).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// inv for every code (0 where the block's codes are all +0), and with `quarter`
// also inv / 4 (exact when the context is fast), for the Hadamard-transformed
// blocks whose 1/4 normalisation is folded into the element scale.  Threads
// 0..127 fill one entry each; the caller synchronises before use.
__device__ __forceinline__ void scale_table_init(float *inv_tab, float *inv4_tab, float s_t) {
    if (threadIdx.x < 128) {
        const uint32_t sb = threadIdx.x;
        const float dec = __fmul_rn(e4m3_value(sb), s_t);
        float inv = __fdiv_rn(1.0f, dec);
        if (sb == 0u || sb == 127u || dec == 0.0f || !isfinite(inv)) inv = 0.0f;
        inv_tab[sb] = inv;
        if (inv4_tab) inv4_tab[sb] = __fmul_rn(inv, 0.25f);
    }
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
// ---------------------------------------------------------------------------
// Packed binary32 pairs: the f32x2 add / sub / mul of sm_100 round each half
// exactly as the scalar operation does, so a pair operation gives the same
// bits as two scalar ones, in one instruction.  Halves live in one 64-bit
// register pair (low half = first element).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ float f2lo(uint64_t d) { return __uint_as_float((uint32_t)d); }
__device__ __forceinline__ float f2hi(uint64_t d) { return __uint_as_float((uint32_t)(d >> 32)); }
__device__ __forceinline__ uint64_t add2_rn(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add2_ru(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rp.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2_rn(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The fixed-order butterfly alone (strides 1, 2, 4, 8), unnormalised: z = H16 v,
// with its outputs as pairs p[k] = (z[2k], z[2k+1]).  Stride 1 runs on scalars
// and writes straight into the pairs; strides 2, 4 and 8 pair element i with
// i + h for both halves at once (pair stride h / 2).  The operations and their
// order are those of the scalar butterfly.
__device__ __forceinline__ void fwht16_x2(const float *v, uint64_t (&p)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) p[k] = f2(__fadd_rn(v[2 * k], v[2 * k + 1]), __fsub_rn(v[2 * k], v[2 * k + 1]));
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k & h) continue;
            const uint64_t a = p[k], b = p[k + h];
            p[k] = add2_rn(a, b);
            p[k + h] = sub2_rn(a, b);
        }
    }
}
// The same butterfly on scalars (for callers that only need max |z|: fewer
// register-pair constraints than the packed form).
__device__ __forceinline__ void fwht16(float *v) {
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
}
__device__ __forceinline__ void rht16(float *v, uint32_t signs) {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((signs >> j) & 1u) << 31));
    fwht16(v);
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
