/*
 * nvfp4_oracle.c -- plain, slow, scalar CPU oracle for the NVFP4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  The product (the CUDA
 * library and its Python binding) never calls it and shares no code with it.
 *
 * Sources (pages are cited by title and section):
 *   [AIS]  aisight.pl, "Koniec marnowania mocy. NVIDIA udowadnia, ze 4 bity
 *          wystarcza do trenowania gigantow":
 *          section "Architektura NVFP4 kontra ograniczenia mikroskalowania"
 *            -> block of 16 elements, E4M3 block scale, extra FP32 per-tensor
 *               scale;
 *          section "Technologie stabilizujace proces treningowy"
 *            -> random Hadamard transforms on the weight-gradient operands,
 *               stochastic rounding against systematic rounding bias.
 *   [ABW]  aibuzzwire.news, Thinking Machines "End-to-End 4-Bit Training":
 *          section "Warum weniger Bits ein schnelleres Training bedeuten"
 *            -> the rounding-error concept (3.2 on the grid {3,4} -> 3, err 0.2);
 *          section "Unterschiedliche Phasen, unterschiedliche Regeln"
 *            -> backward passes tolerate noise but not bias.
 *   [NVN]  nerdman.de, "Nvidia drueckt KI-Training auf 4 Bit runter",
 *          section "Was konkret passiert ist" -> 4-bit NVFP4 on Blackwell
 *          tensor cores.
 *   Formats: E2M1 (+-{0,.5,1,1.5,2,3,4,6}) and E4M3 ("fn": bias 7, max 448,
 *   no infinities) as in the OCP Microscaling / OCP 8-bit floating point
 *   specifications.  Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel
 *   random numbers: as easy as 1, 2, 3", SC'11.
 *
 * The pages give no formula for the tensor scale, the block scale, the tie
 * rule, the stochastic-rounding bit width, the Philox counter mapping, the
 * Hadamard sign generation or its normalisation.  Each reading taken here is
 * marked "Reading:" at the function that implements it.
 *
 * Arithmetic: every float operation is one IEEE-754 binary32 operation with
 * round-to-nearest-even (compiled with -ffp-contract=off, no fast-math, no
 * flush-to-zero); dequantised values and the GEMM are in binary64.
 *
 * Parity status of each function (what pins it, see tests/test_oracle_*.py):
 *   philox4x32_10     pinned: torch's independent header-only Philox engine
 *   e2m1 / e4m3       pinned: brute-force nearest-value scans; torch fp8 casts
 *   rht16             pinned: H.H^T = 16 I, closed-form columns, orthogonality
 *   quantize          pinned: brute-force block-scale choice, format facts,
 *                     storage ratio, tensor-scale bounds, SR unbiasedness
 *   gemm / dot        pinned: exact small-integer case vs numpy, brute force
 *   relu2             pinned: torch CPU float32 ops and bf16 cast
 *   mx (MXFP4)        pinned: E8M0 values, shared exponent on binade
 *                     boundaries, exact round trip of every E2M1 code at many
 *                     exponents, saturation, the RTN error bound
 *   gemm_mx           pinned: closed form K*e2m1*e2m1*2^(xa+xb), one-hot
 *                     indexing across 32-blocks, exact agreement with the
 *                     NVFP4 gemm on scales both formats represent
 *   Readings (tensor-scale constant 2688, the R8 counter mapping, the sign
 *   word of the Hadamard diagonal, multiply-by-reciprocal) are fixed by this
 *   file, not by the pages: "parity unpinned" for those choices themselves.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al. 2011): ten rounds of a multiply-based S-box  */
/* on a 128-bit counter, with a Weyl-sequence key schedule.                  */
/* ------------------------------------------------------------------------ */
static const uint32_t PHILOX_M0 = 0xD2511F53u;
static const uint32_t PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u; /* golden ratio */
static const uint32_t PHILOX_W1 = 0xBB67AE85u; /* sqrt(3) - 1  */

void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t k[2] = {key_in[0], key_in[1]};
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { /* key bump before every round but the first */
            k[0] += PHILOX_W0;
            k[1] += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * c[0];
        uint64_t p1 = (uint64_t)PHILOX_M1 * c[2];
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c[1] ^ k[0];
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c[3] ^ k[1];
        uint32_t n3 = lo0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    }
    out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

/* ------------------------------------------------------------------------ */
/* Element and scale formats                                                 */
/* ------------------------------------------------------------------------ */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * exponent 0 is subnormal: 0.5 * m. */
double oracle_e2m1_value(unsigned code)
{
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* E4M3 "fn": bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa;
 * exponent 0 is subnormal (m * 2^-9); 0x7F / 0xFF are NaN (returned as NaN). */
double oracle_e4m3_value(unsigned code)
{
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Magnitude code of an exactly representable E2M1 magnitude. */
static unsigned e2m1_code_of(float v)
{
    if (v < 1.0f) return (unsigned)(v / 0.5f);          /* 0 -> 0, 0.5 -> 1 */
    int e = 0;
    float f = frexpf(v, &e);                            /* v = f * 2^e, f in [0.5,1) */
    /* v = 2^(e-1) * (1 + m/2) with biased exponent E = e - 1 + 1 = e */
    unsigned m = (unsigned)((f * 2.0f - 1.0f) * 2.0f);  /* 0 or 1 */
    return ((unsigned)e << 1) | m;
}

/* Round-to-nearest, ties to even, saturating to +-6 (the largest E2M1
 * magnitude).  Rounding works on the grid spacing of the binade of |r|:
 * 0.5 below 2, 1 in [2,4), 2 in [4,6].  A tie goes to the even multiple of
 * the spacing, which is the code whose mantissa bit is 0.  The sign of the
 * result is the sign of r, so a negative value that rounds to zero encodes
 * as -0 (0x8), as an IEEE conversion would.  [ABW "Warum weniger Bits ..."]
 * gives the rounding-error concept; the tie rule is round-to-nearest-even. */
unsigned oracle_e2m1_rtn(float r)
{
    unsigned sign = signbit(r) ? 8u : 0u;
    float a = fabsf(r);
    if (a >= 6.0f) return sign | 7u;
    float step = (a < 2.0f) ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
    float n = a / step;                 /* exact: step is a power of two   */
    float lo = floorf(n);
    float frac = n - lo;                /* exact                            */
    float k = lo;
    if (frac > 0.5f || (frac == 0.5f && fmodf(lo, 2.0f) == 1.0f)) k = lo + 1.0f;
    return sign | e2m1_code_of(k * step);
}

/* Stochastic rounding to E2M1.  Reading: with spacing step(|r|) as above,
 * q = step * floor(|r|/step) and f = |r|/step - floor(|r|/step) (both exact);
 * the magnitude rounds up to q + step iff u < f, where u = rnd16 / 2^16 is
 * a 16-bit uniform draw; |r| >= 6 saturates to 6.  A representable |r| has
 * f = 0 and never moves.  [AIS "Technologie stabilizujace ..."] asks for
 * stochastic rounding to remove systematic rounding error. */
unsigned oracle_e2m1_sr(float r, uint32_t rnd16)
{
    unsigned sign = signbit(r) ? 8u : 0u;
    float a = fabsf(r);
    if (a >= 6.0f) return sign | 7u;
    float step = (a < 2.0f) ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
    float n = a / step;
    float lo = floorf(n);
    float f = n - lo;
    float u = (float)(rnd16 & 0xFFFFu) * (1.0f / 65536.0f);   /* exact */
    float k = (u < f) ? lo + 1.0f : lo;
    return sign | e2m1_code_of(k * step);
}

/* Encode a non-negative binary32 t as unsigned E4M3: round to nearest,
 * ties to even, values above 448 saturate to 448 (0x7E).  Rounding works on
 * the spacing of t's binade: 2^(floor(log2 t) - 3) for normal results,
 * 2^-9 below the smallest normal 2^-6. */
unsigned oracle_e4m3_rn_satfinite(float t)
{
    if (!(t > 0.0f)) return 0u;                 /* zero (callers pass t >= 0) */
    if (t >= 448.0f) return 0x7Eu;
    int e2 = 0;
    frexpf(t, &e2);                             /* t in [2^(e2-1), 2^e2)      */
    int ulp_exp = (t < 0.015625f) ? -9 : (e2 - 1) - 3;
    float step = ldexpf(1.0f, ulp_exp);
    float n = t / step;                         /* exact scaling              */
    float lo = floorf(n);
    float frac = n - lo;
    float k = lo;
    if (frac > 0.5f || (frac == 0.5f && fmodf(lo, 2.0f) == 1.0f)) k = lo + 1.0f;
    double v = (double)k * ldexp(1.0, ulp_exp); /* the rounded value, exact   */
    if (v > 448.0) v = 448.0;
    if (v == 0.0) return 0u;
    if (v < 0.015625) return (unsigned)(v / ldexp(1.0, -9));   /* subnormal: m */
    int ev = 0;
    double fv = frexp(v, &ev);                  /* v = fv * 2^ev, fv in [0.5,1) */
    unsigned E = (unsigned)(ev - 1 + 7);
    unsigned m = (unsigned)((fv * 2.0 - 1.0) * 8.0);
    return (E << 3) | m;
}

/* ------------------------------------------------------------------------ */
/* 16-point random Hadamard transform [AIS "Technologie stabilizujace ..."]  */
/* ------------------------------------------------------------------------ */

/* Reading: the sign diagonal is bit j of word 0 of Philox4x32-10 with
 * key (seed_lo, seed_hi) and counter (0, 0, 1, 0); bit set -> -1. */
void oracle_rht_signs(uint64_t seed, float d[16])
{
    uint32_t ctr[4] = {0u, 0u, 1u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    for (int j = 0; j < 16; ++j) d[j] = ((out[0] >> j) & 1u) ? -1.0f : 1.0f;
}

/* Unnormalised Sylvester-Hadamard butterfly in a fixed order: strides
 * 1, 2, 4, 8; the pair (i, i+h) becomes (v_i + v_{i+h}, v_i - v_{i+h}).
 * Result: H16 v with H[i][j] = (-1)^popcount(i & j). */
void oracle_fwht16(float v[16])
{
    for (int h = 1; h < 16; h <<= 1) {
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            float a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
}

/* y = (1/4) H16 D v.  Reading: the 1/4 = 1/sqrt(16) normalisation makes the
 * transform orthonormal, so (Q dY)^T (Q X) = dY^T X; scaling by 0.25 is exact. */
void oracle_rht16(float v[16], const float d[16])
{
    for (int j = 0; j < 16; ++j) v[j] = v[j] * d[j];
    oracle_fwht16(v);
    for (int j = 0; j < 16; ++j) v[j] = v[j] * 0.25f;
}

/* ------------------------------------------------------------------------ */
/* Quantisation [AIS "Architektura NVFP4 kontra ograniczenia ..."]            */
/* ------------------------------------------------------------------------ */

static float widen_bf16(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

/* Element (r, c) of the input, widened exactly to binary32. */
static float load_in(const void *x, int dtype_bf16, int64_t ld, int64_t r, int64_t c)
{
    if (dtype_bf16) return widen_bf16(((const uint16_t *)x)[r * ld + c]);
    return ((const float *)x)[r * ld + c];
}

/* The 16-element block b (0-based) of output row o, as binary32, after the
 * optional Hadamard transform.  Rowwise: output row o is input row o and the
 * block runs along the columns.  Colwise: output row o is input column o and
 * the block runs down the rows (the transposed view). */
static void load_block(const void *x, int dtype_bf16, int64_t ld, int colwise,
                       int64_t o, int64_t b, int rht, const float d[16], float v[16])
{
    for (int j = 0; j < 16; ++j)
        v[j] = colwise ? load_in(x, dtype_bf16, ld, b * 16 + j, o)
                       : load_in(x, dtype_bf16, ld, o, b * 16 + j);
    if (rht) oracle_rht16(v, d);
}

/* Reading of the FP32 per-tensor scale: s_t = amax / (6 * 448), so that the
 * largest block scale lands at the top of the E4M3 range; amax = 0 (or an
 * underflowing quotient) gives s_t = 1.  s_t is the decode scale. */
float oracle_tensor_scale(float amax)
{
    float s = amax / 2688.0f;
    if (amax == 0.0f || s == 0.0f) s = 1.0f;
    return s;
}

/* Reading of the E4M3 block scale: sb = E4M3(amax_b / 6 / s_t), two
 * divisions in this order, round to nearest even, saturating at 448. */
unsigned oracle_block_scale(float amax_b, float s_t)
{
    float t = amax_b / 6.0f;
    t = t / s_t;
    return oracle_e4m3_rn_satfinite(t);
}

/* a1: tensor amax over the (optionally Hadamard-transformed) blocks of the
 * output view.  Returns -1 on bad arguments. */
float oracle_amax(const void *x, int dtype_bf16, int64_t R, int64_t C, int64_t ld,
                  int colwise, int rht, uint64_t seed)
{
    int64_t rows = colwise ? C : R;
    int64_t K = colwise ? R : C;
    if (K % 16 != 0 || (rht && !colwise)) return -1.0f;
    float d[16];
    if (rht) oracle_rht_signs(seed, d);
    float amax = 0.0f, v[16];
    for (int64_t o = 0; o < rows; ++o)
        for (int64_t b = 0; b < K / 16; ++b) {
            load_block(x, dtype_bf16, ld, colwise, o, b, rht, d, v);
            for (int j = 0; j < 16; ++j)
                if (fabsf(v[j]) > amax) amax = fabsf(v[j]);
        }
    return amax;
}

/* a2-a5 for one output row o, given the tensor scale s_t: writes the row's
 * K/2 code bytes and K/16 scale bytes (plain order). */
static void quantize_row(const void *x, int dtype_bf16, int64_t ld, int colwise, int sr, int rht,
                         const float d[16], uint64_t seed, float s_t, int64_t o, int64_t K,
                         uint8_t *codes_row, uint8_t *scales_row)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int64_t b = 0; b < K / 16; ++b) {
        float v[16];
        load_block(x, dtype_bf16, ld, colwise, o, b, rht, d, v);
        /* a3: block amax and E4M3 block scale */
        float amax_b = 0.0f;
        for (int j = 0; j < 16; ++j)
            if (fabsf(v[j]) > amax_b) amax_b = fabsf(v[j]);
        unsigned sb = oracle_block_scale(amax_b, s_t);
        scales_row[b] = (uint8_t)sb;
        /* a4: element scale (reading: one reciprocal per block) */
        float dec = (float)oracle_e4m3_value(sb) * s_t;
        float inv = 1.0f / dec;
        int zero_block = (sb == 0u) || (dec == 0.0f) || !isfinite(inv);
        uint32_t words[4] = {0, 0, 0, 0};
        int64_t have_group = -1;
        for (int j = 0; j < 16; ++j) {
            unsigned q = 0u;
            if (!zero_block) {
                float rr = v[j] * inv;
                if (sr) {
                    int64_t idx = o * K + b * 16 + j;   /* index in the output view */
                    int64_t group = idx >> 3;
                    if (group != have_group) {
                        uint32_t ctr[4] = {(uint32_t)group, (uint32_t)(idx >> 35), 0u, 0u};
                        oracle_philox4x32_10(ctr, key, words);
                        have_group = group;
                    }
                    uint32_t w = words[(idx & 7) >> 1];
                    uint32_t rnd16 = (idx & 1) ? (w >> 16) : (w & 0xFFFFu);
                    q = oracle_e2m1_sr(rr, rnd16);
                } else {
                    q = oracle_e2m1_rtn(rr);
                }
            }
            /* a5: pack, element 2i in the low nibble */
            int64_t e = b * 16 + j;
            uint8_t *byte = &codes_row[e >> 1];
            if ((e & 1) == 0) *byte = (uint8_t)((*byte & 0xF0u) | q);
            else              *byte = (uint8_t)((*byte & 0x0Fu) | (q << 4));
        }
    }
}

/* Quantise an [R x C] tensor (row-major, leading dimension ld, binary32 or
 * bf16 bits) to NVFP4.
 *   colwise = 0: output rows' = R, K = C, blocks along the columns.
 *   colwise = 1: output rows' = C, K = R, blocks down the rows (transposed).
 *   sr = 1: stochastic rounding; idx = o * K + k in the output's row-major
 *     [rows' x K] view; Philox counter (idx>>3 low word, idx>>35, 0, 0), key
 *     (seed_lo, seed_hi); rnd16 = 16-bit half (idx&1: high) of output word
 *     (idx&7)>>1.  (Reading.)
 *   rht = 1: each block goes through the 16-point RHT first (colwise only).
 *   amax_in != NULL: use *amax_in as the tensor amax instead of measuring it.
 * Outputs: codes [rows' x K/2] (element 2i in the low nibble), scales
 * [rows' x K/16] E4M3 bytes in plain row-major order, tensor_scale (1 float)
 * and amax_out (the amax used).  Returns 0, or -1 on bad arguments. */
int oracle_quantize(const void *x, int dtype_bf16, int64_t R, int64_t C, int64_t ld,
                    int colwise, int sr, int rht, uint64_t seed, const float *amax_in,
                    uint8_t *codes, uint8_t *scales, float *tensor_scale, float *amax_out)
{
    int64_t rows = colwise ? C : R;
    int64_t K = colwise ? R : C;
    if (K % 16 != 0 || rows < 0 || K < 0 || (rht && !colwise)) return -1;
    float d[16];
    if (rht) oracle_rht_signs(seed, d);
    float amax = amax_in ? *amax_in : oracle_amax(x, dtype_bf16, R, C, ld, colwise, rht, seed);
    float s_t = oracle_tensor_scale(amax);
    *tensor_scale = s_t;
    if (amax_out) *amax_out = amax;
    for (int64_t o = 0; o < rows; ++o)
        quantize_row(x, dtype_bf16, ld, colwise, sr, rht, d, seed, s_t, o, K,
                     codes + o * (K / 2), scales + o * (K / 16));
    return 0;
}

/* The same quantisation restricted to the output rows out_rows[i], i < n
 * (for sampled checks of full-size tensors); amax is the tensor amax. */
int oracle_quantize_rows(const void *x, int dtype_bf16, int64_t R, int64_t C, int64_t ld,
                         int colwise, int sr, int rht, uint64_t seed, float amax,
                         const int64_t *out_rows, int64_t n, uint8_t *codes, uint8_t *scales)
{
    int64_t K = colwise ? R : C;
    if (K % 16 != 0 || (rht && !colwise)) return -1;
    float d[16];
    if (rht) oracle_rht_signs(seed, d);
    float s_t = oracle_tensor_scale(amax);
    for (int64_t i = 0; i < n; ++i)
        quantize_row(x, dtype_bf16, ld, colwise, sr, rht, d, seed, s_t, out_rows[i], K,
                     codes + i * (K / 2), scales + i * (K / 16));
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MXFP4, the comparison format of [AIS "Architektura NVFP4 kontra           */
/* ograniczenia mikroskalowania"]: blocks of 32 elements, one power-of-two   */
/* scale per block, no per-tensor scale.                                      */
/* ------------------------------------------------------------------------ */

/* E8M0: an unsigned biased exponent, value 2^(code - 127); 0xFF is NaN. */
double oracle_e8m0_value(unsigned code)
{
    return code == 0xFFu ? NAN : ldexp(1.0, (int)code - 127);
}

/* Reading of the MX block scale (the pages name the format, not the rule; this
 * is the OCP Microscaling conversion): shared exponent X = floor(log2 amax_b)
 * - 2, where 2 is the exponent of E2M1's top binade (6 = 1.5 * 2^2), clamped
 * to [-127, 127]; amax_b = 0 gives X = -127.  Returns the E8M0 code X + 127. */
unsigned oracle_mx_scale(float amax_b)
{
    if (amax_b == 0.0f) return 0u;
    int e;
    frexpf(amax_b, &e);          /* amax_b = f * 2^e, f in [0.5, 1): floor(log2) = e - 1 */
    int x = (e - 1) - 2;
    if (x < -127) x = -127;
    if (x > 127) x = 127;
    return (unsigned)(x + 127);
}

/* MXFP4 quantisation of an [R x C] tensor.  Rowwise (colwise = 0, C % 32 ==
 * 0): output row o is input row o, blocks run along the columns.  Colwise
 * (R % 32 == 0): output row o is input column o and blocks run down the rows
 * (the transposed view, as for NVFP4).  Codes packed as for NVFP4 (element 2i
 * in the low nibble), scales plain [rows' x K/32] E8M0 codes.  Each element is
 * E2M1(v * 2^-X) with round-to-nearest-even, saturating at 6; the power-of-two
 * product is exact (it can only lose bits below 2^-126, where every value
 * rounds to zero anyway).  Returns 0, or -1 on bad arguments. */
int oracle_quantize_mx(const void *x, int dtype_bf16, int64_t R, int64_t C, int64_t ld, int colwise,
                       uint8_t *codes, uint8_t *scales)
{
    int64_t rows = colwise ? C : R, K = colwise ? R : C;
    if (K % 32 != 0 || R < 0 || C < 0) return -1;
    for (int64_t o = 0; o < rows; ++o)
        for (int64_t b = 0; b < K / 32; ++b) {
            float v[32], amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                v[j] = colwise ? load_in(x, dtype_bf16, ld, b * 32 + j, o) : load_in(x, dtype_bf16, ld, o, b * 32 + j);
                if (fabsf(v[j]) > amax) amax = fabsf(v[j]);
            }
            unsigned code = oracle_mx_scale(amax);
            float inv = ldexpf(1.0f, 127 - (int)code);   /* 2^-X */
            scales[o * (K / 32) + b] = (uint8_t)code;
            for (int j = 0; j < 32; j += 2) {
                unsigned lo = oracle_e2m1_rtn(v[j] * inv), hi = oracle_e2m1_rtn(v[j + 1] * inv);
                codes[o * (K / 2) + (b * 32 + j) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block-scaled GEMM in binary64 [AIS "Architektura NVFP4 ..."]              */
/* ------------------------------------------------------------------------ */

/* Dequantised element k of a row: e2m1(code) * e4m3(block scale) * s_t. */
static double deq(const uint8_t *codes_row, const uint8_t *scales_row, double s_t, int64_t k)
{
    uint8_t byte = codes_row[k >> 1];
    unsigned q = (k & 1) ? (byte >> 4) : (byte & 0xFu);
    return oracle_e2m1_value(q) * oracle_e4m3_value(scales_row[k >> 4]) * s_t;
}

/* One output element: ref = sum_k a_k b_k and abs = sum_k |a_k b_k| (FP64)
 * for row m of A and row n of B (both K-major NVFP4 with plain scales). */
void oracle_dot(const uint8_t *a_codes, const uint8_t *a_scales, float a_ts,
                const uint8_t *b_codes, const uint8_t *b_scales, float b_ts,
                int64_t K, int64_t m, int64_t n, double *ref, double *absref)
{
    const uint8_t *ac = a_codes + m * (K / 2), *as = a_scales + m * (K / 16);
    const uint8_t *bc = b_codes + n * (K / 2), *bs = b_scales + n * (K / 16);
    double s = 0.0, sa = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double p = deq(ac, as, a_ts, k) * deq(bc, bs, b_ts, k);
        s += p;
        sa += fabs(p);
    }
    *ref = s;
    *absref = sa;
}

/* Full GEMM C[m,n] = sum_k A[m,k] B[n,k] for every (m, n). */
void oracle_gemm(const uint8_t *a_codes, const uint8_t *a_scales, float a_ts,
                 const uint8_t *b_codes, const uint8_t *b_scales, float b_ts,
                 int64_t M, int64_t N, int64_t K, double *ref, double *absref)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            oracle_dot(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, K, m, n,
                       &ref[m * N + n], &absref[m * N + n]);
}

/* Selected output elements (m_i, n_i), i < count. */
void oracle_gemm_sampled(const uint8_t *a_codes, const uint8_t *a_scales, float a_ts,
                         const uint8_t *b_codes, const uint8_t *b_scales, float b_ts,
                         int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                         double *ref, double *absref)
{
    for (int64_t i = 0; i < count; ++i)
        oracle_dot(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, K, ms[i], ns[i],
                   &ref[i], &absref[i]);
}

/* MXFP4 operands [AIS "Architektura NVFP4 kontra ograniczenia ..."]: the
 * same binary64 dot product with E8M0 block scales over blocks of 32 and no
 * tensor scale.  Codes packed as for NVFP4, scales plain [rows x K/32]. */
static double deq_mx(const uint8_t *codes_row, const uint8_t *scales_row, int64_t k)
{
    uint8_t byte = codes_row[k >> 1];
    unsigned q = (k & 1) ? (byte >> 4) : (byte & 0xFu);
    return oracle_e2m1_value(q) * oracle_e8m0_value(scales_row[k >> 5]);
}

void oracle_gemm_mx(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *b_codes,
                    const uint8_t *b_scales, int64_t M, int64_t N, int64_t K, double *ref, double *absref)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t *ac = a_codes + m * (K / 2), *as = a_scales + m * (K / 32);
            const uint8_t *bc = b_codes + n * (K / 2), *bs = b_scales + n * (K / 32);
            double s = 0.0, sa = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = deq_mx(ac, as, k) * deq_mx(bc, bs, k);
                s += p;
                sa += fabs(p);
            }
            ref[m * N + n] = s;
            absref[m * N + n] = sa;
        }
}

/* ------------------------------------------------------------------------ */
/* Squared-ReLU MLP activation and its derivative (bf16 in, bf16 out)         */
/* ------------------------------------------------------------------------ */

/* binary32 -> bf16 bits, round to nearest even (finite inputs). */
static uint16_t bf16_rn(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

uint16_t oracle_bf16_from_f32(float f) { return bf16_rn(f); }

/* relu(y) is y for y > 0 and +0 otherwise (so -0 maps to +0). */
static float relu(float y) { return (y > 0.0f) ? y : 0.0f; }

/* h = relu(y) * relu(y) in binary32, then bf16. */
void oracle_relu2_fwd(const uint16_t *y, int64_t n, uint16_t *h)
{
    for (int64_t i = 0; i < n; ++i) {
        float t = relu(widen_bf16(y[i]));
        h[i] = bf16_rn(t * t);
    }
}

/* dy = dh * (2 * relu(y)) in binary32, then bf16. */
void oracle_relu2_bwd(const uint16_t *dh, const uint16_t *y, int64_t n, uint16_t *dy)
{
    for (int64_t i = 0; i < n; ++i) {
        float g = 2.0f * relu(widen_bf16(y[i]));
        dy[i] = bf16_rn(widen_bf16(dh[i]) * g);
    }
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar encoders (for exhaustive sweeps in the tests)   */
/* ------------------------------------------------------------------------ */
void oracle_e2m1_rtn_array(const float *r, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e2m1_rtn(r[i]);
}

void oracle_e2m1_sr_array(const float *r, const uint32_t *rnd16, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e2m1_sr(r[i], rnd16[i]);
}

void oracle_e4m3_rn_array(const float *t, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e4m3_rn_satfinite(t[i]);
}
