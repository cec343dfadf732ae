/* The quantisation kernels' block-scale division, restated in C for a CPU
 * check against IEEE division (test infrastructure; compiled by
 * tests/test_block_scale_fast.py).
 *
 * The kernels compute t2 = RN(RN(amax_b / 6) / s_t), whose E4M3 rounding is the
 * block scale (aisight.pl, section "Architektura NVFP4 kontra ograniczenia
 * mikroskalowania": E4M3 block scales under an FP32 tensor scale), without a
 * division instruction: with rb = RN(1/b), q0 = RN(a * rb), r = a - q0 * b in
 * one FMA (exact) and q = RN(q0 + r * rb) in another (Markstein's correction
 * step), and with the numerator of the second quotient clamped to s_t * 2^10.
 * Each function returns how many inputs give a quotient that could change the
 * E4M3 code: a different binary32 value where the exact quotient lies in
 * [2^-12, 2^10], a value of at least 2^-11 where it lies below 2^-12 (E4M3
 * rounds everything under 2^-10 to 0), or a value under 464 where it lies above
 * 2^10 (E4M3 saturates everything above 448 to 448).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float as_float(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t as_bits(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }

static float div_corrected(float a, float b, float rb) {
    const float q0 = a * rb;
    const float r = fmaf(-q0, b, a);
    return fmaf(r, rb, q0);
}

/* amax / 6 alone, for every bit pattern from `start` to `stop` (inclusive) in
 * steps of `stride`: the number of differences from IEEE a / 6. */
int64_t div6_mismatches(uint32_t start, uint32_t stop, uint32_t stride) {
    const float rb = 1.0f / 6.0f;
    int64_t bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t i = start; i <= (int64_t)stop; i += stride) {
        const float a = as_float((uint32_t)i);
        if (as_bits(div_corrected(a, 6.0f, rb)) != as_bits(a / 6.0f)) ++bad;
    }
    return bad;
}

/* The whole block-scale quotient for one tensor scale s_t (in [2^-80, 2^100],
 * the kernels' fast range) over amax bit patterns start..stop by stride. */
int64_t t2_mismatches(float s_t, uint32_t start, uint32_t stop, uint32_t stride) {
    const float rb6 = 1.0f / 6.0f, rcp = 1.0f / s_t, hi = s_t * 1024.0f;
    int64_t bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t i = start; i <= (int64_t)stop; i += stride) {
        const float a = as_float((uint32_t)i);
        const float ref = (a / 6.0f) / s_t;
        const float t = fminf(div_corrected(a, 6.0f, rb6), hi);
        const float got = div_corrected(t, s_t, rcp);
        if (ref >= 0x1p-12f && ref <= 1024.0f) {
            if (as_bits(got) != as_bits(ref)) ++bad;
        } else if (ref < 0x1p-12f) {
            if (!(got < 0x1p-11f)) ++bad;
        } else if (!(got >= 464.0f)) {
            ++bad;
        }
    }
    return bad;
}
