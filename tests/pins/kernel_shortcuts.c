/*
 * Exactness checks of two arithmetic shortcuts the quantize kernels take in
 * place of an IEEE division (test code; restates the shortcuts in C, one
 * binary32 operation per step, and compares with the division itself).
 *
 * 1. RN(a / 6) for a BF16 block amax a = (1 + m/128) * 2^k: a table of the
 *    128 values RN((1 + m/128) / 6), scaled by 2^k through the exponent
 *    field.  Exact while the quotient stays a normal number, because scaling
 *    by a power of two commutes with rounding there.
 * 2. RN(a / 6) for a binary32 a whose quotient is normal: q = RN(a * c) with
 *    c = RN(1/6), the remainder r = a - 6q taken exactly by one fused
 *    multiply-add, and the corrected quotient RN(q + r * c) by a second one
 *    (the FMA-based correction step of Markstein, "IA-64 and Elementary
 *    Functions", 2000).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float f32(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t bits(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }

/* Shortcut 1 over every non-negative finite BF16 pattern whose quotient is
 * normal (exponent field e of a in [4, 255)).  Returns mismatches. */
int64_t shortcut_div6_table(void)
{
    float table[128];
    for (int m = 0; m < 128; ++m)
        table[m] = (1.0f + (float)m * 0.0078125f) / 6.0f;
    int64_t bad = 0;
    for (uint32_t h = 0; h < 0x7F80u; ++h) {
        const uint32_t u = h << 16;
        const uint32_t e = u >> 23;
        if (e < 4u)
            continue;
        const float got = f32(bits(table[(u >> 16) & 0x7Fu]) + ((e - 127u) << 23));
        if (bits(got) != bits(f32(u) / 6.0f))
            ++bad;
    }
    return bad;
}

/* Shortcut 2 over the binary32 patterns [lo, hi).  Returns mismatches; the
 * kernel takes the shortcut only for a >= 1.5 * 2^-124 (quotient normal). */
int64_t shortcut_div6_fma(uint32_t lo, uint32_t hi)
{
    const float c = 1.0f / 6.0f;
    int64_t bad = 0;
    for (uint64_t u = lo; u < hi; ++u) {
        const float a = f32((uint32_t)u);
        const float q = a * c;
        const float r = fmaf(-6.0f, q, a);
        const float q1 = fmaf(r, c, q);
        if (bits(q1) != bits(a / 6.0f))
            ++bad;
    }
    return bad;
}
