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
 * 3. Stochastic rounding onto the E2M1 grid evaluated on the binary32 bit
 *    pattern (lower bound by clearing mantissa bits, up-decision by an
 *    integer compare of the draw with the cleared bits), against the
 *    oracle's definition (neighbouring grid values, fraction compared with
 *    u / 2^16 in double).
 * 4. rint(y) of the gated activation's exponential, y = RN(x * RN(log2 e))
 *    for |x| <= 87, by adding and subtracting 1.5 * 2^23 (the sum's unit in
 *    the last place is 1), the integer read from the sum's low mantissa
 *    bits, against rintf.
 * 5. The attention read's split of an FP32 weight p into three TF32 parts
 *    (FP32 values with the low 13 mantissa bits zero) by truncation:
 *    p1 = trunc(p), p2 = trunc(p - p1), p3 = (p - p1) - p2, checked to sum
 *    to p exactly with p3 a TF32 value, for p >= 2^-113 (below, p - p1 may
 *    be a subnormal number whose low 13 bits survive in p3, under 2^-136).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float f32(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }

uint8_t nvo_e2m1_sr(float y, uint32_t u16);
static uint32_t bits(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }
static uint32_t bits_of(float x) { return bits(x); }

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

static uint32_t sr_bits(float y, uint32_t u)
{
    uint32_t bits = bits_of(y);
    uint32_t sign = (bits >> 28) & 8u, mag = bits & 0x7FFFFFFFu;
    uint32_t e = mag >> 23, m = mag & 0x7FFFFFu;
    int ge1 = e >= 127u;
    uint32_t code_n = ge1 ? (((e - 126u) << 1) | (m >> 22)) : 1u;
    int up_n = (u << (ge1 ? 6 : 7)) < (m & (ge1 ? 0x3FFFFFu : 0x7FFFFFu));
    int up_s = (float)u < f32(mag) * 131072.0f;
    uint32_t code = (e >= 126u) ? code_n + (uint32_t)up_n : (uint32_t)up_s;
    return sign | (mag >= 0x40C00000u ? 7u : code);
}

/* Shortcut 3 over the binary32 patterns [lo, hi) (both signs) and the
 * given draws.  Returns mismatches against the oracle's definition. */
int64_t shortcut_sr(uint32_t lo, uint32_t hi, const uint32_t *draws, int n_draws, uint32_t stride)
{
    int64_t bad = 0;
    for (uint64_t p = lo; p < hi; p += stride)
        for (int i = 0; i < n_draws; ++i)
            for (uint32_t s = 0; s < 2; ++s) {
                float y = f32((uint32_t)p | (s << 31));
                if (sr_bits(y, draws[i]) != nvo_e2m1_sr(y, draws[i]))
                    ++bad;
            }
    return bad;
}

/* Shortcut 4 over the binary32 patterns [lo, hi) of x (both signs, |x| <=
 * 87 expected).  Returns mismatches. */
int64_t shortcut_rint_shift(uint32_t lo, uint32_t hi, uint32_t stride)
{
    const float log2e = 0x1.715476p+0f, c = 0x1.8p23f;
    int64_t bad = 0;
    for (uint64_t p = lo; p < hi; p += stride)
        for (uint32_t s = 0; s < 2; ++s) {
            const float x = f32((uint32_t)p | (s << 31));
            const float y = x * log2e;
            const float shifted = y + c;
            const float n = shifted - c;
            const int ni = (int)bits(shifted) - 0x4B400000;
            const float r = rintf(y);
            if (n != r || (float)ni != r) ++bad;
        }
    return bad;
}

/* Shortcut 5 over the binary32 patterns [lo, hi) of p > 0.  Returns the
 * patterns whose three parts do not sum to p exactly or whose third part
 * is not a TF32 value. */
int64_t shortcut_tf32_split(uint32_t lo, uint32_t hi, uint32_t stride)
{
    int64_t bad = 0;
    for (uint64_t q = lo; q < hi; q += stride) {
        const float p = f32((uint32_t)q);
        const float p1 = f32(bits(p) & 0xFFFFE000u);
        const float r1 = p - p1;
        const float p2 = f32(bits(r1) & 0xFFFFE000u);
        const float p3 = r1 - p2;
        if ((double)p1 + (double)p2 + (double)p3 != (double)p || (bits(p3) & 0x1FFFu) != 0) ++bad;
    }
    return bad;
}

