// Device helpers shared by the row-wise (quantize.cu) and column-wise
// (quantize_t.cu) NVFP4 encode kernels: exact block amax, the random
// Hadamard transform, the tensor-scale reduction, the per-block encode and
// the scale-layout offset.  Internal to libnvfp4.so.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t amax_word(uint4 a, uint4 b) {
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t t0 = max_u16x2(a.x & m, a.y & m);
    uint32_t t1 = max_u16x2(a.z & m, a.w & m);
    uint32_t t2 = max_u16x2(b.x & m, b.y & m);
    uint32_t t3 = max_u16x2(b.z & m, b.w & m);
    return max_u16x2(max_u16x2(t0, t1), max_u16x2(t2, t3));
}

// Largest |bf16| bit pattern (sign cleared) as the bit pattern of the same
// value in f32.  Inf/NaN map above every finite pattern.
__device__ __forceinline__ uint32_t halves_to_f32bits(uint32_t w) {
    uint32_t lo = w & 0xFFFFu, hi = w >> 16;
    return (lo > hi ? lo : hi) << 16;
}

__device__ __forceinline__ uint32_t block_reduce_max(uint32_t v, uint32_t *red) {
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
    }
    return v;
}

// Random Hadamard transform of one 16-value block (same pre-training page,
// section "Four stabilisation devices"): y = (1/4) H16 diag(s) x, H16 the
// Sylvester Hadamard matrix, s_j = -1 where bit j of the mask is set.  The
// sign flips act on the BF16 sign bits (exact); the four butterfly stages
// run with strides 1, 2, 4, 8 in that order, each add/sub one FP32 RN
// operation, then an RN multiply by 1/4 -- the evaluation order the
// quantized result is specified with.
//
// Register layout: P[i] = (z_i, z_{i+8}).  Stages 1, 2 and 4 pair P[i]
// with P[i+h] lane-wise (packed f32x2 add/sub); stage 8 pairs the two
// lanes of each P[i].  Output y_i is P[i].x, y_{i+8} is P[i].y.
// Value 2j of a block is the low half of BF16 word j, value 2j + 1 the
// high half.  As an FP32 bit pattern the low value is w << 16 and the high
// one w & 0xFFFF0000; its sign flip is bit 31 of that pattern, applied to
// the low value by adding 2^31 (mod 2^32, the same as flipping the bit) to
// w * 2^16 and to the high value by an XOR before the mask.
struct SignFlips {
    uint32_t lo[8], hi[8];   // 0 or 0x80000000 for values 2j and 2j + 1
};

__device__ __forceinline__ SignFlips sign_flips(uint32_t mask) {
    SignFlips f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f.lo[j] = ((mask >> (2 * j)) & 1u) << 31;
        f.hi[j] = ((mask >> (2 * j + 1)) & 1u) << 31;
    }
    return f;
}

// Sign flips, conversion and butterfly stages 1, 2, 4 (pairs P[i] =
// (z_i, z_{i+8})).
__device__ __forceinline__ void rht16_stages124(uint4 a, uint4 b, const SignFlips &f, float2 P[8]) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t v = w[j], u = w[j + 4];
        P[2 * j] = make_float2(__uint_as_float(v * 65536u + f.lo[j]),
                               __uint_as_float(u * 65536u + f.lo[j + 4]));
        P[2 * j + 1] = make_float2(__uint_as_float((v ^ f.hi[j]) & 0xFFFF0000u),
                                   __uint_as_float((u ^ f.hi[j + 4]) & 0xFFFF0000u));
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if ((i & h) == 0) {
                const float2 u = P[i], v = P[i + h];
                P[i] = add_f32x2(u, v);
                P[i + h] = sub_f32x2(u, v);
            }
        }
    }
}

// The transform without the final quarter: P[i] = (z_i, z_{i+8}), y = z/4.
__device__ __forceinline__ void rht16_unscaled(uint4 a, uint4 b, const SignFlips &f, float2 P[8]) {
    rht16_stages124(a, b, f, P);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float u = P[i].x, v = P[i].y;
        P[i] = make_float2(__fadd_rn(u, v), __fsub_rn(u, v));
    }
}

__device__ __forceinline__ void rht16(uint4 a, uint4 b, const SignFlips &f, float2 P[8]) {
    rht16_unscaled(a, b, f, P);
    const float2 q = make_float2(0.25f, 0.25f);
#pragma unroll
    for (int i = 0; i < 8; ++i) P[i] = mul_f32x2(P[i], q);
}

// max |y_i| of the transformed block without forming y, for the tensor
// amax pass.  The last butterfly stage maps a pair (u, v) to (u + v, u - v);
// one of the two exact values has magnitude |u| + |v|, and rounding is
// symmetric, so max(|RN(u + v)|, |RN(u - v)|) = RN(|u| + |v|).  RN(x / 4) is
// monotone, so the quarter is applied once to the maximum.  Inf and NaN
// reach the result (NaN-propagating max), as in the full transform.
__device__ __forceinline__ uint32_t rht16_abs_max_bits(uint4 a, uint4 b, const SignFlips &f) {
    float2 P[8];
    rht16_stages124(a, b, f, P);
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(fabsf(P[i].x), fabsf(P[i].y));
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = absmax_nan(m[i], m[i + 4]);
    m[0] = absmax_nan(m[0], m[2]);
    m[1] = absmax_nan(m[1], m[3]);
    return __float_as_uint(__fmul_rn(absmax_nan(m[0], m[1]), 0.25f)) & 0x7FFFFFFFu;
}

// max |y_i| as f32 bits; Inf and NaN patterns compare above every finite one.
__device__ __forceinline__ uint32_t abs_max_bits(const float2 P[8]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = absmax_nan(P[i].x, P[i].y);
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = absmax_nan(m[i], m[i + 4]);
    m[0] = absmax_nan(m[0], m[2]);
    m[1] = absmax_nan(m[1], m[3]);
    return __float_as_uint(absmax_nan(m[0], m[1])) & 0x7FFFFFFFu;
}

}  // namespace

// Reduce partial maxima to the tensor scale g; returns false (and records
// the status) for non-finite input or an amax too small for g.
__device__ __forceinline__ bool global_from_partials(const uint32_t *partials, int n,
                                                     uint32_t *status, float *g_out,
                                                     uint32_t *red) {
    uint32_t v = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) v = max(v, partials[i]);
    v = block_reduce_max(v, red);
    __shared__ float g_sh;
    __shared__ int ok_sh;
    if (threadIdx.x == 0) {
        int ok = 1;
        float g = 1.0f;
        if (v > 0x7F7FFFFFu) {  // Inf or NaN somewhere in the tensor
            ok = 0;
            set_status(status, ST_NONFINITE);
        } else if (v != 0u) {
            g = __fdiv_rn(2688.0f, __uint_as_float(v));
            if (!(g <= 0x1p118f)) {
                ok = 0;
                set_status(status, ST_RANGE);
            }
        }
        g_sh = g;
        ok_sh = ok;
    }
    __syncthreads();
    *g_out = g_sh;
    return ok_sh != 0;
}

// ------------------------------------------------------------ block encode
// Exact shortcuts for the two per-block IEEE divisions, filled once per CTA
// into shared memory:
//  * div6[m] = RN((1 + m/128) / 6) for the 128 BF16 mantissas.  For a block
//    amax a = (1 + m/128) * 2^k whose quotient stays a normal number,
//    RN(a / 6) = div6[m] * 2^k exactly (scaling by a power of two commutes
//    with rounding), applied as an exponent-field add; other amax values
//    (zero, subnormal, tiny, non-finite) take the division itself.
//  * inv_s[b] = RN(g / e4m3(b)) for the 127 non-negative finite E4M3 codes
//    (inv_s[0] = 0 gives the zero-scale rule).
struct EncodeTables {
    float div6[128];
    float inv_s[128];
};

__device__ __forceinline__ void fill_tables(EncodeTables &t, float g) {
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
        t.div6[i] = __fdiv_rn(1.0f + (float)i * 0.0078125f, 6.0f);
        t.inv_s[i] = (i == 0 || i == 0x7F) ? 0.0f : __fdiv_rn(g, f32_from_e4m3((uint32_t)i));
    }
}

// RN(a / 6) for a >= 0 given as f32 bits from a BF16 value.
__device__ __forceinline__ float div6_rn(uint32_t bits, const EncodeTables &t) {
    const uint32_t e = bits >> 23;                      // sign is clear
    if (e >= 4u && e < 255u)
        return __uint_as_float(__float_as_uint(t.div6[(bits >> 16) & 0x7Fu]) + ((e - 127u) << 23));
    return __fdiv_rn(__uint_as_float(bits), 6.0f);
}

struct EncodeBlockOut {
    uint2 codes;
    uint32_t scale;
    bool finite;
};

// Block scale code for a block amax given as the f32 bits of a BF16 value
// (sign clear): s = e4m3(RN(RN(amax / 6) * g)).
__device__ __forceinline__ uint32_t scale_code(uint32_t amax_bits, float g, const EncodeTables &tab) {
    return e4m3_from_f32(__fmul_rn(div6_rn(amax_bits, tab), g));
}

// E2M1 codes of eight BF16 values (packed pairs, value 2i low) times e.
__device__ __forceinline__ uint32_t encode8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float e) {
    const uint32_t w[4] = {w0, w1, w2, w3};
    float y[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        y[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), e);
        y[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), e);
    }
    return e2m1x4_from_f32(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
}

// Quantize one 16-value block held in two 16-byte words with the block
// amax `bits` (its own, or that of the 16x16 block it belongs to).
__device__ __forceinline__ EncodeBlockOut encode_block_amax(uint4 a, uint4 b, uint32_t bits, float g,
                                                            const EncodeTables &tab) {
    const uint32_t s = scale_code(bits, g, tab);
    const float e = tab.inv_s[s & 0x7Fu];
    EncodeBlockOut o;
    o.codes.x = encode8(a.x, a.y, a.z, a.w, e);
    o.codes.y = encode8(b.x, b.y, b.z, b.w, e);
    o.scale = s;
    o.finite = bits <= 0x7F7FFFFFu;
    return o;
}

// max |x| of a 16-value BF16 block as f32 bits (Inf/NaN above every finite).
__device__ __forceinline__ uint32_t block_amax_bits(uint4 a, uint4 b) {
    return halves_to_f32bits(amax_word(a, b));
}

// Quantize one 16-value block held in two 16-byte words.
__device__ __forceinline__ EncodeBlockOut encode_block(uint4 a, uint4 b, float g,
                                                       const EncodeTables &tab) {
    return encode_block_amax(a, b, block_amax_bits(a, b), g, tab);
}

// RN(a / 6) for an FP32 a >= 0.  While the quotient is a normal number
// (a >= 1.5 * 2^-124) it is q = RN(a * RN(1/6)) corrected once with the
// exact remainder a - 6q from a fused multiply-add (Markstein's FMA
// correction step, "IA-64 and Elementary Functions", 2000); checked equal
// to the IEEE division on every such input.  Smaller, non-finite and NaN
// inputs take the division.
__device__ __forceinline__ float div6_f32(float a) {
    if (a >= 0x1.8p-124f && a <= 0x1.fffffep127f) {
        const float c = 0x1.555556p-3f;     // RN(1/6)
        const float q = __fmul_rn(a, c);
        return __fmaf_rn(__fmaf_rn(-6.0f, q, a), c, q);
    }
    return __fdiv_rn(a, 6.0f);
}

// Quantize one 16-value block after the random Hadamard transform: the
// same steps on the FP32 values y (amax_b is no longer a BF16 value, so
// RN(amax_b / 6) comes from div6_f32, not the BF16 table).
__device__ __forceinline__ EncodeBlockOut encode_block_rht(uint4 a, uint4 b, const SignFlips &f,
                                                           float g, const EncodeTables &tab) {
    float2 y[8];
    rht16(a, b, f, y);
    const uint32_t bits = abs_max_bits(y);
    float t = __fmul_rn(div6_f32(__uint_as_float(bits)), g);
    uint32_t s = e4m3_from_f32(t);
    const float e = tab.inv_s[s & 0x7Fu];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = mul_f32x2(y[i], make_float2(e, e));
    EncodeBlockOut o;   // y_i = y[i].x, y_{i+8} = y[i].y
    o.codes.x = e2m1x4_from_f32(y[0].x, y[1].x, y[2].x, y[3].x, y[4].x, y[5].x, y[6].x, y[7].x);
    o.codes.y = e2m1x4_from_f32(y[0].y, y[1].y, y[2].y, y[3].y, y[4].y, y[5].y, y[6].y, y[7].y);
    o.scale = s;
    o.finite = bits <= 0x7F7FFFFFu;
    return o;
}

// ------------------------------------------------------ stochastic rounding
// Gradients are rounded stochastically ("NVFP4: how NVIDIA pre-trained a 12B
// model on 10T tokens", section "Four stabilisation devices"): a value goes
// up to the next E2M1 grid point with probability equal to its fractional
// distance.  Random bits: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011) keyed by the
// caller's 64-bit seed, counter (lo32(n), hi32(n), j, 0) for output block n
// = row * (cols / 16) + block column and draws j = 0, 1; value 8j + 2w takes
// the low 16 bits of word w of draw j, value 8j + 2w + 1 the high 16 bits.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t lo0 = c.x * 0xD2511F53u, hi0 = __umulhi(c.x, 0xD2511F53u);
        const uint32_t lo1 = c.z * 0xCD9E8D57u, hi1 = __umulhi(c.z, 0xCD9E8D57u);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// Stochastic E2M1 code of y with a 16-bit draw u: |y| >= 6 saturates;
// otherwise lo <= |y| < hi (neighbouring grid values) and the code of hi
// is taken iff u / 2^16 < (|y| - lo) / (hi - lo).  Evaluated on the FP32
// bit pattern, exactly: for |y| in [1, 6) the grid keeps one mantissa bit,
// so lo is |y| with its lower 22 mantissa bits cleared, its code is
// (exponent - 126) * 2 + top mantissa bit, and the fraction is those 22
// bits / 2^22 (u / 2^16 < f  <=>  u * 64 < bits); on [0.5, 1) lo = 0.5 and
// the fraction is the 23 mantissa bits / 2^23; below 0.5 lo = 0 and the
// fraction is 2|y| (compared as u < |y| * 2^17, exact in FP32).
__device__ __forceinline__ uint32_t e2m1_sr(float y, uint32_t u) {
    const uint32_t bits = __float_as_uint(y);
    const uint32_t sign = (bits >> 28) & 8u;
    const uint32_t mag = bits & 0x7FFFFFFFu;
    const uint32_t e = mag >> 23, m = mag & 0x7FFFFFu;
    // selects, not branches: the lanes of a warp hold values of every range
    const bool ge1 = e >= 127u;
    const uint32_t code_n = ge1 ? (((e - 126u) << 1) | (m >> 22)) : 1u;       // [0.5, 6)
    const bool up_n = (u << (ge1 ? 6 : 7)) < (m & (ge1 ? 0x3FFFFFu : 0x7FFFFFu));
    const bool up_s = (float)u < __fmul_rn(__uint_as_float(mag), 131072.0f);   // [0, 0.5)
    const uint32_t code = (e >= 126u) ? code_n + (up_n ? 1u : 0u) : (up_s ? 1u : 0u);
    return sign | (mag >= 0x40C00000u ? 7u : code);                          // |y| >= 6
}

// The two Philox draws of output block n (see above).
struct BlockDraws {
    uint4 d0, d1;
};

__device__ __forceinline__ BlockDraws block_draws(uint64_t seed, uint64_t n) {
    BlockDraws r;
    r.d0 = philox4x32_10(make_uint4((uint32_t)n, (uint32_t)(n >> 32), 0u, 0u), (uint32_t)seed,
                         (uint32_t)(seed >> 32));
    r.d1 = philox4x32_10(make_uint4((uint32_t)n, (uint32_t)(n >> 32), 1u, 0u), (uint32_t)seed,
                         (uint32_t)(seed >> 32));
    return r;
}

// Codes of 16 values y (already multiplied by the block factor), value i
// of the block in y[i], stochastically rounded with the block's draws.
__device__ __forceinline__ uint2 encode16_sr(const float y[16], const BlockDraws &r) {
    const uint32_t rw[8] = {r.d0.x, r.d0.y, r.d0.z, r.d0.w, r.d1.x, r.d1.y, r.d1.z, r.d1.w};
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {                  // byte i of the block: values 2i, 2i + 1
        const uint32_t lo = e2m1_sr(y[2 * i], rw[i] & 0xFFFFu);
        const uint32_t hi = e2m1_sr(y[2 * i + 1], rw[i] >> 16);
        w[i] = lo | (hi << 4);
    }
    return make_uint2(w[0] | (w[1] << 8) | (w[2] << 16) | (w[3] << 24),
                      w[4] | (w[5] << 8) | (w[6] << 16) | (w[7] << 24));
}

// Stochastically rounded encode of a BF16 block (scale as encode_block).
__device__ __forceinline__ EncodeBlockOut encode_block_sr(uint4 a, uint4 b, float g,
                                                          const EncodeTables &tab,
                                                          const BlockDraws &r) {
    const uint32_t bits = block_amax_bits(a, b);
    const uint32_t s = scale_code(bits, g, tab);
    const float e = tab.inv_s[s & 0x7Fu];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        y[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), e);
        y[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), e);
    }
    EncodeBlockOut o;
    o.codes = encode16_sr(y, r);
    o.scale = s;
    o.finite = bits <= 0x7F7FFFFFu;
    return o;
}

// Stochastically rounded encode after the random Hadamard transform.
__device__ __forceinline__ EncodeBlockOut encode_block_rht_sr(uint4 a, uint4 b, const SignFlips &f,
                                                              float g, const EncodeTables &tab,
                                                              const BlockDraws &r) {
    float2 P[8];
    rht16(a, b, f, P);
    const uint32_t bits = abs_max_bits(P);
    const uint32_t s = e4m3_from_f32(__fmul_rn(div6_f32(__uint_as_float(bits)), g));
    const float e = tab.inv_s[s & 0x7Fu];
    float y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {                  // P[i] = (y_i, y_{i+8})
        y[i] = __fmul_rn(P[i].x, e);
        y[i + 8] = __fmul_rn(P[i].y, e);
    }
    EncodeBlockOut o;
    o.codes = encode16_sr(y, r);
    o.scale = s;
    o.finite = bits <= 0x7F7FFFFFu;
    return o;
}

// The block encoder selected by the compile-time options (r: the block's
// draws, used with kSR only).
template <bool kRht, bool kSR>
__device__ __forceinline__ EncodeBlockOut encode_any(uint4 a, uint4 b, const SignFlips &f, float g,
                                                     const EncodeTables &tab, const BlockDraws &r) {
    if (kSR) return kRht ? encode_block_rht_sr(a, b, f, g, tab, r) : encode_block_sr(a, b, g, tab, r);
    return kRht ? encode_block_rht(a, b, f, g, tab) : encode_block(a, b, g, tab);
}

// Byte offset of scale (row r, scale column c) in either layout.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t sf_cols, int64_t col_tiles,
                                             int32_t layout) {
    if (layout == 1) return r * sf_cols + c;
    return ((r >> 7) * col_tiles + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

}  // namespace nvfp4
