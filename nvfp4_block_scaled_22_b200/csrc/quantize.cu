// NVFP4 two-level quantization and dequantization kernels (sm_100a).
//
// Method ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens",
// section "E2M1 format and two-level scaling"; "NVIDIA shrank GLM-5.2 to 4
// bits", section 3): an FP32 scale per tensor g = 448*6/amax, then per 16
// consecutive values along a row an E4M3 scale s = e4m3(amax_b/6*g) that
// maps the block amax close to the E2M1 maximum 6, and the 4-bit codes
// e2m1(x * g/s).  Every float step is one IEEE RN operation (no fast-math,
// no FMA contraction, no flush-to-zero) so codes and scales are exact.
//
// Kernels
//   k_amax        : per-CTA max|x| over whole rows (optionally gathered).
//   k_amax_rht    : the same over the random-Hadamard-transformed blocks.
//   k_finalize_g  : partial maxima -> g, error status (nvfp4_global_scale).
//   k_encode      : g (from partials or supplied) -> codes + scales; the
//                   kRht instance transforms each block first.
//   k_dequantize  : codes + scales + g -> BF16.
//
// Work split of k_encode/k_dequantize: a warp takes one row's 512-value
// segment, one 16-value block per lane, so every global access of a warp is
// contiguous (see the comment above k_encode).
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
struct SignFlips {
    uint32_t w[8];   // XOR mask of BF16 word j (values 2j, 2j+1 of a block)
};

__device__ __forceinline__ SignFlips sign_flips(uint32_t mask) {
    SignFlips f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        f.w[j] = (((mask >> (2 * j)) & 1u) << 15) | (((mask >> (2 * j + 1)) & 1u) << 31);
    return f;
}

__device__ __forceinline__ void rht16(uint4 a, uint4 b, const SignFlips &f, float2 P[8]) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t v = w[j] ^ f.w[j], u = w[j + 4] ^ f.w[j + 4];
        P[2 * j] = make_float2(__uint_as_float(v << 16), __uint_as_float(u << 16));
        P[2 * j + 1] = make_float2(__uint_as_float(v & 0xFFFF0000u), __uint_as_float(u & 0xFFFF0000u));
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
    const float2 q = make_float2(0.25f, 0.25f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float u = P[i].x, v = P[i].y;
        P[i] = mul_f32x2(make_float2(__fadd_rn(u, v), __fsub_rn(u, v)), q);
    }
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

// ---------------------------------------------------------------- k_amax
// One warp per row (grid-stride over rows), 16-byte loads.  Writes the
// CTA's max|x| as f32 bits (Inf/NaN compare above every finite value).
__global__ void __launch_bounds__(kThreads) k_amax(const uint16_t *__restrict__ x, int64_t ld,
                                                   int64_t rows, int64_t cols,
                                                   const int32_t *__restrict__ gather,
                                                   int64_t src_rows,
                                                   uint32_t *__restrict__ partials,
                                                   uint32_t *status) {
    __shared__ uint32_t red[kThreads / 32];
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t chunks = cols / 8;  // 16-byte chunks per row
    uint32_t m = 0;
    for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        int64_t src = r;
        if (gather != nullptr) {
            src = gather[r];
            if (src < 0) continue;
            if (src >= src_rows) {           // row map points outside x
                if (lane == 0) set_status(status, ST_INVALID_ARG);
                continue;
            }
        }
        const uint4 *p = reinterpret_cast<const uint4 *>(x + src * ld);
        int64_t c = lane;
        for (; c + 96 < chunks; c += 128) {
            uint4 a = __ldg(p + c), b = __ldg(p + c + 32), d = __ldg(p + c + 64),
                  e = __ldg(p + c + 96);
            m = max_u16x2(m, max_u16x2(amax_word(a, b), amax_word(d, e)));
        }
        for (; c < chunks; c += 32) {
            uint4 a = __ldg(p + c);
            m = max_u16x2(m, amax_word(a, a));
        }
    }
    uint32_t v = block_reduce_max(halves_to_f32bits(m), red);
    if (threadIdx.x == 0) partials[blockIdx.x] = v;
}

// ------------------------------------------------------------ k_amax_rht
// One warp per row, one 16-value block per lane (a warp reads 1 KiB
// contiguous per step); the block is transformed in registers and the max
// of |y| over the CTA is written as f32 bits, the format k_amax writes.
__global__ void __launch_bounds__(kThreads) k_amax_rht(const uint16_t *__restrict__ x, int64_t ld,
                                                       int64_t rows, int64_t cols,
                                                       uint32_t rht_mask,
                                                       uint32_t *__restrict__ partials) {
    __shared__ uint32_t red[kThreads / 32];
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t blocks = cols / 16;
    const SignFlips f = sign_flips(rht_mask);
    uint32_t m = 0;
    for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x + r * ld);
        int64_t c = lane;
        for (; c + 32 < blocks; c += 64) {
            uint4 a0 = __ldg(p + 2 * c), b0 = __ldg(p + 2 * c + 1);
            uint4 a1 = __ldg(p + 2 * c + 64), b1 = __ldg(p + 2 * c + 65);
            float2 y[8];
            rht16(a0, b0, f, y);
            m = max(m, abs_max_bits(y));
            rht16(a1, b1, f, y);
            m = max(m, abs_max_bits(y));
        }
        if (c < blocks) {
            float2 y[8];
            rht16(__ldg(p + 2 * c), __ldg(p + 2 * c + 1), f, y);
            m = max(m, abs_max_bits(y));
        }
    }
    uint32_t v = block_reduce_max(m, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = v;
}

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

__global__ void k_finalize_g(const uint32_t *__restrict__ partials, int n, float *global,
                             uint32_t *status) {
    __shared__ uint32_t red[kThreads / 32];
    float g;
    if (global_from_partials(partials, n, status, &g, red) && threadIdx.x == 0) *global = g;
}

// --------------------------------------------------------------- k_encode
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

// Quantize one 16-value block held in two 16-byte words.
__device__ __forceinline__ EncodeBlockOut encode_block(uint4 a, uint4 b, float g,
                                                       const EncodeTables &tab) {
    uint32_t mw = amax_word(a, b);
    const uint32_t bits = halves_to_f32bits(mw);
    float t = __fmul_rn(div6_rn(bits, tab), g);
    uint32_t s = e4m3_from_f32(t);
    float e = tab.inv_s[s & 0x7Fu];
    uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        y[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), e);
        y[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), e);
    }
    EncodeBlockOut o;
    o.codes.x = e2m1x4_from_f32(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
    o.codes.y = e2m1x4_from_f32(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
    o.scale = s;
    o.finite = bits <= 0x7F7FFFFFu;
    return o;
}

// Quantize one 16-value block after the random Hadamard transform: the
// same steps on the FP32 values y (RN(amax_b / 6) by an IEEE division, as
// amax_b is no longer a BF16 value).
__device__ __forceinline__ EncodeBlockOut encode_block_rht(uint4 a, uint4 b, const SignFlips &f,
                                                           float g, const EncodeTables &tab) {
    float2 y[8];
    rht16(a, b, f, y);
    const uint32_t bits = abs_max_bits(y);
    float t = __fmul_rn(__fdiv_rn(__uint_as_float(bits), 6.0f), g);
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

// Byte offset of scale (row r, scale column c) in either layout.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t sf_cols, int64_t col_tiles,
                                             int32_t layout) {
    if (layout == 1) return r * sf_cols + c;
    return ((r >> 7) * col_tiles + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// Work split: a task is one row and one 512-value segment of it; lane l
// owns 16-value block l of the segment (two 16-byte loads, one 8-byte code
// store), so a warp's loads and stores are contiguous.  The four scale
// bytes of blocks 4j..4j+3 are contiguous in both scale layouts; lanes
// 4j..4j+3 combine them with two shuffles and lane 4j stores the word.
// Rows past the end of the last 128-row band (swizzled layout) and scale
// columns past cols/16 up to the next multiple of 4 are written as zero.
constexpr int kUnroll = 4;

// Row of flat task t (tasks laid out row-major, segs per row) without a
// 64-bit division: float reciprocal, then exact integer correction.
__device__ __forceinline__ uint32_t task_row(uint32_t t, uint32_t segs, float inv) {
    uint32_t r = __float2uint_rz((float)t * inv);
    while (r * segs > t) --r;
    while ((r + 1) * segs <= t) ++r;
    return r;
}

template <bool kRht>
__device__ __forceinline__ void encode_body(const EncodeParams &p) {
    __shared__ uint32_t red[kThreads / 32];
    __shared__ EncodeTables tab;
    float g;
    if (p.global_supplied) {
        g = *p.global;
    } else {
        if (!global_from_partials(p.partials, p.n_partials, p.status, &g, red)) return;
        if (blockIdx.x == 0 && threadIdx.x == 0) *p.global = g;
    }
    fill_tables(tab, g);
    __syncthreads();
    const SignFlips flips = sign_flips(kRht ? p.rht_mask : 0u);
    const int lane = threadIdx.x & 31;
    const int64_t sf_cols = p.cols / 16;
    const int64_t sf_cols4 = (sf_cols + 3) / 4 * 4;               // padded scale columns
    const int64_t col_tiles = sf_cols4 / 4;
    const int64_t segs = (sf_cols4 + 31) / 32;                    // 32 blocks per segment
    const int64_t rows_out = (p.layout == 0) ? (p.rows + 127) / 128 * 128 : p.rows;
    const uint32_t tasks = (uint32_t)(rows_out * segs);        // < 2^32 (host-checked)
    const uint32_t warps = gridDim.x * (kThreads / 32);
    const float inv_segs = 1.0f / (float)segs;
    bool finite = true;
    for (uint32_t t0 = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t0 < tasks;
         t0 += warps * kUnroll) {
        uint4 va[kUnroll], vb[kUnroll];
        int64_t rr[kUnroll], bb[kUnroll];
        bool has[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t t = t0 + warps * u;
            const uint32_t row = task_row(t, (uint32_t)segs, inv_segs);
            rr[u] = row;
            bb[u] = (int64_t)(t - row * (uint32_t)segs) * 32 + lane;   // scale column of this lane
            int64_t src = rr[u];
            has[u] = t < tasks && rr[u] < p.rows && bb[u] < sf_cols;
            if (has[u] && p.gather != nullptr) {
                src = p.gather[rr[u]];
                if (src >= p.src_rows) {     // out-of-range map entry: zero row + status
                    set_status(p.status, ST_INVALID_ARG);
                    src = -1;
                }
                if (src < 0) has[u] = false;
            }
            if (has[u]) {
                const uint4 *xp = reinterpret_cast<const uint4 *>(p.x + src * p.ld + bb[u] * 16);
                va[u] = __ldg(xp);
                vb[u] = __ldg(xp + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t t = t0 + warps * u;
            if (t >= tasks) break;                                   // uniform across the warp
            uint32_t s = 0;
            if (has[u]) {
                EncodeBlockOut o = kRht ? encode_block_rht(va[u], vb[u], flips, g, tab)
                                        : encode_block(va[u], vb[u], g, tab);
                finite &= o.finite;
                s = o.scale;
                *reinterpret_cast<uint2 *>(p.codes + rr[u] * (p.cols / 2) + bb[u] * 8) = o.codes;
            } else if (rr[u] < p.rows && bb[u] < sf_cols) {          // gathered padding row
                *reinterpret_cast<uint2 *>(p.codes + rr[u] * (p.cols / 2) + bb[u] * 8) = make_uint2(0, 0);
            }
            uint32_t w = s << (8 * (lane & 3));
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
            if ((lane & 3) == 0 && bb[u] < sf_cols4 && (p.layout == 0 || bb[u] < sf_cols)) {
                uint8_t *sp = p.scales + sf_offset(rr[u], bb[u], sf_cols, col_tiles, p.layout);
                if (p.layout == 0 || ((sf_cols & 3) == 0 && bb[u] + 4 <= sf_cols)) {
                    *reinterpret_cast<uint32_t *>(sp) = w;
                } else {                                             // ragged linear row
                    for (int j = 0; j < 4 && bb[u] + j < sf_cols; ++j) sp[j] = (uint8_t)(w >> (8 * j));
                }
            }
        }
    }
    if (!finite) set_status(p.status, ST_NONFINITE);   // only reachable with a supplied g
}

__global__ void __launch_bounds__(kThreads) k_encode(EncodeParams p) { encode_body<false>(p); }

__global__ void __launch_bounds__(kThreads, 3) k_encode_rht(EncodeParams p) { encode_body<true>(p); }

// ----------------------------------------------------------- k_dequantize
__device__ __forceinline__ void decode_block(uint2 codes, float d, uint4 &o0, uint4 &o1) {
    uint32_t out[8];
    uint32_t cw[2] = {codes.x, codes.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 v = f32x2_from_f16x2(f16x2_from_e2m1x2((cw[h] >> (8 * i)) & 0xFFu));
            out[4 * h + i] = bf16x2_from_f32(__fmul_rn(v.x, d), __fmul_rn(v.y, d));
        }
    }
    o0 = make_uint4(out[0], out[1], out[2], out[3]);
    o1 = make_uint4(out[4], out[5], out[6], out[7]);
}

__global__ void __launch_bounds__(kThreads) k_dequantize(DequantParams p) {
    const float g = *p.global;
    const int lane = threadIdx.x & 31;
    const int64_t sf_cols = p.cols / 16;
    const int64_t col_tiles = (sf_cols + 3) / 4;
    const int64_t segs = (sf_cols + 31) / 32;
    const uint32_t tasks = (uint32_t)(p.rows * segs);          // < 2^32 (host-checked)
    const uint32_t warps = gridDim.x * (kThreads / 32);
    const float inv_segs = 1.0f / (float)segs;
    for (uint32_t t0 = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t0 < tasks;
         t0 += warps * kUnroll) {
        uint2 c[kUnroll];
        uint32_t sb[kUnroll];
        int64_t rr[kUnroll], bb[kUnroll];
        bool has[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t t = t0 + warps * u;
            const uint32_t row = task_row(t, (uint32_t)segs, inv_segs);
            rr[u] = row;
            bb[u] = (int64_t)(t - row * (uint32_t)segs) * 32 + lane;
            has[u] = t < tasks && bb[u] < sf_cols;
            if (has[u]) {
                c[u] = __ldg(reinterpret_cast<const uint2 *>(p.codes + rr[u] * (p.cols / 2) + bb[u] * 8));
                sb[u] = __ldg(p.scales + sf_offset(rr[u], bb[u], sf_cols, col_tiles, p.layout));
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (!has[u]) continue;
            const float d = __fdiv_rn(f32_from_e4m3(sb[u]), g);
            uint4 o0, o1;
            decode_block(c[u], d, o0, o1);
            uint4 *yp = reinterpret_cast<uint4 *>(p.y + rr[u] * p.ld + bb[u] * 16);
            yp[0] = o0;
            yp[1] = o1;
        }
    }
}

}  // namespace nvfp4
