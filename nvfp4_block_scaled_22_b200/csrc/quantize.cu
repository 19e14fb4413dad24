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
//   k_finalize_g  : partial maxima -> g, error status (nvfp4_global_scale).
//   k_encode      : g (from partials or supplied) -> codes + scales.
//   k_dequantize  : codes + scales + g -> BF16.
//
// Work split of k_encode/k_dequantize: one warp owns a 128-row x 64-column
// tile; lane l handles rows l, l+32, l+64, l+96 of the tile, 4 blocks of 16
// each.  Those 4x4 scale bytes are exactly one 16-byte row of the 512-byte
// 128x4 scale tile, so the warp writes its scales as 512 contiguous bytes.
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
struct EncodeBlockOut {
    uint2 codes;
    uint32_t scale;
    bool finite;
};

// Quantize one 16-value block held in two 16-byte words.
__device__ __forceinline__ EncodeBlockOut encode_block(uint4 a, uint4 b, float g) {
    uint32_t mw = amax_word(a, b);
    const uint32_t bits = halves_to_f32bits(mw);
    float amax_b = __uint_as_float(bits);
    float t = __fmul_rn(__fdiv_rn(amax_b, 6.0f), g);
    uint32_t s = e4m3_from_f32(t);
    float e = (s == 0u) ? 0.0f : __fdiv_rn(g, f32_from_e4m3(s));
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

__global__ void __launch_bounds__(kThreads) k_encode(EncodeParams p) {
    __shared__ uint32_t red[kThreads / 32];
    float g;
    if (p.global_supplied) {
        g = *p.global;
    } else {
        if (!global_from_partials(p.partials, p.n_partials, p.status, &g, red)) return;
        if (blockIdx.x == 0 && threadIdx.x == 0) *p.global = g;
    }
    const int lane = threadIdx.x & 31;
    const int64_t row_tiles = (p.rows + 127) / 128;
    const int64_t col_tiles = (p.cols + 63) / 64;   // = padded scale columns / 4
    const int64_t tasks = row_tiles * col_tiles;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t sf_cols = p.cols / 16;
    const bool codes16 = ((p.cols / 2) % 16) == 0;
    for (int64_t t = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < tasks;
         t += warps) {
        const int64_t rt = t / col_tiles, ct = t - rt * col_tiles;
        const int nb = (int)(sf_cols - ct * 4 < 4 ? sf_cols - ct * 4 : 4);  // valid blocks here
        uint32_t sf_rows[4];
        bool finite = true;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t r = rt * 128 + q * 32 + lane;
            uint32_t sfw = 0;
            int64_t src = r;
            if (r < p.rows && p.gather != nullptr) {
                src = p.gather[r];
                if (src >= p.src_rows) {     // out-of-range map entry: zero row + status
                    set_status(p.status, ST_INVALID_ARG);
                    src = -1;
                }
            }
            if (r < p.rows && src >= 0) {
                const uint4 *xp =
                    reinterpret_cast<const uint4 *>(p.x + src * p.ld + ct * 64);
                uint8_t *cp = p.codes + r * (p.cols / 2) + ct * 32;
                if (nb == 4) {
                    uint4 v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = __ldg(xp + i);
                    EncodeBlockOut o[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        o[b] = encode_block(v[2 * b], v[2 * b + 1], g);
                        finite &= o[b].finite;
                    }
                    if (codes16) {
                        uint4 *c4 = reinterpret_cast<uint4 *>(cp);
                        c4[0] = make_uint4(o[0].codes.x, o[0].codes.y, o[1].codes.x, o[1].codes.y);
                        c4[1] = make_uint4(o[2].codes.x, o[2].codes.y, o[3].codes.x, o[3].codes.y);
                    } else {
#pragma unroll
                        for (int b = 0; b < 4; ++b) reinterpret_cast<uint2 *>(cp)[b] = o[b].codes;
                    }
                    sfw = o[0].scale | (o[1].scale << 8) | (o[2].scale << 16) | (o[3].scale << 24);
                } else {
                    for (int b = 0; b < nb; ++b) {
                        EncodeBlockOut o = encode_block(__ldg(xp + 2 * b), __ldg(xp + 2 * b + 1), g);
                        finite &= o.finite;
                        reinterpret_cast<uint2 *>(cp)[b] = o.codes;
                        sfw |= o.scale << (8 * b);
                    }
                }
            } else if (r < p.rows) {  // gathered padding row: zero codes
                uint8_t *cp = p.codes + r * (p.cols / 2) + ct * 32;
                for (int b = 0; b < nb; ++b) reinterpret_cast<uint2 *>(cp)[b] = make_uint2(0, 0);
            }
            sf_rows[q] = sfw;
            if (p.layout == 1 && r < p.rows) {  // linear [rows x cols/16]
                uint8_t *sp = p.scales + r * sf_cols + ct * 4;
                if (nb == 4 && (sf_cols % 4) == 0) {
                    *reinterpret_cast<uint32_t *>(sp) = sfw;
                } else {
                    for (int b = 0; b < nb; ++b) sp[b] = (uint8_t)(sfw >> (8 * b));
                }
            }
        }
        if (!finite) set_status(p.status, ST_NONFINITE);  // only reachable with a supplied g
        if (p.layout == 0) {  // 128x4 tile: this lane's 16 bytes, padding = 0
            uint4 *sp = reinterpret_cast<uint4 *>(p.scales + (rt * col_tiles + ct) * 512) + lane;
            *sp = make_uint4(sf_rows[0], sf_rows[1], sf_rows[2], sf_rows[3]);
        }
    }
}

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
    const int64_t row_tiles = (p.rows + 127) / 128;
    const int64_t col_tiles = (p.cols + 63) / 64;
    const int64_t tasks = row_tiles * col_tiles;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t sf_cols = p.cols / 16;
    for (int64_t t = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < tasks;
         t += warps) {
        const int64_t rt = t / col_tiles, ct = t - rt * col_tiles;
        const int nb = (int)(sf_cols - ct * 4 < 4 ? sf_cols - ct * 4 : 4);
        uint4 sf_tile = make_uint4(0, 0, 0, 0);
        if (p.layout == 0)
            sf_tile = __ldg(reinterpret_cast<const uint4 *>(p.scales + (rt * col_tiles + ct) * 512) + lane);
        const uint32_t sfq[4] = {sf_tile.x, sf_tile.y, sf_tile.z, sf_tile.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t r = rt * 128 + q * 32 + lane;
            if (r >= p.rows) continue;
            const uint8_t *cp = p.codes + r * (p.cols / 2) + ct * 32;
            uint4 *yp = reinterpret_cast<uint4 *>(p.y + r * p.ld + ct * 64);
            for (int b = 0; b < nb; ++b) {
                uint32_t s = (p.layout == 0) ? (sfq[q] >> (8 * b)) & 0xFFu
                                             : (uint32_t)p.scales[r * sf_cols + ct * 4 + b];
                float d = __fdiv_rn(f32_from_e4m3(s), g);
                uint2 c = __ldg(reinterpret_cast<const uint2 *>(cp) + b);
                uint4 o0, o1;
                decode_block(c, d, o0, o1);
                yp[2 * b] = o0;
                yp[2 * b + 1] = o1;
            }
        }
    }
}

}  // namespace nvfp4
