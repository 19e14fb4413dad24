// Consumers of the quantized tensors.
//
// k_moe_combine     : per-token weighted sum of its top-k expert output rows
//                     ("NVIDIA shrank GLM-5.2 to 4 bits", section 2: 8 of
//                     256 experts per token).
// k_dequantize_fp8  : NVFP4 -> FP8 (E4M3) for an attention read ("FP4
//                     KV-cache quantization": current implementations
//                     dequantize the FP4 cache to FP8 before attention).
// k_amax_swiglu,
// k_encode_swiglu   : NVFP4 of the SiLU-gated activation h = silu(gate) * up
//                     between the expert up and down projections.
#include <cstdint>
#include <cuda_runtime.h>

#include "encode_common.cuh"

namespace nvfp4 {

namespace {

// Two f32 -> two E4M3 bytes (lo in bits 0..7), round to nearest even,
// saturating at 448; the sign is kept (also for zero).
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// exp(x) by Cody and Waite's reduction and a degree-7 Taylor polynomial,
// every step one binary32 RN operation in a fixed order (the same steps the
// checker uses, so the bits agree): x clamped to [-87, 87] (NaN kept),
// n = rint(RN(x * RN(log2 e))), r = x - n * ln2 with ln2 split in a 16-bit
// high part and a low correction (two FMAs), Horner with FMA, times 2^n.
__device__ __forceinline__ float exp_ref(float x) {
    if (x != x) return x;
    if (x > 87.0f) x = 87.0f;
    if (x < -87.0f) x = -87.0f;
    const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));           // RN(log2 e)
    float r = __fmaf_rn(-n, 0.693145751953125f, x);                 // ln2 high part
    r = __fmaf_rn(-n, 0x1.7f7d1cp-20f, r);                          // RN(ln2 - high)
    float p = 1.0f / 5040.0f;
    p = __fmaf_rn(p, r, 1.0f / 720.0f);
    p = __fmaf_rn(p, r, 1.0f / 120.0f);
    p = __fmaf_rn(p, r, 1.0f / 24.0f);
    p = __fmaf_rn(p, r, 1.0f / 6.0f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    return __fmul_rn(p, __uint_as_float((uint32_t)((int)n + 127) << 23));   // 2^n, |n| <= 126
}

// h = RN(RN(g * RN(1 / RN(1 + exp(-g)))) * u).  RN(1 / d) is the correctly
// rounded reciprocal (d >= 1, so the result is normal or NaN).
__device__ __forceinline__ float swiglu(float g, float u) {
    const float s = __frcp_rn(__fadd_rn(1.0f, exp_ref(-g)));
    return __fmul_rn(__fmul_rn(g, s), u);
}

// h values of block b (16 columns) of row r: gate at column 16b + i, up at
// inter + 16b + i.
__device__ __forceinline__ void swiglu_block(const uint16_t *row, int64_t inter, int64_t b, float h[16]) {
    const uint4 *gp = reinterpret_cast<const uint4 *>(row + b * 16);
    const uint4 *up = reinterpret_cast<const uint4 *>(row + inter + b * 16);
    const uint4 g0 = __ldg(gp), g1 = __ldg(gp + 1), u0 = __ldg(up), u1 = __ldg(up + 1);
    const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const uint32_t uw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[2 * i] = swiglu(__uint_as_float(gw[i] << 16), __uint_as_float(uw[i] << 16));
        h[2 * i + 1] = swiglu(__uint_as_float(gw[i] & 0xFFFF0000u), __uint_as_float(uw[i] & 0xFFFF0000u));
    }
}

__device__ __forceinline__ uint32_t abs_max16(const float h[16]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = absmax_nan(m, h[i]);
    return __float_as_uint(m) & 0x7FFFFFFFu;
}

}  // namespace

// One CTA per token; thread i covers columns 8i.., 8i + 8 * 256 .. of the
// row (16-byte loads of each of the token's expert rows, coalesced across
// the CTA).  acc = fma(w_k, x_k, acc) for k = 0..topk-1 from 0, slots of -1
// (and any outside the expert rows) skipped, one BF16 rounding.
__global__ void __launch_bounds__(256) k_moe_combine(CombineParams p) {
    __shared__ int32_t s_slot[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < p.topk) {
        s_slot[threadIdx.x] = p.slots[t * p.topk + threadIdx.x];
        s_w[threadIdx.x] = p.weights[t * p.topk + threadIdx.x];
    }
    __syncthreads();
    for (int64_t c = (int64_t)threadIdx.x * 8; c < p.hidden; c += 256 * 8) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < p.topk; ++k) {
            const int32_t s = s_slot[k];
            if (s < 0 || s >= p.out_rows) continue;       // uniform across the CTA
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.out + (int64_t)s * p.ld + c));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            const float wk = s_w[k];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fmaf_rn(wk, __uint_as_float(w4[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = __fmaf_rn(wk, __uint_as_float(w4[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
        }
        *reinterpret_cast<uint4 *>(p.y + t * p.ldy + c) =
            make_uint4(bf16x2_from_f32(acc[0], acc[1]), bf16x2_from_f32(acc[2], acc[3]),
                       bf16x2_from_f32(acc[4], acc[5]), bf16x2_from_f32(acc[6], acc[7]));
    }
}

// Lane per 16-value block: v = e2m1(code) * (s_b / 8) (exact), E4M3 by the
// hardware RN-satfinite conversion, 16 bytes out; block 0 thread 0 writes
// the per-tensor factor RN(8 / g).  Two blocks per thread per step (their
// loads issued together); a block's row and column come from a 32-bit
// division, or none when the tensor is one flat run of blocks (row-major
// scales, output pitch = columns: the KV cache).
namespace {

__device__ __forceinline__ uint4 fp8_block(uint2 codes, float sb8) {
    const uint32_t cw[2] = {codes.x, codes.y};
    uint32_t out[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 v = f32x2_from_f16x2(f16x2_from_e2m1x2((cw[h] >> (8 * j)) & 0xFFu));
            b[j] = e4m3x2_from_f32(__fmul_rn(v.x, sb8), __fmul_rn(v.y, sb8));   // 16 bits
        }
        out[2 * h] = b[0] | (b[1] << 16);
        out[2 * h + 1] = b[2] | (b[3] << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace

__global__ void __launch_bounds__(256) k_dequantize_fp8(Fp8Params p) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.fp8_scale = __fdiv_rn(8.0f, *p.global);
    const int64_t sf_cols = p.cols / 16, col_tiles = (sf_cols + 3) / 4;
    const int64_t blocks = p.rows * sf_cols;
    const bool flat = p.layout == 1 && p.ld == p.cols;
    const bool small = blocks <= 0x7FFFFFFFll;
    auto locate = [&](int64_t i, int64_t &code_off, int64_t &sf_off, int64_t &y_off) {
        if (flat) {
            code_off = i * 8;
            sf_off = i;
            y_off = i * 16;
            return;
        }
        int64_t r, c;
        if (small) {
            const uint32_t q = (uint32_t)i / (uint32_t)sf_cols;
            r = q;
            c = (uint32_t)i - q * (uint32_t)sf_cols;
        } else {
            r = i / sf_cols;
            c = i - r * sf_cols;
        }
        code_off = r * (p.cols / 2) + c * 8;
        sf_off = sf_offset(r, c, sf_cols, col_tiles, p.layout);
        y_off = r * p.ld + c * 16;
    };
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < blocks; i0 += 2 * stride) {
        const int64_t i1 = i0 + stride;
        int64_t co0, so0, yo0, co1 = 0, so1 = 0, yo1 = 0;
        locate(i0, co0, so0, yo0);
        const bool two = i1 < blocks;
        if (two) locate(i1, co1, so1, yo1);
        const uint2 c0 = __ldg(reinterpret_cast<const uint2 *>(p.codes + co0));
        const uint32_t s0 = __ldg(p.scales + so0);
        uint2 c1 = make_uint2(0u, 0u);
        uint32_t s1 = 0u;
        if (two) {
            c1 = __ldg(reinterpret_cast<const uint2 *>(p.codes + co1));
            s1 = __ldg(p.scales + so1);
        }
        *reinterpret_cast<uint4 *>(p.y + yo0) = fp8_block(c0, __fmul_rn(f32_from_e4m3(s0), 0.125f));
        if (two)
            *reinterpret_cast<uint4 *>(p.y + yo1) = fp8_block(c1, __fmul_rn(f32_from_e4m3(s1), 0.125f));
    }
}

// ------------------------------------------------------ gated activation
// Lane per 16-value block of h; tasks = (row, 32-block group), grid-stride.
__global__ void __launch_bounds__(256) k_amax_swiglu(SwigluParams p) {
    __shared__ uint32_t red[8];
    const int lane = threadIdx.x & 31;
    const int64_t blocks = p.inter / 16, groups = (blocks + 31) / 32;
    uint32_t m = 0;
    for (int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); t < p.rows * groups;
         t += (int64_t)gridDim.x * 8) {
        const int64_t r = t / groups, b = (t - r * groups) * 32 + lane;
        if (b >= blocks) continue;
        float h[16];
        swiglu_block(p.gu + r * p.ld, p.inter, b, h);
        m = max(m, abs_max16(h));
    }
    const uint32_t v = block_reduce_max(m, red);
    if (threadIdx.x == 0) p.partials[blockIdx.x] = v;
}

__global__ void __launch_bounds__(256) k_encode_swiglu(SwigluParams p) {
    __shared__ uint32_t red[8];
    __shared__ EncodeTables tab;
    float g;
    if (!global_from_partials(p.partials, p.n_partials, p.status, &g, red)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.global = g;
    fill_tables(tab, g);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t blocks = p.inter / 16, blocks4 = (blocks + 3) / 4 * 4, col_tiles = blocks4 / 4;
    const int64_t rows_out = (p.layout == 0) ? (p.rows + 127) / 128 * 128 : p.rows;
    const int64_t groups = (blocks4 + 31) / 32;
    for (int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); t < rows_out * groups;
         t += (int64_t)gridDim.x * 8) {
        const int64_t r = t / groups, b = (t - r * groups) * 32 + lane;
        uint32_t s = 0;
        if (r < p.rows && b < blocks) {
            float h[16];
            swiglu_block(p.gu + r * p.ld, p.inter, b, h);
            const uint32_t bits = abs_max16(h);
            s = e4m3_from_f32(__fmul_rn(div6_f32(__uint_as_float(bits)), g));
            const float e = tab.inv_s[s & 0x7Fu];
#pragma unroll
            for (int i = 0; i < 16; ++i) h[i] = __fmul_rn(h[i], e);
            *reinterpret_cast<uint2 *>(p.codes + r * (p.inter / 2) + b * 8) =
                make_uint2(e2m1x4_from_f32(h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]),
                           e2m1x4_from_f32(h[8], h[9], h[10], h[11], h[12], h[13], h[14], h[15]));
        }
        uint32_t word = s << (8 * (lane & 3));
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        if ((lane & 3) == 0 && b < blocks4 && (p.layout == 0 || b < blocks)) {
            uint8_t *sp = p.scales + sf_offset(r, b, blocks, col_tiles, p.layout);
            if (p.layout == 0 || ((blocks & 3) == 0 && b + 4 <= blocks)) {
                *reinterpret_cast<uint32_t *>(sp) = word;
            } else {
                for (int j = 0; j < 4 && b + j < blocks; ++j) sp[j] = (uint8_t)(word >> (8 * j));
            }
        }
    }
}

}  // namespace nvfp4
