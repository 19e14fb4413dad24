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
// rint of |y| < 2^22 is taken by adding and subtracting 1.5 * 2^23 (the
// sum's unit in the last place is 1, so the addition rounds y to the
// nearest integer, ties to even), and n's bits are the sum's low mantissa
// bits: no conversion instructions.
__device__ __forceinline__ float exp_ref(float x) {
    if (x != x) return x;
    if (x > 87.0f) x = 87.0f;
    if (x < -87.0f) x = -87.0f;
    const float shifted = __fadd_rn(__fmul_rn(x, 0x1.715476p+0f), 0x1.8p23f);   // RN(log2 e)
    const float n = __fadd_rn(shifted, -0x1.8p23f);
    const int ni = __float_as_int(shifted) - 0x4B400000;                         // n, |n| <= 126
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
    return __fmul_rn(p, __uint_as_float((uint32_t)(ni + 127) << 23));   // 2^n
}

// h = RN(RN(g * RN(1 / RN(1 + exp(-g)))) * u).  RN(1 / d) is the correctly
// rounded reciprocal (d >= 1, so the result is normal or NaN).
__device__ __forceinline__ float swiglu(float g, float u) {
    const float s = __frcp_rn(__fadd_rn(1.0f, exp_ref(-g)));
    return __fmul_rn(__fmul_rn(g, s), u);
}

// Gate and up words of block b (16 columns) of a row: gate at column
// 16b + i, up at inter + 16b + i, two BF16 per word (value 2j in the low
// half of word j).
struct SwigluIn {
    uint32_t gw[8], uw[8];
};

__device__ __forceinline__ SwigluIn swiglu_load(const uint16_t *row, int64_t inter, int64_t b) {
    const uint4 *gp = reinterpret_cast<const uint4 *>(row + b * 16);
    const uint4 *up = reinterpret_cast<const uint4 *>(row + inter + b * 16);
    const uint4 g0 = __ldg(gp), g1 = __ldg(gp + 1), u0 = __ldg(up), u1 = __ldg(up + 1);
    return SwigluIn{{g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w},
                    {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w}};
}

__device__ __forceinline__ float bf16_half(uint32_t w, int hi) {
    return __uint_as_float(hi ? (w & 0xFFFF0000u) : (w << 16));
}

// The defined h of value idx (0..15) of the block; the word is picked by
// selects, so idx may differ between lanes without local memory.
__device__ __forceinline__ float swiglu_at(const SwigluIn &in, int idx) {
    const int w = idx >> 1;
    uint32_t gw = in.gw[0], uw = in.uw[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) {
        gw = (w == j) ? in.gw[j] : gw;
        uw = (w == j) ? in.uw[j] : uw;
    }
    return swiglu(bf16_half(gw, idx & 1), bf16_half(uw, idx & 1));
}

// Screening of a block.  Every value gets a cheap estimate of h (the
// exponential by ex2.approx, the reciprocal by rcp.approx, then the same two
// products), within 2^-15 of the defined h relative to h while g * r is
// zero or a normal number and h is finite: the argument rounding of
// x * log2 e bounds the exponential to ~2^-17 for |x| <= 87, each
// approximate instruction and product adds a few ulps at most.  (The
// flush-to-zero forms change nothing here: 2^y for |y| <= 126 and 1 / d for
// 1 <= d <= 1 + e^87 are normal numbers.)  Only decisions are taken from
// the estimates, each with a relative margin of 2^-11, 64 times that
// bound: the block amax is the max of the defined h over the candidates
// (the values within the margin of the estimated max; the value that
// attains the defined max is one of them), and a code is taken from the
// estimate only when the estimate scaled by 1 - 2^-11 and by 1 + 2^-11
// rounds to the same code (no rounding boundary in between, so the defined
// value rounds to it too).  A block with a subnormal g * r, a non-finite
// estimate or an estimated max below 2^-90 uses the defined h for every
// value.
__device__ __forceinline__ float ex2_approx(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

__device__ __forceinline__ float rcp_approx(float d) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

constexpr float kScreenMargin = 0x1p-11f;
constexpr float kScreenTiny = 0x1p-90f;

// Estimates of the block's 16 values into ha; returns the candidate mask
// for the block amax, all 16 (and `whole` set) when the estimates decide
// nothing.
__device__ __forceinline__ uint32_t swiglu_screen(const SwigluIn &in, float ha[16], bool &whole) {
    float am = 0.0f;
    uint32_t tmin = 0xFFFFFFFFu;   // min over values of |g * r| bits - 1 (zero wraps to the top)
#pragma unroll
    for (int idx = 0; idx < 16; ++idx) {
        const float g = bf16_half(in.gw[idx >> 1], idx & 1), u = bf16_half(in.uw[idx >> 1], idx & 1);
        const float gc = fminf(fmaxf(g, -87.0f), 87.0f);
        const float r = rcp_approx(__fadd_rn(1.0f, ex2_approx(__fmul_rn(gc, -0x1.715476p+0f))));
        const float t = __fmul_rn(g, r);
        const float h = __fmul_rn(t, u);
        ha[idx] = h;
        am = absmax_nan(am, h);
        tmin = min(tmin, (__float_as_uint(t) & 0x7FFFFFFFu) - 1u);
    }
    am = fabsf(am);   // the max keeps magnitudes (its sign is the xor of the operands')
    whole = !(am >= kScreenTiny && am <= 0x1.fffffep127f) || tmin < 0x007FFFFFu;
    if (whole) return 0xFFFFu;
    const float thr = __fmul_rn(am, 1.0f - kScreenMargin);
    uint32_t cand = 0;
#pragma unroll
    for (int idx = 0; idx < 16; ++idx) cand |= (fabsf(ha[idx]) >= thr) ? 1u << idx : 0u;
    return cand;
}

// Row and first block of warp task t (tasks of 32 blocks, `groups` per
// row): a 32-bit division while the task count fits.
__device__ __forceinline__ int64_t task_row(int64_t t, int64_t groups, bool small) {
    return small ? (int64_t)((uint32_t)t / (uint32_t)groups) : t / groups;
}

// Block amax (f32 bits of max |h|, NaN above all) over the candidates.
// Warp-collective: every lane of the warp calls it (cand = 0 for none).
__device__ __forceinline__ uint32_t swiglu_cand_amax(const SwigluIn &in, uint32_t cand) {
    float m = 0.0f;
    while (__any_sync(0xFFFFFFFFu, cand != 0u)) {
        const float h = swiglu_at(in, cand ? __ffs(cand) - 1 : 0);
        m = cand ? absmax_nan(m, h) : m;
        cand &= cand - 1u;
    }
    return __float_as_uint(m) & 0x7FFFFFFFu;
}

// E2M1 code (4 bits) of one value, round to nearest even, saturating.
__device__ __forceinline__ uint32_t e2m1_code(float x) {
    uint16_t r;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u16.u8 %0, b;\n\t}"
        : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFu;
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
// Lane per 16-value block of h; tasks = (row, 32-block group), grid-stride
// per warp (every lane runs every task: the screening loops are
// warp-collective).
__global__ void __launch_bounds__(256) k_amax_swiglu(SwigluParams p) {
    __shared__ uint32_t red[8];
    const int lane = threadIdx.x & 31;
    const int64_t blocks = p.inter / 16, groups = (blocks + 31) / 32, tasks = p.rows * groups;
    const int64_t stride = (int64_t)gridDim.x * 8;
    const bool small = tasks + stride <= 0x7FFFFFFFll;
    auto fetch = [&](int64_t t, SwigluIn &in) {
        const int64_t r = task_row(t, groups, small), b = (t - r * groups) * 32 + lane;
        const bool valid = t < tasks && b < blocks;
        if (valid) in = swiglu_load(p.gu + r * p.ld, p.inter, b);
        return valid;
    };
    uint32_t m = 0;
    int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    SwigluIn nxt = {};
    bool nxt_valid = fetch(t, nxt);
    for (; t < tasks; t += stride) {
        // the next task's loads are in flight during this task's arithmetic
        const SwigluIn in = nxt;
        const bool valid = nxt_valid;
        nxt_valid = fetch(t + stride, nxt);
        float ha[16];
        bool whole;
        const uint32_t cand = valid ? swiglu_screen(in, ha, whole) : 0u;
        m = max(m, swiglu_cand_amax(in, cand));
    }
    const uint32_t v = block_reduce_max(m, red);
    if (threadIdx.x == 0) p.partials[blockIdx.x] = v;
}

__global__ void __launch_bounds__(256, 3) k_encode_swiglu(SwigluParams p) {
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
    const int64_t groups = (blocks4 + 31) / 32, tasks = rows_out * groups;
    const int64_t stride = (int64_t)gridDim.x * 8;
    const bool small = tasks + stride <= 0x7FFFFFFFll;
    auto fetch = [&](int64_t t, SwigluIn &in) {
        const int64_t r = task_row(t, groups, small), b = (t - r * groups) * 32 + lane;
        const bool valid = t < tasks && r < p.rows && b < blocks;
        if (valid) in = swiglu_load(p.gu + r * p.ld, p.inter, b);
        return valid;
    };
    int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    SwigluIn nxt = {};
    bool nxt_valid = fetch(t, nxt);
    for (; t < tasks; t += stride) {
        const int64_t r = task_row(t, groups, small), b = (t - r * groups) * 32 + lane;
        // the next task's loads are in flight during this task's arithmetic
        const SwigluIn in = nxt;
        const bool valid = nxt_valid;
        nxt_valid = fetch(t + stride, nxt);
        float ha[16];
        uint32_t cand = 0;
        bool whole = true;
        if (valid) cand = swiglu_screen(in, ha, whole);
        const uint32_t bits = swiglu_cand_amax(in, cand);
        uint32_t s = 0;
        uint64_t codes = 0, todo = 0;
        float e = 0.0f;
        if (valid) {
            s = e4m3_from_f32(__fmul_rn(div6_f32(__uint_as_float(bits)), g));
            e = tab.inv_s[s & 0x7Fu];
            const float e_lo = __fmul_rn(e, 1.0f - kScreenMargin), e_hi = __fmul_rn(e, 1.0f + kScreenMargin);
            float lo[16], hi[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                lo[i] = __fmul_rn(ha[i], e_lo);
                hi[i] = __fmul_rn(ha[i], e_hi);
            }
            const uint64_t cl = (uint64_t)e2m1x4_from_f32(lo[0], lo[1], lo[2], lo[3], lo[4], lo[5], lo[6], lo[7]) |
                                (uint64_t)e2m1x4_from_f32(lo[8], lo[9], lo[10], lo[11], lo[12], lo[13], lo[14], lo[15]) << 32;
            const uint64_t ch = (uint64_t)e2m1x4_from_f32(hi[0], hi[1], hi[2], hi[3], hi[4], hi[5], hi[6], hi[7]) |
                                (uint64_t)e2m1x4_from_f32(hi[8], hi[9], hi[10], hi[11], hi[12], hi[13], hi[14], hi[15]) << 32;
            codes = cl;
            todo = whole ? ~0ull : (cl ^ ch);
        }
        // codes the estimate does not decide: the defined h, one value per
        // lane and round
        while (__any_sync(0xFFFFFFFFu, todo != 0ull)) {
            const int idx = todo ? (__ffsll((long long)todo) - 1) >> 2 : 0;
            const uint32_t c = e2m1_code(__fmul_rn(swiglu_at(in, idx), e));
            if (todo) {
                const uint64_t mask = 0xFull << (4 * idx);
                codes = (codes & ~mask) | ((uint64_t)c << (4 * idx));
                todo &= ~mask;
            }
        }
        if (valid)
            *reinterpret_cast<uint2 *>(p.codes + r * (p.inter / 2) + b * 8) =
                make_uint2((uint32_t)codes, (uint32_t)(codes >> 32));
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
