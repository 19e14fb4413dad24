// Consumers of the quantized tensors.
//
// k_moe_combine     : per-token weighted sum of its top-k expert output rows
//                     ("NVIDIA shrank GLM-5.2 to 4 bits", section 2: 8 of
//                     256 experts per token).
// k_dequantize_fp8  : NVFP4 -> FP8 (E4M3) for an attention read ("FP4
//                     KV-cache quantization": current implementations
//                     dequantize the FP4 cache to FP8 before attention).
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
// the per-tensor factor RN(8 / g).
__global__ void __launch_bounds__(256) k_dequantize_fp8(Fp8Params p) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.fp8_scale = __fdiv_rn(8.0f, *p.global);
    const int64_t sf_cols = p.cols / 16, col_tiles = (sf_cols + 3) / 4;
    const int64_t blocks = p.rows * sf_cols;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < blocks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / sf_cols, c = i - r * sf_cols;
        const uint2 codes = __ldg(reinterpret_cast<const uint2 *>(p.codes + r * (p.cols / 2) + c * 8));
        const float sb8 = __fmul_rn(f32_from_e4m3(__ldg(p.scales + sf_offset(r, c, sf_cols, col_tiles, p.layout))),
                                    0.125f);
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
        *reinterpret_cast<uint4 *>(p.y + r * p.ld + c * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

}  // namespace nvfp4
