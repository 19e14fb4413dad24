// MXFP4 quantization and dequantization (the format the pages compare
// NVFP4 with: "NVIDIA shrank GLM-5.2 to 4 bits" section 3 -- blocks of 32
// with a power-of-two E8M0 scale; "FP4 KV-cache quantization", section "FP4
// formats compared" -- about 4.25 bits per value).  No tensor scale.
//
// Per 32 consecutive values of a row: X = floor(log2(amax)) - 2 clamped to
// [-127, 127] (the OCP microscaling shared-exponent rule; -127 for an
// all-zero or subnormal-only block), stored as the UE8M0 byte X + 127, and
// codes e2m1_rne_satfinite(x * 2^-X) (the power-of-two product is exact).
//
// Work split: a warp task is one row and 32 consecutive blocks (1024
// values); lane l owns block l (four 16-byte loads, one 16-byte code
// store); lanes 4i..4i+3 combine their scale bytes into one word.
#include <cstdint>
#include <cuda_runtime.h>

#include "encode_common.cuh"

namespace nvfp4 {

namespace {

// X for a block amax given as the f32 bits of a BF16 magnitude.
__device__ __forceinline__ int mx_exponent(uint32_t amax_bits) {
    const int e = (int)(amax_bits >> 23);                 // biased exponent
    if (e == 0) return -127;                              // zero or subnormal
    const int X = (e - 127) - 2;
    return X < -127 ? -127 : (X > 127 ? 127 : X);
}

__device__ __forceinline__ int64_t mx_sf_offset(int64_t r, int64_t c, int64_t sf_cols, int32_t layout) {
    if (layout == 1) return r * sf_cols + c;
    const int64_t tiles = (sf_cols + 3) / 4;
    return ((r >> 7) * tiles + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

}  // namespace

// p.rows x p.cols BF16 -> MXFP4 (codes + UE8M0 scales); p.global unused.
__global__ void __launch_bounds__(kThreads) k_encode_mx(EncodeParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t sf_cols = p.cols / 32, sf_cols4 = (sf_cols + 3) / 4 * 4;
    const int64_t rows_out = (p.layout == 0) ? (p.rows + 127) / 128 * 128 : p.rows;
    const uint32_t segs = (uint32_t)((sf_cols4 + 31) / 32);
    const uint32_t tasks = (uint32_t)rows_out * segs;
    bool finite = true;
    for (uint32_t t = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < tasks;
         t += gridDim.x * (kThreads / 32)) {
        const int64_t row = t / segs;
        const int64_t c = (int64_t)(t % segs) * 32 + lane;          // this lane's block
        uint32_t s = 0;
        if (row < p.rows && c < sf_cols) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(p.x + row * p.ld + c * 32);
            const uint4 v0 = __ldg(xp), v1 = __ldg(xp + 1), v2 = __ldg(xp + 2), v3 = __ldg(xp + 3);
            const uint32_t bits = halves_to_f32bits(max_u16x2(amax_word(v0, v1), amax_word(v2, v3)));
            finite &= bits <= 0x7F7FFFFFu;
            const int X = mx_exponent(bits);
            const float inv = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X, normal
            uint4 out;
            out.x = encode8(v0.x, v0.y, v0.z, v0.w, inv);
            out.y = encode8(v1.x, v1.y, v1.z, v1.w, inv);
            out.z = encode8(v2.x, v2.y, v2.z, v2.w, inv);
            out.w = encode8(v3.x, v3.y, v3.z, v3.w, inv);
            *reinterpret_cast<uint4 *>(p.codes + row * (p.cols / 2) + c * 16) = out;
            s = (uint32_t)(X + 127);
        }
        uint32_t word = s << (8 * (lane & 3));
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        if ((lane & 3) == 0 && c < sf_cols4 && (p.layout == 0 || c < sf_cols)) {
            uint8_t *sp = p.scales + mx_sf_offset(row, c, sf_cols, p.layout);
            if (p.layout == 0 || ((sf_cols & 3) == 0 && c + 4 <= sf_cols)) {
                *reinterpret_cast<uint32_t *>(sp) = word;
            } else {                                                  // ragged linear row
                for (int j = 0; j < 4 && c + j < sf_cols; ++j) sp[j] = (uint8_t)(word >> (8 * j));
            }
        }
    }
    if (!finite) set_status(p.status, ST_NONFINITE);
}

// MXFP4 -> BF16: x_hat = bf16(e2m1(code) * 2^X).
__global__ void __launch_bounds__(kThreads) k_dequantize_mx(DequantParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t sf_cols = p.cols / 32;
    const uint32_t segs = (uint32_t)((sf_cols + 31) / 32);
    const uint32_t tasks = (uint32_t)p.rows * segs;
    for (uint32_t t = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < tasks;
         t += gridDim.x * (kThreads / 32)) {
        const int64_t row = t / segs;
        const int64_t c = (int64_t)(t % segs) * 32 + lane;
        if (c >= sf_cols) continue;
        const uint4 codes = __ldg(reinterpret_cast<const uint4 *>(p.codes + row * (p.cols / 2) + c * 16));
        const uint32_t sb = __ldg(p.scales + mx_sf_offset(row, c, sf_cols, p.layout));
        // 2^(sb - 127) as f32: a normal number down to 2^-126, else subnormal
        const float scale = sb >= 1u ? __uint_as_float(sb << 23) : __uint_as_float(0x00400000u);
        const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
        uint32_t o[16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 v = f32x2_from_f16x2(f16x2_from_e2m1x2((cw[h] >> (8 * i)) & 0xFFu));
                o[4 * h + i] = bf16x2_from_f32(__fmul_rn(v.x, scale), __fmul_rn(v.y, scale));
            }
        }
        uint16_t *yp = p.y + row * p.ld + c * 32;
        store_32b(yp, make_uint4(o[0], o[1], o[2], o[3]), make_uint4(o[4], o[5], o[6], o[7]), p.y_vec32 != 0);
        store_32b(yp + 16, make_uint4(o[8], o[9], o[10], o[11]), make_uint4(o[12], o[13], o[14], o[15]),
                  p.y_vec32 != 0);
    }
}

}  // namespace nvfp4
