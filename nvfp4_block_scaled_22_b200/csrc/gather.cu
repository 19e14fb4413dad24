// Row gather of an NVFP4 tensor into MoE expert slots.
//
// Output row r is source row map[r] -- its packed codes and its block scales
// -- or a zero row for map[r] == -1; the tensor scale is copied.  With the
// tensor scale of the whole source, quantizing rows one by one is row-wise
// (a row's codes and scales depend on the row and g only), so gathering the
// quantized rows of x gives exactly the NVFP4 tensor of the gathered rows
// of x ("NVIDIA shrank GLM-5.2 to 4 bits", section 1: the expert linears'
// activations are NVFP4; section 2: each token goes to 8 of 256 experts, so
// a token's row appears 8 times in the expert-grouped batch).  The gather
// moves 0.5625 bytes per value instead of quantizing every copy.
//
// One warp per output row (grid-stride over the output's rows, including
// the zero padding rows of the 128x4 scale layout): codes in 16-byte (or
// 8-byte) pieces, scales as 4-byte words of four blocks when both tensors
// use the 128x4 layout with whole words, else byte by byte.
#include <cstdint>
#include <cuda_runtime.h>

#include "encode_common.cuh"

namespace nvfp4 {

__global__ void __launch_bounds__(256) k_gather_rows(GatherParams p) {
    const int lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.dst_global = *p.src_global;
    const int64_t sf_cols = p.cols / 16;
    const int64_t col_tiles = (sf_cols + 3) / 4;                      // 128x4 tiles per row band
    const int64_t code_bytes = p.cols / 2;
    const int64_t rows_pad = p.dst_layout == 0 ? (p.rows + 127) / 128 * 128 : p.rows;
    const bool words = p.src_layout == 0 && p.dst_layout == 0;     // 4-scale words on both sides
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < rows_pad;
         r += warps) {
        int64_t src = -1;
        if (r < p.rows) {
            src = __ldg(p.map + r);
            if (src >= p.src_rows) {
                if (lane == 0) set_status(p.status, ST_INVALID_ARG);
                src = -1;
            }
        }
        if (r < p.rows) {
            uint8_t *dst = p.dst_codes + r * code_bytes;
            const uint8_t *s = p.src_codes + (src < 0 ? 0 : src) * code_bytes;
            if (code_bytes % 16 == 0) {
                for (int64_t i = lane; i < code_bytes / 16; i += 32)
                    reinterpret_cast<uint4 *>(dst)[i] =
                        src < 0 ? make_uint4(0, 0, 0, 0) : __ldg(reinterpret_cast<const uint4 *>(s) + i);
            } else {
                for (int64_t i = lane; i < code_bytes / 8; i += 32)
                    reinterpret_cast<uint2 *>(dst)[i] =
                        src < 0 ? make_uint2(0, 0) : __ldg(reinterpret_cast<const uint2 *>(s) + i);
            }
        }
        if (words) {
            const int64_t nwords = (sf_cols + 3) / 4;                 // incl. zero padding columns
            for (int64_t w = lane; w < nwords; w += 32) {
                const uint32_t v = src < 0 ? 0u
                    : __ldg(reinterpret_cast<const uint32_t *>(p.src_scales + sf_offset(src, 4 * w, sf_cols, col_tiles, 0)));
                *reinterpret_cast<uint32_t *>(p.dst_scales + sf_offset(r, 4 * w, sf_cols, col_tiles, 0)) = v;
            }
        } else {
            const int64_t ncols = p.dst_layout == 0 ? (sf_cols + 3) / 4 * 4 : sf_cols;
            for (int64_t c = lane; c < ncols; c += 32) {
                const uint8_t v = (src < 0 || c >= sf_cols) ? 0
                    : __ldg(p.src_scales + sf_offset(src, c, sf_cols, col_tiles, p.src_layout));
                p.dst_scales[sf_offset(r, c, sf_cols, col_tiles, p.dst_layout)] = v;
            }
        }
    }
}

}  // namespace nvfp4
