// Row gather of an NVFP4 tensor into MoE expert slots.
//
// Output row r is source row map[r] -- its packed codes and its block scales
// -- or a zero row for map[r] < 0; the tensor scale is copied.  With the
// tensor scale of the whole source, quantizing rows one by one is row-wise
// (a row's codes and scales depend on the row and g only), so gathering the
// quantized rows of x gives exactly the NVFP4 tensor of the gathered rows
// of x ("NVIDIA shrank GLM-5.2 to 4 bits", section 1: the expert linears'
// activations are NVFP4; section 2: each token goes to 8 of 256 experts, so
// a token's row appears 8 times in the expert-grouped batch).  The gather
// moves 0.5625 bytes per value instead of quantizing every copy.
//
// Work unit: one 128-row band of the output (one row of 512-byte tiles in the
// 128x4 scale layout), split over kSplit CTAs.  CTA y of a band copies the
// codes of 128 / kSplit of its rows (a warp per row, 16-byte pieces, eight
// loads in flight per lane) and builds 1 / kSplit of its scale tiles: the
// band's 128 source rows' scale words are staged in shared memory, then each
// warp writes whole 512-byte tiles, so the scattered side of the gather is
// the read (one 4-byte word per source row and tile from 128x4 tiles, whole
// row pieces from linear rows), not the write.  Scales move as words
// of four blocks whenever both layouts allow it (128x4 tiles, or linear rows
// of a multiple of four blocks), else byte by byte.
#include <cstdint>
#include <cuda_runtime.h>

#include "encode_common.cuh"

namespace nvfp4 {

namespace {

constexpr int kSplit = kGatherSplit;   // CTAs per 128-row band
constexpr int kChunk = 32;          // scale words per row staged at once
constexpr int kUnroll = 8;          // code pieces in flight per lane

__device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// One warp per row: lane l moves pieces l, l + 32, ... of the row's codes,
// kUnroll of them in flight.
template <typename V>
__device__ __forceinline__ void copy_code_rows(const GatherParams &p, const int32_t *smap,
                                               int64_t r0, int i_lo, int i_hi, int units) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    for (int i = i_lo + warp; i < i_hi; i += nwarps) {
        const int32_t s = smap[i];
        const V *srow = reinterpret_cast<const V *>(p.src_codes) + (int64_t)(s < 0 ? 0 : s) * units;
        V *drow = reinterpret_cast<V *>(p.dst_codes) + (r0 + i) * units;
        for (int c0 = lane; c0 < units; c0 += 32 * kUnroll) {
            V v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int c = c0 + 32 * u;
                if (s >= 0 && c < units) v[u] = __ldg(srow + c);
                else memset(&v[u], 0, sizeof(V));
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int c = c0 + 32 * u;
                if (c < units) drow[c] = v[u];
            }
        }
    }
}

}  // namespace

__global__ void __launch_bounds__(256) k_gather_rows(GatherParams p) {
    __shared__ int32_t smap[128];
    __shared__ uint32_t sw[128 * (kChunk + 1)];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nwarps = blockDim.x >> 5;
    if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *p.dst_global = *p.src_global;
    const int64_t sf_cols = p.cols / 16;
    const int64_t col_tiles = (sf_cols + 3) / 4;                      // 128x4 tiles per band
    const int64_t code_bytes = p.cols / 2;
    const bool swz_dst = p.dst_layout == 0;
    const int64_t rows_pad = swz_dst ? (p.rows + 127) / 128 * 128 : p.rows;
    const int64_t bands = (rows_pad + 127) / 128;
    const bool words = (p.src_layout == 0 || sf_cols % 4 == 0) &&
                       (p.dst_layout == 0 || sf_cols % 4 == 0);
    const int y = (int)blockIdx.y;
    // This CTA's share of the band's scale words (per row): [w_lo, w_hi).
    const int64_t w_per = (col_tiles + kSplit - 1) / kSplit;
    const int64_t w_lo = imin64(col_tiles, y * w_per);
    const int64_t w_hi = imin64(col_tiles, w_lo + w_per);

    for (int64_t band = blockIdx.x; band < bands; band += gridDim.x) {
        const int64_t r0 = band * 128;
        __syncthreads();                       // the previous band's reads of smem are done
        if (tid < 128) {
            int32_t s = -1;
            if (r0 + tid < p.rows) {
                s = __ldg(p.map + r0 + tid);
                if (s >= p.src_rows) {
                    set_status(p.status, ST_INVALID_ARG);
                    s = -1;
                }
                if (s < 0) s = -1;
            }
            smap[tid] = s;
        }
        __syncthreads();

        // Codes of this CTA's rows of the band that exist.
        const int i_lo = (128 / kSplit) * y;
        const int i_hi = (int)imin64(i_lo + 128 / kSplit, p.rows - r0);
        if (i_hi > i_lo) {
            if (code_bytes % 16 == 0) copy_code_rows<uint4>(p, smap, r0, i_lo, i_hi, (int)(code_bytes / 16));
            else copy_code_rows<uint2>(p, smap, r0, i_lo, i_hi, (int)(code_bytes / 8));
        }

        if (words) {
            for (int64_t w0 = w_lo; w0 < w_hi; w0 += kChunk) {
                const int cw = (int)imin64(kChunk, w_hi - w0);
                __syncthreads();               // the previous chunk's tiles are written
                for (int j = tid; j < 128 * cw; j += blockDim.x) {
                    const int i = j / cw, t = j % cw;
                    const int32_t s = smap[i];
                    uint32_t v = 0;
                    if (s >= 0) {
                        const int64_t off = p.src_layout == 1
                            ? (int64_t)s * sf_cols + 4 * (w0 + t)
                            : sf_offset(s, 4 * (w0 + t), sf_cols, col_tiles, 0);
                        v = __ldg(reinterpret_cast<const uint32_t *>(p.src_scales + off));
                    }
                    sw[i * (kChunk + 1) + t] = v;
                }
                __syncthreads();
                if (swz_dst) {
                    // One warp per 512-byte tile: lane l holds row slot l of the
                    // four 32-row groups (rows l, l+32, l+64, l+96).
                    for (int t = warp; t < cw; t += nwarps) {
                        const uint4 v = make_uint4(sw[lane * (kChunk + 1) + t],
                                                   sw[(lane + 32) * (kChunk + 1) + t],
                                                   sw[(lane + 64) * (kChunk + 1) + t],
                                                   sw[(lane + 96) * (kChunk + 1) + t]);
                        *reinterpret_cast<uint4 *>(p.dst_scales + (band * col_tiles + w0 + t) * 512 +
                                                   16 * lane) = v;
                    }
                } else {
                    for (int j = tid; j < 128 * cw; j += blockDim.x) {
                        const int i = j / cw, t = j % cw;
                        if (r0 + i < p.rows)
                            *reinterpret_cast<uint32_t *>(p.dst_scales + (r0 + i) * sf_cols +
                                                          4 * (w0 + t)) = sw[i * (kChunk + 1) + t];
                    }
                }
            }
        } else {
            // Byte by byte: this CTA's rows of the band, padding included.
            const int64_t ncols = swz_dst ? col_tiles * 4 : sf_cols;
            const int nrows = (int)imin64(128 / kSplit, rows_pad - r0 - (128 / kSplit) * y);
            for (int64_t j = tid; j < (int64_t)max(nrows, 0) * ncols; j += blockDim.x) {
                const int i = (128 / kSplit) * y + (int)(j / ncols);
                const int64_t c = j % ncols;
                const int32_t s = smap[i];
                const uint8_t v = (s < 0 || c >= sf_cols) ? 0
                    : __ldg(p.src_scales + sf_offset(s, c, sf_cols, col_tiles, p.src_layout));
                p.dst_scales[sf_offset(r0 + i, c, sf_cols, col_tiles, p.dst_layout)] = v;
            }
        }
    }
}

}  // namespace nvfp4
