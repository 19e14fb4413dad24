// Kernel parameter blocks and launch entry points shared by the host API
// (api.cu) and the kernel files.  Internal to libnvfp4.so.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm.h"

namespace nvfp4 {

struct EncodeParams {
    const uint16_t *x;      // BF16 source, row pitch ld elements
    int64_t ld;
    int64_t rows, cols;     // output (gathered) shape
    const int32_t *gather;  // optional row map (output row -> source row, -1 = zero row)
    int64_t src_rows;       // rows of x (gathered indices must lie below)
    uint8_t *codes;
    uint8_t *scales;
    int32_t layout;         // 0 swizzled 128x4, 1 linear
    float *global;
    int32_t global_supplied;
    const uint32_t *partials;
    int32_t n_partials;
    uint32_t *status;
    uint32_t rht_mask = 0;  // random Hadamard transform: sign bit j negates value j of a block
    uint64_t sr_seed = 0;   // stochastic rounding: Philox key
};

// Quantize / dequantize work unit: one row and kChunkBlocks consecutive
// 16-value blocks of it per warp task.
constexpr int kChunkBlocks = 128;

// Warp tasks of the encode kernel (rows padded to 128 in the swizzled
// layout; scale columns padded to a multiple of 4): rows of at least
// kChunkBlocks blocks split into chunks of kChunkBlocks, narrower rows into
// 32-block groups.
inline int64_t encode_tasks(int64_t rows, int64_t cols, int32_t layout) {
    const int64_t rows_out = (layout == 0) ? (rows + 127) / 128 * 128 : rows;
    const int64_t groups = ((cols / 16 + 3) / 4 * 4 + 31) / 32;
    return rows_out * (groups >= kChunkBlocks / 32 ? (groups + 3) / 4 : groups);
}

// True when rows are split into 32-block groups (a warp then takes four
// tasks per pass) rather than chunks.
inline bool tasks_are_groups(int64_t cols) {
    return ((cols / 16 + 3) / 4 * 4 + 31) / 32 < kChunkBlocks / 32;
}

// Warp tasks of the dequantize kernel (same split, unpadded).
inline int64_t decode_tasks(int64_t rows, int64_t cols) {
    const int64_t groups = (cols / 16 + 31) / 32;
    return rows * (groups >= kChunkBlocks / 32 ? (groups + 3) / 4 : groups);
}

struct DequantParams {
    const uint8_t *codes;
    const uint8_t *scales;
    int32_t layout;
    const float *global;
    int64_t rows, cols;
    uint16_t *y;
    int64_t ld;
    int32_t y_vec32 = 0;    // 1: y and ld * 2 bytes are 32-byte aligned (one 256-bit store per block)
};

// Row gather of an NVFP4 tensor (gather.cu).
struct GatherParams {
    const uint8_t *src_codes, *src_scales;
    const float *src_global;
    int32_t src_layout;
    int64_t src_rows;
    uint8_t *dst_codes, *dst_scales;
    float *dst_global;
    int32_t dst_layout;
    int64_t rows, cols;      // output rows, columns (values per row)
    const int32_t *map;      // output row -> source row, -1 = zero row
    uint32_t *status;
};
constexpr int kGatherSplit = 2;   // CTAs per 128-row output band (grid.y of k_gather_rows)
__global__ void k_gather_rows(GatherParams p);

__global__ void k_amax(const uint16_t *x, int64_t ld, int64_t rows, int64_t cols,
                       const int32_t *gather, int64_t src_rows, uint32_t *partials,
                       uint32_t *status);
__global__ void k_amax_rht(const uint16_t *x, int64_t ld, int64_t rows, int64_t cols,
                           uint32_t rht_mask, uint32_t *partials);
__global__ void k_finalize_g(const uint32_t *partials, int n, float *global, uint32_t *status);
__global__ void k_encode(EncodeParams p);
__global__ void k_encode_narrow(EncodeParams p);
__global__ void k_encode_rht(EncodeParams p);
__global__ void k_encode_rht_narrow(EncodeParams p);
__global__ void k_encode_sr(EncodeParams p);
__global__ void k_encode_sr_narrow(EncodeParams p);
__global__ void k_encode_rht_sr(EncodeParams p);
__global__ void k_encode_rht_sr_narrow(EncodeParams p);
// Column-wise quantization (out = NVFP4 of x^T): p.rows = columns of x,
// p.cols = rows of x (a multiple of 16), x is p.cols x p.rows with pitch
// p.ld; 128 threads per CTA.
constexpr int kTransposeThreads = 128;
constexpr int kTransposeSmemBytes = (kTransposeThreads / 32) * 2 * 64 * 64 * 2;   // 64 KiB
cudaError_t launch_transpose_kernel(const void *kernel, int grid, void **args, cudaStream_t stream);
__global__ void k_amax_t_rht(const uint16_t *x, int64_t ld, int64_t R, int64_t C, uint32_t rht_mask,
                             uint32_t *partials);
__global__ void k_encode_t(EncodeParams p);
__global__ void k_encode_t_rht(EncodeParams p);
__global__ void k_encode_t_2d(EncodeParams p);
__global__ void k_encode_t_sr(EncodeParams p);
__global__ void k_encode_t_rht_sr(EncodeParams p);
// 2D (16x16 block) row-wise encode: 256 threads; tasks of 16 rows x 256 columns.
__global__ void k_encode_2d(EncodeParams p);
inline int64_t transpose_tasks(int64_t x_rows, int64_t out_rows_padded) {
    return ((x_rows + 63) / 64) * ((out_rows_padded + 63) / 64);
}

// Consumers.  MoE combine: one CTA of 256 threads per token.
constexpr int kMaxTopk = 32;
struct CombineParams {
    const uint16_t *out;     // expert outputs, BF16, pitch ld
    int64_t ld;
    int64_t out_rows;        // rows of out: slots at or past it are skipped
    const int32_t *slots;    // [tokens x topk] rows of out (-1 = none)
    const float *weights;    // [tokens x topk]
    int32_t topk;
    int64_t hidden;
    uint16_t *y;             // [tokens x hidden] BF16, pitch ldy
    int64_t ldy;
};
__global__ void k_moe_combine(CombineParams p);

// NVFP4 -> E4M3 bytes (pitch ld) and the per-tensor factor RN(8 / g).
struct Fp8Params {
    const uint8_t *codes;
    const uint8_t *scales;
    int32_t layout;
    const float *global;
    int64_t rows, cols;
    uint8_t *y;
    int64_t ld;
    float *fp8_scale;
};
__global__ void k_dequantize_fp8(Fp8Params p);

// SiLU-gated activation + quantize: gu = [gate | up] BF16 rows x 2*inter.
struct SwigluParams {
    const uint16_t *gu;
    int64_t ld;
    int64_t rows, inter;
    uint8_t *codes;
    uint8_t *scales;
    int32_t layout;
    float *global;
    uint32_t *partials;
    int32_t n_partials;
    uint32_t *status;
};
__global__ void k_amax_swiglu(SwigluParams p);
__global__ void k_encode_swiglu(SwigluParams p);

// MXFP4 (block 32, UE8M0 scales, no tensor scale); 256 threads.
__global__ void k_encode_mx(EncodeParams p);
__global__ void k_dequantize_mx(DequantParams p);

__global__ void k_dequantize(DequantParams p);
__global__ void k_dequantize_narrow(DequantParams p);

// Decode attention over an NVFP4 KV cache: one query token, grouped query
// heads, head_dim 128, K and V [tokens x heads_kv * 128] in the linear
// scale layout.  Pass 1 (grid chunks x heads_kv, kAttnThreads threads):
// per chunk of tokens and KV head, the running score maximum m, the weight
// sum l and the unnormalised output O of each of the group's query heads.
// Pass 2 (grid heads_q, 128 threads): merge the chunks, o = O / l / g_V.
constexpr int kAttnDim = 128;        // head_dim
constexpr int kAttnMaxGroup = 8;     // query heads per KV head
constexpr int kAttnThreads = 256;
constexpr int kAttnSub = 256;        // tokens per sub-tile (one per thread)
struct AttnParams {
    const uint16_t *q;               // BF16 [heads_q x 128], pitch ldq
    int64_t ldq;
    const uint8_t *kc, *ks;          // K codes [tokens x cols/2], scales [tokens x cols/16]
    const uint8_t *vc, *vs;
    const float *gk, *gv;            // tensor scales
    int64_t tokens, cols;            // cols = heads_kv * 128
    int32_t heads_kv, group;         // heads_q = group * heads_kv
    float scale;                     // softmax scale
    int64_t chunk;                   // tokens per pass-1 CTA, a multiple of kAttnSub
    int32_t n_chunks;
    float *part_o;                   // [n_chunks][heads_q][128]
    float *part_ml;                  // [n_chunks][heads_q][2]: m (log2 units), l
    uint16_t *o;                     // BF16 [heads_q x 128], pitch ldo
    int64_t ldo;
};
__global__ void k_attn_partial(AttnParams p);
__global__ void k_attn_combine(AttnParams p);

}  // namespace nvfp4
