// Kernel parameter blocks and launch entry points shared by the host API
// (api.cu) and the kernel files.  Internal to libnvfp4.so.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

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
};

// Block-scaled GEMM tiling: 128 x 256 output tile; each pipeline stage
// holds 256 K-values (one 128-byte swizzle column of packed codes).  The
// MMA issuer takes stages in pairs, synchronising once per eight MMAs.
constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 256;                         // K values per stage
constexpr int kBoxK = 256;                       // K values per TMA box (128 bytes)
constexpr int kStages = 4;
constexpr int kStageA = kBM * kBK / 2;           // 16 KiB
constexpr int kStageB = kBN * kBK / 2;           // 32 KiB
constexpr int kStageSFA = kBM * kBK / 16;        // 2 KiB: four 512-byte 128x4 scale tiles
constexpr int kStageSFB = kBN * kBK / 16;        // 4 KiB: two 128-row bands
constexpr int kStageBytes = kStageA + kStageB + kStageSFA + kStageSFB;
constexpr int kSfWarps = 4;                      // write block scales into TMEM
constexpr int kEpiWarps = 8;                     // two per TMEM lane quarter
constexpr int kMaxGroups = 512;
constexpr int kGemmThreads = 32 * (2 + kSfWarps + kEpiWarps);   // 448
constexpr int kGemmSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 512 /*barriers*/ +
                               2 * (kMaxGroups + 1) * 4 /*group tables*/;

struct GemmParams {
    const uint8_t *sfa;       // A scales, 128x4 layout
    const uint8_t *sfb;       // W scales, 128x4 layout
    uint16_t *d;              // BF16 output
    int64_t ldd;
    int32_t d_vec16;          // 1: D and ldd allow 16-byte stores
    int32_t m;                // dense: rows of A (and D)
    int32_t n;                // columns of D (per group when grouped)
    int32_t k;
    int32_t groups;           // 0 = dense
    const int32_t *slot_offsets;  // grouped: groups+1 padded row offsets
    const int32_t *group_rows;    // grouped: real rows per group
    const float *ga;          // A tensor scale (device)
    const float *gw;          // W tensor scale(s) (device), one per group
    int32_t a_row_blocks;     // ceil(A rows / 128), bounds the grouped slots
    int32_t b_row_blocks;     // ceil(W rows / 128), bounds the SFB reads
    int32_t n_fastest;        // tile order: 0 = M fastest, 1 = N fastest
    uint32_t *status;
    long long timeout_cycles;
};

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
__global__ void k_dequantize(DequantParams p);
__global__ void k_dequantize_narrow(DequantParams p);

cudaError_t launch_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                        int grid, cudaStream_t stream);

// Dense GEMM on CTA pairs (256x256 tiles); tmB must use 128-row boxes.
cudaError_t launch_gemm_pair(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                             int clusters, cudaStream_t stream);

// Tile order: N fastest when A's codes exceed this many bytes and W's do
// not (the operand swept by the CTAs working at one time must stay in L2).
constexpr int64_t kL2SweepBytes = 48ll << 20;

// Dense GEMMs with at least this many rows run on CTA pairs.
constexpr int64_t kPairMinRows = 256;

}  // namespace nvfp4
