// Block-scaled FP4 GEMM (tcgen05 kind::mxf4nvf4): tiling constants,
// kernel parameters and launch entry points.  Internal to libnvfp4.so.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nvfp4 {

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
    int32_t splits;           // K splits (1 = none); > 1: FP32 slices to `partial`
    float *partial;           // splits x m x n FP32 partial sums (split-K only)
    uint32_t *status;
    long long timeout_cycles;
};

// mx: MXFP4 operands (UE8M0 scales per 32 values, no tensor scales).
cudaError_t launch_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                        int grid, cudaStream_t stream, bool mx = false);

// Dense GEMM on CTA pairs (256x256 tiles); tmB must use 128-row boxes.
cudaError_t launch_gemm_pair(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                             int clusters, cudaStream_t stream);

// Tile order: the CTAs working at one time sweep one operand, which must
// stay in L2.  M fastest sweeps A; when A's codes exceed this many bytes
// and W is the smaller operand, N fastest sweeps W instead.
constexpr int64_t kL2SweepBytes = 48ll << 20;

// Split-K finalize: D = bf16(RN(sum_s partial[s] * alpha)), sums in split
// order; 256 threads.
__global__ void k_splitk_finalize(const float *partial, int splits, int m, int n, const float *ga,
                                  const float *gw, uint16_t *d, int64_t ldd);

// Dense GEMMs with at least this many rows run on CTA pairs.
constexpr int64_t kPairMinRows = 256;

}  // namespace nvfp4
