// Block-scaled FP4 GEMM (tcgen05 kind::mxf4nvf4): tiling constants,
// kernel parameters and launch entry points.  Internal to libnvfp4.so.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// Block-scaled GEMM tiling: 128 x 256 output tile per CTA.
constexpr int kBM = 128;
constexpr int kBN = 256;

// Pipeline of the single-CTA kernel: each stage holds kSK K-values (one TMA
// box row of kSK/2 bytes, 128- or 64-byte swizzle), kNS stages in shared
// memory, and the MMA issuer waits once per kGrp stages.  Measured on B200:
// eight 128-value stages (64-byte swizzle rows) run the FFN GEMM at 0.64 ms
// against 0.41 ms for four 256-value stages, while the MMA itself runs at
// the same rate on either layout (also under 64-byte-box TMA traffic), so
// the loss is in the stage traffic and the default keeps 256-value stages.
#ifndef NVFP4_GEMM_STAGE_K
#define NVFP4_GEMM_STAGE_K 256
#endif
#ifndef NVFP4_GEMM_STAGES
#define NVFP4_GEMM_STAGES 4
#endif
#ifndef NVFP4_GEMM_GROUP
#define NVFP4_GEMM_GROUP 2
#endif
// Block scales into TMEM: 0 = four scale-writer warps read the tiles from
// shared memory and write every lane quarter with tcgen05.st (each warp
// reads all of a stage's 6 KiB); 1 = the MMA issuer copies each 512-byte
// tile once with tcgen05.cp (32x128b, broadcast to the four quarters).
#ifndef NVFP4_GEMM_SF_CP
#define NVFP4_GEMM_SF_CP 0
#endif
constexpr bool kSfCp = NVFP4_GEMM_SF_CP != 0;
constexpr int kSK = NVFP4_GEMM_STAGE_K;
constexpr int kNS = NVFP4_GEMM_STAGES;
constexpr int kGrp = NVFP4_GEMM_GROUP;
constexpr int kKB = kSK / 64;                    // 64-value MMA steps per stage
constexpr int kBoxBytes = kSK / 2;               // TMA box row (bytes of packed codes)
constexpr int kStageA = kBM * kSK / 2;
constexpr int kStageB = kBN * kSK / 2;
constexpr int kStageSFA = kBM * kSK / 16;        // kKB 512-byte 128x4 scale tiles
constexpr int kStageSFB = kBN * kSK / 16;        // two 128-row bands of kKB tiles
constexpr int kStageBytes = kStageA + kStageB + kStageSFA + kStageSFB;
constexpr int kReadyBufs = kNS / kGrp;           // one ready barrier per group slot of the ring
static_assert(kSK == 128 || kSK == 256, "stage K must fill a 64- or 128-byte swizzle row");
static_assert(kNS % kGrp == 0, "stages must form whole groups");
static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
constexpr int kSfWarps = 4;                      // write block scales into TMEM
constexpr int kEpiWarps = 8;                     // two per TMEM lane quarter
constexpr int kMaxGroups = 512;
constexpr int kGemmThreads = 32 * (2 + kSfWarps + kEpiWarps);   // 448
constexpr int kGemmSmemBytes = kNS * kStageBytes + 1024 /*align*/ + 512 /*barriers*/ +
                               2 * (kMaxGroups + 1) * 4 /*group tables*/;
static_assert(kGemmSmemBytes <= 232448, "shared memory per CTA");
static_assert(kBN + kNS * kKB * 12 <= 512, "accumulator + scale columns fit TMEM");

// The CTA-pair kernel keeps 256-value stages (128-byte swizzle rows).
constexpr int kBK = 256;

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
    // when set (grouped NVFP4, unsplit): max |D| over the real rows, as f32
    // bits, atomically maxed into this word (zeroed before the launch)
    uint32_t *out_amax;
    uint32_t *status;
    long long timeout_cycles;
};

// TMA box of the single-CTA kernel's operands: kBoxBytes x rows, swizzled
// to match the MMA descriptors.
constexpr int kSingleBoxBytes = kBoxBytes;
constexpr int kPairBoxBytes = 128;

// mx: MXFP4 operands (UE8M0 scales per 32 values, no tensor scales).
cudaError_t launch_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                        int grid, cudaStream_t stream, bool mx = false);

// Dense GEMM with few rows of A (m <= kSwapMaxRows): W on the MMA's M side,
// A's rows (padded to a multiple of 16) on its N side.  tmW: 128-row boxes of
// W; tmX: boxes of A's padded row count; both 128-byte rows.
constexpr int kSwapMaxRows = 64;
constexpr int kSwapThreads = 32 * (2 + kSfWarps + 4);   // 320
cudaError_t launch_gemm_swap(const CUtensorMap &tmW, const CUtensorMap &tmX, const GemmParams &p,
                             int grid, cudaStream_t stream);

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

// k_splitk_finalize launched with programmatic stream serialization: it is
// scheduled while the split GEMM runs and waits on the device for it.
cudaError_t launch_splitk_finalize(const float *partial, int splits, int m, int n, const float *ga,
                                   const float *gw, uint16_t *d, int64_t ldd, int grid,
                                   cudaStream_t stream);

// Dense GEMMs with at least this many rows run on CTA pairs.
constexpr int64_t kPairMinRows = 256;

}  // namespace nvfp4
