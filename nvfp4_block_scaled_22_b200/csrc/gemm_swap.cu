// Block-scaled NVFP4 GEMM for few rows of A (M <= 64): the operand roles of
// the tensor-core MMA are swapped, D^T = W_q * A_q^T.
//
// Same arithmetic as the kernel in gemm.cu (D = bf16(alpha * A_q * W_q^T),
// E4M3 scales per 16 values, FP32 accumulation, alpha = RN(1 / RN(gA*gW)))
// for the W4A4 linear layer of "NVFP4: how NVIDIA pre-trained a 12B model on
// 10T tokens" (sections "MXFP4 vs 36% token efficiency and Blackwell speed"
// and "Four stabilisation devices") at decode-like batch sizes, where the
// layer is a stream of the weight matrix from HBM.
//
// Why swap: the MMA's M side is 128 rows.  With A on that side a 16-token
// batch fills 16 of 128 rows, and the 128 x 256 FP32 accumulator must be
// drained before the next tile starts.  With W on the M side every MMA row
// is a real weight row, the tokens are the N side (16..64 columns, a
// multiple of 16), and two tiles' accumulators fit in TMEM at once, so the
// epilogue of one tile overlaps the MMAs of the next.
//
// Work unit = (128-row tile of W, K split).  One persistent CTA per SM walks
// units u = blockIdx.x, += gridDim.x; unit u is tile u % ntiles of split
// u / ntiles, so the CTAs running at one time stream different W tiles and W
// is read from HBM once.  With one split the epilogue writes BF16 directly;
// with several, each split writes its FP32 sums to its own slice of the
// workspace and k_splitk_finalize adds the slices in split order.
//
// Roles (10 warps): warp 0 TMA producer (W box 128 rows x 128 B, A box MP
// rows x 128 B, their 512-byte scale tiles); warp 1 MMA issuer
// (tcgen05.mma kind::mxf4nvf4, M128 N=MP K64); warps 2-5 scale writers (W
// and A scales into TMEM with tcgen05.st); warps 6-9 epilogue, one per TMEM
// lane quarter.  Every wait is bounded; a timeout records
// NVFP4_ERR_TIMEOUT, stops all roles, lets issued copies and MMAs finish and
// frees TMEM.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr int kSwStageW = 128 * 128;              // 16 KiB: 128 W rows x 256 K values
constexpr int kSwStageX = kSwapMaxRows * 128;     // 8 KiB: up to 64 A rows
constexpr int kSwStageSFW = 2048;                 // four 512-byte scale tiles
constexpr int kSwStageSFX = 2048;
constexpr int kSwStageBytes = kSwStageW + kSwStageX + kSwStageSFW + kSwStageSFX;
constexpr int kSwStages = 7;
constexpr int kSwSfCols = 32;                     // per stage: 16 W + 16 A scale columns
constexpr uint32_t kSwAccCols = 2 * kSwapMaxRows; // two accumulator slots
constexpr uint32_t kSwTmemCols = 512;
constexpr int kSwEpiWarps = 4;
constexpr long long kSwDrainCycles = 2000000000ll;
static_assert(kSwStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
static_assert(kSwAccCols + kSwStages * kSwSfCols <= kSwTmemCols, "TMEM columns");
static_assert(kSwStages * kSwStageBytes + 1024 + 512 <= 232448, "shared memory per CTA");

struct SwShared {
    uint64_t tma_ready[kSwStages];
    uint64_t sf_landed[kSwStages];
    uint64_t ready[kSwStages];      // scales of the stage in TMEM and its codes landed
    uint64_t empty[kSwStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort_flag;
};

__device__ __forceinline__ bool sw_wait(uint64_t *bar, uint32_t parity, SwShared *sh,
                                        const GemmParams &p) {
    if (mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (sh->abort_flag) return false;
        if (clock64() - t0 > p.timeout_cycles) {
            sh->abort_flag = 1;
            set_status(p.status, ST_TIMEOUT);
            return false;
        }
    }
}

}  // namespace

// p.m = rows of A (<= kSwapMaxRows), p.n = rows of W; mp = p.m rounded up to
// 16 (the MMA's N).  p.splits >= 1; p.partial when p.splits > 1.
__global__ void __launch_bounds__(kSwapThreads, 1)
k_gemm_nvf4_swap(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SwShared *sh = reinterpret_cast<SwShared *>(smem + kSwStages * kSwStageBytes);
    static_assert(sizeof(SwShared) <= 512, "barrier block");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int mp = (p.m + 15) & ~15;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSwStages; ++s) {
            mbar_init(&sh->tma_ready[s], 1);
            mbar_init(&sh->sf_landed[s], 1);
            mbar_init(&sh->ready[s], kSfWarps);
            mbar_init(&sh->empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sh->acc_full[j], 1);
            mbar_init(&sh->acc_empty[j], kSwEpiWarps);
        }
        mbar_init(&sh->drain, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kSwTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (p.splits > 1) grid_dependents_launch();   // the finalize may become resident and wait
    const uint32_t tmem = sh->tmem_base;

    const int ntiles = (p.n + 127) / 128;
    const int splits = p.splits;
    const int units = ntiles * splits;
    const int kblocks = p.k / 64;
    const int ktiles = (kblocks + 3) / 4;             // 256-value stages
    const int64_t sf_rowblock_bytes = (int64_t)kblocks * 512;
    auto krange = [&](int u, int &kt0, int &kt1) {
        const int sp = u / ntiles;
        kt0 = (sp * ktiles) / splits;
        kt1 = ((sp + 1) * ktiles) / splits;
    };
    int total_k = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        int a, b;
        krange(u, a, b);
        total_k += b - a;
    }

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed_phase[kSwStages];
            bool armed[kSwStages];
            for (int s = 0; s < kSwStages; ++s) armed[s] = false;
            bool ok = true;
            const uint32_t x_bytes = (uint32_t)mp * 128;
            for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
                const int t = u % ntiles;
                int kt0, kt1;
                krange(u, kt0, kt1);
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!sw_wait(&sh->empty[stage], phase ^ 1, sh, p)) { ok = false; break; }
                    const int nkb = min(4, kblocks - 4 * kt);
                    const uint32_t sf_bytes = (uint32_t)nkb * 512;
                    uint8_t *sW = smem + stage * kSwStageBytes;
                    uint8_t *sX = sW + kSwStageW;
                    uint8_t *sSFW = sX + kSwStageX;
                    uint8_t *sSFX = sSFW + kSwStageSFW;
                    mbar_arrive_expect_tx(&sh->tma_ready[stage], kSwStageW + x_bytes);
                    mbar_arrive_expect_tx(&sh->sf_landed[stage], 2 * sf_bytes);
                    armed[stage] = true;
                    armed_phase[stage] = phase;
                    bulk_load(sSFW, p.sfb + (int64_t)t * sf_rowblock_bytes + (int64_t)kt * 2048, sf_bytes,
                              &sh->sf_landed[stage]);
                    bulk_load(sSFX, p.sfa + (int64_t)kt * 2048, sf_bytes, &sh->sf_landed[stage]);
                    tma_load_2d(sW, &tmW, &sh->tma_ready[stage], kt * 128, t * 128);
                    tma_load_2d(sX, &tmX, &sh->tma_ready[stage], kt * 128, 0);
                    if (++stage == kSwStages) { stage = 0; phase ^= 1; }
                }
            }
            // Every issued copy lands before the CTA can exit (a no-op unless
            // some role aborted before consuming the last stages).
            for (int s = 0; s < kSwStages; ++s) {
                if (!armed[s]) continue;
                const long long t0 = clock64();
                while (!mbar_try_wait(&sh->sf_landed[s], armed_phase[s]) &&
                       clock64() - t0 < kSwDrainCycles) {
                }
                while (!mbar_try_wait(&sh->tma_ready[s], armed_phase[s]) &&
                       clock64() - t0 < kSwDrainCycles) {
                }
            }
        }
    } else if (warp >= 2 && warp < 2 + kSfWarps) {
        // -------------------------------------------------- scale writers
        // Stage s's scale columns start at kSwAccCols + s * kSwSfCols: W (the
        // MMA's A side) at +4*kb, A rows (its B side) at +16+4*kb.  Lane i of
        // each 32-lane quarter holds in column c the four scales of row
        // 32c+i: row i of the 512-byte 128x4 tile; every quarter gets all.
        const int quarter = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        int stage = 0;
        uint32_t phase = 0;
        for (int g = 0; g < total_k; ++g) {
            if (!sw_wait(&sh->sf_landed[stage], phase, sh, p)) break;
            const uint8_t *sSFW = smem + stage * kSwStageBytes + kSwStageW + kSwStageX;
            const uint8_t *sSFX = sSFW + kSwStageSFW;
            const uint32_t col = lane_base + kSwAccCols + (uint32_t)stage * kSwSfCols;
            uint32_t v[16], u[16];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const uint4 w = *reinterpret_cast<const uint4 *>(sSFW + 512 * kb + 16 * lane);
                const uint4 x = *reinterpret_cast<const uint4 *>(sSFX + 512 * kb + 16 * lane);
                v[4 * kb] = w.x; v[4 * kb + 1] = w.y; v[4 * kb + 2] = w.z; v[4 * kb + 3] = w.w;
                u[4 * kb] = x.x; u[4 * kb + 1] = x.y; u[4 * kb + 2] = x.z; u[4 * kb + 3] = x.w;
            }
            tmem_st_32x32b(col, v);
            tmem_st_32x32b(col + 16, u);
            if (!sw_wait(&sh->tma_ready[stage], phase, sh, p)) break;
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->ready[stage]);
            if (++stage == kSwStages) { stage = 0; phase ^= 1; }
        }
        tmem_st_wait();
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            // tcgen05.mma kind::mxf4nvf4: A/B E2M1, K-major, N = mp, UE4M3
            // scales, M = 128.
            const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(mp >> 3) << 17) |
                                   ((uint32_t)(128 >> 4) << 24);
            const uint64_t wdesc0 = smem_desc(smem_u32(smem), 16, 1024, 2);
            const uint64_t xdesc0 = smem_desc(smem_u32(smem) + kSwStageW, 16, 1024, 2);
            const int last_nkb = kblocks - 4 * (ktiles - 1);
            int stage = 0;
            uint32_t phase = 0;
            int unit = blockIdx.x, j = 0, kt0, kt1;       // j: unit count of this CTA
            krange(unit, kt0, kt1);
            int kt = kt0;
            for (int g = 0; g < total_k; ++g) {
                if (!sw_wait(&sh->ready[stage], phase, sh, p)) break;
                tc_fence_after();
                const int slot = j & 1;
                if (kt == kt0) {   // first stage of a unit: its accumulator slot must be free
                    if (!sw_wait(&sh->acc_empty[slot], ((uint32_t)(j >> 1) & 1u) ^ 1u, sh, p)) break;
                    tc_fence_after();
                }
                const uint32_t acc = tmem + (uint32_t)(slot * kSwapMaxRows);
                const uint32_t sfc = tmem + kSwAccCols + (uint32_t)stage * kSwSfCols;
                const uint32_t off = (uint32_t)(stage * kSwStageBytes / 16);
                const int nkb = (kt == ktiles - 1) ? last_nkb : 4;
                for (int kb = 0; kb < nkb; ++kb)
                    mma_nvf4(acc, wdesc0 + off + 2 * kb, xdesc0 + off + 2 * kb, idesc, sfc + 4 * kb,
                             sfc + 16 + 4 * kb, (kt != kt0 || kb != 0) ? 1u : 0u);
                tc_commit(&sh->empty[stage]);
                if (kt == kt1 - 1) {
                    tc_commit(&sh->acc_full[slot]);
                    ++j;
                    unit += gridDim.x;
                    krange(unit, kt0, kt1);
                    kt = kt0;
                } else {
                    ++kt;
                }
                if (++stage == kSwStages) { stage = 0; phase ^= 1; }
            }
            tc_commit(&sh->drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(&sh->drain, 0) && clock64() - t0 < kSwDrainCycles) {
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        // Lane l of quarter q holds W row 32q + l of the tile (output column
        // j) and, in TMEM column c of its slot, token row c.
        const int quarter = warp & 3;
        const float alpha = __frcp_rn(__fmul_rn(*p.ga, *p.gw));
        int j = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++j) {
            const int slot = j & 1;
            if (!sw_wait(&sh->acc_full[slot], (uint32_t)(j >> 1) & 1u, sh, p)) break;
            tc_fence_after();
            const int t = u % ntiles, sp = u / ntiles;
            const int col = t * 128 + quarter * 32 + lane;
            const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(slot * kSwapMaxRows);
            uint32_t r[kSwapMaxRows];
#pragma unroll
            for (int c = 0; c < kSwapMaxRows / 16; ++c) {
                if (16 * c < mp) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(base + 16 * c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[16 * c + i] = v[i];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty[slot]);
            if (col < p.n) {
                if (splits > 1) {
                    float *dst = p.partial + (int64_t)sp * p.m * p.n + col;
#pragma unroll
                    for (int i = 0; i < kSwapMaxRows; ++i)
                        if (i < p.m) dst[(int64_t)i * p.n] = __uint_as_float(r[i]);
                } else {
                    uint16_t *dst = p.d + col;
#pragma unroll
                    for (int i = 0; i < kSwapMaxRows; ++i)
                        if (i < p.m)
                            dst[(int64_t)i * p.ldd] = (uint16_t)bf16x2_from_f32(
                                __fmul_rn(__uint_as_float(r[i]), alpha), 0.0f);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kSwTmemCols);
    }
}

cudaError_t launch_gemm_swap(const CUtensorMap &tmW, const CUtensorMap &tmX, const GemmParams &p,
                             int grid, cudaStream_t stream) {
    constexpr int smem_bytes = kSwStages * kSwStageBytes + 1024 + 512;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_gemm_nvf4_swap, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_bytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    k_gemm_nvf4_swap<<<grid, kSwapThreads, smem_bytes, stream>>>(tmW, tmX, p);
    return cudaGetLastError();
}

}  // namespace nvfp4
