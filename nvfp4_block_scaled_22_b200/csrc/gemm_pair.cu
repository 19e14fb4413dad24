// Block-scaled NVFP4 GEMM on CTA pairs (tcgen05 cta_group::2), dense only.
//
// Same arithmetic as the single-CTA kernel in gemm.cu (D = bf16(alpha *
// A_q * W_q^T) with E4M3 scales per 16 values), for the W4A4 linear layer of
// "NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens" (sections "MXFP4
// vs 36% token efficiency and Blackwell speed" and "Four stabilisation
// devices").
//
// Why pairs: a 128x256 tile per SM needs 54 KiB of operands and scales from
// L2 for every 512 tensor-core cycles, which is more than L2 delivers to all
// 148 SMs at once.  Two SMs of a cluster share one 256x256 tile instead:
// each loads its own 128 rows of A and its own 128 rows (half of N) of W, and
// one MMA instruction issued by the leader CTA multiplies across the pair
// (M = 256 split by rows, N = 256 split by W rows), writing each CTA's 128
// accumulator rows into its own TMEM.  Per SM that is 38 KiB per 512 cycles.
//
// Roles per CTA (14 warps):
//   warp 0     TMA producer of this CTA's halves (A box, W box, scale tiles).
//   warps 2-5  scale writers: this CTA's A scales and both W bands into its
//              TMEM with tcgen05.st; after the codes of a stage pair landed
//              they arrive on the leader's `pair_ready`.
//   warp 1     leader only: pair MMAs (kind::mxf4nvf4, M256 N256 K64); commits
//              multicast to both CTAs' `empty` and `acc_full` barriers.
//   warps 6-13 epilogue of this CTA's 128 rows x 256 columns; release by
//              arriving on the leader's `acc_empty`.
// All waits are bounded (NVFP4_ERR_TIMEOUT); a cluster barrier at start and
// end keeps either CTA from touching the other's barriers before they exist
// or after it exits.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr int kPBM = 256;                         // pair tile rows (128 per CTA)
constexpr int kPBN = 256;                         // pair tile columns (W rows, 128 per CTA)
constexpr int kPStages = 5;
constexpr int kPStageA = 128 * kBK / 2;           // 16 KiB
constexpr int kPStageB = 128 * kBK / 2;           // 16 KiB (this CTA's half of N)
constexpr int kPStageSFA = 128 * kBK / 16;        // 2 KiB
constexpr int kPStageSFB = 256 * kBK / 16;        // 4 KiB (both W bands)
constexpr int kPStageBytes = kPStageA + kPStageB + kPStageSFA + kPStageSFB;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kSfCols = 48;
constexpr int kFirstEpiWarp = 2 + kSfWarps;
// Instruction descriptor: E2M1 x E2M1, K-major, N = 256, UE4M3 scales, M = 256.
constexpr uint32_t kIdescPair = (1u << 7) | (1u << 10) | ((uint32_t)(kPBN >> 3) << 17) |
                                ((uint32_t)(kPBM >> 4) << 24);
constexpr long long kDrainCycles = 2000000000ll;

struct PairShared {
    uint64_t tma_ready[kPStages];
    uint64_t sf_landed[kPStages];
    uint64_t empty[kPStages];     // arrived on by the leader's multicast commit
    uint64_t pair_ready[2];       // leader: 4 scale-writer warps per CTA
    uint64_t acc_full;            // arrived on by the leader's multicast commit
    uint64_t acc_empty;           // leader: 8 epilogue warps per CTA
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort_flag;
};

template <bool kCluster>
__device__ __forceinline__ bool pwait(uint64_t *bar, uint32_t parity, PairShared *sh,
                                      const GemmParams &p) {
    // Barriers the other CTA arrives on are waited on like local ones: its
    // arrives carry their own release, and the waits' default acquire pairs
    // with them (the same pattern as for CTA-local barriers).
    (void)kCluster;
    auto test = [&]() { return mbar_try_wait(bar, parity); };
    if (mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (test()) return true;
        if (sh->abort_flag) return false;
        if (clock64() - t0 > p.timeout_cycles) {
            sh->abort_flag = 1;
            set_status(p.status, ST_TIMEOUT);
            return false;
        }
    }
}


// Pair tile order: M fastest, or N fastest when the CTAs running at one time
// should share A's rows and sweep W (the same rule as the single-CTA kernel:
// chosen when A's codes are too large to stay in L2 across a sweep).
__device__ __forceinline__ void pair_tile(int tile, int mtiles, int ntiles, int n_fastest, int &mt,
                                          int &nt) {
    const int fast = n_fastest ? ntiles : mtiles;
    const int q = tile / fast, r = tile - q * fast;
    mt = n_fastest ? q : r;
    nt = n_fastest ? r : q;
}

}  // namespace

constexpr int kPairSmemBytes = kPStages * kPStageBytes + 1024 + 512;
constexpr int kPairThreads = kGemmThreads;

__global__ void __launch_bounds__(kPairThreads, 1)
k_gemm_nvf4_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairShared *sh = reinterpret_cast<PairShared *>(smem + kPStages * kPStageBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&sh->tma_ready[s], 1);
            mbar_init(&sh->sf_landed[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) mbar_init(&sh->pair_ready[j], 2 * kSfWarps);
        mbar_init(&sh->acc_full, 1);
        mbar_init(&sh->acc_empty, 2 * kEpiWarps);
        mbar_init(&sh->drain, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(&sh->tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                 // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    const uint32_t leader_pair_ready0 = mapa_shared(smem_u32(&sh->pair_ready[0]), 0);
    const uint32_t leader_pair_ready1 = mapa_shared(smem_u32(&sh->pair_ready[1]), 0);
    const uint32_t leader_acc_empty = mapa_shared(smem_u32(&sh->acc_empty), 0);

    const int mtiles = (p.m + kPBM - 1) / kPBM;
    const int ntiles = (p.n + kPBN - 1) / kPBN;
    const int tiles = mtiles * ntiles;
    const int cluster = (int)blockIdx.x >> 1;
    const int nclusters = (int)gridDim.x >> 1;
    const int kblocks = p.k / 64;
    const int ktiles = (kblocks + 3) / 4;
    const int64_t sf_rowblock_bytes = (int64_t)kblocks * 512;
    const int my_tiles = cluster < tiles ? (tiles - 1 - cluster) / nclusters + 1 : 0;
    const int total_k = my_tiles * ktiles;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed_phase[kPStages];
            bool armed[kPStages];
            for (int s = 0; s < kPStages; ++s) armed[s] = false;
            bool ok = true;
            for (int tile = cluster; ok && tile < tiles; tile += nclusters) {
                int mt, nt;
                pair_tile(tile, mtiles, ntiles, p.n_fastest, mt, nt);
                const int a_row0 = mt * kPBM + 128 * (int)rank;
                const int b_pair0 = nt * kPBN;
                const int b_row0 = b_pair0 + 128 * (int)rank;
                const int64_t sfa_base = (int64_t)(a_row0 / 128) * sf_rowblock_bytes;
                const int brb = b_pair0 / 128;
                const int halves = (brb + 1 < p.b_row_blocks) ? 2 : 1;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!pwait<false>(&sh->empty[stage], phase ^ 1, sh, p)) { ok = false; break; }
                    const int nkb = min(4, kblocks - 4 * kt);
                    const uint32_t sf_bytes = (uint32_t)nkb * 512;
                    uint8_t *sA = smem + stage * kPStageBytes;
                    uint8_t *sB = sA + kPStageA;
                    uint8_t *sSFA = sB + kPStageB;
                    uint8_t *sSFB = sSFA + kPStageSFA;
                    mbar_arrive_expect_tx(&sh->tma_ready[stage], kPStageA + kPStageB);
                    const bool sfa_ok = a_row0 / 128 < p.a_row_blocks;
                    mbar_arrive_expect_tx(&sh->sf_landed[stage],
                                          sf_bytes * ((sfa_ok ? 1 : 0) + halves));
                    armed[stage] = true;
                    armed_phase[stage] = phase;
                    if (sfa_ok)
                        bulk_load(sSFA, p.sfa + sfa_base + (int64_t)kt * 2048, sf_bytes,
                                  &sh->sf_landed[stage]);
                    for (int h = 0; h < halves; ++h)
                        bulk_load(sSFB + h * 2048,
                                  p.sfb + (int64_t)(brb + h) * sf_rowblock_bytes + (int64_t)kt * 2048,
                                  sf_bytes, &sh->sf_landed[stage]);
                    tma_load_2d(sA, &tmA, &sh->tma_ready[stage], kt * (kBK / 2), a_row0);
                    tma_load_2d(sB, &tmB, &sh->tma_ready[stage], kt * (kBK / 2), b_row0);
                    if (++stage == kPStages) { stage = 0; phase ^= 1; }
                }
            }
            // Let every copy already issued land before the CTA can exit: after
            // an abort (here or in another role) the consumers may never wait
            // on the last stages armed; in a normal run those phases have
            // completed and each check returns at once.
            {
                for (int s = 0; s < kPStages; ++s) {
                    if (!armed[s]) continue;
                    const long long t0 = clock64();
                    while (!mbar_try_wait(&sh->sf_landed[s], armed_phase[s]) &&
                           clock64() - t0 < kDrainCycles) {
                    }
                    while (!mbar_try_wait(&sh->tma_ready[s], armed_phase[s]) &&
                           clock64() - t0 < kDrainCycles) {
                    }
                }
            }
        }
    } else if (warp >= 2 && warp < kFirstEpiWarp) {
        // -------------------------------------------------- scale writers
        // As in the single-CTA kernel: column c of lane i (any quarter) holds
        // the four scales of row 32c+i; A covers this CTA's 128 rows (4
        // columns per K block), W all 256 rows of the pair tile (8 columns).
        const int quarter = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        int stage = 0;
        uint32_t phase = 0;
        for (int g = 0; g < total_k; ++g) {
            if (!pwait<false>(&sh->sf_landed[stage], phase, sh, p)) break;
            const uint8_t *sSFA = smem + stage * kPStageBytes + kPStageA + kPStageB;
            const uint8_t *sSFB = sSFA + kPStageSFA;
            const uint32_t col = lane_base + kAccCols + (uint32_t)stage * kSfCols;
            uint32_t v[16];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const uint4 w = *reinterpret_cast<const uint4 *>(sSFA + 512 * kb + 16 * lane);
                v[4 * kb] = w.x; v[4 * kb + 1] = w.y; v[4 * kb + 2] = w.z; v[4 * kb + 3] = w.w;
            }
            tmem_st_32x32b_x16(col, v);
            uint32_t u[32];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(sSFB + 2048 * h + 512 * kb + 16 * lane);
                    const int o = 8 * kb + 4 * h;
                    u[o] = w.x; u[o + 1] = w.y; u[o + 2] = w.z; u[o + 3] = w.w;
                }
            }
            tmem_st_32x32b_x32(col + 16, u);
            if (!pwait<false>(&sh->tma_ready[stage], phase, sh, p)) break;
            if ((g & 1) || g == total_k - 1) {
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(((g >> 1) & 1) ? leader_pair_ready1 : leader_pair_ready0);
            }
            if (++stage == kPStages) { stage = 0; phase ^= 1; }
        }
        tmem_st_wait();   // no store in flight when TMEM is released (abort path)
    } else if (warp == 1) {
        // -------------------------------------------- MMA (leader CTA only)
        if (lane == 0 && leader) {
            const uint64_t adesc0 = smem_desc(smem_u32(smem), 16, 1024, 2);
            const uint64_t bdesc0 = smem_desc(smem_u32(smem) + kPStageA, 16, 1024, 2);
            const int last_nkb = kblocks - 4 * (ktiles - 1);
            uint32_t acc_phase = 0;
            int stage = 0, kt = 0;
            uint32_t stage_off = 0;
            uint32_t sfa = tmem + kAccCols;
            for (int g = 0; g < total_k; ++g) {
                if ((g & 1) == 0) {
                    const int pj = g >> 1;
                    if (!pwait<true>(&sh->pair_ready[pj & 1], (uint32_t)(pj >> 1) & 1u, sh, p)) break;
                    tc_fence_after();
                }
                if (kt == 0) {
                    if (!pwait<true>(&sh->acc_empty, acc_phase ^ 1, sh, p)) break;
                    tc_fence_after();
                }
                const uint32_t first = kt != 0 ? 1u : 0u;
                if (kt != ktiles - 1 || last_nkb == 4) {
                    mma_nvf4_pair(tmem, adesc0 + stage_off, bdesc0 + stage_off, kIdescPair, sfa, sfa + 16, first);
                    mma_nvf4_pair(tmem, adesc0 + stage_off + 2, bdesc0 + stage_off + 2, kIdescPair, sfa + 4, sfa + 24, 1u);
                    mma_nvf4_pair(tmem, adesc0 + stage_off + 4, bdesc0 + stage_off + 4, kIdescPair, sfa + 8, sfa + 32, 1u);
                    mma_nvf4_pair(tmem, adesc0 + stage_off + 6, bdesc0 + stage_off + 6, kIdescPair, sfa + 12, sfa + 40, 1u);
                } else {
                    for (int kb = 0; kb < last_nkb; ++kb)
                        mma_nvf4_pair(tmem, adesc0 + stage_off + 2 * kb, bdesc0 + stage_off + 2 * kb,
                                      kIdescPair, sfa + 4 * kb, sfa + 16 + 8 * kb,
                                      (kt | kb) != 0 ? 1u : 0u);
                }
                tc_commit_pair(&sh->empty[stage], 0x3);
                if (kt == ktiles - 1) {
                    tc_commit_pair(&sh->acc_full, 0x3);
                    acc_phase ^= 1;
                    kt = 0;
                } else {
                    ++kt;
                }
                if (++stage == kPStages) {
                    stage = 0;
                    stage_off = 0;
                    sfa = tmem + kAccCols;
                } else {
                    stage_off += kPStageBytes / 16;
                    sfa += kSfCols;
                }
            }
            tc_commit_pair(&sh->drain, 0x1);
            const long long t0 = clock64();
            while (!mbar_try_wait(&sh->drain, 0) && clock64() - t0 < kDrainCycles) {
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int chalf = (warp - kFirstEpiWarp) / 4;
        uint32_t acc_phase = 0;
        for (int tile = cluster; tile < tiles; tile += nclusters) {
            int mt, nt;
            pair_tile(tile, mtiles, ntiles, p.n_fastest, mt, nt);
            if (!pwait<false>(&sh->acc_full, acc_phase, sh, p)) break;
            tc_fence_after();
            const float alpha = __frcp_rn(__fmul_rn(*p.ga, *p.gw));
            uint32_t o[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) +
                                       (uint32_t)(chalf * 128 + 32 * c), r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    o[16 * c + i] = bf16x2_from_f32(__fmul_rn(__uint_as_float(r[2 * i]), alpha),
                                                    __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty);
            acc_phase ^= 1;

            // One warp stores its 32 rows x 128 columns; a register transpose
            // makes every store instruction cover one row's 128 bytes.
            const int row0 = mt * kPBM + 128 * (int)rank + quarter * 32;
            const int col0 = nt * kPBN + chalf * 128;
            if (row0 < p.m && col0 < p.n)
                store_rows_coalesced(o, p.d + (int64_t)row0 * p.ldd + col0, p.ldd,
                                     p.m - row0, min(128, p.n - col0), p.d_vec16 != 0, lane);
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();                 // the leader's MMAs into this CTA's TMEM are drained
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

cudaError_t launch_gemm_pair(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                             int clusters, cudaStream_t stream) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_gemm_nvf4_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPairSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_gemm_nvf4_pair, tmA, tmB, p);
}

}  // namespace nvfp4
