// Block-scaled NVFP4 GEMM on the sm_100a tensor cores (tcgen05).
//
//   D[i, j] = bf16( alpha * sum_k e2m1(a_ik) s^A_{i,k/16} * e2m1(w_jk) s^W_{j,k/16} )
//   alpha   = RN(1 / RN(gA * gW))
//
// The W4A4 linear layer of "NVFP4: how NVIDIA pre-trained a 12B model on
// 10T tokens" (sections "MXFP4 vs 36% token efficiency and Blackwell speed"
// and "Four stabilisation devices": Fprop/Dgrad/Wgrad in NVFP4 on the
// Blackwell FP4 tensor cores) and of the MoE expert linears of "NVIDIA
// shrank GLM-5.2 to 4 bits" (section 1, weights and activations in NVFP4;
// section 2, 256 experts with 8 active per token).
//
// Design (one persistent CTA per SM, 6 warps):
//   warp 0   TMA producer: per stage a 128x256 A box and a 256x256 W box of
//            packed codes (128-byte swizzle) plus the matching 128x4 scale
//            tiles by bulk copy, all completing on one mbarrier.
//   warp 1   MMA issuer: copies the stage's scales into TMEM (tcgen05.cp)
//            and issues tcgen05.mma kind::mxf4nvf4 (M128 N256 K64, E4M3
//            scale per 16) into a 128x256 FP32 accumulator in TMEM; commits
//            free the stage and, after the last K step, signal the epilogue.
//   warps 2-5 epilogue: tcgen05.ld the accumulator (each warp its 32-lane
//            quarter), scale by alpha, round to BF16, store with row/column
//            masks, then hand the accumulator back.
// The grouped variant walks (group, M tile, N tile) with the group taken
// from the device-side slot offsets, so no host synchronisation is needed.
// Every mbarrier wait is bounded; a timeout records NVFP4_ERR_TIMEOUT, stops
// all roles, drains in-flight copies and MMAs, and frees TMEM before exit.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = kBN;          // 256 FP32 columns
constexpr uint32_t kSfCols = 48;            // per buffer: 16 (A) + 32 (W)
// tcgen05.mma instruction descriptor, kind::mxf4nvf4: A/B E2M1 (format 1),
// K-major, N = 256 (>> 3), UE4M3 scales (bit 23 = 0), M = 128 (>> 4).
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

struct Shared {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Shared *sh,
                                              const GemmParams &p) {
    if (mbar_try_wait(bar, parity)) return true;
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

struct TileInfo {
    int mt, nt, group;
    int a_row0, b_row0;
    int row_end;      // first row (exclusive) of real output rows for this tile
};

__device__ __forceinline__ TileInfo tile_info(int tile, int mtiles, const GemmParams &p,
                                              const int *s_off, const int *s_rows) {
    TileInfo t;
    t.mt = tile % mtiles;
    t.nt = tile / mtiles;
    t.a_row0 = t.mt * kBM;
    if (p.groups == 0) {
        t.group = 0;
        t.b_row0 = t.nt * kBN;
        t.row_end = p.m;
    } else {
        int lo = 0, hi = p.groups - 1;   // last group whose slot starts at or before a_row0
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (s_off[mid] <= t.a_row0) lo = mid; else hi = mid - 1;
        }
        // skip empty slots that share the same offset
        while (lo + 1 < p.groups && s_off[lo + 1] <= t.a_row0) ++lo;
        t.group = lo;
        t.b_row0 = lo * p.n + t.nt * kBN;
        t.row_end = s_off[lo] + s_rows[lo];
    }
    return t;
}

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm_nvf4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Shared *sh = reinterpret_cast<Shared *>(smem + kStages * kStageBytes);
    int *s_off = reinterpret_cast<int *>(smem + kStages * kStageBytes + 512);
    int *s_rows = s_off + (kMaxGroups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        mbar_init(&sh->acc_full, 1);
        mbar_init(&sh->acc_empty, 4);
        mbar_init(&sh->drain, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (p.groups > 0) {
        for (int i = threadIdx.x; i <= p.groups; i += blockDim.x) s_off[i] = p.slot_offsets[i];
        for (int i = threadIdx.x; i < p.groups; i += blockDim.x) s_rows[i] = p.group_rows[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    if (p.groups > 0 && threadIdx.x == 0) {
        // Offsets must start at 0, rise in multiples of 128 within A's rows,
        // and every group's real rows must fit its slot; else no tile runs.
        bool good = s_off[0] == 0;
        for (int g = 0; g < p.groups && good; ++g)
            good = (s_off[g + 1] % kBM) == 0 && s_off[g + 1] >= s_off[g] && s_rows[g] >= 0 &&
                   s_rows[g] <= s_off[g + 1] - s_off[g];
        good = good && s_off[p.groups] <= p.a_row_blocks * kBM;
        if (!good) {
            set_status(p.status, ST_SHAPE);
            s_off[p.groups] = 0;
        }
    }
    __syncthreads();

    const int mtiles = (p.groups == 0) ? (p.m + kBM - 1) / kBM : s_off[p.groups] / kBM;
    const int ntiles = (p.n + kBN - 1) / kBN;
    const int tiles = mtiles * ntiles;
    const int kblocks = p.k / 64;                    // 64-value MMA steps
    const int ktiles = (kblocks + 3) / 4;
    const int64_t sf_rowblock_bytes = (int64_t)kblocks * 512;   // one 128-row band

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed_phase[kStages];
            bool armed[kStages];
            for (int s = 0; s < kStages; ++s) armed[s] = false;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
                const TileInfo t = tile_info(tile, mtiles, p, s_off, s_rows);
                const int64_t sfa_base = (int64_t)(t.a_row0 / kBM) * sf_rowblock_bytes;
                const int brb = t.b_row0 / kBM;
                const int halves = (brb + 1 < p.b_row_blocks) ? 2 : 1;
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!wait_or_abort(&sh->empty[stage], phase ^ 1, sh, p)) { ok = false; break; }
                    const int nkb = min(4, kblocks - 4 * kt);
                    const uint32_t sf_bytes = (uint32_t)nkb * 512;
                    uint8_t *sA = smem + stage * kStageBytes;
                    uint8_t *sB = sA + kStageA;
                    uint8_t *sSFA = sB + kStageB;
                    uint8_t *sSFB = sSFA + kStageSFA;
                    mbar_arrive_expect_tx(&sh->full[stage],
                                          kStageA + kStageB + sf_bytes * (1 + halves));
                    armed[stage] = true;
                    armed_phase[stage] = phase;
                    tma_load_2d(sA, &tmA, &sh->full[stage], kt * (kBK / 2), t.a_row0);
                    tma_load_2d(sB, &tmB, &sh->full[stage], kt * (kBK / 2), t.b_row0);
                    bulk_load(sSFA, p.sfa + sfa_base + (int64_t)kt * 2048, sf_bytes,
                              &sh->full[stage]);
                    for (int h = 0; h < halves; ++h)
                        bulk_load(sSFB + h * 2048,
                                  p.sfb + (int64_t)(brb + h) * sf_rowblock_bytes + (int64_t)kt * 2048,
                                  sf_bytes, &sh->full[stage]);
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // Let every copy already issued land before the CTA can exit.
                for (int s = 0; s < kStages; ++s) {
                    if (!armed[s]) continue;
                    const long long t0 = clock64();
                    while (!mbar_try_wait(&sh->full[s], armed_phase[s]) &&
                           clock64() - t0 < 2000000000ll) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0, kiter = 0;
            bool ok = true;
            const uint32_t sf_lbo = 0, sf_sbo = 128;    // 8-row x 16-byte core matrices
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
                if (!wait_or_abort(&sh->acc_empty, acc_phase ^ 1, sh, p)) { ok = false; break; }
                tc_fence_after();
                for (int kt = 0; kt < ktiles; ++kt) {
                    if (!wait_or_abort(&sh->full[stage], phase, sh, p)) { ok = false; break; }
                    tc_fence_after();
                    const int nkb = min(4, kblocks - 4 * kt);
                    const uint32_t sA = smem_u32(smem + stage * kStageBytes);
                    const uint32_t sB = sA + kStageA;
                    const uint32_t sSFA = sB + kStageB;
                    const uint32_t sSFB = sSFA + kStageSFA;
                    const uint32_t sfa_col = kAccCols + (kiter & 1) * kSfCols;
                    const uint32_t sfb_col = sfa_col + 16;
                    for (int kb = 0; kb < nkb; ++kb) {
                        tc_cp_32x128b_x4(tmem + sfa_col + 4 * kb,
                                         smem_desc(sSFA + 512 * kb, sf_lbo, sf_sbo, 0));
                        tc_cp_32x128b_x4(tmem + sfb_col + 8 * kb,
                                         smem_desc(sSFB + 512 * kb, sf_lbo, sf_sbo, 0));
                        tc_cp_32x128b_x4(tmem + sfb_col + 8 * kb + 4,
                                         smem_desc(sSFB + 2048 + 512 * kb, sf_lbo, sf_sbo, 0));
                    }
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint64_t ad = smem_desc(sA + 32 * kb, 16, 1024, 2);
                        const uint64_t bd = smem_desc(sB + 32 * kb, 16, 1024, 2);
                        mma_nvf4(tmem, ad, bd, kIdesc, tmem + sfa_col + 4 * kb,
                                 tmem + sfb_col + 8 * kb, (kt | kb) != 0 ? 1u : 0u);
                    }
                    tc_commit(&sh->empty[stage]);
                    ++kiter;
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(&sh->acc_full);
                acc_phase ^= 1;
            }
            // Wait for every issued MMA/copy before TMEM can be released.
            tc_commit(&sh->drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(&sh->drain, 0) && clock64() - t0 < 2000000000ll) {
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;                  // TMEM lane quarter of this warp
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const TileInfo t = tile_info(tile, mtiles, p, s_off, s_rows);
            if (!wait_or_abort(&sh->acc_full, acc_phase, sh, p)) break;
            tc_fence_after();
            const float gw = p.gw[t.group];
            const float alpha = __frcp_rn(__fmul_rn(*p.ga, gw));
            const int row = t.a_row0 + quarter * 32 + lane;
            const bool row_ok = row < t.row_end;
            uint16_t *drow = p.d + (int64_t)row * p.ldd;
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, r);
                tmem_ld_wait();
                const int col = t.nt * kBN + c0;
                if (!row_ok || col >= p.n) continue;
                uint32_t o[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    o[i] = bf16x2_from_f32(__fmul_rn(__uint_as_float(r[2 * i]), alpha),
                                           __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha));
                if (col + 32 <= p.n) {
                    uint4 *dst = reinterpret_cast<uint4 *>(drow + col);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                } else {
                    for (int i = 0; i < 32 && col + i < p.n; ++i)
                        drow[col + i] = (uint16_t)(o[i >> 1] >> (16 * (i & 1)));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty);
            acc_phase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

cudaError_t launch_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                        int grid, cudaStream_t stream) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_gemm_nvf4, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    k_gemm_nvf4<<<grid, kGemmThreads, kGemmSmemBytes, stream>>>(tmA, tmB, p);
    return cudaGetLastError();
}

}  // namespace nvfp4
