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
// Design (one persistent CTA per SM, 14 warps, a ring of kNS stages of kSK
// K-values each; gemm.h sets the geometry):
//   warp 0     TMA producer: per stage a 128-row A box and a 256-row W box of
//              packed codes (kSK/2-byte rows, swizzled to match the MMA
//              descriptors) on `tma_ready`, and the matching 512-byte 128x4
//              scale tiles by bulk copy on `sf_landed`.
//   warps 2-5  scale writers, one per 32-lane TMEM quarter.  The tensor core
//              reads block scales from TMEM, and tcgen05.cp spends
//              tensor-pipe time on every instruction, so these warps read
//              their rows of the scale tiles from shared memory and write the
//              MMA's scale layout into TMEM with tcgen05.st.  They also wait
//              for the stage's codes, and arrive on `ready` once per group of
//              kGrp stages, so the MMA issuer synchronises once per group
//              (a completed mbarrier wait costs the issuing thread about as
//              long as one MMA).
//   warp 1     MMA issuer: tcgen05.mma kind::mxf4nvf4 (M128 N256 K64, E4M3
//              scale per 16 values) into a 128x256 FP32 accumulator in TMEM;
//              a commit per stage frees it (and its TMEM scale columns), and
//              a commit after the last K step of a tile wakes the epilogue.
//   warps 6-13 epilogue: two warps per TMEM lane quarter, 128 columns each;
//              tcgen05.ld the accumulator, scale by alpha, round to BF16 in
//              registers, hand the accumulator back at once, then store with
//              row/column masks while the next tile's main loop runs.
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
constexpr uint32_t kSfCols = kKB * 12;      // per stage: kKB K blocks x (4 A + 8 W) columns
constexpr uint32_t kSfbCol0 = kKB * 4;      // W scales after the stage's A scales
// Shared-memory descriptor of a K-major operand in a stage: 128- or 64-byte
// swizzle rows, 8-row groups kBoxBytes * 8 apart.
constexpr uint32_t kSwizzleMode = kBoxBytes == 128 ? 2u : 4u;
constexpr uint32_t kSbo = 8u * kBoxBytes;
constexpr int kFirstEpiWarp = 2 + kSfWarps;
// tcgen05.mma instruction descriptor, kind::mxf4nvf4: A/B E2M1 (format 1),
// K-major, N = 256 (>> 3), UE4M3 scales (bit 23 = 0), M = 128 (>> 4).
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);
// The same for MXFP4 operands: UE8M0 scales (bit 23 = 1), scale vector 2X.
constexpr uint32_t kIdescMx = kIdesc | (1u << 23);
constexpr long long kDrainCycles = 2000000000ll;

struct Shared {
    uint64_t tma_ready[kNS];      // packed codes of the stage landed (tx)
    uint64_t sf_landed[kNS];      // scale tiles of the stage landed (tx)
    uint64_t ready[kReadyBufs];   // every stage of a group loaded, scales in TMEM
    uint64_t empty[kNS];          // MMAs of the stage done (commit)
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Shared *sh,
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

struct TileInfo {
    int mt, nt, group;
    int a_row0, b_row0;
    int row_end;      // first row (exclusive) of real output rows for this tile
};

// Tile order: M fastest (the CTAs working at one time share a few W
// column tiles and sweep all of A, which then has to stay in L2), or, when
// A is large and W is the smaller operand, N fastest (they share a few A
// row tiles and sweep all of W).
__device__ __forceinline__ TileInfo tile_info(int tile, int mtiles, int ntiles,
                                              const GemmParams &p, const int *s_off,
                                              const int *s_rows) {
    TileInfo t;
    const int fast = p.n_fastest ? ntiles : mtiles;
    const int q = tile / fast, r = tile - q * fast;
    t.mt = p.n_fastest ? q : r;
    t.nt = p.n_fastest ? r : q;
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
        t.group = lo;
        t.b_row0 = lo * p.n + t.nt * kBN;
        t.row_end = s_off[lo] + s_rows[lo];
    }
    return t;
}


}  // namespace

// kMx: MXFP4 operands (one UE8M0 scale per 32 values, 512-byte 128x4 tiles
// covering 128 K values; no tensor scales, alpha = 1).  The MMA reads two
// scale bytes per row and K=64 step; the scale writers put them in bytes
// 0-1 of the same TMEM words the NVFP4 path fills with four.
// kSplit: split-K instance (p.splits > 1, dense only); the other instances
// take the whole K range per tile and compile without that bookkeeping.
template <bool kMx, bool kSplit>
__device__ __forceinline__ void gemm_body(const CUtensorMap &tmA, const CUtensorMap &tmB,
                                          const GemmParams &p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Shared *sh = reinterpret_cast<Shared *>(smem + kNS * kStageBytes);
    static_assert(sizeof(Shared) <= 512, "barrier block");
    int *s_off = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(sh) + 512);
    int *s_rows = s_off + (kMaxGroups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&sh->tma_ready[s], 1);
            mbar_init(&sh->sf_landed[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int j = 0; j < kReadyBufs; ++j) mbar_init(&sh->ready[j], kSfWarps);
        mbar_init(&sh->acc_full, 1);
        mbar_init(&sh->acc_empty, kEpiWarps);
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
    // Launched with programmatic stream serialization: the setup above
    // overlaps the previous kernel (e.g. the quantize of A); every global
    // input is read after this wait.
    grid_dependency_wait();
    if (p.groups > 0) {
        for (int i = threadIdx.x; i <= p.groups; i += blockDim.x) s_off[i] = p.slot_offsets[i];
        for (int i = threadIdx.x; i < p.groups; i += blockDim.x) s_rows[i] = p.group_rows[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (kSplit) grid_dependents_launch();   // the finalize may become resident and wait
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
    // Split-K (dense, small M): tile index = split * (mtiles * ntiles) + output
    // tile; split s covers stages [s * ktiles / splits, (s + 1) * ktiles / splits).
    const int tiles_mn = mtiles * ntiles;
    const int splits = kSplit ? p.splits : 1;
    const int tiles = tiles_mn * splits;
    const int kblocks = p.k / 64;                    // 64-value MMA steps
    const int ktiles = (kblocks + kKB - 1) / kKB;    // kSK-value stages
    // one 128-row band of scale tiles; a tile covers 64 (NVFP4) or 128 (MX) K
    const int64_t sf_rowblock_bytes = (int64_t)(kMx ? (kblocks + 1) / 2 : kblocks) * 512;
    constexpr int64_t kSfStageStride = (kMx ? kKB / 2 : kKB) * 512;   // scale bytes per band and stage
    constexpr int kSfBand = kKB * 512;              // smem offset of the second W band
    auto krange = [&](int tile, int &kt0, int &kt1) {
        if (!kSplit) {
            kt0 = 0;
            kt1 = ktiles;
            return;
        }
        const int sp = tile / tiles_mn;
        kt0 = (sp * ktiles) / splits;
        kt1 = ((sp + 1) * ktiles) / splits;
    };
    int total_k = 0;                                  // stages this CTA runs, in order
    if (kSplit) {
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            int a, b;
            krange(tile, a, b);
            total_k += b - a;
        }
    } else {
        total_k = ((int)blockIdx.x < tiles ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0) * ktiles;
    }

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed_phase[kNS];
            bool armed[kNS];
            for (int s = 0; s < kNS; ++s) armed[s] = false;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
                const TileInfo t = tile_info(kSplit ? tile % tiles_mn : tile, mtiles, ntiles, p, s_off, s_rows);
                const int64_t sfa_base = (int64_t)(t.a_row0 / kBM) * sf_rowblock_bytes;
                const int brb = t.b_row0 / kBM;
                const int halves = (brb + 1 < p.b_row_blocks) ? 2 : 1;
                int kt0, kt1;
                krange(tile, kt0, kt1);
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!wait_or_abort(&sh->empty[stage], phase ^ 1, sh, p)) { ok = false; break; }
                    const int nkb = min(kKB, kblocks - kKB * kt);
                    const uint32_t sf_bytes = (uint32_t)(kMx ? (nkb + 1) / 2 : nkb) * 512;
                    uint8_t *sA = smem + stage * kStageBytes;
                    uint8_t *sB = sA + kStageA;
                    uint8_t *sSFA = sB + kStageB;
                    uint8_t *sSFB = sSFA + kStageSFA;
                    mbar_arrive_expect_tx(&sh->tma_ready[stage], kStageA + kStageB);
                    mbar_arrive_expect_tx(&sh->sf_landed[stage], sf_bytes * (1 + halves));
                    armed[stage] = true;
                    armed_phase[stage] = phase;
                    bulk_load(sSFA, p.sfa + sfa_base + (int64_t)kt * kSfStageStride, sf_bytes,
                              &sh->sf_landed[stage]);
                    for (int h = 0; h < halves; ++h)
                        bulk_load(sSFB + h * kSfBand,
                                  p.sfb + (int64_t)(brb + h) * sf_rowblock_bytes +
                                      (int64_t)kt * kSfStageStride,
                                  sf_bytes, &sh->sf_landed[stage]);
                    tma_load_2d(sA, &tmA, &sh->tma_ready[stage], kt * kBoxBytes, t.a_row0);
                    tma_load_2d(sB, &tmB, &sh->tma_ready[stage], kt * kBoxBytes, t.b_row0);
                    if (++stage == kNS) { stage = 0; phase ^= 1; }
                }
            }
            // Let every copy already issued land before the CTA can exit: after
            // an abort (here or in another role) the consumers may never wait
            // on the last stages armed; in a normal run those phases have
            // completed and each check returns at once.
            {
                for (int s = 0; s < kNS; ++s) {
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
        // TMEM scale columns of stage s start at kAccCols + s * kSfCols: A at
        // +4*kb (K block kb), W at +kSfbCol0+8*kb.  Lane i of every 32-lane
        // quarter holds, in column c, the four scales of row 32c+i: exactly
        // row i of the 512-byte 128x4 scale tile (16 bytes = four columns).
        // Every quarter needs the full set, so each writer warp stores all
        // kSfCols columns of its own 32 lanes.
        const int quarter = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        int stage = 0;
        uint32_t phase = 0;
        for (int g = 0; g < total_k; ++g) {
            if (!wait_or_abort(&sh->sf_landed[stage], phase, sh, p)) break;
            if (kSfCp && !kMx) {
                // scales reach TMEM by the MMA issuer's tcgen05.cp: only
                // signal that the stage's codes and scale tiles landed
                if (!wait_or_abort(&sh->tma_ready[stage], phase, sh, p)) break;
                if ((g % kGrp) == kGrp - 1 || g == total_k - 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh->ready[(g / kGrp) % kReadyBufs]);
                }
                if (++stage == kNS) { stage = 0; phase ^= 1; }
                continue;
            }
            const uint8_t *sSFA = smem + stage * kStageBytes + kStageA + kStageB;
            const uint8_t *sSFB = sSFA + kStageSFA;
            const uint32_t col = lane_base + kAccCols + (uint32_t)stage * kSfCols;
            // NVFP4: word q of tile kb is the four scales of row 32q+i for K
            // block kb.  MX: tile kb/2 covers K blocks 2t, 2t+1 with two
            // scales each (bytes 0-1 and 2-3 of the word).
            auto pick = [](uint32_t w, int kb) -> uint32_t {
                return kMx ? (w >> (16 * (kb & 1))) & 0xFFFFu : w;
            };
            uint32_t v[kKB * 4];
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb) {
                const int tile = kMx ? kb / 2 : kb;
                const uint4 w = *reinterpret_cast<const uint4 *>(sSFA + 512 * tile + 16 * lane);
                v[4 * kb] = pick(w.x, kb); v[4 * kb + 1] = pick(w.y, kb);
                v[4 * kb + 2] = pick(w.z, kb); v[4 * kb + 3] = pick(w.w, kb);
            }
            tmem_st_32x32b(col, v);
            uint32_t u[kKB * 8];
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int tile = kMx ? kb / 2 : kb;
                    const uint4 w = *reinterpret_cast<const uint4 *>(sSFB + kSfBand * h + 512 * tile + 16 * lane);
                    const int o = 8 * kb + 4 * h;
                    u[o] = pick(w.x, kb); u[o + 1] = pick(w.y, kb);
                    u[o + 2] = pick(w.z, kb); u[o + 3] = pick(w.w, kb);
                }
            }
            tmem_st_32x32b(col + kSfbCol0, u);
            if (!wait_or_abort(&sh->tma_ready[stage], phase, sh, p)) break;
            if ((g % kGrp) == kGrp - 1 || g == total_k - 1) {
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh->ready[(g / kGrp) % kReadyBufs]);
            }
            if (++stage == kNS) { stage = 0; phase ^= 1; }
        }
        tmem_st_wait();   // no store in flight when TMEM is released (abort path)
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            // Descriptors are linear in the start address (field = address >> 4),
            // so stage s and K block kb are plain additions to the stage-0 value.
            const uint64_t adesc0 = smem_desc(smem_u32(smem), 16, kSbo, kSwizzleMode);
            const uint64_t bdesc0 = smem_desc(smem_u32(smem) + kStageA, 16, kSbo, kSwizzleMode);
            static_assert(kStageBytes % 16 == 0, "stage stride must be 16-byte granular");
            // The tensor pipe queues very few MMAs, so everything between two
            // MMA issues is on the critical path: per-stage bookkeeping below
            // is incremental (no divisions), and the MMA waits once per group.
            const int last_nkb = kblocks - kKB * (ktiles - 1);
            uint32_t acc_phase = 0;
            int stage = 0;
            int mma_tile = blockIdx.x, kt0, kt1;           // current tile and its stage range
            krange(mma_tile, kt0, kt1);
            int kt = kt0;
            uint32_t stage_off = 0;                       // stage * kStageBytes / 16
            uint32_t sfa = tmem + kAccCols;               // stage's TMEM scale columns
            for (int g = 0; g < total_k; ++g) {
                if (g % kGrp == 0) {
                    const int j = g / kGrp;
                    if (!wait_or_abort(&sh->ready[j % kReadyBufs], (uint32_t)(j / kReadyBufs) & 1u, sh, p))
                        break;
                    tc_fence_after();
                }
                if (kt == kt0) {   // first stage of a tile: the accumulator must be free
                    if (!wait_or_abort(&sh->acc_empty, acc_phase ^ 1, sh, p)) break;
                    tc_fence_after();
                }
                const uint32_t first = kt != kt0 ? 1u : 0u;
                if (kSfCp && !kMx) {
                    // this stage's scale tiles: A tile kb -> columns 4kb, W band h
                    // tile kb -> kSfbCol0 + 8kb + 4h; each 512-byte tile is
                    // 32 rows x 16 bytes (no swizzle, 8-row core matrices 128
                    // bytes apart), copied to lanes 0-31 of every quarter
                    const uint32_t sf0 = smem_u32(smem) + (uint32_t)(stage * kStageBytes + kStageA + kStageB);
#pragma unroll
                    for (int kb = 0; kb < kKB; ++kb) {
                        tc_cp_32x128b_x4(sfa + 4 * kb, smem_desc(sf0 + 512 * kb, 128, 128, 0));
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tc_cp_32x128b_x4(sfa + kSfbCol0 + 8 * kb + 4 * h,
                                             smem_desc(sf0 + kStageSFA + kSfBand * h + 512 * kb, 128, 128, 0));
                    }
                }
                auto mma = [&](int kb, uint32_t acc) {
                    if (kMx)
                        mma_mxf4(tmem, adesc0 + stage_off + 2 * kb, bdesc0 + stage_off + 2 * kb,
                                 kIdescMx, sfa + 4 * kb, sfa + kSfbCol0 + 8 * kb, acc);
                    else
                        mma_nvf4(tmem, adesc0 + stage_off + 2 * kb, bdesc0 + stage_off + 2 * kb,
                                 kIdesc, sfa + 4 * kb, sfa + kSfbCol0 + 8 * kb, acc);
                };
                if (kt != ktiles - 1 || last_nkb == kKB) {
                    mma(0, first);
#pragma unroll
                    for (int kb = 1; kb < kKB; ++kb) mma(kb, 1u);
                } else {
                    for (int kb = 0; kb < last_nkb; ++kb) mma(kb, (kt != kt0 || kb != 0) ? 1u : 0u);
                }
                tc_commit(&sh->empty[stage]);
                if (kt == kt1 - 1) {
                    tc_commit(&sh->acc_full);
                    acc_phase ^= 1;
                    mma_tile += gridDim.x;
                    krange(mma_tile, kt0, kt1);
                    kt = kt0;
                } else {
                    ++kt;
                }
                if (++stage == kNS) {
                    stage = 0;
                    stage_off = 0;
                    sfa = tmem + kAccCols;
                } else {
                    stage_off += kStageBytes / 16;
                    sfa += kSfCols;
                }
            }
            // Wait for every issued MMA before TMEM can be released.
            tc_commit(&sh->drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(&sh->drain, 0) && clock64() - t0 < kDrainCycles) {
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;                          // TMEM lane quarter
        const int chalf = (warp - kFirstEpiWarp) / 4;          // column half of the tile
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            if (kSplit) {
                // split-K: this split's FP32 sums, unscaled, into its slice;
                // each lane holds one row (16 columns per TMEM load)
                if (!wait_or_abort(&sh->acc_full, acc_phase, sh, p)) break;
                tc_fence_after();
                const TileInfo t = tile_info(tile % tiles_mn, mtiles, ntiles, p, s_off, s_rows);
                const int row = t.a_row0 + quarter * 32 + lane;
                const int col0 = t.nt * kBN + chalf * 128;
                float *dst = p.partial + ((int64_t)(tile / tiles_mn) * p.m + row) * p.n + col0;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(tmem + ((uint32_t)(quarter * 32) << 16) +
                                           (uint32_t)(chalf * 128 + 16 * c), r);
                    tmem_ld_wait();
                    if (row < p.m && col0 + 16 * c < p.n) {        // n % 16 == 0 in this mode
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            reinterpret_cast<uint4 *>(dst + 16 * c)[q] =
                                make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh->acc_empty);
                acc_phase ^= 1;
                continue;
            }
            // Only alpha is held across the accumulator loads; the tile's
            // coordinates are derived again for the stores (fewer live
            // registers next to the 64 output words).
            const float alpha =
                kMx ? 1.0f
                    : __frcp_rn(__fmul_rn(*p.ga, p.gw[tile_info(tile, mtiles, ntiles, p, s_off, s_rows).group]));
            // Output max wanted (grouped NVFP4, see out_amax): the number of
            // this lane's columns that count (its row must be a real row);
            // -1 when not wanted.
            int amax_lim = -1;
            uint32_t amax_m = 0;
            if (!kMx && !kSplit && p.out_amax != nullptr) {
                const TileInfo ta = tile_info(tile, mtiles, ntiles, p, s_off, s_rows);
                const int ca = ta.nt * kBN + chalf * 128;
                amax_lim = ta.a_row0 + quarter * 32 + lane < ta.row_end ? max(0, min(128, p.n - ca)) : 0;
            }
            if (!wait_or_abort(&sh->acc_full, acc_phase, sh, p)) break;
            tc_fence_after();
            // Four 32-column loads per warp: each wait is a TMEM round trip
            // during which the next tile's MMAs cannot start.
            uint32_t o[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) +
                                       (uint32_t)(chalf * 128 + 32 * c), r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    o[16 * c + i] = bf16x2_from_f32(__fmul_rn(__uint_as_float(r[2 * i]), alpha),
                                                    __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha));
                    // BF16 magnitudes order as their bit patterns (Inf, NaN above all finite)
                    if (2 * (16 * c + i) < amax_lim) amax_m = max_u16x2(amax_m, o[16 * c + i] & 0x7FFF7FFFu);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->acc_empty);    // accumulator free for the next tile
            acc_phase ^= 1;

            const TileInfo t = tile_info(tile, mtiles, ntiles, p, s_off, s_rows);
            // One warp stores its 32 rows x 128 columns; a register transpose
            // makes every store instruction cover one row's 128 bytes.
            const int row0 = t.a_row0 + quarter * 32;
            const int col0 = t.nt * kBN + chalf * 128;
            if (amax_lim >= 0) {
                const uint32_t lo = amax_m & 0xFFFFu, hi = amax_m >> 16;
                const uint32_t v = __reduce_max_sync(0xFFFFFFFFu, (lo > hi ? lo : hi) << 16);
                if (lane == 0 && v != 0u) atomicMax(p.out_amax, v);
            }
            if (row0 < t.row_end && col0 < p.n)
                store_rows_coalesced(o, p.d + (int64_t)row0 * p.ldd + col0, p.ldd,
                                     t.row_end - row0, min(128, p.n - col0), p.d_vec16 != 0, lane);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// D = bf16(RN(RN(sum of the split slices in split order) * alpha)), alpha =
// RN(1 / RN(gA * gW)); four columns per thread (n % 16 == 0).
__global__ void __launch_bounds__(256) k_splitk_finalize(const float *partial, int splits, int m,
                                                         int n, const float *ga, const float *gw,
                                                         uint16_t *d, int64_t ldd) {
    grid_dependency_wait();   // the GEMM that wrote the slices (launched ahead of it)
    const float alpha = __frcp_rn(__fmul_rn(*ga, *gw));
    const int64_t quads = (int64_t)m * (n / 4);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < quads;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / (n / 4), col = (i - row * (n / 4)) * 4;
        float4 acc = __ldg(reinterpret_cast<const float4 *>(partial + row * n + col));
        for (int s = 1; s < splits; ++s) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(partial + ((int64_t)s * m + row) * n + col));
            acc.x = __fadd_rn(acc.x, v.x);
            acc.y = __fadd_rn(acc.y, v.y);
            acc.z = __fadd_rn(acc.z, v.z);
            acc.w = __fadd_rn(acc.w, v.w);
        }
        uint32_t *dp = reinterpret_cast<uint32_t *>(d + row * ldd + col);
        dp[0] = bf16x2_from_f32(__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha));
        dp[1] = bf16x2_from_f32(__fmul_rn(acc.z, alpha), __fmul_rn(acc.w, alpha));
    }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm_nvf4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const GemmParams p) {
    gemm_body<false, false>(tmA, tmB, p);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm_nvf4_splitk(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
    gemm_body<false, true>(tmA, tmB, p);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm_mxf4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const GemmParams p) {
    gemm_body<true, false>(tmA, tmB, p);
}

cudaError_t launch_splitk_finalize(const float *partial, int splits, int m, int n, const float *ga,
                                   const float *gw, uint16_t *d, int64_t ldd, int grid,
                                   cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_splitk_finalize, partial, splits, m, n, ga, gw, d, ldd);
}

cudaError_t launch_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p,
                        int grid, cudaStream_t stream, bool mx) {
    static bool attr_set[64][3] = {};
    const int which = mx ? 1 : (p.splits > 1 ? 2 : 0);
    void (*kernel)(const CUtensorMap, const CUtensorMap, const GemmParams) =
        mx ? k_gemm_mxf4 : (p.splits > 1 ? k_gemm_nvf4_splitk : k_gemm_nvf4);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev][which]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev][which] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = kGemmSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, p);
}

}  // namespace nvfp4
