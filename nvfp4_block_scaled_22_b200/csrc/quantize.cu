// NVFP4 two-level quantization and dequantization kernels (sm_100a).
//
// Method ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens",
// section "E2M1 format and two-level scaling"; "NVIDIA shrank GLM-5.2 to 4
// bits", section 3): an FP32 scale per tensor g = 448*6/amax, then per 16
// consecutive values along a row an E4M3 scale s = e4m3(amax_b/6*g) that
// maps the block amax close to the E2M1 maximum 6, and the 4-bit codes
// e2m1(x * g/s).  Every float step is one IEEE RN operation (no fast-math,
// no FMA contraction, no flush-to-zero) so codes and scales are exact.
//
// Kernels
//   k_amax        : per-CTA max|x| over whole rows (optionally gathered).
//   k_amax_rht    : the same over the random-Hadamard-transformed blocks.
//   k_finalize_g  : partial maxima -> g, error status (nvfp4_global_scale).
//   k_encode      : g (from partials or supplied) -> codes + scales; the
//                   kRht instance transforms each block first.
//   k_dequantize  : codes + scales + g -> BF16.
//
// Work split of k_encode/k_dequantize: a warp task is a 2048-value chunk of
// one row (narrow rows: a 32-block group), one 16-value block per lane per
// step, so every global access of a warp is contiguous (see the comment
// above TaskWalk).  Shared block-level helpers: encode_common.cuh.
#include <cstdint>
#include <cuda_runtime.h>

#include "encode_common.cuh"

namespace nvfp4 {

// ---------------------------------------------------------------- k_amax
// One warp per row (grid-stride over rows), 16-byte loads.  Writes the
// CTA's max|x| as f32 bits (Inf/NaN compare above every finite value).
__global__ void __launch_bounds__(kThreads) k_amax(const uint16_t *__restrict__ x, int64_t ld,
                                                   int64_t rows, int64_t cols,
                                                   const int32_t *__restrict__ gather,
                                                   int64_t src_rows,
                                                   uint32_t *__restrict__ partials,
                                                   uint32_t *status) {
    __shared__ uint32_t red[kThreads / 32];
    grid_dependents_launch();   // the encode pass may be scheduled and wait on the device
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t chunks = cols / 8;  // 16-byte chunks per row
    uint32_t m = 0;
    for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        int64_t src = r;
        if (gather != nullptr) {
            src = gather[r];
            if (src < 0) continue;
            if (src >= src_rows) {           // row map points outside x
                if (lane == 0) set_status(status, ST_INVALID_ARG);
                continue;
            }
        }
        const uint4 *p = reinterpret_cast<const uint4 *>(x + src * ld);
        int64_t c = lane;
        for (; c + 96 < chunks; c += 128) {
            uint4 a = __ldg(p + c), b = __ldg(p + c + 32), d = __ldg(p + c + 64),
                  e = __ldg(p + c + 96);
            m = max_u16x2(m, max_u16x2(amax_word(a, b), amax_word(d, e)));
        }
        for (; c < chunks; c += 32) {
            uint4 a = __ldg(p + c);
            m = max_u16x2(m, amax_word(a, a));
        }
    }
    uint32_t v = block_reduce_max(halves_to_f32bits(m), red);
    if (threadIdx.x == 0) partials[blockIdx.x] = v;
}

// ------------------------------------------------------------ k_amax_rht
// One warp per row, one 16-value block per lane (a warp reads 1 KiB
// contiguous per step); the block is transformed in registers and the max
// of |y| over the CTA is written as f32 bits, the format k_amax writes.
__global__ void __launch_bounds__(kThreads) k_amax_rht(const uint16_t *__restrict__ x, int64_t ld,
                                                       int64_t rows, int64_t cols,
                                                       uint32_t rht_mask,
                                                       uint32_t *__restrict__ partials) {
    __shared__ uint32_t red[kThreads / 32];
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t blocks = cols / 16;
    const SignFlips f = sign_flips(rht_mask);
    uint32_t m = 0;
    for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x + r * ld);
        int64_t c = lane;
        for (; c + 32 < blocks; c += 64) {
            uint4 a0 = __ldg(p + 2 * c), b0 = __ldg(p + 2 * c + 1);
            uint4 a1 = __ldg(p + 2 * c + 64), b1 = __ldg(p + 2 * c + 65);
            m = max(m, rht16_abs_max_bits(a0, b0, f));
            m = max(m, rht16_abs_max_bits(a1, b1, f));
        }
        if (c < blocks) m = max(m, rht16_abs_max_bits(__ldg(p + 2 * c), __ldg(p + 2 * c + 1), f));
    }
    uint32_t v = block_reduce_max(m, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = v;
}

__global__ void k_finalize_g(const uint32_t *__restrict__ partials, int n, float *global,
                             uint32_t *status) {
    __shared__ uint32_t red[kThreads / 32];
    float g;
    if (global_from_partials(partials, n, status, &g, red) && threadIdx.x == 0) *global = g;
}

// Work split: a task is one row and one chunk of kChunkBlocks = 128
// consecutive 16-value blocks (2048 values) of it; lane l owns blocks
// l, l + 32, l + 64, l + 96 of the chunk (two 16-byte loads and one 8-byte
// code store each), so every load and store instruction of a warp is
// contiguous, and the row's addresses are formed once per task.  The four
// scale bytes of blocks 4i..4i+3 are contiguous in both scale layouts;
// lanes 4i..4i+3 combine them with two shuffles and lane 4i stores the
// word.  Rows past the end of the last 128-row band (swizzled layout) and
// scale columns past cols/16 up to the next multiple of 4 are written as
// zero.
constexpr int kUnroll = kChunkBlocks / 32;

// Row of flat task t (tasks laid out row-major, segs per row) without a
// 64-bit division: float reciprocal, then exact integer correction.
__device__ __forceinline__ uint32_t task_row(uint32_t t, uint32_t segs, float inv) {
    uint32_t r = __float2uint_rz((float)t * inv);
    while (r * segs > t) --r;
    while ((r + 1) * segs <= t) ++r;
    return r;
}

// The tasks a warp takes, t, t + stride, t + 2 stride, ..., as (row,
// chunk) pairs of the row-major task grid (chunks per row): one division
// for the first task, then an add with carry per step.
struct TaskWalk {
    uint32_t row, seg, segs, step_rows, step_segs;
    __device__ __forceinline__ TaskWalk(uint32_t t, uint32_t stride, uint32_t segs_)
        : row(t / segs_), seg(t - (t / segs_) * segs_), segs(segs_), step_rows(stride / segs_),
          step_segs(stride - (stride / segs_) * segs_) {}
    __device__ __forceinline__ void next() {
        seg += step_segs;
        row += step_rows;
        if (seg >= segs) {
            seg -= segs;
            ++row;
        }
    }
};

// Shape constants of one encode launch.
struct EncodeShape {
    int64_t sf_cols, sf_cols4, col_tiles, rows_out, sf_step;
};

// Block column c of one row: quantize it (or write zero codes for a
// gathered padding row), store its codes at cp, and let lanes 4i store the
// scale word of blocks 4i..4i+3 at sp.  Every lane of the warp takes part
// (two shuffles).
template <bool kRht, bool kSR>
__device__ __forceinline__ void emit_block(const EncodeParams &p, const EncodeShape &sh,
                                           const SignFlips &flips, float g, const EncodeTables &tab,
                                           bool real, bool load, int64_t c, uint4 a, uint4 b,
                                           const BlockDraws &r, uint2 *cp, uint8_t *sp, int lane,
                                           bool &finite) {
    uint32_t s = 0;
    if (real && c < sh.sf_cols) {
        if (load) {
            EncodeBlockOut o = encode_any<kRht, kSR>(a, b, flips, g, tab, r);
            finite &= o.finite;
            s = o.scale;
            *cp = o.codes;
        } else {                                                      // gathered padding row
            *cp = make_uint2(0, 0);
        }
    }
    uint32_t word = s << (8 * (lane & 3));
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
    if ((lane & 3) == 0 && c < sh.sf_cols4 && (p.layout == 0 || c < sh.sf_cols)) {
        if (p.layout == 0 || ((sh.sf_cols & 3) == 0 && c + 4 <= sh.sf_cols)) {
            *reinterpret_cast<uint32_t *>(sp) = word;
        } else {                                                      // ragged linear row
            for (int i = 0; i < 4 && c + i < sh.sf_cols; ++i) sp[i] = (uint8_t)(word >> (8 * i));
        }
    }
}

// Source row of output row `row` (gathered or not); load = false for band
// padding rows, gathered padding rows (-1) and invalid map entries.  `mapped`
// is the row map's entry for `row`, already loaded by the caller.
__device__ __forceinline__ int64_t source_row(const EncodeParams &p, int64_t row, int32_t mapped,
                                              bool &real, bool &load) {
    real = row < p.rows;
    load = real;
    int64_t src = row;
    if (real && p.gather != nullptr) {
        src = mapped;
        if (src >= p.src_rows) {             // out-of-range map entry: zero row + status
            set_status(p.status, ST_INVALID_ARG);
            src = -1;
        }
        load = src >= 0;
    }
    return load ? src : 0;
}

template <bool kRht, bool kNarrow, bool kSR>
__device__ __forceinline__ void encode_body(const EncodeParams &p) {
    __shared__ uint32_t red[kThreads / 32];
    __shared__ EncodeTables tab;
    // Launched with programmatic stream serialization after the amax pass:
    // let the next kernel (the GEMM) be scheduled as this grid drains, and
    // wait for the previous kernel's partial maxima before reading them.
    grid_dependents_launch();
    grid_dependency_wait();
    float g;
    if (p.global_supplied) {
        g = *p.global;
    } else {
        if (!global_from_partials(p.partials, p.n_partials, p.status, &g, red)) return;
        if (blockIdx.x == 0 && threadIdx.x == 0) *p.global = g;
    }
    fill_tables(tab, g);
    __syncthreads();
    const SignFlips flips = sign_flips(kRht ? p.rht_mask : 0u);
    const int lane = threadIdx.x & 31;
    EncodeShape sh;
    sh.sf_cols = p.cols / 16;
    sh.sf_cols4 = (sh.sf_cols + 3) / 4 * 4;                        // padded scale columns
    sh.col_tiles = sh.sf_cols4 / 4;
    sh.rows_out = (p.layout == 0) ? (p.rows + 127) / 128 * 128 : p.rows;
    sh.sf_step = (p.layout == 0) ? 4096 : 32;                      // scale bytes per 32 blocks
    const uint32_t groups = (uint32_t)((sh.sf_cols4 + 31) / 32);   // 32-block groups per row
    const uint32_t warps = gridDim.x * (kThreads / 32);
    const uint32_t warp_id = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (groups == 0) return;                                       // no columns
    bool finite = true;
    if (!kNarrow) {
        // Wide rows: a task is kChunkBlocks consecutive blocks of one row,
        // lane l taking blocks l, l+32, l+64, l+96; addresses once per task.
        // With a row map, the next task's map entry is loaded one task ahead
        // so that its latency overlaps this task's loads.
        const uint32_t chunks = (groups + kUnroll - 1) / kUnroll;
        TaskWalk w(warp_id, warps, chunks);
        int32_t map_next = (p.gather != nullptr && w.row < p.rows) ? __ldg(p.gather + w.row) : 0;
        for (; w.row < sh.rows_out; w.next()) {
            const int64_t row = w.row;
            const int32_t mapped = map_next;
            if (p.gather != nullptr) {
                TaskWalk nx = w;
                nx.next();
                if (nx.row < p.rows) map_next = __ldg(p.gather + nx.row);
            }
            const int64_t c0 = (int64_t)w.seg * kChunkBlocks + lane;   // this lane's first block
            bool real, load;
            const int64_t src = source_row(p, row, mapped, real, load);
            const uint4 *xp = reinterpret_cast<const uint4 *>(p.x + src * p.ld + c0 * 16);
            uint4 va[kUnroll], vb[kUnroll];
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                if (load && c0 + 32 * j < sh.sf_cols) {
                    va[j] = __ldg(xp + 64 * j);
                    vb[j] = __ldg(xp + 64 * j + 1);
                }
            }
            // stochastic rounding: all draws of the task first (independent
            // Philox chains, so their latencies overlap)
            BlockDraws rnd[kUnroll];
            if (kSR) {
#pragma unroll
                for (int j = 0; j < kUnroll; ++j)
                    rnd[j] = block_draws(p.sr_seed, (uint64_t)row * (uint64_t)sh.sf_cols +
                                                        (uint64_t)(c0 + 32 * j));
            }
            uint2 *cp = reinterpret_cast<uint2 *>(p.codes + row * (p.cols / 2) + c0 * 8);
            uint8_t *sp = p.scales + sf_offset(row, c0, sh.sf_cols, sh.col_tiles, p.layout);
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                if (c0 - lane + 32 * j >= sh.sf_cols4) break;           // uniform across the warp
                emit_block<kRht, kSR>(p, sh, flips, g, tab, real, load, c0 + 32 * j, va[j], vb[j],
                                      rnd[j], cp + 32 * j, sp + sh.sf_step * j, lane, finite);
            }
        }
    } else {
        // Narrow rows (fewer than 128 blocks): a task is one 32-block group
        // of one row (lane l owns block l); a warp keeps kUnroll tasks in
        // flight, tasks t0, t0 + warps, ... of the row-major task grid.
        const uint32_t tasks = (uint32_t)(sh.rows_out * groups);   // < 2^32 (host-checked)
        const float inv_groups = 1.0f / (float)groups;
        for (uint32_t t0 = warp_id; t0 < tasks; t0 += warps * kUnroll) {
            uint4 va[kUnroll], vb[kUnroll];
            int64_t rr[kUnroll], bb[kUnroll];
            bool has[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const uint32_t t = t0 + warps * u;
                const uint32_t row = task_row(t, groups, inv_groups);
                rr[u] = row;
                bb[u] = (int64_t)(t - row * groups) * 32 + lane;   // scale column of this lane
                int64_t src = rr[u];
                has[u] = t < tasks && rr[u] < p.rows && bb[u] < sh.sf_cols;
                if (has[u] && p.gather != nullptr) {
                    src = p.gather[rr[u]];
                    if (src >= p.src_rows) {     // out-of-range map entry: zero row + status
                        set_status(p.status, ST_INVALID_ARG);
                        src = -1;
                    }
                    if (src < 0) has[u] = false;
                }
                if (has[u]) {
                    const uint4 *xp = reinterpret_cast<const uint4 *>(p.x + src * p.ld + bb[u] * 16);
                    va[u] = __ldg(xp);
                    vb[u] = __ldg(xp + 1);
                }
            }
            BlockDraws rnd[kUnroll];
            if (kSR) {
#pragma unroll
                for (int u = 0; u < kUnroll; ++u)
                    rnd[u] = block_draws(p.sr_seed, (uint64_t)rr[u] * (uint64_t)sh.sf_cols + (uint64_t)bb[u]);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const uint32_t t = t0 + warps * u;
                if (t >= tasks) break;                               // uniform across the warp
                uint32_t s = 0;
                if (has[u]) {
                    EncodeBlockOut o = encode_any<kRht, kSR>(va[u], vb[u], flips, g, tab, rnd[u]);
                    finite &= o.finite;
                    s = o.scale;
                    *reinterpret_cast<uint2 *>(p.codes + rr[u] * (p.cols / 2) + bb[u] * 8) = o.codes;
                } else if (rr[u] < p.rows && bb[u] < sh.sf_cols) {      // gathered padding row
                    *reinterpret_cast<uint2 *>(p.codes + rr[u] * (p.cols / 2) + bb[u] * 8) =
                        make_uint2(0, 0);
                }
                uint32_t w = s << (8 * (lane & 3));
                w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
                w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
                if ((lane & 3) == 0 && bb[u] < sh.sf_cols4 && (p.layout == 0 || bb[u] < sh.sf_cols)) {
                    uint8_t *sp = p.scales + sf_offset(rr[u], bb[u], sh.sf_cols, sh.col_tiles, p.layout);
                    if (p.layout == 0 || ((sh.sf_cols & 3) == 0 && bb[u] + 4 <= sh.sf_cols)) {
                        *reinterpret_cast<uint32_t *>(sp) = w;
                    } else {                                         // ragged linear row
                        for (int j = 0; j < 4 && bb[u] + j < sh.sf_cols; ++j)
                            sp[j] = (uint8_t)(w >> (8 * j));
                    }
                }
            }
        }
    }
    if (!finite) set_status(p.status, ST_NONFINITE);   // only reachable with a supplied g
}

// The host launches the *_narrow kernels for rows of fewer than
// kChunkBlocks blocks (tasks_are_groups).
__global__ void __launch_bounds__(kThreads) k_encode(EncodeParams p) {
    encode_body<false, false, false>(p);
}

__global__ void __launch_bounds__(kThreads) k_encode_narrow(EncodeParams p) {
    encode_body<false, true, false>(p);
}

__global__ void __launch_bounds__(kThreads, 3) k_encode_rht(EncodeParams p) {
    encode_body<true, false, false>(p);
}

__global__ void __launch_bounds__(kThreads, 3) k_encode_rht_narrow(EncodeParams p) {
    encode_body<true, true, false>(p);
}

// Stochastically rounded codes (p.sr_seed), with or without the transform.
__global__ void __launch_bounds__(kThreads) k_encode_sr(EncodeParams p) {
    encode_body<false, false, true>(p);
}

__global__ void __launch_bounds__(kThreads) k_encode_sr_narrow(EncodeParams p) {
    encode_body<false, true, true>(p);
}

__global__ void __launch_bounds__(kThreads) k_encode_rht_sr(EncodeParams p) {
    encode_body<true, false, true>(p);
}

__global__ void __launch_bounds__(kThreads) k_encode_rht_sr_narrow(EncodeParams p) {
    encode_body<true, true, true>(p);
}

// ------------------------------------------------------------ k_encode_2d
// 2D weight blocks ("NVFP4: how NVIDIA pre-trained a 12B model on 10T
// tokens", section "Four stabilisation devices"): one scale per 16 rows x
// 16 columns.  A warp task is one 16-row group x 256 columns; lane l holds
// columns 8l..8l+7 of all 16 rows (each load instruction reads 512
// contiguous bytes of one row), lanes 2m and 2m+1 share a block and combine
// their maxima with one shuffle, and each code store writes 128 contiguous
// bytes of one row.  Every row of the group gets the block's scale.
__global__ void __launch_bounds__(kThreads) k_encode_2d(EncodeParams p) {
    __shared__ uint32_t red[kThreads / 32];
    __shared__ EncodeTables tab;
    float g;
    if (p.global_supplied) {
        g = *p.global;
    } else {
        if (!global_from_partials(p.partials, p.n_partials, p.status, &g, red)) return;
        if (blockIdx.x == 0 && threadIdx.x == 0) *p.global = g;
    }
    fill_tables(tab, g);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t sf_cols = p.cols / 16, sf_cols4 = (sf_cols + 3) / 4 * 4, col_tiles = sf_cols4 / 4;
    const int64_t rows_out = (p.layout == 0) ? (p.rows + 127) / 128 * 128 : p.rows;
    const uint32_t chunks = (uint32_t)((sf_cols4 + 15) / 16);          // 16 blocks per task
    const uint32_t tasks = (uint32_t)((rows_out + 15) / 16) * chunks;
    bool finite = true;
    for (uint32_t t = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < tasks;
         t += gridDim.x * (kThreads / 32)) {
        const int64_t r0 = (int64_t)(t / chunks) * 16;
        const int64_t blk = (int64_t)(t % chunks) * 16 + (lane >> 1);   // this lane's block column
        const int64_t c0 = blk * 16 + (lane & 1) * 8;                   // its first element column
        const bool col_ok = blk < sf_cols;
        uint4 v[16];
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            v[i] = (col_ok && r0 + i < p.rows)
                       ? __ldg(reinterpret_cast<const uint4 *>(p.x + (r0 + i) * p.ld + c0))
                       : make_uint4(0, 0, 0, 0);
            m = max_u16x2(m, amax_word(v[i], v[i]));
        }
        uint32_t bits = halves_to_f32bits(m);
        bits = max(bits, __shfl_xor_sync(0xFFFFFFFFu, bits, 1));
        const uint32_t s = scale_code(bits, g, tab);
        const float e = tab.inv_s[s & 0x7Fu];
        finite &= bits <= 0x7F7FFFFFu;
        if (col_ok) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (r0 + i < p.rows)
                    *reinterpret_cast<uint32_t *>(p.codes + (r0 + i) * (p.cols / 2) + c0 / 2) =
                        encode8(v[i].x, v[i].y, v[i].z, v[i].w, e);
        }
        // scale word of blocks blk..blk+3 (lanes 8q, 8q+2, 8q+4, 8q+6)
        uint32_t word = s;
        word |= __shfl_down_sync(0xFFFFFFFFu, s, 2) << 8;
        word |= __shfl_down_sync(0xFFFFFFFFu, s, 4) << 16;
        word |= __shfl_down_sync(0xFFFFFFFFu, s, 6) << 24;
        if ((lane & 7) == 0 && blk < sf_cols4 && (p.layout == 0 || blk < sf_cols)) {
            for (int i = 0; i < 16 && r0 + i < rows_out; ++i) {
                const uint32_t wr = (r0 + i < p.rows) ? word : 0u;  // band padding rows: zero
                uint8_t *sp = p.scales + sf_offset(r0 + i, blk, sf_cols, col_tiles, p.layout);
                if (p.layout == 0 || ((sf_cols & 3) == 0 && blk + 4 <= sf_cols)) {
                    *reinterpret_cast<uint32_t *>(sp) = wr;
                } else {                                               // ragged linear row
                    for (int j = 0; j < 4 && blk + j < sf_cols; ++j) sp[j] = (uint8_t)(wr >> (8 * j));
                }
            }
        }
    }
    if (!finite) set_status(p.status, ST_NONFINITE);   // only reachable with a supplied g
}

// ----------------------------------------------------------- k_dequantize
__device__ __forceinline__ void decode_block(uint2 codes, float d, uint4 &o0, uint4 &o1) {
    uint32_t out[8];
    uint32_t cw[2] = {codes.x, codes.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 v = f32x2_from_f16x2(f16x2_from_e2m1x2((cw[h] >> (8 * i)) & 0xFFu));
            out[4 * h + i] = bf16x2_from_f32(__fmul_rn(v.x, d), __fmul_rn(v.y, d));
        }
    }
    o0 = make_uint4(out[0], out[1], out[2], out[3]);
    o1 = make_uint4(out[4], out[5], out[6], out[7]);
}

template <bool kNarrow>
__device__ __forceinline__ void dequantize_body(const DequantParams &p) {
    // Wide rows: d = RN(f32(s) / g) for each of the 128 non-negative E4M3
    // codes s (stored scales are never negative), one table per CTA; narrow
    // rows divide per block.
    __shared__ float dtab[128];
    const float g = *p.global;
    if (!kNarrow) {
        for (int i = threadIdx.x; i < 128; i += blockDim.x)
            dtab[i] = __fdiv_rn(f32_from_e4m3((uint32_t)i), g);
        __syncthreads();
    }
    const int lane = threadIdx.x & 31;
    const int64_t sf_cols = p.cols / 16;
    const int64_t col_tiles = (sf_cols + 3) / 4;
    const uint32_t groups = (uint32_t)((sf_cols + 31) / 32);
    const uint32_t warps = gridDim.x * (kThreads / 32);
    const uint32_t warp_id = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int64_t sf_step = (p.layout == 0) ? 4096 : 32;         // scale bytes per 32 blocks
    if (groups == 0) return;                                      // no columns
    if (!kNarrow) {
        // Wide rows: kChunkBlocks blocks of one row per task (as in k_encode).
        const uint32_t chunks = (groups + kUnroll - 1) / kUnroll;
        for (TaskWalk w(warp_id, warps, chunks); w.row < p.rows; w.next()) {
            const int64_t row = w.row;
            const int64_t c0 = (int64_t)w.seg * kChunkBlocks + lane;
            const uint2 *cp = reinterpret_cast<const uint2 *>(p.codes + row * (p.cols / 2) + c0 * 8);
            const uint8_t *sp = p.scales + sf_offset(row, c0, sf_cols, col_tiles, p.layout);
            uint2 c[kUnroll];
            uint32_t sb[kUnroll];
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                if (c0 + 32 * j < sf_cols) {
                    c[j] = __ldg(cp + 32 * j);
                    sb[j] = __ldg(sp + sf_step * j);
                }
            }
            uint16_t *yp = p.y + row * p.ld + c0 * 16;
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                if (c0 + 32 * j >= sf_cols) continue;
                uint4 o0, o1;
                decode_block(c[j], dtab[sb[j] & 0x7Fu], o0, o1);
                store_32b(yp + 512 * j, o0, o1, p.y_vec32 != 0);
            }
        }
    } else {
        // Narrow rows: one 32-block group per task, kUnroll tasks in flight.
        const uint32_t tasks = (uint32_t)(p.rows * groups);       // < 2^32 (host-checked)
        const float inv_groups = 1.0f / (float)groups;
        for (uint32_t t0 = warp_id; t0 < tasks; t0 += warps * kUnroll) {
            uint2 c[kUnroll];
            uint32_t sb[kUnroll];
            int64_t rr[kUnroll], bb[kUnroll];
            bool has[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const uint32_t t = t0 + warps * u;
                const uint32_t row = task_row(t, groups, inv_groups);
                rr[u] = row;
                bb[u] = (int64_t)(t - row * groups) * 32 + lane;
                has[u] = t < tasks && bb[u] < sf_cols;
                if (has[u]) {
                    c[u] = __ldg(reinterpret_cast<const uint2 *>(p.codes + rr[u] * (p.cols / 2) + bb[u] * 8));
                    sb[u] = __ldg(p.scales + sf_offset(rr[u], bb[u], sf_cols, col_tiles, p.layout));
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (!has[u]) continue;
                const float d = __fdiv_rn(f32_from_e4m3(sb[u]), g);
                uint4 o0, o1;
                decode_block(c[u], d, o0, o1);
                store_32b(p.y + rr[u] * p.ld + bb[u] * 16, o0, o1, p.y_vec32 != 0);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads) k_dequantize(DequantParams p) { dequantize_body<false>(p); }

__global__ void __launch_bounds__(kThreads) k_dequantize_narrow(DequantParams p) {
    dequantize_body<true>(p);
}

}  // namespace nvfp4
