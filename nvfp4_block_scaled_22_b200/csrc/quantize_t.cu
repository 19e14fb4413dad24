// Column-wise NVFP4 quantization: the NVFP4 tensor of x^T straight from a
// row-major x, without a BF16 transpose in memory.
//
// The Dgrad and Wgrad GEMMs of a linear layer contract over the axes the
// forward pass keeps contiguous ("NVFP4: how NVIDIA pre-trained a 12B model
// on 10T tokens", section "Four stabilisation devices": Fprop, Dgrad and
// Wgrad all run in NVFP4); the block-scaled GEMM wants both operands with
// 16-value blocks along the contraction axis.  For x [R x C] this produces
// out = NVFP4(x^T) [C x R]: output row j holds column j of x, blocked by 16
// consecutive rows of x, with exactly the codes and scales that quantizing
// an explicit BF16 x^T would give.
//
// Kernels
//   k_amax_t_rht : tensor amax of the Hadamard-transformed column blocks
//                  (the plain tensor amax of x^T is k_amax over x itself).
//   k_encode_t   : codes + scales of x^T (kRht: of its transformed blocks).
//
// Work split: a warp task is a 64 x 64 tile of x (4 output blocks of 64
// output rows).  The warp copies the tile into shared memory with cp.async
// (each instruction moves four 128-byte row pieces), double-buffered so the
// next tile's copy overlaps the current tile's encode, then lane
// l takes columns 2l and 2l + 1: a 32-bit shared read per tile row gives
// both columns' values, two byte permutes per pair of rows regroup them
// into each column's packed BF16 pairs, and the row-wise block encoder
// does the rest.  Each lane stores 32 contiguous code bytes and one scale
// word per output row.
#include <cstdint>
#include <cuda_runtime.h>

#include "encode_common.cuh"

namespace nvfp4 {

namespace {

constexpr int kTThreads = kTransposeThreads;   // 4 warps per CTA
constexpr int kTile = 64;                 // tile rows (of x) and columns (of x)
constexpr int kTileWords = kTile * kTile / 2;   // BF16 pairs per tile

// Tile (r0, c0) of x copied asynchronously into shared memory as [64 rows]
// [32 words] (cp.async, 16 bytes per lane per step, four 128-byte row
// pieces per warp instruction); values outside x are zero-filled without a
// global read.  Requires C % 8 == 0 (whole 16-byte pieces).
__device__ __forceinline__ void issue_tile(const uint16_t *__restrict__ x, int64_t ld, int64_t R,
                                           int64_t C, int64_t r0, int64_t c0, uint32_t *tile,
                                           int lane) {
    const int pr = lane >> 3, pc = lane & 7;          // row within a 4-row step, 16-byte piece
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(tile);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int64_t r = r0 + pr + 4 * i, c = c0 + pc * 8;
        const bool in = r < R && c < C;
        const void *src = in ? (const void *)(x + r * ld + c) : (const void *)x;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                     :: "r"(base + (uint32_t)(((pr + 4 * i) * 8 + pc) * 16)), "l"(src),
                        "r"(in ? 16 : 0)
                     : "memory");
    }
}

__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

// Wait until at most one committed group (the newest) is still in flight.
__device__ __forceinline__ void async_wait_all_but_newest() {
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}

// Double-buffered walk over a warp's tiles t0, t0 + stride, ...: the copy of
// the next tile runs while `work(tile_words, r0, c0)` handles the current one.
template <typename Work>
__device__ __forceinline__ void walk_tiles(const uint16_t *x, int64_t ld, int64_t R, int64_t C,
                                           uint32_t t0, uint32_t stride, uint32_t tasks, uint32_t ct,
                                           uint32_t *buf0, uint32_t *buf1, int lane, Work work) {
    uint32_t t = t0;
    if (t < tasks) issue_tile(x, ld, R, C, (int64_t)(t / ct) * kTile, (int64_t)(t % ct) * kTile, buf0, lane);
    async_commit();
    for (int i = 0; t < tasks; ++i, t += stride) {
        uint32_t *cur = (i & 1) ? buf1 : buf0, *nxt = (i & 1) ? buf0 : buf1;
        const uint32_t tn = t + stride;
        if (tn < tasks)
            issue_tile(x, ld, R, C, (int64_t)(tn / ct) * kTile, (int64_t)(tn % ct) * kTile, nxt, lane);
        async_commit();
        async_wait_all_but_newest();
        __syncwarp();
        work(cur, (int64_t)(t / ct) * kTile, (int64_t)(t % ct) * kTile);
        __syncwarp();                            // cur is refilled two steps later
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// Rows 16k .. 16k+15 of the lane's two columns as the row-wise encoder's
// packed input: a/b for column 2l, c/d for column 2l + 1 (value 2i in the
// low half of word i).
__device__ __forceinline__ void column_blocks(const uint32_t *tile, int k, int lane, uint4 &a,
                                              uint4 &b, uint4 &c, uint4 &d) {
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t w0 = tile[(16 * k + 2 * i) * 32 + lane];       // row 2i:   (col 2l, col 2l+1)
        const uint32_t w1 = tile[(16 * k + 2 * i + 1) * 32 + lane];   // row 2i+1
        lo[i] = __byte_perm(w0, w1, 0x5410);                           // (row 2i, row 2i+1) of col 2l
        hi[i] = __byte_perm(w0, w1, 0x7632);                           // same for col 2l + 1
    }
    a = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    b = make_uint4(lo[4], lo[5], lo[6], lo[7]);
    c = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    d = make_uint4(hi[4], hi[5], hi[6], hi[7]);
}

// Codes (up to four blocks) and the scale word of output row j at scale
// column b0; rows in [C, rows_out) are band padding and get zero scales.
// 16-byte code stores only where the row pitch R/2 keeps them aligned.
__device__ __forceinline__ void store_row(const EncodeParams &p, int64_t j, int64_t C,
                                          int64_t rows_out, int64_t R, int64_t b0, int nblk,
                                          int64_t sf_cols, int64_t col_tiles, const uint2 (&cw)[4],
                                          uint32_t sw) {
    if (j >= rows_out) return;
    if (j < C) {
        uint8_t *cp = p.codes + j * (R / 2) + b0 * 8;
        if (nblk == 4 && (R & 31) == 0) {
            reinterpret_cast<uint4 *>(cp)[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
            reinterpret_cast<uint4 *>(cp)[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < nblk) reinterpret_cast<uint2 *>(cp)[k] = cw[k];
        }
    }
    const uint32_t word = (j < C) ? sw : 0u;
    uint8_t *sp = p.scales + sf_offset(j, b0, sf_cols, col_tiles, p.layout);
    if (p.layout == 0 || ((sf_cols & 3) == 0 && b0 + 4 <= sf_cols)) {
        *reinterpret_cast<uint32_t *>(sp) = word;
    } else {                                                   // ragged linear row
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < nblk) sp[k] = (uint8_t)(word >> (8 * k));
    }
}

}  // namespace

// ----------------------------------------------------------- k_amax_t_rht
// x is R x C (pitch ld); writes the CTA's max |y| as f32 bits.  Dynamic
// shared memory: two tile buffers per warp.
__global__ void __launch_bounds__(kTThreads) k_amax_t_rht(const uint16_t *__restrict__ x, int64_t ld,
                                                          int64_t R, int64_t C, uint32_t rht_mask,
                                                          uint32_t *__restrict__ partials) {
    extern __shared__ uint4 dyn_smem[];
    __shared__ uint32_t red[kTThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t *buf0 = reinterpret_cast<uint32_t *>(dyn_smem) + warp * 2 * kTileWords;
    const uint32_t rt = (uint32_t)((R + kTile - 1) / kTile), ct = (uint32_t)((C + kTile - 1) / kTile);
    const SignFlips f = sign_flips(rht_mask);
    uint32_t m = 0;
    walk_tiles(x, ld, R, C, blockIdx.x * (kTThreads / 32) + warp, gridDim.x * (kTThreads / 32),
               rt * ct, ct, buf0, buf0 + kTileWords, lane,
               [&](const uint32_t *tile, int64_t r0, int64_t) {
#pragma unroll
                   for (int k = 0; k < 4; ++k) {
                       if (r0 + 16 * k >= R) break;                    // uniform across the warp
                       uint4 a, b, c, d;
                       column_blocks(tile, k, lane, a, b, c, d);
                       m = max(m, rht16_abs_max_bits(a, b, f));        // zero columns stay zero
                       m = max(m, rht16_abs_max_bits(c, d, f));
                   }
               });
    const uint32_t v = block_reduce_max(m, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = v;
}

// -------------------------------------------------------------- k_encode_t
// kTwoD: one scale per 16x16 block of x (16 rows x 16 columns, the 2D
// weight blocks), so the output is the 2D quantization of x^T.
template <bool kRht, bool kTwoD, bool kSR>
__device__ __forceinline__ void encode_t_body(const EncodeParams &p) {
    extern __shared__ uint4 dyn_smem[];
    __shared__ uint32_t red[kTThreads / 32];
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
    const SignFlips f = sign_flips(kRht ? p.rht_mask : 0u);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t *buf0 = reinterpret_cast<uint32_t *>(dyn_smem) + warp * 2 * kTileWords;
    const int64_t R = p.cols, C = p.rows;
    const int64_t sf_cols = R / 16, sf_cols4 = (sf_cols + 3) / 4 * 4, col_tiles = sf_cols4 / 4;
    const int64_t rows_out = (p.layout == 0) ? (C + 127) / 128 * 128 : C;
    const uint32_t rt = (uint32_t)((R + kTile - 1) / kTile);
    const uint32_t ct = (uint32_t)((rows_out + kTile - 1) / kTile);
    bool finite = true;
    walk_tiles(p.x, p.ld, R, C, blockIdx.x * (kTThreads / 32) + warp, gridDim.x * (kTThreads / 32),
               rt * ct, ct, buf0, buf0 + kTileWords, lane,
               [&](const uint32_t *tile, int64_t r0, int64_t c0) {
                   uint2 code0[4], code1[4];           // columns 2l, 2l+1; blocks k = 0..3
                   uint32_t sw0 = 0, sw1 = 0;          // their scale words
#pragma unroll
                   for (int k = 0; k < 4; ++k) {
                       code0[k] = code1[k] = make_uint2(0, 0);
                       if (r0 + 16 * k >= R) continue; // uniform across the warp
                       uint4 a, b, c, d;
                       column_blocks(tile, k, lane, a, b, c, d);
                       EncodeBlockOut o0, o1;
                       if (kTwoD) {
                           // lanes 8m..8m+7 hold columns 16m..16m+15: one 16x16 block
                           uint32_t m = max(block_amax_bits(a, b), block_amax_bits(c, d));
                           m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                           m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                           m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                           o0 = encode_block_amax(a, b, m, g, tab);
                           o1 = encode_block_amax(c, d, m, g, tab);
                       } else {
                           // output block n = output row * (R / 16) + block column
                           BlockDraws r0d, r1d;
                           if (kSR) {
                               const uint64_t n0 = (uint64_t)(c0 + 2 * lane) * (uint64_t)sf_cols +
                                                   (uint64_t)(r0 / 16 + k);
                               r0d = block_draws(p.sr_seed, n0);
                               r1d = block_draws(p.sr_seed, n0 + (uint64_t)sf_cols);
                           }
                           o0 = encode_any<kRht, kSR>(a, b, f, g, tab, r0d);
                           o1 = encode_any<kRht, kSR>(c, d, f, g, tab, r1d);
                       }
                       finite &= o0.finite && o1.finite;
                       code0[k] = o0.codes;
                       code1[k] = o1.codes;
                       sw0 |= o0.scale << (8 * k);
                       sw1 |= o1.scale << (8 * k);
                   }
                   const int64_t b0 = r0 / 16;         // first scale column of the tile
                   const int nblk = (sf_cols - b0 < 4) ? (int)(sf_cols - b0) : 4;
                   const int64_t j = c0 + 2 * lane;    // output rows j, j + 1
                   store_row(p, j, C, rows_out, R, b0, nblk, sf_cols, col_tiles, code0, sw0);
                   store_row(p, j + 1, C, rows_out, R, b0, nblk, sf_cols, col_tiles, code1, sw1);
               });
    if (!finite) set_status(p.status, ST_NONFINITE);   // only reachable with a supplied g
}

__global__ void __launch_bounds__(kTThreads) k_encode_t(EncodeParams p) {
    encode_t_body<false, false, false>(p);
}

__global__ void __launch_bounds__(kTThreads) k_encode_t_rht(EncodeParams p) {
    encode_t_body<true, false, false>(p);
}

__global__ void __launch_bounds__(kTThreads) k_encode_t_2d(EncodeParams p) {
    encode_t_body<false, true, false>(p);
}

__global__ void __launch_bounds__(kTThreads) k_encode_t_sr(EncodeParams p) {
    encode_t_body<false, false, true>(p);
}

__global__ void __launch_bounds__(kTThreads) k_encode_t_rht_sr(EncodeParams p) {
    encode_t_body<true, false, true>(p);
}

// Launch with the dynamic shared memory of two tile buffers per warp (the
// size limit is raised once per device).
cudaError_t launch_transpose_kernel(const void *kernel, int grid, void **args, cudaStream_t stream) {
    constexpr int kKernels = 6;
    static bool attr_set[64][kKernels] = {};
    const void *kernels[kKernels] = {(const void *)k_amax_t_rht, (const void *)k_encode_t,
                                     (const void *)k_encode_t_rht, (const void *)k_encode_t_2d,
                                     (const void *)k_encode_t_sr, (const void *)k_encode_t_rht_sr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int which = -1;
    for (int i = 0; i < kKernels; ++i)
        if (kernels[i] == kernel) which = i;
    if (which < 0) return cudaErrorInvalidDeviceFunction;
    if (dev < 0 || dev >= 64 || !attr_set[dev][which]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTransposeSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev][which] = true;
    }
    return cudaLaunchKernel(kernel, dim3(grid), dim3(kTThreads), args, kTransposeSmemBytes, stream);
}

}  // namespace nvfp4
