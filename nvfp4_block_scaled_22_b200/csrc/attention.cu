// Decode attention over an NVFP4 KV cache ("FP4 KV-cache quantization":
// every generated token re-reads the whole cache, so reading it is the cost
// of a decode step; the FP4 values are restored before the attention
// arithmetic).  The cache is read once in its 0.5625-byte form and restored
// in registers (e2m1 * s_b, exact in FP32); no FP8 or BF16 copy is written.
//
// Grouped-query attention for one query token: query head h uses KV head
// h / group.  One CTA takes one KV head and one chunk of tokens and keeps
// all of the group's query heads (up to 8), so each K and V byte is read
// once and serves every head of the group.  Scores are kept in log2 units:
// c = scale * log2(e) / g_K is folded into the query, and the weights are
// exp2(score - running max) with the running maximum and the rescale of
// what was summed before (the online softmax of flash-decoding).
//
// k_attn_partial, per sub-tile of 256 tokens of the CTA's chunk:
//   A  scores on the tensor cores (mma.sync m16n8k16, BF16 operands, FP32
//      accumulation): each warp takes two 16-token tiles; the K values
//      restored to BF16 (e2m1 * s_b has at most 6 significant bits, so the
//      restore is exact) are the A operand and the query (BF16, exact) the
//      B operand, 8 query heads as the 8 columns.  The 128 dims are dealt
//      to the eight 16-wide k-steps so that each lane's A values come from
//      one 16-byte piece of the token's code row (lane column pair c holds
//      dims 32c .. 32c + 31); the query columns follow the same order.
//      Scores times c, the CTA maximum per head -> new running maximum and
//      rescale factor; weights -> shared memory.
//   B  O^T[dim][head] += V^T[dim][token] P^T[token][head] on the tensor
//      cores too (mma.sync m16n8k8, TF32 operands, FP32 accumulation), each
//      warp over its own 32 tokens: the restored V values (6 significant
//      bits) are exact TF32, and each FP32 weight is split exactly into
//      three TF32 parts (p = p1 + p2 + p3, 11 + 11 + 2 bits), one MMA per
//      part, so every product is exact as in the FP32 reading.  Lane
//      (g, c) restores the 16 dims 16g .. 16g + 15 (one 8-byte piece and
//      one scale of its token row) of tokens c and c + 4 of each 8-token
//      k-step; M-tile j row r is dim 16(r mod 8) + 2j + r / 8.
// After the chunk the warps' accumulators are summed in a fixed order
// (three halvings through shared memory) and the chunk's O, m and l are
// written.  k_attn_combine merges the chunks in chunk order:
//   o = (sum_c 2^(m_c - M) O_c) / (sum_c 2^(m_c - M) l_c) / g_V.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr float kLog2e = 1.44269504088896340736f;

__device__ __forceinline__ float neg_inf() { return __uint_as_float(0xFF800000u); }

// The two values of one code byte (low nibble first) times the block scale
// s2 = (s, s): exact, e2m1 has 2 significant bits and E4M3 has 4.
__device__ __forceinline__ float2 restore_pair(uint32_t byte, float2 s2) {
    return mul_f32x2(f32x2_from_f16x2(f16x2_from_e2m1x2(byte & 0xFFu)), s2);
}

// The same two values as BF16 (exact: at most 6 significant bits, within
// 2^-10 .. 2688), low nibble in the low half.
__device__ __forceinline__ uint32_t restore_bf16x2(uint32_t byte, float s) {
    const float2 v = f32x2_from_f16x2(f16x2_from_e2m1x2(byte & 0xFFu));
    return bf16x2_from_f32(__fmul_rn(v.x, s), __fmul_rn(v.y, s));
}

// D += A B for one 16x8x8 tile: A 16x8 row-major, B 8x8 column-major, TF32
// operands (FP32 bit patterns whose low 13 bits are zero), FP32
// accumulators (fragments of the PTX mma.sync m16n8k8 shape).
__device__ __forceinline__ void mma_tf32_1688(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// p = w[0] + w[1] + w[2] exactly, each part a TF32 value (FP32 with the low
// 13 mantissa bits zero), for p >= 2^-113: truncation leaves remainders that
// FP32 holds exactly (13, then 2 significant bits).  Below that p - p1 can
// be subnormal and the third part keeps low bits that the TF32 operand
// drops: an absolute error under 2^-136 per weight.
__device__ __forceinline__ void split_tf32x3(float p, uint32_t (&w)[3]) {
    const float p1 = __uint_as_float(__float_as_uint(p) & 0xFFFFE000u);
    const float r1 = __fsub_rn(p, p1);
    const float p2 = __uint_as_float(__float_as_uint(r1) & 0xFFFFE000u);
    w[0] = __float_as_uint(p1);
    w[1] = __float_as_uint(p2);
    w[2] = __float_as_uint(__fsub_rn(r1, p2));
}

// D += A B for one 16x8x16 tile: A 16x16 row-major, B 16x8 column-major,
// BF16 operands, FP32 accumulators (thread fragments of the PTX mma.sync
// m16n8k16 shape: a row group g = lane / 4 and a column pair c = lane % 4).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace

__global__ void __launch_bounds__(kAttnThreads, 1) k_attn_partial(AttnParams p) {
    // weights p[head][token of the sub-tile] (rows padded: the B-fragment
    // reads of a warp hit 32 banks); reused for the warps' final sums
    constexpr int kPwPitch = kAttnSub + 4;
    __shared__ __align__(16) float sbuf[4 * 32 * 32];
    static_assert(kAttnMaxGroup * kPwPitch <= 4 * 32 * 32, "weights fit the reduction buffer");
    float(*pw)[kPwPitch] = reinterpret_cast<float(*)[kPwPitch]>(sbuf);
    __shared__ float wred[kAttnThreads / 32][kAttnMaxGroup];
    __shared__ float m_sh[kAttnMaxGroup], alpha_sh[kAttnMaxGroup];

    // the combine (launched with programmatic stream serialization) may be
    // scheduled now; it waits on the device for this whole grid
    grid_dependents_launch();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;    // pass A: MMA fragment row group, column pair
    const int hk = blockIdx.y, G = p.group;
    const int heads_q = p.group * p.heads_kv;
    const int64_t t0 = (int64_t)blockIdx.x * p.chunk;
    const int64_t t1 = min(p.tokens, t0 + p.chunk);
    const int64_t row_codes = p.cols / 2, row_scales = p.cols / 16;
    const float ck = __fdiv_rn(__fmul_rn(p.scale, kLog2e), *p.gk);

    // B operand of the score MMAs: query head g, dims 32c .. 32c + 31 as
    // BF16 pairs; step j uses dims 32c + 4j .. + 3 (qb[2j], qb[2j + 1]).
    uint32_t qb[16];
#pragma unroll
    for (int n = 0; n < 16; ++n) qb[n] = 0u;
    if (g < G) {
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(p.q + (int64_t)(hk * G + g) * p.ldq + 32 * c);
#pragma unroll
        for (int n = 0; n < 16; ++n) qb[n] = __ldg(qrow + n);
    }
    if (tid < kAttnMaxGroup) m_sh[tid] = neg_inf();
    __syncthreads();

    float lsum[2] = {0.0f, 0.0f};             // heads 2c, 2c + 1 over this lane's tokens
    // pass B accumulators: M-tile j, (dim 16g + 2j, head 2c), (.., 2c + 1),
    // (dim 16g + 2j + 1, head 2c), (.., 2c + 1)
    float oacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) oacc[j][i] = 0.0f;

    // Pass A rows of this lane: tokens 32 warp + 16 u + g + 8 r of the
    // sub-tile (u = MMA tile 0/1, r = fragment row half), code bytes
    // 16c .. 16c + 15 of the KV head's 64 (dims 32c .. 32c + 31) and the
    // scales of blocks 2c, 2c + 1.  Loaded one sub-tile ahead.
    uint4 kw[4];
    uint32_t ksw[4];
    auto load_k = [&](int64_t base) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t t = base + 32 * warp + 16 * (e >> 1) + g + 8 * (e & 1);
            kw[e] = make_uint4(0u, 0u, 0u, 0u);
            ksw[e] = 0u;
            if (t < t1) {
                kw[e] = __ldg(reinterpret_cast<const uint4 *>(p.kc + t * row_codes + hk * 64 + 16 * c));
                ksw[e] = __ldg(reinterpret_cast<const uint16_t *>(p.ks + t * row_scales + hk * 8 + 2 * c));
            }
        }
    };
    load_k(t0);

    for (int64_t base = t0; base < t1; base += kAttnSub) {
        const int64_t n_sub = min((int64_t)kAttnSub, t1 - base);
        // pass B operands of this lane: tokens 32 warp + 8 kk + c (+ 4) of
        // the sub-tile, dims 16g .. 16g + 15 (code bytes 8g .. 8g + 7 of the
        // KV head's 64, scale block g)
        uint2 vw[8];
        uint32_t vsb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int tl = 32 * warp + 8 * (e >> 1) + c + 4 * (e & 1);
            vw[e] = make_uint2(0u, 0u);
            vsb[e] = 0u;
            if (tl < n_sub) {   // tokens past the end keep code 0 and scale 0, weight 0
                const int64_t tv = base + tl;
                vw[e] = __ldg(reinterpret_cast<const uint2 *>(p.vc + tv * row_codes + hk * 64 + 8 * g));
                vsb[e] = __ldg(p.vs + tv * row_scales + hk * 8 + g);
            }
        }

        // ---- A: scores S[token][head] = sum_d (e2m1 * s_b)[token][d] q[head][d]
        // on the tensor cores (BF16 operands, both exact; FP32 accumulate):
        // two 16-token tiles per warp, eight k-steps of 16 dims each.
        float sc[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const uint4 w0 = kw[2 * u], w1 = kw[2 * u + 1];          // rows g, g + 8
            const uint32_t r0[4] = {w0.x, w0.y, w0.z, w0.w}, r1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {                            // dims 32c + 4j .. + 3
                const float s0 = f32_from_e4m3((ksw[2 * u] >> (8 * (j >> 2))) & 0xFFu);
                const float s1 = f32_from_e4m3((ksw[2 * u + 1] >> (8 * (j >> 2))) & 0xFFu);
                const uint32_t b0 = r0[j >> 1] >> (16 * (j & 1)), b1 = r1[j >> 1] >> (16 * (j & 1));
                uint32_t a[4];
                a[0] = restore_bf16x2(b0, s0);          // row g,     dims +0, +1
                a[1] = restore_bf16x2(b1, s1);          // row g + 8, dims +0, +1
                a[2] = restore_bf16x2(b0 >> 8, s0);     // row g,     dims +2, +3
                a[3] = restore_bf16x2(b1 >> 8, s1);     // row g + 8, dims +2, +3
                mma_bf16_16816(d, a, qb[2 * j], qb[2 * j + 1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {    // d: (g, 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1)
                const int tl = 32 * warp + 16 * u + g + 8 * (e >> 1);
                sc[u][e] = tl < n_sub ? __fmul_rn(d[e], ck) : neg_inf();
            }
        }
        if (base + kAttnSub < t1) load_k(base + kAttnSub);
#pragma unroll
        for (int e = 0; e < 2; ++e) {        // heads 2c + e
            float v = fmaxf(fmaxf(sc[0][e], sc[0][e + 2]), fmaxf(sc[1][e], sc[1][e + 2]));
#pragma unroll
            for (int off = 4; off <= 16; off <<= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
            if (g == 0) wred[warp][2 * c + e] = v;
        }
        __syncthreads();
        if (tid < kAttnMaxGroup) {
            float mt = wred[0][tid];
#pragma unroll
            for (int w = 1; w < kAttnThreads / 32; ++w) mt = fmaxf(mt, wred[w][tid]);
            const float mo = m_sh[tid];
            const float mn = fmaxf(mo, mt);
            alpha_sh[tid] = (mo == neg_inf()) ? 0.0f : exp2f(mo - mn);
            m_sh[tid] = mn;
        }
        __syncthreads();
        {
            const float m0 = m_sh[2 * c], m1 = m_sh[2 * c + 1];
            float l0 = 0.0f, l1 = 0.0f;
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int tl = 32 * warp + 16 * u + g + 8 * r;
                    const bool ok = tl < n_sub;
                    const float p0 = ok ? exp2f(sc[u][2 * r] - m0) : 0.0f;
                    const float p1 = ok ? exp2f(sc[u][2 * r + 1] - m1) : 0.0f;
                    l0 += p0;
                    l1 += p1;
                    pw[2 * c][tl] = p0;
                    pw[2 * c + 1][tl] = p1;
                }
            lsum[0] = __fmaf_rn(lsum[0], alpha_sh[2 * c], l0);
            lsum[1] = __fmaf_rn(lsum[1], alpha_sh[2 * c + 1], l1);
        }
        __syncthreads();

        // ---- B: O^T += V^T P^T over this warp's 32 tokens (exact products)
        {
            const float a0 = alpha_sh[2 * c], a1 = alpha_sh[2 * c + 1];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                oacc[j][0] = __fmul_rn(oacc[j][0], a0);
                oacc[j][1] = __fmul_rn(oacc[j][1], a1);
                oacc[j][2] = __fmul_rn(oacc[j][2], a0);
                oacc[j][3] = __fmul_rn(oacc[j][3], a1);
            }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int ta = 32 * warp + 8 * kk + c;          // B rows c and c + 4
            uint32_t wa[3], wb[3];
            split_tf32x3(pw[g][ta], wa);
            split_tf32x3(pw[g][ta + 4], wb);
            const float sa = f32_from_e4m3(vsb[2 * kk]), sb = f32_from_e4m3(vsb[2 * kk + 1]);
            const uint2 ca = vw[2 * kk], cb = vw[2 * kk + 1];
#pragma unroll
            for (int j = 0; j < 8; ++j) {                   // M-tile j: dims 16r + 2j (+1)
                const uint32_t byte_a = (j < 4 ? ca.x : ca.y) >> (8 * (j & 3));
                const uint32_t byte_b = (j < 4 ? cb.x : cb.y) >> (8 * (j & 3));
                const float2 va = restore_pair(byte_a, make_float2(sa, sa));
                const float2 vb = restore_pair(byte_b, make_float2(sb, sb));
                const uint32_t a[4] = {__float_as_uint(va.x), __float_as_uint(va.y),
                                       __float_as_uint(vb.x), __float_as_uint(vb.y)};
#pragma unroll
                for (int q = 0; q < 3; ++q) mma_tf32_1688(oacc[j], a, wa[q], wb[q]);
            }
        }
        __syncthreads();   // pw and alpha_sh are rewritten by the next sub-tile
    }

    // ---- chunk totals: weight sums per head (lanes of one column pair c)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float v = lsum[e];
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if (g == 0) wred[warp][2 * c + e] = v;
    }
    // O: warps 4..7 onto 0..3, 2..3 onto 0..1, 1 onto 0, through the (now
    // free) weight buffer
#pragma unroll
    for (int half = 4; half >= 1; half >>= 1) {
        if (warp >= half && warp < 2 * half) {
            float *dst = sbuf + (warp - half) * 1024 + lane;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[(4 * j + i) * 32] = oacc[j][i];
        }
        __syncthreads();
        if (warp < half) {
            const float *src = sbuf + warp * 1024 + lane;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) oacc[j][i] = __fadd_rn(oacc[j][i], src[(4 * j + i) * 32]);
        }
        __syncthreads();
    }
    const int64_t slot0 = (int64_t)blockIdx.x * heads_q + (int64_t)hk * G;
    if (warp == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {                        // heads 2c + e
            if (2 * c + e < G) {
                float *dst = p.part_o + (slot0 + 2 * c + e) * kAttnDim + 16 * g;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float2 *>(dst + 2 * j) = make_float2(oacc[j][e], oacc[j][2 + e]);
            }
        }
    }
    if (tid < G) {
        float l = 0.0f;
#pragma unroll
        for (int w = 0; w < kAttnThreads / 32; ++w) l += wred[w][tid];
        p.part_ml[(slot0 + tid) * 2] = m_sh[tid];
        p.part_ml[(slot0 + tid) * 2 + 1] = l;
    }
}

// The chunks' values are loaded eight at a time before they are used, so
// that a batch costs one memory round trip; the sums still run in chunk
// order.  Launched behind k_attn_partial with programmatic stream
// serialization: the wait below returns once that grid has completed.
__global__ void __launch_bounds__(kAttnDim) k_attn_combine(AttnParams p) {
    constexpr int kBatch = 8;
    grid_dependency_wait();
    const int qh = blockIdx.x, d = threadIdx.x;
    const int64_t heads_q = (int64_t)p.group * p.heads_kv;
    const int n = p.n_chunks;
    float r = 0.0f;
    if (n > 0) {
        float M = neg_inf();
        for (int c0 = 0; c0 < n; c0 += kBatch) {
            float m[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                m[j] = c0 + j < n ? p.part_ml[((c0 + j) * heads_q + qh) * 2] : neg_inf();
#pragma unroll
            for (int j = 0; j < kBatch; ++j) M = fmaxf(M, m[j]);
        }
        float L = 0.0f, O = 0.0f;
        for (int c0 = 0; c0 < n; c0 += kBatch) {
            float m[kBatch], l[kBatch], o[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int64_t slot = (c0 + j) * heads_q + qh;
                const bool ok = c0 + j < n;
                m[j] = ok ? p.part_ml[slot * 2] : 0.0f;
                l[j] = ok ? p.part_ml[slot * 2 + 1] : 0.0f;
                o[j] = ok ? p.part_o[slot * kAttnDim + d] : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                if (c0 + j < n) {
                    const float w = exp2f(m[j] - M);
                    L = __fmaf_rn(w, l[j], L);
                    O = __fmaf_rn(w, o[j], O);
                }
            }
        }
        r = __fdiv_rn(__fdiv_rn(O, L), *p.gv);
    }
    p.o[(int64_t)qh * p.ldo + d] = (uint16_t)(bf16x2_from_f32(r, 0.0f) & 0xFFFFu);
}

}  // namespace nvfp4
