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
//   B  thread = (8 dims, token phase 0..15): the V values of its dims for
//      every 16th token of the sub-tile times the weights of all 8 heads,
//      into 64 FP32 accumulators (rescaled first, packed FP32 FMAs).
// After the chunk the token phases are summed in a fixed order (a shuffle,
// then three halvings through shared memory) and the chunk's O, m and l
// are written.  k_attn_combine merges the chunks in chunk order:
//   o = (sum_c 2^(m_c - M) O_c) / (sum_c 2^(m_c - M) l_c) / g_V.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr float kLog2e = 1.44269504088896340736f;
constexpr int kPhases = kAttnThreads / 16;     // token phases of pass B

__device__ __forceinline__ float neg_inf() { return __uint_as_float(0xFF800000u); }

// d = a * b + c lane-wise, one rounding per lane (one instruction).
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

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
    // ps[t][hp] = (p[2hp], p[2hp], p[2hp+1], p[2hp+1]) of token t of the sub-tile
    __shared__ float4 ps[kAttnSub][kAttnMaxGroup / 2];
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
    float2 oacc[kAttnMaxGroup][4];
#pragma unroll
    for (int h = 0; h < kAttnMaxGroup; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) oacc[h][i] = make_float2(0.0f, 0.0f);
    const int dg = tid & 15, tp = tid >> 4;   // pass B: dims 8dg .. 8dg + 7, token phase

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
        uint32_t vw[kAttnSub / kPhases], vsb[kAttnSub / kPhases];
#pragma unroll
        for (int s = 0; s < kAttnSub / kPhases; ++s) {
            const int tl = tp + kPhases * s;
            vw[s] = 0u;
            vsb[s] = 0u;
            if (tl < n_sub) {   // tokens past the end keep code 0 and scale 0, weight 0
                const int64_t tv = base + tl;
                vw[s] = __ldg(reinterpret_cast<const uint32_t *>(p.vc + tv * row_codes + hk * 64 + dg * 4));
                vsb[s] = __ldg(p.vs + tv * row_scales + hk * 8 + (dg >> 1));
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
                    ps[tl][c] = make_float4(p0, p0, p1, p1);
                }
            lsum[0] = __fmaf_rn(lsum[0], alpha_sh[2 * c], l0);
            lsum[1] = __fmaf_rn(lsum[1], alpha_sh[2 * c + 1], l1);
        }
        __syncthreads();

        // ---- B: weighted V of tokens tp, tp + 16, ... of the sub-tile
#pragma unroll
        for (int h = 0; h < kAttnMaxGroup; ++h) {
            const float a = alpha_sh[h];
#pragma unroll
            for (int i = 0; i < 4; ++i) oacc[h][i] = mul_f32x2(oacc[h][i], make_float2(a, a));
        }
#pragma unroll
        for (int s = 0; s < kAttnSub / kPhases; ++s) {
            const int tl = tp + kPhases * s;
            const float sv = f32_from_e4m3(vsb[s]);
            const float2 sv2 = make_float2(sv, sv);
            float2 v2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) v2[i] = restore_pair(vw[s] >> (8 * i), sv2);
#pragma unroll
            for (int hp = 0; hp < kAttnMaxGroup / 2; ++hp) {
                const float4 pp = ps[tl][hp];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    oacc[2 * hp][i] = fma_f32x2(v2[i], make_float2(pp.x, pp.y), oacc[2 * hp][i]);
                    oacc[2 * hp + 1][i] = fma_f32x2(v2[i], make_float2(pp.z, pp.w), oacc[2 * hp + 1][i]);
                }
            }
        }
        __syncthreads();   // ps and alpha_sh are rewritten by the next sub-tile
    }

    // ---- chunk totals: weight sums per head (lanes of one column pair c)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float v = lsum[e];
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if (g == 0) wred[warp][2 * c + e] = v;
    }
    // O: the two token phases of a warp, then warps 4..7 onto 0..3, 2..3
    // onto 0..1, 1 onto 0, through the (now free) weight buffer.
#pragma unroll
    for (int h = 0; h < kAttnMaxGroup; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            oacc[h][i].x += __shfl_xor_sync(0xFFFFFFFFu, oacc[h][i].x, 16);
            oacc[h][i].y += __shfl_xor_sync(0xFFFFFFFFu, oacc[h][i].y, 16);
        }
    float *red = reinterpret_cast<float *>(&ps[0][0]);   // [4 warps][64 values][16 lanes]
#pragma unroll
    for (int half = 4; half >= 1; half >>= 1) {
        if (warp >= half && warp < 2 * half && lane < 16) {
            float *dst = red + (warp - half) * 1024 + lane;
#pragma unroll
            for (int h = 0; h < kAttnMaxGroup; ++h)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dst[(h * 8 + 2 * i) * 16] = oacc[h][i].x;
                    dst[(h * 8 + 2 * i + 1) * 16] = oacc[h][i].y;
                }
        }
        __syncthreads();
        if (warp < half && lane < 16) {
            const float *src = red + warp * 1024 + lane;
#pragma unroll
            for (int h = 0; h < kAttnMaxGroup; ++h)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    oacc[h][i].x += src[(h * 8 + 2 * i) * 16];
                    oacc[h][i].y += src[(h * 8 + 2 * i + 1) * 16];
                }
        }
        __syncthreads();
    }
    const int64_t slot0 = (int64_t)blockIdx.x * heads_q + (int64_t)hk * G;
    if (warp == 0 && lane < 16) {
#pragma unroll
        for (int h = 0; h < kAttnMaxGroup; ++h) {
            if (h < G) {
                float4 *dst = reinterpret_cast<float4 *>(p.part_o + (slot0 + h) * kAttnDim + 8 * lane);
                dst[0] = make_float4(oacc[h][0].x, oacc[h][0].y, oacc[h][1].x, oacc[h][1].y);
                dst[1] = make_float4(oacc[h][2].x, oacc[h][2].y, oacc[h][3].x, oacc[h][3].y);
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
