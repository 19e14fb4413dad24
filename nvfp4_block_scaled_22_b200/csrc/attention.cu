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
//   A  thread = token: its 128 K values restored, the 8 head scores by
//      packed FP32 FMAs against the query in shared memory (every lane reads
//      the same query word: broadcast); CTA maximum per head -> new running
//      maximum and rescale factor; weights -> shared memory.
//   B  thread = (8 dims, token phase 0..15): the V values of its dims for
//      every 16th token of the sub-tile times the weights of all 8 heads,
//      into 64 FP32 accumulators (rescaled first).
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

}  // namespace

__global__ void __launch_bounds__(kAttnThreads, 1) k_attn_partial(AttnParams p) {
    // qs[i][hp] = (q[2hp][2i], q[2hp][2i+1], q[2hp+1][2i], q[2hp+1][2i+1]) * c
    __shared__ float4 qs[kAttnDim / 2][kAttnMaxGroup / 2];
    // ps[t][hp] = (p[2hp], p[2hp], p[2hp+1], p[2hp+1]) of token t of the sub-tile
    __shared__ float4 ps[kAttnSub][kAttnMaxGroup / 2];
    __shared__ float wred[kAttnThreads / 32][kAttnMaxGroup];
    __shared__ float m_sh[kAttnMaxGroup], alpha_sh[kAttnMaxGroup];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hk = blockIdx.y, G = p.group;
    const int heads_q = p.group * p.heads_kv;
    const int64_t t0 = (int64_t)blockIdx.x * p.chunk;
    const int64_t t1 = min(p.tokens, t0 + p.chunk);
    const int64_t row_codes = p.cols / 2, row_scales = p.cols / 16;

    {
        const float c = __fdiv_rn(__fmul_rn(p.scale, kLog2e), *p.gk);
        float *qf = reinterpret_cast<float *>(&qs[0][0]);
        for (int e = tid; e < (kAttnDim / 2) * kAttnMaxGroup; e += kAttnThreads) {
            const int i = e >> 3, h = e & 7;     // float pair e: dims 2i, 2i + 1 of head h
            float lo = 0.0f, hi = 0.0f;
            if (h < G) {
                const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(
                    p.q + (int64_t)(hk * G + h) * p.ldq + 2 * i));
                lo = __fmul_rn(__uint_as_float(w << 16), c);
                hi = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), c);
            }
            qf[i * 16 + 2 * h] = lo;
            qf[i * 16 + 2 * h + 1] = hi;
        }
        if (tid < kAttnMaxGroup) m_sh[tid] = neg_inf();
    }
    __syncthreads();

    float lsum[kAttnMaxGroup];
    float2 oacc[kAttnMaxGroup][4];
#pragma unroll
    for (int h = 0; h < kAttnMaxGroup; ++h) {
        lsum[h] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) oacc[h][i] = make_float2(0.0f, 0.0f);
    }
    const int dg = tid & 15, tp = tid >> 4;   // pass B: dims 8dg .. 8dg + 7, token phase

    // K words of the first sub-tile; each later sub-tile's are loaded while
    // the previous one is in pass B, and a sub-tile's V words while its
    // scores are computed, so HBM latency overlaps the arithmetic.
    uint4 kw[4];
    uint2 ksw;
    auto load_k = [&](int64_t base) {
        const int64_t t = base + tid;
        ksw = make_uint2(0u, 0u);
#pragma unroll
        for (int n = 0; n < 4; ++n) kw[n] = make_uint4(0u, 0u, 0u, 0u);
        if (t < t1) {
            const uint4 *kp = reinterpret_cast<const uint4 *>(p.kc + t * row_codes + hk * 64);
#pragma unroll
            for (int n = 0; n < 4; ++n) kw[n] = __ldg(kp + n);
            ksw = __ldg(reinterpret_cast<const uint2 *>(p.ks + t * row_scales + hk * 8));
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

        // ---- A: scores of token base + tid for the 8 heads
        const bool valid = tid < n_sub;
        float2 acc[kAttnMaxGroup];
#pragma unroll
        for (int h = 0; h < kAttnMaxGroup; ++h) acc[h] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int b = 0; b < 8; ++b) {                 // block b: dims 16b .. 16b + 15
            const float sf = f32_from_e4m3(((b < 4 ? ksw.x : ksw.y) >> (8 * (b & 3))) & 0xFFu);
            const float2 sf2 = make_float2(sf, sf);
            const uint32_t w0 = (b & 1) ? kw[b >> 1].z : kw[b >> 1].x;
            const uint32_t w1 = (b & 1) ? kw[b >> 1].w : kw[b >> 1].y;
#pragma unroll
            for (int j = 0; j < 8; ++j) {             // byte j: dims 16b + 2j, 16b + 2j + 1
                const float2 k2 = restore_pair((j < 4 ? w0 : w1) >> (8 * (j & 3)), sf2);
                const int i = 8 * b + j;
#pragma unroll
                for (int hp = 0; hp < kAttnMaxGroup / 2; ++hp) {
                    const float4 qq = qs[i][hp];
                    acc[2 * hp] = fma_f32x2(k2, make_float2(qq.x, qq.y), acc[2 * hp]);
                    acc[2 * hp + 1] = fma_f32x2(k2, make_float2(qq.z, qq.w), acc[2 * hp + 1]);
                }
            }
        }
        if (base + kAttnSub < t1) load_k(base + kAttnSub);
        float s2[kAttnMaxGroup];
#pragma unroll
        for (int h = 0; h < kAttnMaxGroup; ++h) {
            s2[h] = valid ? __fadd_rn(acc[h].x, acc[h].y) : neg_inf();
            float v = s2[h];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
            if (lane == 0) wred[warp][h] = v;
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
        float pv[kAttnMaxGroup];
#pragma unroll
        for (int h = 0; h < kAttnMaxGroup; ++h) {
            pv[h] = valid ? exp2f(s2[h] - m_sh[h]) : 0.0f;
            lsum[h] = __fmaf_rn(lsum[h], alpha_sh[h], pv[h]);
        }
#pragma unroll
        for (int hp = 0; hp < kAttnMaxGroup / 2; ++hp)
            ps[tid][hp] = make_float4(pv[2 * hp], pv[2 * hp], pv[2 * hp + 1], pv[2 * hp + 1]);
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

    // ---- chunk totals: weight sums per head
#pragma unroll
    for (int h = 0; h < kAttnMaxGroup; ++h) {
        float v = lsum[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if (lane == 0) wred[warp][h] = v;
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

__global__ void __launch_bounds__(kAttnDim) k_attn_combine(AttnParams p) {
    const int qh = blockIdx.x, d = threadIdx.x;
    const int64_t heads_q = (int64_t)p.group * p.heads_kv;
    float r = 0.0f;
    if (p.n_chunks > 0) {
        float M = neg_inf();
        for (int c = 0; c < p.n_chunks; ++c) M = fmaxf(M, p.part_ml[(c * heads_q + qh) * 2]);
        float L = 0.0f, O = 0.0f;
        for (int c = 0; c < p.n_chunks; ++c) {
            const int64_t slot = c * heads_q + qh;
            const float w = exp2f(p.part_ml[slot * 2] - M);
            L = __fmaf_rn(w, p.part_ml[slot * 2 + 1], L);
            O = __fmaf_rn(w, p.part_o[slot * kAttnDim + d], O);
        }
        r = __fdiv_rn(__fdiv_rn(O, L), *p.gv);
    }
    p.o[(int64_t)qh * p.ldo + d] = (uint16_t)(bf16x2_from_f32(r, 0.0f) & 0xFFFFu);
}

}  // namespace nvfp4
