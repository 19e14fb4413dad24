/*
 * NVFP4 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct restatement of what the NVFP4 hot path
 * computes.  Only the test suite, the package's smoke check and the CPU
 * baseline leg of the benchmark may load this library; the product path
 * never does.  It shares no code, header or table with the CUDA kernels.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -msse2
 *        -mfpmath=sse -fPIC -shared  (so every float operation below is one
 *        IEEE binary32 operation rounded to nearest-even; no FMA contraction,
 *        no flush-to-zero).
 *
 * Sources (web pages; section in parentheses):
 *  [P1] "NVIDIA shrank GLM-5.2 to 4 bits" (iwan.kr), section 3 "Glossary --
 *       quantization and NVFP4": 15 distinct 4-bit values, 16-value blocks
 *       with one FP8 scale each, one FP32 scale per tensor.
 *  [P2] "NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens"
 *       (axbrief.com), section "E2M1 format and two-level scaling": E2M1 =
 *       1 sign, 2 exponent, 1 mantissa bit with values +-0, 0.5, 1, 1.5, 2,
 *       3, 4, 6; blocks of 16 with an E4M3 scale; FP32 tensor-level scale;
 *       block amax mapped close to the FP4 maximum.
 *  [P5] "FP4 KV-cache quantization" (theddari.com), section "FP4 formats
 *       compared": 0.5625 bytes per value (4.5 bits) including scales.
 *  [P2'] same pre-training page, section "Four stabilisation devices": the
 *       Wgrad inputs are multiplied by a 16x16 Hadamard matrix and a random
 *       +-1 sign vector before quantization; weights use 16x16 (2D) blocks
 *       so that the transposed weight holds the same quantized values;
 *       gradients are rounded stochastically (a value 0.7 of the way from
 *       one grid point to the next goes up with probability 0.7).
 *  [PM] MXFP4, the format the pages compare NVFP4 with: "NVIDIA shrank
 *       GLM-5.2 to 4 bits" section 3 (blocks of 32, power-of-two E8M0
 *       scale), pre-training page section "E2M1 format and two-level
 *       scaling" (32 values per UE8M0 scale, no tensor scale), KV page
 *       section "FP4 formats compared" (about 4.25 bits per value).
 *  [PC] consumers of the quantized tensors: "NVIDIA shrank GLM-5.2 to 4
 *       bits" section 2 (256 experts, 8 active per token: the expert
 *       outputs are combined per token); "FP4 KV-cache quantization",
 *       section on current implementations (the FP4 KV cache is
 *       dequantized to FP8 before attention).
 *  [PG] gated activation between the expert up and down projections (the
 *       MoE expert block of the GLM page, section 2): SiLU-gated linear
 *       unit h = silu(gate) * up.
 *  [PE] Cody and Waite, "Software Manual for the Elementary Functions"
 *       (1980): exp by reduction x = n ln2 + r with ln2 split in a high part
 *       exact in few bits and a low correction, then a polynomial in r.
 *  [PX] Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
 *       1, 2, 3" (SC 2011): the Philox4x32-10 counter-based generator.
 *  The FP32 evaluation order below is the convention the hot path is
 *  specified with: global g = 448*6/amax_tensor, block scale
 *  s = e4m3_rne(amax_block/6*g), code = e2m1_rne(x*g/s), with x*g/s taken as
 *  x*(g/s) (one division per block).  Every point the pages leave open is
 *  marked READING below.
 *
 * Parity status: every function here is pinned by the oracle tests
 * (exhaustive sweeps against brute-force nearest-value search, the pages'
 * value list and storage figures, exact round trips, integer-exact GEMM).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define NVO_OK 0
#define NVO_ERR_SHAPE 3
#define NVO_ERR_NONFINITE 4
#define NVO_ERR_RANGE 5

#define NVO_SF_SWIZZLED 0
#define NVO_SF_LINEAR 1

/* ---------------------------------------------------------------- BF16 */

float nvo_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a binary32 to bfloat16, nearest-even on the 16 dropped bits. */
uint16_t nvo_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x0040u);          /* quiet NaN */
    uint32_t low = u & 0xFFFFu;
    uint32_t hi = u >> 16;
    if (low > 0x8000u || (low == 0x8000u && (hi & 1u)))
        hi += 1u;
    return (uint16_t)hi;
}

/* ---------------------------------------------------------------- E2M1 */

/* [P2] value list; code bits s.ee.m, bias 1, exponent field 0 = subnormal
 * (m * 0.5).  Both 0x0 and 0x8 decode to zero: 16 codes, 15 values [P1]. */
float nvo_e2m1_decode(uint8_t code)
{
    int e = (code >> 1) & 3, m = code & 1;
    float mag = (e == 0) ? 0.5f * (float)m
                         : ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return (code & 8) ? -mag : mag;
}

/* Round y to the nearest E2M1 value, ties to the even code (mantissa bit
 * 0), magnitudes at or above 6 saturate to 6 (E2M1 has no infinity).  The
 * sign bit is copied from y, so -0 and tiny negatives give code 0x8
 * (READING: the pages do not say which zero a negative underflow keeps). */
uint8_t nvo_e2m1_rne_satfinite(float y)
{
    uint8_t sign = signbit(y) ? 8 : 0;
    double a = fabs((double)y);
    if (a >= 6.0)
        return sign | 7;
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                /* floor(log2 a) for a > 0 */
    if (a == 0.0 || E < 0)
        E = 0;                     /* [0, 2) shares the quantum 0.5 */
    double q = ldexp(1.0, E - 1);  /* spacing of the grid in this binade */
    double r = nearbyint(a / q) * q;  /* default mode: half to even */
    if (r >= 6.0)
        return sign | 7;
    uint8_t code;
    if (r < 1.0) {
        code = (uint8_t)(r / 0.5);             /* 0 or 1 (subnormal) */
    } else {
        int e2;
        frexp(r, &e2);
        int E2 = e2 - 1;                       /* 0, 1 or 2 */
        int m = (int)((r / ldexp(1.0, E2) - 1.0) * 2.0);
        code = (uint8_t)(((E2 + 1) << 1) | m);
    }
    return sign | code;
}

/* ---------------------------------------------------------------- E4M3 */

/* E4M3 (the block-scale format named in [P2]): bias 7, exponent field 0 is
 * subnormal m/8 * 2^-6, S.1111.111 is NaN, largest finite 448. */
float nvo_e4m3_decode(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    float mag;
    if (e == 15 && m == 7)
        mag = NAN;
    else if (e == 0)
        mag = ldexpf((float)m / 8.0f, -6);
    else
        mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return (b & 0x80) ? -mag : mag;
}

/* Round v >= 0 to the nearest finite E4M3 value, ties to even mantissa,
 * subnormals kept, values past the largest finite (448) saturate to it. */
uint8_t nvo_e4m3_rne_satfinite(float v)
{
    if (!(v > 0.0f))
        return 0;                  /* +0, -0 (and NaN, never passed) */
    if (v >= 448.0f)
        return 0x7E;
    int ex;
    frexp((double)v, &ex);
    int E = ex - 1;
    if (E < -6)
        E = -6;                    /* subnormals share binade -6's quantum */
    double q = ldexp(1.0, E - 3);
    double r = nearbyint((double)v / q) * q;
    if (r == 0.0)
        return 0;
    if (r >= 448.0)
        return 0x7E;
    int e2;
    frexp(r, &e2);
    int E2 = e2 - 1;
    if (E2 < -6)
        return (uint8_t)(r / ldexp(1.0, -9));        /* subnormal m */
    int m = (int)((r / ldexp(1.0, E2) - 1.0) * 8.0);
    return (uint8_t)(((E2 + 7) << 3) | m);
}

/* ------------------------------------------------------- scale layouts */

/* READING (pages silent): GEMM operands keep their block scales in the
 * 128x4 tiled layout the block-scaled tensor-core MMA consumes -- per 128
 * rows and 4 scale columns one 512-byte tile, row r%32 at 16-byte stride,
 * (r%128)/32 at 4-byte stride, scale column c%4 at 1-byte stride; tiles run
 * along the scale columns first.  Rows pad to 128 and scale columns to 4,
 * padding holds zero.  The KV cache uses the plain row-major
 * [rows x cols/16] layout. */
int64_t nvo_sf_cols(int64_t cols) { return cols / 16; }

int64_t nvo_scales_bytes(int64_t rows, int64_t cols, int layout)
{
    int64_t s = cols / 16;
    if (layout == NVO_SF_LINEAR)
        return rows * s;
    int64_t sp = (s + 3) / 4 * 4;
    int64_t rp = (rows + 127) / 128 * 128;
    return rp * sp;
}

int64_t nvo_sf_offset(int64_t r, int64_t c, int64_t rows, int64_t cols, int layout)
{
    (void)rows;
    int64_t s = cols / 16;
    if (layout == NVO_SF_LINEAR)
        return r * s + c;
    int64_t sp = (s + 3) / 4 * 4;
    return ((r / 128) * (sp / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

int64_t nvo_codes_bytes(int64_t rows, int64_t cols) { return rows * cols / 2; }

/* ------------------------------------------------------------ quantize */

/* Tensor amax: max |x| over all elements, exact (a max of BF16 values).
 * Returns NVO_ERR_NONFINITE if any element is Inf or NaN. */
int nvo_tensor_amax(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, float *amax)
{
    float m = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float v = fabsf(nvo_bf16_to_f32(x[r * ld + c]));
            if (!isfinite(v))
                return NVO_ERR_NONFINITE;
            if (v > m)
                m = v;
        }
    *amax = m;
    return NVO_OK;
}

/* Global (tensor) scale g = RN(448*6 / amax).  READINGS: amax == 0 gives
 * g = 1 (all blocks then quantize to zero); g must stay at or below 2^118 so
 * that every per-block factor g/s (s >= 2^-9) is finite -- smaller amax is
 * reported as NVO_ERR_RANGE. */
int nvo_global_scale(float amax, float *g)
{
    if (!isfinite(amax))
        return NVO_ERR_NONFINITE;
    if (amax == 0.0f) {
        *g = 1.0f;
        return NVO_OK;
    }
    float v = 2688.0f / amax;
    *g = v;
    if (!(v <= 0x1p118f))
        return NVO_ERR_RANGE;
    return NVO_OK;
}

/* Encode one row-major BF16 tensor with a given global scale g:
 * per 16-block along the row, s = e4m3(RN(RN(amax_b/6)*g)),
 * e = s ? RN(g/f32(s)) : 0, code = e2m1(RN(x*e)).  Codes pack two per byte,
 * element 2i in the low nibble (READING: the pages give no nibble order;
 * this is the order the FP4 tensor-core operand uses).  `scales` must hold
 * nvo_scales_bytes() bytes; padding entries are written as zero. */
void nvo_quantize_with_global(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                              float g, uint8_t *codes, uint8_t *scales, int layout)
{
    memset(scales, 0, (size_t)nvo_scales_bytes(rows, cols, layout));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 16; ++b) {
            const uint16_t *xb = x + r * ld + b * 16;
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float v = fabsf(nvo_bf16_to_f32(xb[i]));
                if (v > amax_b)
                    amax_b = v;
            }
            float t = amax_b / 6.0f;
            t = t * g;
            uint8_t s = nvo_e4m3_rne_satfinite(t);
            float sf = nvo_e4m3_decode(s);
            float e = (s == 0) ? 0.0f : g / sf;
            scales[nvo_sf_offset(r, b, rows, cols, layout)] = s;
            uint8_t *cb = codes + r * (cols / 2) + b * 8;
            for (int i = 0; i < 8; ++i) {
                float y0 = nvo_bf16_to_f32(xb[2 * i]) * e;
                float y1 = nvo_bf16_to_f32(xb[2 * i + 1]) * e;
                uint8_t c0 = nvo_e2m1_rne_satfinite(y0);
                uint8_t c1 = nvo_e2m1_rne_satfinite(y1);
                cb[i] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
}

/* Full two-level quantize: amax -> g -> encode.  Returns a status; on error
 * the outputs are unspecified.  *g_out receives the global scale. */
int nvo_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                 uint8_t *codes, uint8_t *scales, int layout, float *g_out)
{
    if (cols % 16 != 0 || rows < 0 || cols < 0)
        return NVO_ERR_SHAPE;
    float amax, g;
    int st = nvo_tensor_amax(x, rows, cols, ld, &amax);
    if (st != NVO_OK)
        return st;
    st = nvo_global_scale(amax, &g);
    *g_out = g;
    if (st != NVO_OK)
        return st;
    nvo_quantize_with_global(x, rows, cols, ld, g, codes, scales, layout);
    return NVO_OK;
}

/* ---------------------------------------------------------- dequantize */

/* x_hat = bf16(RN(f32(e2m1(code)) * d)), d = RN(f32(s) / g) per block: the
 * block scale restores the block's range and the tensor scale is divided
 * back out ([P1] section 3, [P2] two-level scaling). */
void nvo_dequantize(const uint8_t *codes, const uint8_t *scales, int layout, float g,
                    int64_t rows, int64_t cols, uint16_t *y, int64_t ld)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 16; ++b) {
            float sf = nvo_e4m3_decode(scales[nvo_sf_offset(r, b, rows, cols, layout)]);
            float d = sf / g;
            for (int i = 0; i < 16; ++i) {
                int64_t c = b * 16 + i;
                uint8_t byte = codes[r * (cols / 2) + c / 2];
                uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
                float v = nvo_e2m1_decode(code) * d;
                y[r * ld + c] = nvo_f32_to_bf16(v);
            }
        }
}

/* ----------------------------------------------------------------- GEMM */

/* Exact real value of one quantized element as a double:
 * e2m1(code) * s / g.  Both factors are exact in double. */
static double elem_f64(const uint8_t *codes, const uint8_t *scales, int layout, double g,
                       int64_t rows, int64_t cols, int64_t r, int64_t c)
{
    uint8_t byte = codes[r * (cols / 2) + c / 2];
    uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
    double s = (double)nvo_e4m3_decode(scales[nvo_sf_offset(r, c / 16, rows, cols, layout)]);
    return (double)nvo_e2m1_decode(code) * s / g;
}

/* Reference W4A4 linear, sampled: for t < count,
 *   ref[t] = sum_k Ahat[i_t,k] * What[j_t,k]     (FP64)
 *   abs[t] = sum_k |Ahat[i_t,k] * What[j_t,k]|   (FP64, for the tolerance)
 * with Ahat/What the dequantized operands in FP64 (A is M x K, W is N x K,
 * both row-major over K; D = A * W^T).  gw holds one tensor scale per
 * sample so grouped (per-expert) weights use the same routine. */
void nvo_gemm_ref(const uint8_t *a_codes, const uint8_t *a_sf, int a_layout, float ga, int64_t m,
                  const uint8_t *w_codes, const uint8_t *w_sf, int w_layout, const float *gw,
                  int64_t n, int64_t k, const int64_t *i_idx, const int64_t *j_idx,
                  int64_t count, double *ref, double *abs_sum)
{
    for (int64_t t = 0; t < count; ++t) {
        int64_t i = i_idx[t], j = j_idx[t];
        double acc = 0.0, aacc = 0.0;
        for (int64_t kk = 0; kk < k; ++kk) {
            double p = elem_f64(a_codes, a_sf, a_layout, (double)ga, m, k, i, kk) *
                       elem_f64(w_codes, w_sf, w_layout, (double)gw[t], n, k, j, kk);
            acc += p;
            aacc += fabs(p);
        }
        ref[t] = acc;
        abs_sum[t] = aacc;
    }
}

/* Integer-exact form of the same dot product, before the tensor scales:
 *   sum_k (2*e2m1(a)) * (512*sA) * (2*e2m1(w)) * (512*sW)
 * Every factor is an integer (codes*2 in [-12,12], E4M3*512 in [0,229376]),
 * so the int64 sum is exact for K up to ~1.2e6.  The real value is this
 * sum / 2^20 / (gA*gW). */
int64_t nvo_dot_exact_i64(const uint8_t *a_codes, const uint8_t *a_sf, int a_layout, int64_t m,
                          const uint8_t *w_codes, const uint8_t *w_sf, int w_layout, int64_t n,
                          int64_t k, int64_t i, int64_t j)
{
    int64_t acc = 0;
    for (int64_t kk = 0; kk < k; ++kk) {
        uint8_t ab = a_codes[i * (k / 2) + kk / 2];
        uint8_t wb = w_codes[j * (k / 2) + kk / 2];
        uint8_t ac = (kk & 1) ? (ab >> 4) : (ab & 15);
        uint8_t wc = (kk & 1) ? (wb >> 4) : (wb & 15);
        int64_t a2 = (int64_t)(2.0f * nvo_e2m1_decode(ac));
        int64_t w2 = (int64_t)(2.0f * nvo_e2m1_decode(wc));
        int64_t sa = (int64_t)(512.0f * nvo_e4m3_decode(a_sf[nvo_sf_offset(i, kk / 16, m, k, a_layout)]));
        int64_t sw = (int64_t)(512.0f * nvo_e4m3_decode(w_sf[nvo_sf_offset(j, kk / 16, n, k, w_layout)]));
        acc += a2 * sa * w2 * sw;
    }
    return acc;
}

/* ------------------------------------------- random Hadamard transform */

/* [P2'] 16x16 random Hadamard transform of one block.  READINGS (the page
 * names the matrices only): y = (1/4) * H16 * diag(s) * x with H16 the
 * Sylvester Hadamard matrix, H[i][j] = (-1)^popcount(i & j), scaled by 1/4 so
 * that the transform is orthonormal; s_j = -1 where bit j of sign_mask is
 * set.  FP32 evaluation: z_j = s_j x_j (exact), then the in-place fast
 * Walsh-Hadamard butterfly with strides 1, 2, 4, 8 -- each pair (z_i, z_{i+h})
 * becomes (RN(z_i + z_{i+h}), RN(z_i - z_{i+h})) -- then y_i = RN(z_i / 4). */
void nvo_rht16(const float *x, uint32_t sign_mask, float *y)
{
    float z[16];
    for (int j = 0; j < 16; ++j)
        z[j] = ((sign_mask >> j) & 1u) ? -x[j] : x[j];
    for (int h = 1; h < 16; h <<= 1)
        for (int i = 0; i < 16; ++i)
            if ((i & h) == 0) {
                float a = z[i], b = z[i + h];
                z[i] = a + b;
                z[i + h] = a - b;
            }
    for (int i = 0; i < 16; ++i)
        y[i] = z[i] * 0.25f;
}

/* Inverse of nvo_rht16 in exact arithmetic: x = diag(s) * (1/4) * H16 * y
 * (H16 is symmetric and H16 * H16 = 16 I).  Same butterfly, signs after. */
void nvo_rht16_inverse(const float *y, uint32_t sign_mask, float *x)
{
    float z[16];
    for (int j = 0; j < 16; ++j)
        z[j] = y[j];
    for (int h = 1; h < 16; h <<= 1)
        for (int i = 0; i < 16; ++i)
            if ((i & h) == 0) {
                float a = z[i], b = z[i + h];
                z[i] = a + b;
                z[i + h] = a - b;
            }
    for (int j = 0; j < 16; ++j) {
        float v = z[j] * 0.25f;
        x[j] = ((sign_mask >> j) & 1u) ? -v : v;
    }
}

/* Two-level NVFP4 quantization of the transformed tensor: every 16-block
 * of each row goes through nvo_rht16 first (FP32 values, not rounded back
 * to BF16), then amax, g, block scales and codes follow the same steps as
 * nvo_quantize on those FP32 values.  global_supplied = 1 uses *g_io. */
int nvo_quantize_rht(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, uint32_t sign_mask,
                     uint8_t *codes, uint8_t *scales, int layout, int global_supplied, float *g_io)
{
    if (cols % 16 != 0 || rows < 0 || cols < 0)
        return NVO_ERR_SHAPE;
    float g = *g_io;
    if (!global_supplied) {
        float m = 0.0f;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t b = 0; b < cols / 16; ++b) {
                float in[16], y[16];
                for (int i = 0; i < 16; ++i)
                    in[i] = nvo_bf16_to_f32(x[r * ld + b * 16 + i]);
                nvo_rht16(in, sign_mask, y);
                for (int i = 0; i < 16; ++i) {
                    float v = fabsf(y[i]);
                    if (!isfinite(v))
                        return NVO_ERR_NONFINITE;
                    if (v > m)
                        m = v;
                }
            }
        int st = nvo_global_scale(m, &g);
        *g_io = g;
        if (st != NVO_OK)
            return st;
    }
    memset(scales, 0, (size_t)nvo_scales_bytes(rows, cols, layout));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 16; ++b) {
            float in[16], y[16];
            for (int i = 0; i < 16; ++i)
                in[i] = nvo_bf16_to_f32(x[r * ld + b * 16 + i]);
            nvo_rht16(in, sign_mask, y);
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i)
                if (fabsf(y[i]) > amax_b)
                    amax_b = fabsf(y[i]);
            float t = amax_b / 6.0f;
            t = t * g;
            uint8_t s = nvo_e4m3_rne_satfinite(t);
            float e = (s == 0) ? 0.0f : g / nvo_e4m3_decode(s);
            scales[nvo_sf_offset(r, b, rows, cols, layout)] = s;
            uint8_t *cb = codes + r * (cols / 2) + b * 8;
            for (int i = 0; i < 8; ++i) {
                uint8_t c0 = nvo_e2m1_rne_satfinite(y[2 * i] * e);
                uint8_t c1 = nvo_e2m1_rne_satfinite(y[2 * i + 1] * e);
                cb[i] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return NVO_OK;
}

/* ------------------------------------------------------ 2D (16x16) blocks */

/* [P2'] 2D block scaling of a weight: one E4M3 scale per 16x16 block (16
 * rows x 16 columns), so that W and W^T are quantized identically.
 * READINGS: the block amax is max |x| over the block's values (a partial
 * block at the bottom edge covers the rows present); s, e and the codes
 * follow the 1D steps with that amax; the result is stored as an ordinary
 * NVFP4 tensor (1x16 scale positions along each row) whose scale entry for
 * row r, scale column b is the scale of block (r / 16, b).  g comes from the
 * plain tensor amax (or is supplied). */
int nvo_quantize_2d(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, uint8_t *codes,
                    uint8_t *scales, int layout, int global_supplied, float *g_io)
{
    if (cols % 16 != 0 || rows < 0 || cols < 0)
        return NVO_ERR_SHAPE;
    float g = *g_io;
    if (!global_supplied) {
        float amax;
        int st = nvo_tensor_amax(x, rows, cols, ld, &amax);
        if (st != NVO_OK)
            return st;
        st = nvo_global_scale(amax, &g);
        *g_io = g;
        if (st != NVO_OK)
            return st;
    }
    memset(scales, 0, (size_t)nvo_scales_bytes(rows, cols, layout));
    for (int64_t a = 0; a * 16 < rows; ++a)
        for (int64_t b = 0; b < cols / 16; ++b) {
            const int64_t r_end = (a * 16 + 16 < rows) ? a * 16 + 16 : rows;
            float amax_b = 0.0f;
            for (int64_t r = a * 16; r < r_end; ++r)
                for (int i = 0; i < 16; ++i) {
                    float v = fabsf(nvo_bf16_to_f32(x[r * ld + b * 16 + i]));
                    if (v > amax_b)
                        amax_b = v;
                }
            float t = amax_b / 6.0f;
            t = t * g;
            uint8_t s = nvo_e4m3_rne_satfinite(t);
            float e = (s == 0) ? 0.0f : g / nvo_e4m3_decode(s);
            for (int64_t r = a * 16; r < r_end; ++r) {
                scales[nvo_sf_offset(r, b, rows, cols, layout)] = s;
                uint8_t *cb = codes + r * (cols / 2) + b * 8;
                for (int i = 0; i < 8; ++i) {
                    uint8_t c0 = nvo_e2m1_rne_satfinite(nvo_bf16_to_f32(x[r * ld + b * 16 + 2 * i]) * e);
                    uint8_t c1 = nvo_e2m1_rne_satfinite(nvo_bf16_to_f32(x[r * ld + b * 16 + 2 * i + 1]) * e);
                    cb[i] = (uint8_t)(c0 | (c1 << 4));
                }
            }
        }
    return NVO_OK;
}

/* ---------------------------------------------- counter-based random bits */

/* [PX] Philox4x32-10: ten rounds on a 128-bit counter under a 64-bit key.
 * A round multiplies words 0 and 2 by 0xD2511F53 and 0xCD9E8D57 (full
 * 64-bit products), then sets (c0, c1, c2, c3) = (hi(c2*M1) ^ c1 ^ k0,
 * lo(c2*M1), hi(c0*M0) ^ c3 ^ k1, lo(c0*M0)); the key gains the Weyl
 * constants 0x9E3779B9 and 0xBB67AE85 after every round. */
void nvo_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c[1] ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c[3] ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    for (int i = 0; i < 4; ++i)
        out[i] = c[i];
}

/* ----------------------------------------------------- stochastic rounding */

/* [P2'] Stochastic rounding onto the E2M1 grid.  READINGS: |y| >= 6
 * saturates to 6; otherwise with lo <= |y| < hi the neighbouring grid
 * values, |y| rounds up to hi with probability (|y| - lo) / (hi - lo),
 * decided by a 16-bit uniform draw u (up iff u / 2^16 < that fraction, so
 * the probability is ceil(2^16 * fraction) / 2^16); grid values stay put;
 * the sign is copied from y (as in the round-to-nearest encode).  Returns
 * the 4-bit code. */
uint8_t nvo_e2m1_sr(float y, uint32_t u16)
{
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    uint8_t sign = signbit(y) ? 8 : 0;
    double a = fabs((double)y);
    if (a >= 6.0)
        return sign | 7;
    int k = 0;
    while (k < 7 && grid[k + 1] <= a)
        ++k;                                   /* grid[k] <= a < grid[k + 1] */
    double frac = (a - grid[k]) / (grid[k + 1] - grid[k]);
    int up = ((double)u16 / 65536.0) < frac;
    return sign | (uint8_t)(k + up);
}

/* Random 16-bit draws of the 16 values of output block (row r, block b) of
 * an R x C NVFP4 tensor, for the caller's 64-bit seed.  READING (the pages
 * fix no generator): block index n = r * (C / 16) + b; Philox4x32-10 with
 * counter (lo32(n), hi32(n), j, 0), j = 0, 1, and key (lo32(seed),
 * hi32(seed)); value 8j + 2w takes the low 16 bits of word w of draw j,
 * value 8j + 2w + 1 its high 16 bits. */
void nvo_sr_block_draws(uint64_t seed, int64_t r, int64_t b, int64_t cols, uint32_t u[16])
{
    uint64_t n = (uint64_t)r * (uint64_t)(cols / 16) + (uint64_t)b;
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (uint32_t j = 0; j < 2; ++j) {
        uint32_t ctr[4] = {(uint32_t)n, (uint32_t)(n >> 32), j, 0u}, w[4];
        nvo_philox4x32_10(ctr, key, w);
        for (int i = 0; i < 4; ++i) {
            u[8 * j + 2 * i] = w[i] & 0xFFFFu;
            u[8 * j + 2 * i + 1] = w[i] >> 16;
        }
    }
}

/* Two-level quantization with stochastic rounding of the codes (the block
 * scales and g as in nvo_quantize; rht = 1 transforms every block first as
 * in nvo_quantize_rht). */
int nvo_quantize_sr(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int rht,
                    uint32_t sign_mask, uint64_t seed, uint8_t *codes, uint8_t *scales, int layout,
                    int global_supplied, float *g_io)
{
    if (cols % 16 != 0 || rows < 0 || cols < 0)
        return NVO_ERR_SHAPE;
    float g = *g_io;
    if (!global_supplied) {
        float m = 0.0f;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t b = 0; b < cols / 16; ++b) {
                float in[16], y[16];
                for (int i = 0; i < 16; ++i)
                    in[i] = nvo_bf16_to_f32(x[r * ld + b * 16 + i]);
                if (rht)
                    nvo_rht16(in, sign_mask, y);
                else
                    memcpy(y, in, sizeof y);
                for (int i = 0; i < 16; ++i) {
                    float v = fabsf(y[i]);
                    if (!isfinite(v))
                        return NVO_ERR_NONFINITE;
                    if (v > m)
                        m = v;
                }
            }
        int st = nvo_global_scale(m, &g);
        *g_io = g;
        if (st != NVO_OK)
            return st;
    }
    memset(scales, 0, (size_t)nvo_scales_bytes(rows, cols, layout));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 16; ++b) {
            float in[16], y[16];
            uint32_t u[16];
            for (int i = 0; i < 16; ++i)
                in[i] = nvo_bf16_to_f32(x[r * ld + b * 16 + i]);
            if (rht)
                nvo_rht16(in, sign_mask, y);
            else
                memcpy(y, in, sizeof y);
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i)
                if (fabsf(y[i]) > amax_b)
                    amax_b = fabsf(y[i]);
            float t = amax_b / 6.0f;
            t = t * g;
            uint8_t s = nvo_e4m3_rne_satfinite(t);
            float e = (s == 0) ? 0.0f : g / nvo_e4m3_decode(s);
            scales[nvo_sf_offset(r, b, rows, cols, layout)] = s;
            nvo_sr_block_draws(seed, r, b, cols, u);
            uint8_t *cb = codes + r * (cols / 2) + b * 8;
            for (int i = 0; i < 8; ++i) {
                uint8_t c0 = nvo_e2m1_sr(y[2 * i] * e, u[2 * i]);
                uint8_t c1 = nvo_e2m1_sr(y[2 * i + 1] * e, u[2 * i + 1]);
                cb[i] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return NVO_OK;
}

/* ------------------------------------------------------------------ MXFP4 */

/* [PM] UE8M0 block scale: byte b encodes 2^(b - 127); 255 is NaN. */
double nvo_ue8m0_decode(uint8_t b)
{
    return (b == 255) ? NAN : ldexp(1.0, (int)b - 127);
}

int64_t nvo_mx_scales_bytes(int64_t rows, int64_t cols, int layout)
{
    int64_t s = cols / 32;
    if (layout == NVO_SF_LINEAR)
        return rows * s;
    return (rows + 127) / 128 * 128 * ((s + 3) / 4 * 4);
}

/* Scale positions: the 128x4 tiled layout (or row-major) over the
 * cols / 32 scale columns, as for NVFP4 over cols / 16. */
int64_t nvo_mx_sf_offset(int64_t r, int64_t c, int64_t cols, int layout)
{
    int64_t s = cols / 32;
    if (layout == NVO_SF_LINEAR)
        return r * s + c;
    int64_t sp = (s + 3) / 4 * 4;
    return ((r / 128) * (sp / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* [PM] Shared exponent of a 32-value block.  READING (the pages fix only
 * "power of two"): the OCP microscaling rule X = floor(log2(amax)) - 2,
 * 2 being the exponent of the largest E2M1 value (6 = 1.5 * 2^2), so the
 * block amax lands in [4, 8) after scaling (values above 6 saturate);
 * clamped to [-127, 127]; an all-zero block takes X = -127. */
int nvo_mx_exponent(float amax)
{
    if (amax == 0.0f)
        return -127;
    int ex;
    frexp((double)amax, &ex);          /* amax = f * 2^ex, f in [0.5, 1) */
    int X = ex - 1 - 2;
    if (X < -127)
        X = -127;
    if (X > 127)
        X = 127;
    return X;
}

/* [PM] MXFP4 quantization: per 32 consecutive values of a row, the scale
 * byte X + 127 and codes e2m1_rne_satfinite(RN(x * 2^-X)) (the product by
 * a power of two is exact unless it underflows).  No tensor scale.  Returns
 * NVO_ERR_NONFINITE for Inf/NaN input (outputs unspecified). */
int nvo_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, uint8_t *codes,
                    uint8_t *scales, int layout)
{
    if (cols % 32 != 0 || rows < 0 || cols < 0)
        return NVO_ERR_SHAPE;
    memset(scales, 0, (size_t)nvo_mx_scales_bytes(rows, cols, layout));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 32; ++b) {
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float v = fabsf(nvo_bf16_to_f32(x[r * ld + b * 32 + i]));
                if (!isfinite(v))
                    return NVO_ERR_NONFINITE;
                if (v > amax)
                    amax = v;
            }
            int X = nvo_mx_exponent(amax);
            scales[nvo_mx_sf_offset(r, b, cols, layout)] = (uint8_t)(X + 127);
            float inv = ldexpf(1.0f, -X);
            uint8_t *cb = codes + r * (cols / 2) + b * 16;
            for (int i = 0; i < 16; ++i) {
                uint8_t c0 = nvo_e2m1_rne_satfinite(nvo_bf16_to_f32(x[r * ld + b * 32 + 2 * i]) * inv);
                uint8_t c1 = nvo_e2m1_rne_satfinite(nvo_bf16_to_f32(x[r * ld + b * 32 + 2 * i + 1]) * inv);
                cb[i] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return NVO_OK;
}

/* x_hat = bf16(e2m1(code) * 2^X), exact before the BF16 rounding. */
void nvo_dequantize_mx(const uint8_t *codes, const uint8_t *scales, int layout, int64_t rows,
                       int64_t cols, uint16_t *y, int64_t ld)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
            double v = (double)nvo_e2m1_decode(code) *
                       nvo_ue8m0_decode(scales[nvo_mx_sf_offset(r, c / 32, cols, layout)]);
            y[r * ld + c] = nvo_f32_to_bf16((float)v);
        }
}

/* Sampled FP64 reference of D = Ahat * What^T for MXFP4 operands (no
 * tensor scales): ref[t] and abs[t] as in nvo_gemm_ref. */
void nvo_gemm_ref_mx(const uint8_t *a_codes, const uint8_t *a_scales, int a_layout, int64_t m,
                     const uint8_t *w_codes, const uint8_t *w_scales, int w_layout, int64_t n,
                     int64_t k, const int64_t *i_idx, const int64_t *j_idx, int64_t count,
                     double *ref, double *abs_out)
{
    (void)m;
    (void)n;
    for (int64_t t = 0; t < count; ++t) {
        double acc = 0.0, aacc = 0.0;
        for (int64_t c = 0; c < k; ++c) {
            uint8_t ab = a_codes[i_idx[t] * (k / 2) + c / 2], wb = w_codes[j_idx[t] * (k / 2) + c / 2];
            double av = nvo_e2m1_decode((c & 1) ? (ab >> 4) : (ab & 15)) *
                        nvo_ue8m0_decode(a_scales[nvo_mx_sf_offset(i_idx[t], c / 32, k, a_layout)]);
            double wv = nvo_e2m1_decode((c & 1) ? (wb >> 4) : (wb & 15)) *
                        nvo_ue8m0_decode(w_scales[nvo_mx_sf_offset(j_idx[t], c / 32, k, w_layout)]);
            acc += av * wv;
            aacc += fabs(av * wv);
        }
        ref[t] = acc;
        abs_out[t] = aacc;
    }
}

/* ------------------------------------------------------------ consumers */

/* [PC] MoE combine: y[t] = bf16(sum_k w[t][k] * out[slot[t][k]]) over the
 * token's topk expert rows.  READINGS: the weights are the caller's
 * (routing) combine weights; FP32 accumulation in k order, each step one
 * fused multiply-add (acc = fma(w, x, acc), starting from 0); a slot of -1
 * contributes nothing; one BF16 rounding at the end. */
void nvo_moe_combine(const uint16_t *out, int64_t ld, const int32_t *slots, const float *w,
                     int64_t tokens, int64_t topk, int64_t hidden, uint16_t *y, int64_t ldy)
{
    for (int64_t t = 0; t < tokens; ++t)
        for (int64_t c = 0; c < hidden; ++c) {
            float acc = 0.0f;
            for (int64_t k = 0; k < topk; ++k) {
                int32_t s = slots[t * topk + k];
                if (s < 0)
                    continue;
                acc = fmaf(w[t * topk + k], nvo_bf16_to_f32(out[(int64_t)s * ld + c]), acc);
            }
            y[t * ldy + c] = nvo_f32_to_bf16(acc);
        }
}

/* [PC] NVFP4 -> FP8 (E4M3) for an attention read.  READING (the page says
 * only that the FP4 cache is dequantized to FP8): each value becomes
 * e4m3_rne_satfinite(e2m1(code) * s_b / 8), with one per-tensor dequant
 * factor RN(8 / g) returned in *fp8_scale, so x_hat ~= fp8 * fp8_scale.
 * e2m1 * s_b / 8 is exact in FP32 (the 1/8 keeps 6 * 448 = 2688 inside the
 * E4M3 range); the E4M3 rounding is the only one.  Sign kept. */
void nvo_dequantize_fp8(const uint8_t *codes, const uint8_t *scales, int layout, float g,
                        int64_t rows, int64_t cols, uint8_t *y, int64_t ld, float *fp8_scale)
{
    *fp8_scale = 8.0f / g;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
            float sb = nvo_e4m3_decode(scales[nvo_sf_offset(r, c / 16, rows, cols, layout)]);
            float v = nvo_e2m1_decode(code) * sb / 8.0f;
            uint8_t e = nvo_e4m3_rne_satfinite(fabsf(v));
            y[r * ld + c] = (uint8_t)(e | (signbit(v) ? 0x80 : 0));
        }
}

/* ------------------------------------------------------- gated activation */

/* [PE] exp(x) for the SiLU, with every step an IEEE binary32 operation in a
 * fixed order (so any implementation of these steps gives the same bits):
 * x clamped to [-87, 87]; n = rint(RN(x * RN(log2 e))); r = fma(-n, L_hi, x),
 * r = fma(-n, L_lo, r) with L_hi = ln 2 rounded to a multiple of 2^-16 and
 * L_lo = RN(ln 2 - L_hi); p = the degree-7 Taylor polynomial of e^r in
 * Horner form with fma (coefficients RN(1/k!)); result RN(p * 2^n). */
float nvo_exp_ref(float x)
{
    const float l2e = 1.44269504088896340736f;
    const float l_hi = 0.693145751953125f;               /* 45426 / 65536 */
    const float l_lo = (float)(0.69314718055994530942 - 0.693145751953125);
    if (x > 87.0f)
        x = 87.0f;
    if (x < -87.0f)
        x = -87.0f;
    float n = rintf(x * l2e);
    float r = fmaf(-n, l_hi, x);
    r = fmaf(-n, l_lo, r);
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    return p * ldexpf(1.0f, (int)n);
}

/* [PG] h = silu(g) * u = RN(RN(g * RN(1 / RN(1 + exp(-g)))) * u). */
float nvo_swiglu(float g, float u)
{
    float e = nvo_exp_ref(-g);
    float s = 1.0f / (1.0f + e);
    return (g * s) * u;
}

/* Quantize h = silu(gate) * up of a [rows x 2I] BF16 tensor (gate in
 * columns 0..I-1, up in I..2I-1: READING, the pages give no layout) to
 * NVFP4 [rows x I], the FP32 values h quantized with the plain two-level
 * steps (amax over h; RN(amax_b / 6) by division). */
int nvo_quantize_swiglu(const uint16_t *gu, int64_t rows, int64_t inter, int64_t ld, uint8_t *codes,
                        uint8_t *scales, int layout, float *g_out)
{
    if (inter % 16 != 0 || rows < 0 || inter < 0)
        return NVO_ERR_SHAPE;
    float m = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < inter; ++c) {
            float h = fabsf(nvo_swiglu(nvo_bf16_to_f32(gu[r * ld + c]), nvo_bf16_to_f32(gu[r * ld + inter + c])));
            if (!isfinite(h))
                return NVO_ERR_NONFINITE;
            if (h > m)
                m = h;
        }
    float g;
    int st = nvo_global_scale(m, &g);
    *g_out = g;
    if (st != NVO_OK)
        return st;
    memset(scales, 0, (size_t)nvo_scales_bytes(rows, inter, layout));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < inter / 16; ++b) {
            float y[16], amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                int64_t c = b * 16 + i;
                y[i] = nvo_swiglu(nvo_bf16_to_f32(gu[r * ld + c]), nvo_bf16_to_f32(gu[r * ld + inter + c]));
                if (fabsf(y[i]) > amax_b)
                    amax_b = fabsf(y[i]);
            }
            float t = amax_b / 6.0f;
            t = t * g;
            uint8_t s = nvo_e4m3_rne_satfinite(t);
            float e = (s == 0) ? 0.0f : g / nvo_e4m3_decode(s);
            scales[nvo_sf_offset(r, b, rows, inter, layout)] = s;
            uint8_t *cb = codes + r * (inter / 2) + b * 8;
            for (int i = 0; i < 8; ++i) {
                uint8_t c0 = nvo_e2m1_rne_satfinite(y[2 * i] * e);
                uint8_t c1 = nvo_e2m1_rne_satfinite(y[2 * i + 1] * e);
                cb[i] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    return NVO_OK;
}

/* ------------------------------------------------------- attention read */

/* [PC] One decode step of attention over an NVFP4 KV cache (the KV page:
 * every generated token re-reads the cache, and the FP4 values are
 * restored to higher precision before the attention arithmetic).
 * READINGS: K and V are NVFP4 tensors [tokens x heads_kv * head_dim] (one
 * row per cached token, head h in columns h*head_dim .. +head_dim-1,
 * blocks of 16 along head_dim) with tensor scales gk, gv; query head h
 * (BF16 row h of q, pitch ldq) attends with KV head h / (heads_q /
 * heads_kv) (grouped-query attention); the restored values are the exact
 * reals e2m1 * s_b / g (no intermediate FP8 rounding); the scores are
 * scale * q . k and the weights their softmax over all tokens.  Computed in
 * FP64 with the maximum score subtracted before exp, for the query heads
 * h_begin <= h < h_end (rows h - h_begin of the outputs):
 *   o[h][d]      = sum_t p_t v[t][d] / sum_t p_t
 *   abs_o[h][d]  = sum_t p_t |v[t][d]| / sum_t p_t   (for the tolerance)
 *   score_abs[h] = max_t |scale| * sum_d |q_d k[t][d]| (for the tolerance)
 * tokens == 0 gives o = abs_o = 0.  Returns NVO_ERR_SHAPE for a head count
 * that does not divide, head_dim % 16 != 0 or a bad size or head range. */
int nvo_attention_decode(const uint16_t *q, int64_t ldq, int64_t heads_q, const uint8_t *kc,
                         const uint8_t *ks, float gk, const uint8_t *vc, const uint8_t *vs,
                         float gv, int layout, int64_t tokens, int64_t heads_kv, int64_t head_dim,
                         double scale, int64_t h_begin, int64_t h_end, double *o, double *abs_o,
                         double *score_abs)
{
    if (heads_kv <= 0 || heads_q <= 0 || heads_q % heads_kv != 0 || head_dim <= 0 ||
        head_dim % 16 != 0 || tokens < 0 || h_begin < 0 || h_end > heads_q || h_begin > h_end)
        return NVO_ERR_SHAPE;
    const int64_t group = heads_q / heads_kv, cols = heads_kv * head_dim;
    double *p = (double *)malloc((size_t)(tokens + 1) * sizeof(double));
    double *num = (double *)malloc((size_t)head_dim * 2 * sizeof(double));
    if (p == NULL || num == NULL) {
        free(p);
        free(num);
        return NVO_ERR_SHAPE;
    }
    double *anum = num + head_dim;
    for (int64_t h = h_begin; h < h_end; ++h) {
        const int64_t c0 = (h / group) * head_dim, row = h - h_begin;
        double mx = -INFINITY, amax = 0.0;
        for (int64_t t = 0; t < tokens; ++t) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t d = 0; d < head_dim; ++d) {
                double qd = (double)nvo_bf16_to_f32(q[h * ldq + d]);
                double kd = elem_f64(kc, ks, layout, (double)gk, tokens, cols, t, c0 + d);
                acc += qd * kd;
                aacc += fabs(qd * kd);
            }
            p[t] = scale * acc;
            if (p[t] > mx)
                mx = p[t];
            if (fabs(scale) * aacc > amax)
                amax = fabs(scale) * aacc;
        }
        score_abs[row] = amax;
        double den = 0.0;
        for (int64_t t = 0; t < tokens; ++t) {
            p[t] = exp(p[t] - mx);
            den += p[t];
        }
        for (int64_t d = 0; d < head_dim; ++d)
            num[d] = anum[d] = 0.0;
        for (int64_t t = 0; t < tokens; ++t)
            for (int64_t d = 0; d < head_dim; ++d) {
                double vd = elem_f64(vc, vs, layout, (double)gv, tokens, cols, t, c0 + d);
                num[d] += p[t] * vd;
                anum[d] += p[t] * fabs(vd);
            }
        for (int64_t d = 0; d < head_dim; ++d) {
            o[row * head_dim + d] = tokens > 0 ? num[d] / den : 0.0;
            abs_o[row * head_dim + d] = tokens > 0 ? anum[d] / den : 0.0;
        }
    }
    free(p);
    free(num);
    return NVO_OK;
}
