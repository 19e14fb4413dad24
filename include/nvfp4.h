/*
 * nvfp4.h -- C ABI of libnvfp4.so, the B200 (sm_100a) NVFP4 hot path.
 *
 * NVFP4 stores a tensor as 4-bit E2M1 codes (values +-0, 0.5, 1, 1.5, 2, 3,
 * 4, 6), one E4M3 scale per 16 consecutive values along the last dimension,
 * and one FP32 scale per tensor.  Sources: "NVFP4: how NVIDIA pre-trained a
 * 12B model on 10T tokens" (axbrief.com), section "E2M1 format and
 * two-level scaling"; "NVIDIA shrank GLM-5.2 to 4 bits" (iwan.kr), section 3;
 * "FP4 KV-cache quantization" (theddari.com), sections "KV cache size
 * example" and "FP4 formats compared".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Memory: every pointer named d_* or held in an nvfp4_tensor is DEVICE
 *   memory owned by the caller.  The library allocates no device memory and
 *   keeps no handle to caller buffers after a call returns.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *   default stream).  Work is enqueued asynchronously; argument errors are
 *   returned synchronously before anything is enqueued.
 * - Device-side errors (non-finite input, out-of-range tensor amax, a
 *   pipeline wait that exceeded its bound) are recorded in the 32-bit status
 *   word at the start of the caller's workspace.  The first error sticks
 *   until nvfp4_check_status() reads and clears it.  A workspace must be
 *   zero-filled once before its first use.
 * - Alignment: tensor base pointers and row pitches 16-byte aligned.
 * - Device: compute capability 10.0 (B200, sm_100a) is required; any other
 *   device gives NVFP4_ERR_UNSUPPORTED_DEVICE.  There is no fallback.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad enum */
    NVFP4_ERR_ALIGNMENT = 2,        /* pointer or pitch not 16-byte aligned */
    NVFP4_ERR_SHAPE = 3,            /* shape rule of the call violated */
    NVFP4_ERR_NONFINITE = 4,        /* input holds Inf or NaN (device-side) */
    NVFP4_ERR_RANGE = 5,            /* tensor amax so small that g > 2^118 */
    NVFP4_ERR_WORKSPACE = 6,        /* workspace missing or too small */
    NVFP4_ERR_TIMEOUT = 7,          /* a device pipeline wait gave up */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 8,
    NVFP4_ERR_CUDA = 9              /* a CUDA runtime/driver call failed */
} nvfp4_status;

/* Block-scale layouts.
 * SWIZZLED_128x4: the tiled layout the block-scaled tensor-core MMA reads.
 *   For row r and scale column c (= element column / 16), with
 *   S4 = ceil(cols/16 / 4) * 4 padded scale columns:
 *     offset = ((r/128) * (S4/4) + c/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + c%4
 *   The buffer covers ceil(rows/128)*128 rows x S4 columns; padding holds 0.
 * LINEAR: row-major [rows x cols/16], offset = r * (cols/16) + c. */
typedef enum {
    NVFP4_SF_SWIZZLED_128x4 = 0,
    NVFP4_SF_LINEAR = 1
} nvfp4_sf_layout;

/* An NVFP4 tensor of `rows` x `cols` logical values.
 * codes : rows x cols/2 bytes, row-major, two codes per byte, element 2i in
 *         the low nibble and 2i+1 in the high nibble.  Sign in bit 3.
 * scales: nvfp4_scales_bytes(rows, cols, sf_layout) bytes of E4M3 scales.
 * global: one float, the tensor scale g = 448*6 / amax(tensor) (g = 1 for an
 *         all-zero tensor).  A value x is represented as
 *         e2m1(code) * e4m3(scale) / g. */
typedef struct {
    void *codes;
    void *scales;
    float *global;
    int64_t rows;
    int64_t cols;
    int32_t sf_layout;
} nvfp4_tensor;

/* Operation ids for nvfp4_workspace_bytes(). */
typedef enum {
    NVFP4_OP_QUANTIZE = 0,
    NVFP4_OP_DEQUANTIZE = 1,
    NVFP4_OP_GEMM = 2,
    NVFP4_OP_GROUPED_GEMM = 3,
    NVFP4_OP_QUANTIZE_GATHER = 4,
    NVFP4_OP_ATTENTION = 5          /* a = tokens, b = query heads, c = KV heads */
} nvfp4_op;

/* ---- sizes ------------------------------------------------------------ */

/* Bytes of the packed code array: rows * cols / 2. */
NVFP4_API size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);

/* Bytes of the block-scale array for the given layout (see above). */
NVFP4_API size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout);

/* Bytes of workspace the operation can use (the first 4 bytes are the
 * status word).  The arguments are the operation's sizes (rows/cols, or
 * m/n/k) and the group count for grouped calls.  Quantize calls need the
 * returned amount.  A dense GEMM needs only 256 bytes; with M <= 128 the
 * returned amount also holds the FP32 partial sums of the split-K path (K
 * split over up to 8 SMs per output tile when there are fewer output tiles
 * than SMs), which a smaller workspace turns off without changing what is
 * computed beyond the FP32 summation order. */
NVFP4_API size_t nvfp4_workspace_bytes(int32_t op, int64_t a, int64_t b, int64_t c, int32_t groups);

/* ---- quantize --------------------------------------------------------- */

/* Two-level NVFP4 quantization of a row-major BF16 matrix.
 * ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens", section
 * "E2M1 format and two-level scaling": a per-tensor FP32 scale sets the
 * range, an E4M3 scale per 16-value block maps each block's amax close to
 * the FP4 maximum.)
 *   amax = max |x|;  g = RN(2688 / amax)            (skipped if global_supplied)
 *   per 16-block b of a row:  s_b = e4m3_rne_satfinite(RN(RN(amax_b / 6) * g))
 *                             e_b = s_b ? RN(g / s_b) : 0
 *   code = e2m1_rne_satfinite(RN(x * e_b)), sign kept (-0 -> 0x8)
 * x        : device BF16, out->rows x out->cols, row pitch `ld` elements.
 * out      : destination; codes/scales/global are written.  out->cols must
 *            be a multiple of 16, out->rows >= 0.
 * global_supplied: 0 = compute amax and g and store g to *out->global;
 *            1 = use the g already stored at *out->global (one pass).
 * Errors: argument checks synchronously; Inf/NaN in x -> NVFP4_ERR_NONFINITE
 *   and amax below 2688 * 2^-118 -> NVFP4_ERR_RANGE, both via the status word
 *   (outputs then unspecified). */
NVFP4_API nvfp4_status nvfp4_quantize(const void *x, int64_t ld, const nvfp4_tensor *out,
                            int32_t global_supplied, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Row gather of an NVFP4 tensor, for MoE expert batches: output row r is
 * source row d_gather[r] -- its packed codes and its block scales -- and
 * d_gather[r] == -1 makes row r a zero padding row (codes and scales 0);
 * *out->global = *src->global.  Quantization is row-wise once the tensor
 * scale is fixed, so gathering the rows of nvfp4_quantize(x) gives the same
 * bytes as nvfp4_quantize_gather(x, d_gather, global_supplied with x's
 * tensor scale) while moving 0.5625 instead of 2 bytes per gathered value.
 * ("NVIDIA shrank GLM-5.2 to 4 bits", section 1: the MoE expert linears take
 * NVFP4 activations; section 2: each token goes to 8 of 256 experts.)
 * src      : NVFP4 tensor, src->rows x src->cols, either scale layout.
 * d_gather : device int32[out->rows].  An entry >= src->rows is not read:
 *            its row is zeroed and NVFP4_ERR_INVALID_ARG is recorded in the
 *            status word.
 * out      : out->cols == src->cols; either scale layout (the 128x4 layout's
 *            padding rows are zeroed).
 * workspace: only its 256-byte status block is used.
 * Errors: argument checks synchronously. */
NVFP4_API nvfp4_status nvfp4_gather_rows(const nvfp4_tensor *src, const int32_t *d_gather,
                                         const nvfp4_tensor *out, void *workspace,
                                         size_t workspace_bytes, void *stream);

/* Tensor scale only: *d_global = RN(2688 / max|x|) over a rows x cols BF16
 * matrix with pitch ld (1.0 if all zero).  Same status rules as
 * nvfp4_quantize.  Lets a caller share one g between tensors or take g from
 * a tensor other than the one encoded (nvfp4_quantize_gather). */
NVFP4_API nvfp4_status nvfp4_global_scale(const void *x, int64_t ld, int64_t rows, int64_t cols,
                                float *d_global, void *workspace, size_t workspace_bytes,
                                void *stream);

/* Quantize rows gathered through a row map, for MoE expert batches.
 * Output row r takes source row d_gather[r] of x (src_rows x out->cols,
 * pitch ld); d_gather[r] == -1 makes row r a zero padding row (all codes
 * and scales 0).  out->rows is the number of gathered rows.  A map entry
 * >= src_rows is not read: its row is zeroed and NVFP4_ERR_INVALID_ARG is
 * recorded in the status word.
 * global_supplied: 1 = use *out->global (e.g. from nvfp4_global_scale over
 *   the whole source), 0 = amax over the gathered (non -1) rows.
 * ("NVIDIA shrank GLM-5.2 to 4 bits", section 1: weights and activations of
 * the MoE expert linears are NVFP4; section 2: 256 experts, 8 per token.) */
NVFP4_API nvfp4_status nvfp4_quantize_gather(const void *x, int64_t ld, int64_t src_rows,
                                   const int32_t *d_gather, const nvfp4_tensor *out,
                                   int32_t global_supplied, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* Quantize after a 16x16 random Hadamard transform of every 16-value block
 * ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens", section
 * "Four stabilisation devices": the Wgrad GEMM inputs are multiplied by a
 * 16x16 Hadamard matrix and a random +-1 sign vector before quantization).
 * Per block of 16 consecutive values along a row:
 *   y = (1/4) * H16 * diag(s) * x,  H16[i][j] = (-1)^popcount(i & j),
 *   s_j = -1 where bit j of sign_mask is set, else +1,
 * evaluated in FP32 as an in-place butterfly with strides 1, 2, 4, 8 (each
 * add/sub rounded to nearest even) and an exact-order multiply by 1/4.  The
 * FP32 values y (not rounded to BF16) are then quantized as nvfp4_quantize
 * quantizes x: g = RN(2688 / max|y|) unless supplied, s_b, codes.  The
 * transform is orthogonal, so an NVFP4 GEMM of two operands transformed
 * with the same sign_mask along the contraction axis approximates the
 * product of the untransformed operands.
 * sign_mask: the random sign vector drawn by the caller, bits 0..15
 *   (NVFP4_ERR_INVALID_ARG if any higher bit is set).
 * Other arguments, the workspace, the status word and the errors are those
 * of nvfp4_quantize; an input whose transform overflows FP32 reports
 * NVFP4_ERR_NONFINITE. */
NVFP4_API nvfp4_status nvfp4_quantize_rht(const void *x, int64_t ld, uint32_t sign_mask,
                                          const nvfp4_tensor *out, int32_t global_supplied,
                                          void *workspace, size_t workspace_bytes, void *stream);

/* Column-wise quantization: out = NVFP4 of x^T, read straight from a
 * row-major x without a BF16 transpose in memory.  The Dgrad and Wgrad GEMMs
 * ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens", section
 * "Four stabilisation devices": Fprop, Dgrad and Wgrad all in NVFP4)
 * contract over the axes the forward pass keeps contiguous, and the
 * block-scaled GEMM wants 16-value blocks along its contraction axis: for
 * Wgrad dW = dY^T X both dY and X are quantized column-wise.
 * x: BF16, out->cols rows x out->rows columns, row pitch ld elements.
 *   out->cols % 16 == 0 (blocks of 16 rows of x); out->rows % 8 == 0
 *   (NVFP4_ERR_SHAPE otherwise); x and ld 16-byte aligned.
 * out: [out->rows x out->cols]; output row j is column j of x.  Codes,
 *   scales and the tensor scale equal those of nvfp4_quantize (rht = 0) or
 *   nvfp4_quantize_rht (rht = 1, sign_mask as there) applied to an explicit
 *   BF16 copy of x^T.
 * Workspace, status word, global_supplied and errors as nvfp4_quantize. */
NVFP4_API nvfp4_status nvfp4_quantize_t(const void *x, int64_t ld, int32_t rht, uint32_t sign_mask,
                                        const nvfp4_tensor *out, int32_t global_supplied,
                                        void *workspace, size_t workspace_bytes, void *stream);

/* 2D (16x16 block) quantization of a weight ("NVFP4: how NVIDIA pre-trained
 * a 12B model on 10T tokens", section "Four stabilisation devices": weights
 * use 16x16 blocks so that W and W^T hold the same quantized values, which
 * the Fprop and Dgrad GEMMs then share).
 * One E4M3 scale per block of 16 rows x 16 columns of w, from the block's
 * amax (a partial block at the bottom edge covers the rows present); the
 * codes of each value follow the 1D steps under that scale.  g as in
 * nvfp4_quantize (plain tensor amax, or supplied in *out->global).
 * w: BF16 out->rows x out->cols, pitch ld, 16-byte aligned.
 * out: W's NVFP4 tensor (16 rows of a group share each scale entry).
 * out_t: NULL, or W^T's NVFP4 tensor [out->cols x out->rows] (requires
 *   out->rows % 16 == 0 and out->cols % 8 == 0): the same quantized values
 *   transposed, scales of block (a, b) at row k, column a for every k in
 *   column group b; its tensor scale receives the same g.
 * Workspace, status word and errors as nvfp4_quantize. */
NVFP4_API nvfp4_status nvfp4_quantize_2d(const void *w, int64_t ld, const nvfp4_tensor *out,
                                         const nvfp4_tensor *out_t, int32_t global_supplied,
                                         void *workspace, size_t workspace_bytes, void *stream);

/* Quantization with stochastically rounded codes, for gradients ("NVFP4:
 * how NVIDIA pre-trained a 12B model on 10T tokens", section "Four
 * stabilisation devices": gradients are rounded stochastically -- a value
 * 0.7 of the way to the next grid point goes up with probability 0.7).
 * Scales and g are those of the round-to-nearest path; each value y = x*e
 * (after the optional transform) goes to the E2M1 grid point above it with
 * probability (|y| - lo) / (hi - lo), decided by a 16-bit draw u (up iff
 * u / 2^16 < that fraction; grid values stay, |y| >= 6 saturates, the sign
 * is kept).  Draws: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 * random numbers: as easy as 1, 2, 3", SC 2011) keyed by `seed`, counter
 * (lo32(n), hi32(n), j, 0) for output block n = row * (cols / 16) + block
 * column and j = 0, 1; value 8j + 2w uses the low 16 bits of word w of draw
 * j, value 8j + 2w + 1 the high 16 bits.  The same seed gives the same
 * codes on every call.
 * transposed: 0 = row-wise (x is out->rows x out->cols, as nvfp4_quantize),
 *   1 = column-wise (x is out->cols x out->rows, as nvfp4_quantize_t).
 * rht, sign_mask: apply the random Hadamard transform first (as
 *   nvfp4_quantize_rht); rht = 0 ignores sign_mask.
 * Other arguments, workspace and errors as nvfp4_quantize / _t. */
NVFP4_API nvfp4_status nvfp4_quantize_sr(const void *x, int64_t ld, int32_t transposed, int32_t rht,
                                         uint32_t sign_mask, uint64_t seed, const nvfp4_tensor *out,
                                         int32_t global_supplied, void *workspace,
                                         size_t workspace_bytes, void *stream);

/* ---- consumers -------------------------------------------------------- */
/* MoE combine ("NVIDIA shrank GLM-5.2 to 4 bits", section 2: 8 of 256
 * experts per token): y[t] = bf16(sum_k w[t][k] * out[slot[t][k]]), an FP32
 * fused multiply-add chain in k order starting from 0; slot -1 contributes
 * nothing, and so does any slot >= out_rows.  expert_out: out_rows BF16
 * rows (the expert outputs, e.g. the padded expert-major layout of
 * nvfp4_grouped_gemm), pitch ld; d_slots, d_weights:
 * [tokens x topk] int32 / float (device); y: [tokens x hidden] BF16, pitch
 * ldy.  hidden % 8 == 0, 1 <= topk <= 32, pointers and pitches 16-byte
 * aligned. */
NVFP4_API nvfp4_status nvfp4_moe_combine(const void *expert_out, int64_t ld, int64_t out_rows,
                                         const int32_t *d_slots, const float *d_weights,
                                         int64_t tokens, int32_t topk, int64_t hidden, void *y,
                                         int64_t ldy, void *stream);

/* Gated activation between the expert up and down projections, quantized
 * for the down projection: out = NVFP4 of h = silu(gate) * up, where row r
 * of gate_up holds gate in columns [0, out->cols) and up in [out->cols,
 * 2 * out->cols) (BF16, pitch ld >= 2 * out->cols).  silu(g) = g / (1 +
 * exp(-g)) with every step one binary32 RN operation in a fixed order: exp
 * by Cody and Waite's reduction (x clamped to [-87, 87]; n = rint(x *
 * RN(log2 e)); r = x - n ln2 with ln2 split into 0.693145751953125 and
 * RN(ln2 - that); the degree-7 Taylor polynomial of e^r in Horner form with
 * fused multiply-adds; times 2^n), then RN(1 / RN(1 + e)), RN(g * s),
 * RN(. * up).  h (FP32) is quantized with the two-level steps of
 * nvfp4_quantize (its own tensor amax).  Workspace and errors as
 * nvfp4_quantize. */
NVFP4_API nvfp4_status nvfp4_quantize_swiglu(const void *gate_up, int64_t ld, const nvfp4_tensor *out,
                                             void *workspace, size_t workspace_bytes, void *stream);

/* NVFP4 -> FP8 (E4M3) for an attention read ("FP4 KV-cache quantization":
 * current implementations dequantize the FP4 cache to FP8 before
 * attention): y = e4m3_rne_satfinite(e2m1(code) * s_b / 8) per value (one
 * byte, row-major, pitch ld bytes, ld % 16 == 0) and *d_fp8_scale =
 * RN(8 / g), so x_hat ~= e4m3(y) * (*d_fp8_scale).  Values below half the
 * smallest E4M3 subnormal become signed zeros. */
NVFP4_API nvfp4_status nvfp4_dequantize_fp8(const nvfp4_tensor *in, void *y, int64_t ld,
                                            float *d_fp8_scale, void *stream);

/* Decode attention read straight from an NVFP4 KV cache ("FP4 KV-cache
 * quantization": each decode step re-reads the whole cache; the FP4 values
 * are restored before the attention arithmetic).  One query token,
 * grouped-query attention: query head h (BF16 row h of q, 128 values,
 * pitch ldq elements) attends with KV head h / (heads_q / heads_kv) over
 * all K->rows cached tokens:
 *   s_t = scale * q_h . k_t,  p = softmax(s),  o_h = sum_t p_t v_t
 * with k, v the exact restored values e2m1(code) * s_b / g (no FP8 or BF16
 * copy of the cache is made; the values are restored in registers).
 * K, V  : NVFP4 [tokens x heads_kv * 128], LINEAR scale layout (the KV
 *         cache layout of nvfp4_quantize), equal shapes; head j of a token
 *         in columns 128j .. 128j + 127.
 * heads_q: a multiple of heads_kv with heads_q / heads_kv <= 8.
 * o     : BF16 [heads_q x 128], pitch ldo elements (round to nearest even of
 *         the FP32 result).  tokens == 0 gives o = 0.
 * q 4-byte aligned with even ldq; o 2-byte aligned.  Workspace:
 *   nvfp4_workspace_bytes(NVFP4_OP_ATTENTION, tokens, heads_q, heads_kv, 0)
 *   (per chunk of tokens and query head: the running maximum, the weight sum
 *   and the 128 unnormalised outputs in FP32).
 * Arithmetic: scores q . (e2m1 * s_b) on the tensor cores (BF16 operands,
 *   both exact; FP32 accumulation) times RN(RN(scale * log2(e)) / g_K), so
 *   in log2 units; exp2 and an online softmax over token chunks merged in
 *   chunk order; the weighted V sum on the tensor cores as well, with exact
 *   products (TF32 operands: the restored V values, and each FP32 weight
 *   split exactly into three TF32 parts; FP32 accumulation).  Deterministic
 *   for given sizes.
 *   Non-finite q or scale bytes give unspecified (NaN) outputs; no status
 *   is recorded. */
NVFP4_API nvfp4_status nvfp4_attention_decode(const void *q, int64_t ldq, int32_t heads_q,
                                              const nvfp4_tensor *K, const nvfp4_tensor *V,
                                              int32_t heads_kv, float scale, void *o, int64_t ldo,
                                              void *workspace, size_t workspace_bytes,
                                              void *stream);

/* ---- MXFP4 ------------------------------------------------------------ */
/* MXFP4, the format the pages compare NVFP4 with ("NVIDIA shrank GLM-5.2 to
 * 4 bits", section 3: blocks of 32 with a power-of-two E8M0 scale; "NVFP4:
 * how NVIDIA pre-trained a 12B model on 10T tokens", section "E2M1 format
 * and two-level scaling": 32 values per UE8M0 scale; "FP4 KV-cache
 * quantization", section "FP4 formats compared": about 4.25 bits/value).
 * An nvfp4_tensor holds an MXFP4 tensor with: the same E2M1 codes and
 * nibble order; one UE8M0 byte per 32 values (2^(byte - 127)) at the
 * positions of the same two layouts over cols / 32 scale columns
 * (nvfp4_mx_scales_bytes); `global` unused (may be NULL); cols % 32 == 0.
 * Quantize: per block X = floor(log2(amax)) - 2 clamped to [-127, 127] (the
 * OCP microscaling shared-exponent rule; -127 for a block of zeros or
 * subnormals), byte X + 127, codes e2m1_rne_satfinite(x * 2^-X).
 * Dequantize: bf16(e2m1(code) * 2^X).  Non-finite input is recorded as
 * NVFP4_ERR_NONFINITE in the workspace status word (outputs unspecified). */
NVFP4_API size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout);
NVFP4_API nvfp4_status nvfp4_quantize_mx(const void *x, int64_t ld, const nvfp4_tensor *out,
                                         void *workspace, size_t workspace_bytes, void *stream);
NVFP4_API nvfp4_status nvfp4_dequantize_mx(const nvfp4_tensor *in, void *y, int64_t ld,
                                           void *stream);

/* MXFP4 W4A4 linear: D = A_hat * W_hat^T with A, W MXFP4 tensors (block 32,
 * UE8M0 scales, swizzled layout, no tensor scales: alpha = 1), on the same
 * block-scaled tensor-core MMA as nvfp4_gemm with scale vector 2X.  Shapes,
 * output and errors as nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_gemm_mx(const nvfp4_tensor *A, const nvfp4_tensor *W, void *D,
                                     int64_t ldd, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Same quantization as nvfp4_quantize, for callers that cannot allocate
 * device memory when they quantize: code recorded into a CUDA graph (device
 * allocation cannot be captured), latency-critical paths that cannot afford
 * the device synchronisation cudaMalloc implies, and host frameworks whose
 * memory pool already owns the device.  (The pages have no counterpart to
 * this entry point; it changes where scratch lives, not what is computed.)
 * It takes no workspace: its scratch (status word plus up to 1024 per-block
 * partial maxima, 4352 bytes) is a fixed device array inside the library
 * that every GPU loading the library keeps until the process exits.  The
 * scratch does not grow with the tensor (the amax pass runs at most four
 * blocks per SM, each striding over rows), so every size nvfp4_quantize
 * accepts is accepted here; a device with more than 256 SMs would need more
 * than the 1024 partial slots and is refused with NVFP4_ERR_WORKSPACE.
 * - The first call in a CUDA context looks up the array's device address
 *   (with that device current) and caches it against the context; make that
 *   first call before any stream capture.  After cudaDeviceReset the new
 *   context looks the address up again on its first call (again before any
 *   capture).
 * - All calls share the array and the status word is cleared by every call:
 *   calls whose kernels can overlap on the GPU (unordered streams) race and
 *   must not be issued.
 * - Device-detected errors (non-finite input, amax out of range) are
 *   reported in band: *out->global is set to NaN.
 * Arguments and the other return codes are those of nvfp4_quantize. */
NVFP4_API nvfp4_status nvfp4_quantize_noalloc(const void *x, int64_t ld, const nvfp4_tensor *out,
                                              int32_t global_supplied, void *stream);

/* ---- dequantize ------------------------------------------------------- */

/* NVFP4 -> BF16:  y = bf16_rne(RN(e2m1(code) * d_b)),  d_b = RN(s_b / g).
 * (The block scale and tensor scale restore each value's range; "NVIDIA
 * shrank GLM-5.2 to 4 bits", section 3.)  y: device BF16 in->rows x in->cols,
 * pitch ld.  Both scale layouts are accepted. */
NVFP4_API nvfp4_status nvfp4_dequantize(const nvfp4_tensor *in, void *y, int64_t ld, void *stream);

/* ---- GEMM ------------------------------------------------------------- */

/* W4A4 linear layer on the FP4 tensor cores (block-scaled MMA, FP32
 * accumulation; for small M with a large enough workspace the K range is
 * split over several SMs and the FP32 partial sums are added in split order
 * by a second kernel):  D[i,j] = bf16_rne(alpha * sum_k a_ik * w_jk), where a and w
 * are the E2M1 codes times their E4M3 block scales and
 * alpha = RN(1 / RN(gA * gW)) is formed on the device from *A->global and
 * *W->global.  ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens",
 * section "MXFP4 vs 36% token efficiency and Blackwell speed": FP4 GEMM on
 * Blackwell; section "Four stabilisation devices": Fprop/Dgrad/Wgrad GEMMs
 * in NVFP4.)
 * A: M x K, W: N x K (both K-major, i.e. D = A * W^T), both with
 *    NVFP4_SF_SWIZZLED_128x4 scales.  K % 64 == 0; M, N >= 1 arbitrary.
 * D: device BF16 M x N, row pitch ldd >= N (any; 16-byte aligned D with
 *    ldd % 8 == 0 takes the vectorised store path).
 * Accuracy: |D - exact| <= 1e-3 * sum_k |a_ik w_jk| / (gA gW) + BF16 rounding. */
NVFP4_API nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *W, void *D, int64_t ldd,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Grouped W4A4 GEMM over MoE experts (one launch for all groups).
 * A: stacked activation rows, group g occupying padded rows
 *    [d_slot_offsets[g], d_slot_offsets[g+1]) -- every offset a multiple of
 *    128 -- of which the first d_group_rows[g] are real rows.  Padding rows
 *    must hold zero codes and scales (nvfp4_quantize_gather writes them).
 *    A->rows (the padded capacity) must be a multiple of 128; at most 512
 *    groups.  Offsets that break these rules are caught on the device: the
 *    call then computes nothing and records NVFP4_ERR_SHAPE.
 * W: groups stacked weights, [groups * n] x K; group g uses rows
 *    [g*n, (g+1)*n) and tensor scale d_w_globals[g].  n % 128 == 0.
 * D: BF16 rows in the same padded layout as A, pitch ldd >= n; only real
 *    rows are written.  alpha_g = RN(1 / RN(gA * d_w_globals[g])).
 * Offsets and row counts stay on the device (no host synchronisation). */
NVFP4_API nvfp4_status nvfp4_grouped_gemm(int32_t groups, const int32_t *d_slot_offsets,
                                const int32_t *d_group_rows, const nvfp4_tensor *A,
                                const nvfp4_tensor *W, const float *d_w_globals, int64_t n,
                                void *D, int64_t ldd, void *workspace, size_t workspace_bytes,
                                void *stream);

/* nvfp4_grouped_gemm that also writes, to *d_out_global, the NVFP4 tensor
 * scale g = RN(2688 / amax) of its BF16 output, amax = max |D| over the real
 * rows and the n columns (the padding rows are not part of the tensor; g = 1
 * when every value is zero).  That is the g nvfp4_quantize_gather computes
 * in its own amax pass over the same rows, so the next projection's
 * quantize can take it as supplied (global_supplied = 1) and skip that pass
 * ("NVIDIA shrank GLM-5.2 to 4 bits", §1: the expert linears' activations
 * are NVFP4; "NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens",
 * "E2M1 format and two-level scaling": the FP32 tensor scale from the
 * tensor's amax).  The maximum is taken in the GEMM's epilogue over the
 * rounded BF16 values it stores.  Arguments and errors as
 * nvfp4_grouped_gemm; d_out_global: device float, 4-byte aligned.
 * Non-finite output records NVFP4_ERR_NONFINITE, an amax too small for a
 * finite g NVFP4_ERR_RANGE (as nvfp4_quantize).  Uses bytes 8..11 of the
 * workspace's status block. */
NVFP4_API nvfp4_status nvfp4_grouped_gemm_out_scale(int32_t groups, const int32_t *d_slot_offsets,
                                                    const int32_t *d_group_rows, const nvfp4_tensor *A,
                                                    const nvfp4_tensor *W, const float *d_w_globals,
                                                    int64_t n, void *D, int64_t ldd, float *d_out_global,
                                                    void *workspace, size_t workspace_bytes, void *stream);

/* ---- status ----------------------------------------------------------- */

/* Synchronise `stream`, return the workspace's status word and reset it to
 * NVFP4_OK.  Returns NVFP4_ERR_CUDA if the synchronisation itself failed. */
NVFP4_API nvfp4_status nvfp4_check_status(void *workspace, void *stream);

/* Static, human-readable name of a status code. */
NVFP4_API const char *nvfp4_status_string(nvfp4_status s);

/* Library version as 10000*major + 100*minor + patch. */
NVFP4_API int32_t nvfp4_version(void);

/* Number of kernels this library has enqueued since load (all entry points;
 * for accounting in benchmarks). */
NVFP4_API int64_t nvfp4_launch_count(void);

/* Bound, in SM clock cycles, on every pipeline wait inside the GEMM kernels
 * (default 2e9, about one second).  A wait that runs past it makes the
 * kernel record NVFP4_ERR_TIMEOUT, drain what it issued and exit instead of
 * hanging.  cycles <= 0 restores the default.  Returns the previous bound.
 * Meant for tests of the timeout path. */
NVFP4_API long long nvfp4_set_wait_limit_cycles(long long cycles);

/* Kernel choice for dense NVFP4 nvfp4_gemm calls with M >= 256: enable = 1
 * (the default; 3-8 % faster at the measured shapes) runs them on pairs of
 * SMs sharing 256x256 output tiles (half the operand traffic from L2 per
 * SM), enable = 0 on one SM per 128x256 tile.  Smaller M, MXFP4 operands and
 * the grouped GEMM always use one SM per tile.  Both give results within the
 * same bound.  Process-wide; returns the previous setting. */
NVFP4_API int32_t nvfp4_set_gemm_pairs(int32_t enable);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
