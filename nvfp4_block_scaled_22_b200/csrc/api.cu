// Host side of libnvfp4.so: the C ABI declared in include/nvfp4.h.
// Argument validation, device check, tensor-map encoding and launches.
// No device memory is allocated here; every buffer belongs to the caller.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "kernels.h"
#include "nvfp4.h"

using namespace nvfp4;

namespace {

std::atomic<int64_t> g_launches{0};

constexpr int kMaxDevices = 64;
constexpr size_t kStatusBytes = 256;          // status word + reserved
constexpr size_t kOutAmaxOffset = 8;          // in the status block: nvfp4_grouped_gemm_out_scale's max
constexpr int kMaxPartials = 1024;            // CTAs of the amax pass
constexpr long long kDefaultTimeoutCycles = 2000000000ll;   // ~1 s at 1.9 GHz
constexpr int64_t kFlatCols = 2048;           // row width for contiguous row-major-scale tensors
// Most K splits of the few-row GEMM: each split costs an accumulator
// hand-off and FP32 partials; measured at M = 16, N = 20480, K = 5120, a cap
// of 4 beats 16 (29.7 vs 33.8 us).
#ifndef NVFP4_SWAP_MAX_SPLITS
#define NVFP4_SWAP_MAX_SPLITS 4
#endif
constexpr int kSwapMaxSplits = NVFP4_SWAP_MAX_SPLITS;

struct DeviceInfo {
    bool checked = false;
    bool supported = false;
    int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
long long g_timeout_cycles = kDefaultTimeoutCycles;
bool g_use_pairs = true;

nvfp4_status current_device(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.checked) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.supported = (major == 10 && minor == 0);
        d.sms = sms;
        d.checked = true;
    }
    if (!d.supported) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    *sms = d.sms;
    return NVFP4_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

nvfp4_status launched(cudaError_t e, int n = 1) {
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    g_launches.fetch_add(n, std::memory_order_relaxed);
    return NVFP4_OK;
}

nvfp4_status check_tensor(const nvfp4_tensor *t) {
    if (t == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (t->rows < 0 || t->cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (t->sf_layout != NVFP4_SF_SWIZZLED_128x4 && t->sf_layout != NVFP4_SF_LINEAR)
        return NVFP4_ERR_INVALID_ARG;
    if (t->cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (t->global == nullptr) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(t->global) & 3u) != 0) return NVFP4_ERR_ALIGNMENT;
    if (t->rows > 0 && t->cols > 0) {
        if (t->codes == nullptr || t->scales == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(t->codes) || !aligned16(t->scales)) return NVFP4_ERR_ALIGNMENT;
    }
    return NVFP4_OK;
}

nvfp4_status check_mx_tensor(const nvfp4_tensor *t) {
    if (t == nullptr || t->rows < 0 || t->cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (t->sf_layout != NVFP4_SF_SWIZZLED_128x4 && t->sf_layout != NVFP4_SF_LINEAR)
        return NVFP4_ERR_INVALID_ARG;
    if (t->cols % 32 != 0) return NVFP4_ERR_SHAPE;
    if (t->rows > 0 && t->cols > 0) {
        if (t->codes == nullptr || t->scales == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(t->codes) || !aligned16(t->scales)) return NVFP4_ERR_ALIGNMENT;
    }
    return NVFP4_OK;
}

nvfp4_status check_workspace(void *ws, size_t bytes, size_t need) {
    if (ws == nullptr || bytes < need) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGNMENT;
    return NVFP4_OK;
}

// ---------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

nvfp4_status get_encode() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Packed-code matrix [rows x cols/2 bytes] as a 2-D uint8 tensor, boxes of
// box_bytes (128 or 64) x box_rows, swizzled over the box row (the MMA's
// K-major operand layout).
nvfp4_status encode_codes_map(CUtensorMap *m, const void *codes, int64_t rows, int64_t cols,
                              uint32_t box_rows, uint32_t box_bytes) {
    cuuint64_t dims[2] = {(cuuint64_t)(cols / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols / 2)};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t estr[2] = {1, 1};
    if (box_bytes != 128 && box_bytes != 64) return NVFP4_ERR_INVALID_ARG;
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Launch a kernel with programmatic stream serialization: it may be
// scheduled while the previous kernel on the stream finishes, and waits on
// the device (griddepcontrol.wait) before reading that kernel's results.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), int grid, int block, size_t smem,
                       cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3((unsigned)block, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

nvfp4_status run_encode(const void *x, int64_t ld, int64_t src_rows, const int32_t *gather,
                        const nvfp4_tensor *out, int32_t global_supplied, void *ws,
                        cudaStream_t stream, int sms, bool rht = false, uint32_t rht_mask = 0,
                        bool sr = false, uint64_t sr_seed = 0) {
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    uint32_t *partials = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + kStatusBytes);
    int n_partials = 0;
    if (!global_supplied) {
        int64_t warps_needed = ceil_div(out->rows, 1);
        int grid = (int)std::min<int64_t>(std::min<int64_t>(ceil_div(warps_needed, 8), 4 * sms),
                                          kMaxPartials);
        if (grid < 1) grid = 1;
        if (rht)
            k_amax_rht<<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(x), ld, out->rows,
                                                 out->cols, rht_mask, partials);
        else
            k_amax<<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(x), ld, out->rows,
                                             out->cols, gather, src_rows, partials, status);
        nvfp4_status st = launched(cudaGetLastError());
        if (st != NVFP4_OK) return st;
        n_partials = grid;
    }
    EncodeParams p;
    p.x = static_cast<const uint16_t *>(x);
    p.ld = ld;
    p.rows = out->rows;
    p.cols = out->cols;
    p.gather = gather;
    p.src_rows = src_rows;
    p.codes = static_cast<uint8_t *>(out->codes);
    p.scales = static_cast<uint8_t *>(out->scales);
    p.layout = out->sf_layout;
    p.global = out->global;
    p.global_supplied = global_supplied;
    p.partials = partials;
    p.n_partials = n_partials;
    p.status = status;
    p.rht_mask = rht_mask;
    p.sr_seed = sr_seed;
    // Narrow rows with row-major scales and no row padding (the KV cache) are
    // one contiguous run of 16-value blocks in x, codes and scales alike:
    // encode them as 2048-value rows, which the chunked kernel streams
    // faster.  Same bytes at the same offsets.  (Not for stochastic rounding,
    // whose draws are keyed by the row and block column, nor for gathers.)
    if (!sr && gather == nullptr && out->sf_layout == NVFP4_SF_LINEAR && ld == out->cols &&
        tasks_are_groups(out->cols) && (out->rows * out->cols) % kFlatCols == 0) {
        p.rows = out->rows * out->cols / kFlatCols;
        p.cols = kFlatCols;
        p.ld = kFlatCols;
    }
    const int64_t tasks = encode_tasks(p.rows, p.cols, out->sf_layout);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    const bool narrow = tasks_are_groups(p.cols);
    void (*kernel)(EncodeParams) =
        sr ? (rht ? (narrow ? k_encode_rht_sr_narrow : k_encode_rht_sr)
                  : (narrow ? k_encode_sr_narrow : k_encode_sr))
           : (rht ? (narrow ? k_encode_rht_narrow : k_encode_rht)
                  : (narrow ? k_encode_narrow : k_encode));
    int grid = (int)std::min<int64_t>(ceil_div(tasks, 8 * (narrow ? 4 : 1)), 8LL * sms);
    if (grid < 1) grid = 1;
    return launched(launch_pdl(kernel, grid, 256, 0, stream, p));
}

// Column-wise quantize (out = NVFP4 of x^T); arguments already validated.
nvfp4_status run_encode_t(const void *x, int64_t ld, bool rht, uint32_t sign_mask, bool sr,
                          uint64_t sr_seed, const nvfp4_tensor *out, int32_t global_supplied,
                          void *workspace, cudaStream_t s, int sms) {
    nvfp4_status st = NVFP4_OK;
    const int64_t R = out->cols, C = out->rows;        // x is R x C
    uint32_t *status = reinterpret_cast<uint32_t *>(workspace);
    uint32_t *partials = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    const int64_t rows_out = (out->sf_layout == NVFP4_SF_SWIZZLED_128x4) ? ceil_div(C, 128) * 128 : C;
    const int64_t tasks = transpose_tasks(R, rows_out);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    const int per_cta = kTransposeThreads / 32;
    int n_partials = 0;
    if (!global_supplied) {
        if (rht) {
            int grid = (int)std::min<int64_t>(std::min<int64_t>(ceil_div(transpose_tasks(R, C), per_cta),
                                                                8LL * sms), kMaxPartials);
            if (grid < 1) grid = 1;
            const uint16_t *xp = static_cast<const uint16_t *>(x);
            int64_t ld_ = ld, R_ = R, C_ = C;
            uint32_t mask_ = sign_mask;
            uint32_t *part_ = partials;
            void *args[] = {&xp, &ld_, &R_, &C_, &mask_, &part_};
            st = launched(launch_transpose_kernel((const void *)k_amax_t_rht, grid, args, s));
            if (st != NVFP4_OK) return st;
            n_partials = grid;
        } else {
            int grid = (int)std::min<int64_t>(std::min<int64_t>(ceil_div(R, 8), 4 * sms), kMaxPartials);
            if (grid < 1) grid = 1;
            k_amax<<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(x), ld, R, C, nullptr, R,
                                        partials, status);
            st = launched(cudaGetLastError());
            if (st != NVFP4_OK) return st;
            n_partials = grid;
        }
    }
    EncodeParams p;
    p.x = static_cast<const uint16_t *>(x);
    p.ld = ld;
    p.rows = C;
    p.cols = R;
    p.gather = nullptr;
    p.src_rows = 0;
    p.codes = static_cast<uint8_t *>(out->codes);
    p.scales = static_cast<uint8_t *>(out->scales);
    p.layout = out->sf_layout;
    p.global = out->global;
    p.global_supplied = global_supplied;
    p.partials = partials;
    p.n_partials = n_partials;
    p.status = status;
    p.rht_mask = sign_mask;
    p.sr_seed = sr_seed;
    int grid = (int)std::min<int64_t>(ceil_div(tasks, per_cta), 8LL * sms);
    if (grid < 1) grid = 1;
    const void *kernel = sr ? (rht ? (const void *)k_encode_t_rht_sr : (const void *)k_encode_t_sr)
                            : (rht ? (const void *)k_encode_t_rht : (const void *)k_encode_t);
    void *args[] = {&p};
    return launched(launch_transpose_kernel(kernel, grid, args, s));
}

// Shared argument checks of the column-wise entry points.
nvfp4_status check_transposed(const void *x, int64_t ld, const nvfp4_tensor *out,
                              int32_t global_supplied, void *workspace, size_t workspace_bytes) {
    nvfp4_status st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    if (global_supplied != 0 && global_supplied != 1) return NVFP4_ERR_INVALID_ARG;
    const int64_t R = out->cols, C = out->rows;
    if (C % 8 != 0) return NVFP4_ERR_SHAPE;
    if (R > 0 && C > 0) {
        if (x == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < C) return NVFP4_ERR_SHAPE;
    }
    return check_workspace(workspace, workspace_bytes,
                           nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, out->rows, out->cols, 0, 0));
}

}  // namespace

extern "C" {

// Token chunks of the attention read: about one CTA per SM of a B200 (148
// SMs) over all KV heads, at least one 256-token sub-tile per chunk.  Fixed
// by the sizes alone, so the workspace size and the summation order do not
// depend on the device.
static int64_t attn_chunk_tokens(int64_t tokens, int64_t heads_kv) {
    const int64_t subs = ceil_div(tokens, kAttnSub);
    const int64_t want = std::max<int64_t>(1, std::min<int64_t>(subs, 148 / heads_kv));
    return ceil_div(subs, want) * kAttnSub;
}

static int64_t attn_chunks(int64_t tokens, int64_t heads_kv) {
    return tokens > 0 ? ceil_div(tokens, attn_chunk_tokens(tokens, heads_kv)) : 0;
}

size_t nvfp4_codes_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return (size_t)(rows * (cols / 2));
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout) {
    if (rows < 0 || cols < 0) return 0;
    const int64_t s = cols / 16;
    if (sf_layout == NVFP4_SF_LINEAR) return (size_t)(rows * s);
    return (size_t)(ceil_div(rows, 128) * 128 * ceil_div(s, 4) * 4);
}

size_t nvfp4_workspace_bytes(int32_t op, int64_t m, int64_t n, int64_t k, int32_t groups) {
    switch (op) {
        case NVFP4_OP_QUANTIZE:
        case NVFP4_OP_QUANTIZE_GATHER:
            return kStatusBytes + 4 * kMaxPartials;
        case NVFP4_OP_GEMM:
            // dense GEMMs with few output tiles may split K into up to 8 FP32
            // slices; a smaller workspace only turns the split off
            if (groups == 0 && m > 0 && n > 0 && k > 0 && m <= kBM)
                return kStatusBytes + (size_t)std::min<int64_t>(8, ceil_div(k / 64, 4)) * m * n * 4;
            return kStatusBytes;
        case NVFP4_OP_ATTENTION:
            // m = tokens, n = query heads, k = KV heads
            if (m > 0 && n > 0 && k > 0)
                return kStatusBytes + (size_t)attn_chunks(m, k) * n * (kAttnDim + 2) * 4;
            return kStatusBytes;
        default:
            return kStatusBytes;
    }
}

nvfp4_status nvfp4_quantize(const void *x, int64_t ld, const nvfp4_tensor *out,
                            int32_t global_supplied, void *workspace, size_t workspace_bytes,
                            void *stream) {
    nvfp4_status st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    if (global_supplied != 0 && global_supplied != 1) return NVFP4_ERR_INVALID_ARG;
    if (out->rows > 0 && out->cols > 0) {
        if (x == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < out->cols) return NVFP4_ERR_SHAPE;
    }
    st = check_workspace(workspace, workspace_bytes,
                         nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, out->rows, out->cols, 0, 0));
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return run_encode(x, ld, out->rows, nullptr, out, global_supplied, workspace,
                      static_cast<cudaStream_t>(stream), sms);
}

nvfp4_status nvfp4_quantize_rht(const void *x, int64_t ld, uint32_t sign_mask,
                                const nvfp4_tensor *out, int32_t global_supplied, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (sign_mask > 0xFFFFu) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    if (global_supplied != 0 && global_supplied != 1) return NVFP4_ERR_INVALID_ARG;
    if (out->rows > 0 && out->cols > 0) {
        if (x == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < out->cols) return NVFP4_ERR_SHAPE;
    }
    st = check_workspace(workspace, workspace_bytes,
                         nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, out->rows, out->cols, 0, 0));
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return run_encode(x, ld, out->rows, nullptr, out, global_supplied, workspace,
                      static_cast<cudaStream_t>(stream), sms, true, sign_mask);
}

nvfp4_status nvfp4_quantize_t(const void *x, int64_t ld, int32_t rht, uint32_t sign_mask,
                              const nvfp4_tensor *out, int32_t global_supplied, void *workspace,
                              size_t workspace_bytes, void *stream) {
    if (rht != 0 && rht != 1) return NVFP4_ERR_INVALID_ARG;
    if (sign_mask > 0xFFFFu) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_transposed(x, ld, out, global_supplied, workspace, workspace_bytes);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return run_encode_t(x, ld, rht != 0, sign_mask, false, 0, out, global_supplied, workspace,
                        static_cast<cudaStream_t>(stream), sms);
}

nvfp4_status nvfp4_quantize_sr(const void *x, int64_t ld, int32_t transposed, int32_t rht,
                               uint32_t sign_mask, uint64_t seed, const nvfp4_tensor *out,
                               int32_t global_supplied, void *workspace, size_t workspace_bytes,
                               void *stream) {
    if ((transposed != 0 && transposed != 1) || (rht != 0 && rht != 1)) return NVFP4_ERR_INVALID_ARG;
    if (sign_mask > 0xFFFFu) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st;
    if (transposed) {
        st = check_transposed(x, ld, out, global_supplied, workspace, workspace_bytes);
    } else {
        st = check_tensor(out);
        if (st == NVFP4_OK && global_supplied != 0 && global_supplied != 1) st = NVFP4_ERR_INVALID_ARG;
        if (st == NVFP4_OK && out->rows > 0 && out->cols > 0) {
            if (x == nullptr) st = NVFP4_ERR_INVALID_ARG;
            else if (!aligned16(x) || ld % 8 != 0) st = NVFP4_ERR_ALIGNMENT;
            else if (ld < out->cols) st = NVFP4_ERR_SHAPE;
        }
        if (st == NVFP4_OK)
            st = check_workspace(workspace, workspace_bytes,
                                 nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, out->rows, out->cols, 0, 0));
    }
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (transposed)
        return run_encode_t(x, ld, rht != 0, sign_mask, true, seed, out, global_supplied, workspace, s,
                            sms);
    return run_encode(x, ld, out->rows, nullptr, out, global_supplied, workspace, s, sms, rht != 0,
                      sign_mask, true, seed);
}

nvfp4_status nvfp4_quantize_2d(const void *w, int64_t ld, const nvfp4_tensor *out,
                               const nvfp4_tensor *out_t, int32_t global_supplied, void *workspace,
                               size_t workspace_bytes, void *stream) {
    nvfp4_status st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    if (global_supplied != 0 && global_supplied != 1) return NVFP4_ERR_INVALID_ARG;
    const int64_t R = out->rows, C = out->cols;
    if (out_t != nullptr) {
        st = check_tensor(out_t);
        if (st != NVFP4_OK) return st;
        if (out_t->rows != C || out_t->cols != R) return NVFP4_ERR_SHAPE;
        if (R % 16 != 0) return NVFP4_ERR_SHAPE;
    }
    if (R > 0 && C > 0) {
        if (w == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(w) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < C) return NVFP4_ERR_SHAPE;
    }
    st = check_workspace(workspace, workspace_bytes,
                         nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, R, C, 0, 0));
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(workspace);
    uint32_t *partials = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    int n_partials = 0;
    if (!global_supplied) {
        int grid = (int)std::min<int64_t>(std::min<int64_t>(ceil_div(R, 8), 4 * sms), kMaxPartials);
        if (grid < 1) grid = 1;
        k_amax<<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(w), ld, R, C, nullptr, R, partials,
                                    status);
        st = launched(cudaGetLastError());
        if (st != NVFP4_OK) return st;
        n_partials = grid;
    } else if (out_t != nullptr && out_t->global != out->global) {
        if (cudaMemcpyAsync(out_t->global, out->global, sizeof(float), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
            return NVFP4_ERR_CUDA;
    }
    EncodeParams p;
    p.x = static_cast<const uint16_t *>(w);
    p.ld = ld;
    p.rows = R;
    p.cols = C;
    p.gather = nullptr;
    p.src_rows = 0;
    p.codes = static_cast<uint8_t *>(out->codes);
    p.scales = static_cast<uint8_t *>(out->scales);
    p.layout = out->sf_layout;
    p.global = out->global;
    p.global_supplied = global_supplied;
    p.partials = partials;
    p.n_partials = n_partials;
    p.status = status;
    const int64_t rows_out = (out->sf_layout == NVFP4_SF_SWIZZLED_128x4) ? ceil_div(R, 128) * 128 : R;
    const int64_t tasks = ceil_div(rows_out, 16) * ceil_div(ceil_div(C / 16, 4) * 4, 16);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    int grid = (int)std::min<int64_t>(ceil_div(tasks, 8), 8LL * sms);
    if (grid < 1) grid = 1;
    k_encode_2d<<<grid, 256, 0, s>>>(p);
    st = launched(cudaGetLastError());
    if (st != NVFP4_OK || out_t == nullptr) return st;
    // W^T: column-wise with 16x16 blocks (x = W is R x C; out_t is C x R)
    EncodeParams q = p;
    q.rows = C;
    q.cols = R;
    q.codes = static_cast<uint8_t *>(out_t->codes);
    q.scales = static_cast<uint8_t *>(out_t->scales);
    q.layout = out_t->sf_layout;
    q.global = out_t->global;
    const int64_t rows_out_t = (out_t->sf_layout == NVFP4_SF_SWIZZLED_128x4) ? ceil_div(C, 128) * 128 : C;
    const int64_t tasks_t = transpose_tasks(R, rows_out_t);
    if (tasks_t >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    int grid_t = (int)std::min<int64_t>(ceil_div(tasks_t, kTransposeThreads / 32), 8LL * sms);
    if (grid_t < 1) grid_t = 1;
    void *args[] = {&q};
    return launched(launch_transpose_kernel((const void *)k_encode_t_2d, grid_t, args, s));
}

size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout) {
    if (rows < 0 || cols < 0) return 0;
    const int64_t s = cols / 32;
    if (sf_layout == NVFP4_SF_LINEAR) return (size_t)(rows * s);
    return (size_t)(ceil_div(rows, 128) * 128 * ceil_div(s, 4) * 4);
}


nvfp4_status nvfp4_quantize_mx(const void *x, int64_t ld, const nvfp4_tensor *out, void *workspace,
                               size_t workspace_bytes, void *stream) {
    nvfp4_status st = check_mx_tensor(out);
    if (st != NVFP4_OK) return st;
    if (out->rows > 0 && out->cols > 0) {
        if (x == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < out->cols) return NVFP4_ERR_SHAPE;
    }
    st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    const int64_t rows_out = (out->sf_layout == NVFP4_SF_SWIZZLED_128x4) ? ceil_div(out->rows, 128) * 128
                                                                         : out->rows;
    const int64_t tasks = rows_out * ceil_div(ceil_div(out->cols / 32, 4) * 4, 32);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    EncodeParams p;
    p.x = static_cast<const uint16_t *>(x);
    p.ld = ld;
    p.rows = out->rows;
    p.cols = out->cols;
    p.gather = nullptr;
    p.src_rows = 0;
    p.codes = static_cast<uint8_t *>(out->codes);
    p.scales = static_cast<uint8_t *>(out->scales);
    p.layout = out->sf_layout;
    p.global = nullptr;
    p.global_supplied = 1;
    p.partials = nullptr;
    p.n_partials = 0;
    p.status = reinterpret_cast<uint32_t *>(workspace);
    int grid = (int)std::min<int64_t>(ceil_div(tasks, 8), 8LL * sms);
    if (grid < 1) grid = 1;
    k_encode_mx<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_dequantize_mx(const nvfp4_tensor *in, void *y, int64_t ld, void *stream) {
    nvfp4_status st = check_mx_tensor(in);
    if (st != NVFP4_OK) return st;
    if (in->rows > 0 && in->cols > 0) {
        if (y == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(y) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < in->cols) return NVFP4_ERR_SHAPE;
    }
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    if (in->rows == 0 || in->cols == 0) return NVFP4_OK;
    DequantParams p;
    p.codes = static_cast<const uint8_t *>(in->codes);
    p.scales = static_cast<const uint8_t *>(in->scales);
    p.layout = in->sf_layout;
    p.global = nullptr;
    p.rows = in->rows;
    p.cols = in->cols;
    p.y = static_cast<uint16_t *>(y);
    p.ld = ld;
    p.y_vec32 = ((reinterpret_cast<uintptr_t>(y) & 31u) == 0 && ld % 16 == 0) ? 1 : 0;
    const int64_t tasks = in->rows * ceil_div(in->cols / 32, 32);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    int grid = (int)std::min<int64_t>(ceil_div(tasks, 8), 8LL * sms);
    if (grid < 1) grid = 1;
    k_dequantize_mx<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_moe_combine(const void *expert_out, int64_t ld, int64_t out_rows,
                               const int32_t *d_slots, const float *d_weights, int64_t tokens,
                               int32_t topk, int64_t hidden, void *y, int64_t ldy, void *stream) {
    if (tokens < 0 || hidden < 0 || out_rows < 0 || topk < 1 || topk > kMaxTopk)
        return NVFP4_ERR_INVALID_ARG;
    if (hidden % 8 != 0) return NVFP4_ERR_SHAPE;
    if (tokens == 0 || hidden == 0) return NVFP4_OK;
    if (expert_out == nullptr || d_slots == nullptr || d_weights == nullptr || y == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(expert_out) || !aligned16(y) || ld % 8 != 0 || ldy % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (ld < hidden || ldy < hidden) return NVFP4_ERR_SHAPE;
    if (tokens > INT32_MAX) return NVFP4_ERR_SHAPE;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    CombineParams p;
    p.out = static_cast<const uint16_t *>(expert_out);
    p.ld = ld;
    p.out_rows = out_rows;
    p.slots = d_slots;
    p.weights = d_weights;
    p.topk = topk;
    p.hidden = hidden;
    p.y = static_cast<uint16_t *>(y);
    p.ldy = ldy;
    k_moe_combine<<<(unsigned)tokens, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_dequantize_fp8(const nvfp4_tensor *in, void *y, int64_t ld, float *d_fp8_scale,
                                  void *stream) {
    nvfp4_status st = check_tensor(in);
    if (st != NVFP4_OK) return st;
    if (d_fp8_scale == nullptr) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_fp8_scale) & 3u) != 0) return NVFP4_ERR_ALIGNMENT;
    if (in->rows > 0 && in->cols > 0) {
        if (y == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(y) || ld % 16 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < in->cols) return NVFP4_ERR_SHAPE;
    }
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    Fp8Params p;
    p.codes = static_cast<const uint8_t *>(in->codes);
    p.scales = static_cast<const uint8_t *>(in->scales);
    p.layout = in->sf_layout;
    p.global = in->global;
    p.rows = in->rows;
    p.cols = in->cols;
    p.y = static_cast<uint8_t *>(y);
    p.ld = ld;
    p.fp8_scale = d_fp8_scale;
    const int64_t blocks = in->rows * (in->cols / 16);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(blocks, 256), 8LL * sms));
    k_dequantize_fp8<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_attention_decode(const void *q, int64_t ldq, int32_t heads_q,
                                    const nvfp4_tensor *K, const nvfp4_tensor *V, int32_t heads_kv,
                                    float scale, void *o, int64_t ldo, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    nvfp4_status st = check_tensor(K);
    if (st != NVFP4_OK) return st;
    st = check_tensor(V);
    if (st != NVFP4_OK) return st;
    if (heads_q < 1 || heads_kv < 1 || !(scale == scale) || scale > 3.4e38f || scale < -3.4e38f)
        return NVFP4_ERR_INVALID_ARG;
    if (heads_q % heads_kv != 0 || heads_q / heads_kv > kAttnMaxGroup) return NVFP4_ERR_SHAPE;
    if (K->sf_layout != NVFP4_SF_LINEAR || V->sf_layout != NVFP4_SF_LINEAR) return NVFP4_ERR_SHAPE;
    if (K->rows != V->rows || K->cols != V->cols || K->cols != (int64_t)heads_kv * kAttnDim)
        return NVFP4_ERR_SHAPE;
    if (q == nullptr || o == nullptr) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) & 3u) != 0 || ldq % 2 != 0 ||
        (reinterpret_cast<uintptr_t>(o) & 1u) != 0)
        return NVFP4_ERR_ALIGNMENT;
    if (ldq < kAttnDim || ldo < kAttnDim) return NVFP4_ERR_SHAPE;
    const int64_t tokens = K->rows;
    const int64_t chunks = attn_chunks(tokens, heads_kv);
    st = check_workspace(workspace, workspace_bytes,
                         kStatusBytes + (size_t)chunks * heads_q * (kAttnDim + 2) * 4);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    AttnParams p;
    p.q = static_cast<const uint16_t *>(q);
    p.ldq = ldq;
    p.kc = static_cast<const uint8_t *>(K->codes);
    p.ks = static_cast<const uint8_t *>(K->scales);
    p.vc = static_cast<const uint8_t *>(V->codes);
    p.vs = static_cast<const uint8_t *>(V->scales);
    p.gk = K->global;
    p.gv = V->global;
    p.tokens = tokens;
    p.cols = K->cols;
    p.heads_kv = heads_kv;
    p.group = heads_q / heads_kv;
    p.scale = scale;
    p.chunk = tokens > 0 ? attn_chunk_tokens(tokens, heads_kv) : kAttnSub;
    p.n_chunks = (int32_t)chunks;
    p.part_o = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    p.part_ml = p.part_o + chunks * heads_q * kAttnDim;
    p.o = static_cast<uint16_t *>(o);
    p.ldo = ldo;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (chunks > 0) {
        k_attn_partial<<<dim3((unsigned)chunks, (unsigned)heads_kv), kAttnThreads, 0, s>>>(p);
        st = launched(cudaGetLastError());
        if (st != NVFP4_OK) return st;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)heads_q, 1, 1);
    cfg.blockDim = dim3(kAttnDim, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return launched(cudaLaunchKernelEx(&cfg, k_attn_combine, p));
}

nvfp4_status nvfp4_quantize_swiglu(const void *gate_up, int64_t ld, const nvfp4_tensor *out,
                                   void *workspace, size_t workspace_bytes, void *stream) {
    nvfp4_status st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    const int64_t rows = out->rows, inter = out->cols;
    if (rows > 0 && inter > 0) {
        if (gate_up == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(gate_up) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < 2 * inter) return NVFP4_ERR_SHAPE;
    }
    st = check_workspace(workspace, workspace_bytes,
                         nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, inter, 0, 0));
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SwigluParams p;
    p.gu = static_cast<const uint16_t *>(gate_up);
    p.ld = ld;
    p.rows = rows;
    p.inter = inter;
    p.codes = static_cast<uint8_t *>(out->codes);
    p.scales = static_cast<uint8_t *>(out->scales);
    p.layout = out->sf_layout;
    p.global = out->global;
    p.partials = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    p.status = reinterpret_cast<uint32_t *>(workspace);
    const int64_t tasks = rows * ceil_div(inter / 16, 32);
    int grid = (int)std::min<int64_t>(std::min<int64_t>(ceil_div(tasks, 8), 4LL * sms), kMaxPartials);
    if (grid < 1) grid = 1;
    p.n_partials = grid;
    k_amax_swiglu<<<grid, 256, 0, s>>>(p);
    st = launched(cudaGetLastError());
    if (st != NVFP4_OK) return st;
    const int64_t rows_out = (out->sf_layout == NVFP4_SF_SWIZZLED_128x4) ? ceil_div(rows, 128) * 128 : rows;
    const int64_t etasks = rows_out * ceil_div(ceil_div(inter / 16, 4) * 4, 32);
    int egrid = (int)std::min<int64_t>(ceil_div(etasks, 8), 8LL * sms);
    if (egrid < 1) egrid = 1;
    k_encode_swiglu<<<egrid, 256, 0, s>>>(p);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_quantize_gather(const void *x, int64_t ld, int64_t src_rows,
                                   const int32_t *d_gather, const nvfp4_tensor *out,
                                   int32_t global_supplied, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    nvfp4_status st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    if (global_supplied != 0 && global_supplied != 1) return NVFP4_ERR_INVALID_ARG;
    if (src_rows < 0) return NVFP4_ERR_INVALID_ARG;
    if (out->rows > 0 && out->cols > 0) {
        if (x == nullptr || d_gather == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < out->cols) return NVFP4_ERR_SHAPE;
    }
    st = check_workspace(workspace, workspace_bytes,
                         nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE_GATHER, out->rows, out->cols, 0, 0));
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return run_encode(x, ld, src_rows, d_gather, out, global_supplied, workspace,
                      static_cast<cudaStream_t>(stream), sms);
}

nvfp4_status nvfp4_gather_rows(const nvfp4_tensor *src, const int32_t *d_gather,
                               const nvfp4_tensor *out, void *workspace, size_t workspace_bytes,
                               void *stream) {
    nvfp4_status st = check_tensor(src);
    if (st != NVFP4_OK) return st;
    st = check_tensor(out);
    if (st != NVFP4_OK) return st;
    if (out->cols != src->cols) return NVFP4_ERR_SHAPE;
    if (out->rows > 0 && out->cols > 0 && d_gather == nullptr) return NVFP4_ERR_INVALID_ARG;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    GatherParams p;
    p.src_codes = static_cast<const uint8_t *>(src->codes);
    p.src_scales = static_cast<const uint8_t *>(src->scales);
    p.src_global = src->global;
    p.src_layout = src->sf_layout;
    p.src_rows = src->rows;
    p.dst_codes = static_cast<uint8_t *>(out->codes);
    p.dst_scales = static_cast<uint8_t *>(out->scales);
    p.dst_global = out->global;
    p.dst_layout = out->sf_layout;
    p.rows = out->rows;
    p.cols = out->cols;
    p.map = d_gather;
    p.status = reinterpret_cast<uint32_t *>(workspace);
    if (out->cols == 0) {           // only the tensor scale moves
        p.rows = 0;
    }
    const int64_t rows_pad = out->sf_layout == NVFP4_SF_SWIZZLED_128x4 ? ceil_div(out->rows, 128) * 128
                                                                      : out->rows;
    // One 128-row band per grid column, kGatherSplit CTAs per band
    // (grid-stride beyond 64 bands per SM).
    const int64_t bands = std::max<int64_t>(ceil_div(rows_pad, 128), 1);
    const dim3 grid((unsigned)std::min<int64_t>(bands, 64LL * sms), kGatherSplit, 1);
    k_gather_rows<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_global_scale(const void *x, int64_t ld, int64_t rows, int64_t cols,
                                float *d_global, void *workspace, size_t workspace_bytes,
                                void *stream) {
    if (rows < 0 || cols < 0 || d_global == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(d_global) & 3u) != 0) return NVFP4_ERR_ALIGNMENT;
    if (rows > 0 && cols > 0) {
        if (x == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < cols) return NVFP4_ERR_SHAPE;
    }
    nvfp4_status st = check_workspace(workspace, workspace_bytes,
                                      nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE, rows, cols, 0, 0));
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(workspace);
    uint32_t *partials =
        reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    int grid = (int)std::min<int64_t>(std::min<int64_t>(ceil_div(rows, 8), 4 * sms), kMaxPartials);
    if (grid < 1) grid = 1;
    k_amax<<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(x), ld, rows, cols, nullptr, rows,
                                partials, status);
    st = launched(cudaGetLastError());
    if (st != NVFP4_OK) return st;
    k_finalize_g<<<1, 256, 0, s>>>(partials, grid, d_global, status);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor *in, void *y, int64_t ld, void *stream) {
    nvfp4_status st = check_tensor(in);
    if (st != NVFP4_OK) return st;
    if (in->rows > 0 && in->cols > 0) {
        if (y == nullptr) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(y) || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
        if (ld < in->cols) return NVFP4_ERR_SHAPE;
    }
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    if (in->rows == 0 || in->cols == 0) return NVFP4_OK;
    DequantParams p;
    p.codes = static_cast<const uint8_t *>(in->codes);
    p.scales = static_cast<const uint8_t *>(in->scales);
    p.layout = in->sf_layout;
    p.global = in->global;
    p.rows = in->rows;
    p.cols = in->cols;
    p.y = static_cast<uint16_t *>(y);
    p.ld = ld;
    p.y_vec32 = ((reinterpret_cast<uintptr_t>(y) & 31u) == 0 && ld % 16 == 0) ? 1 : 0;
    const int64_t tasks = decode_tasks(p.rows, p.cols);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;
    const bool narrow = tasks_are_groups(p.cols);
    void (*kernel)(DequantParams) = narrow ? k_dequantize_narrow : k_dequantize;
    int grid = (int)std::min<int64_t>(ceil_div(tasks, 8 * (narrow ? 4 : 1)), 8LL * sms);
    if (grid < 1) grid = 1;
    kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launched(cudaGetLastError());
}


// Few rows of A: the swapped-operand kernel over units of (128-row W tile,
// K split).  Split count: fewest stages on the busiest SM (plus one for the
// finalize pass when split), ties to fewer splits, if the FP32 slices fit in
// the workspace and the output allows the finalize's 4-column stores.
static nvfp4_status gemm_swap(const nvfp4_tensor *A, const nvfp4_tensor *W, int64_t m, int64_t n,
                              int64_t k, void *D, int64_t ldd, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream, int sms) {
    const uint32_t mp = (uint32_t)((m + 15) / 16 * 16);
    CUtensorMap tmW, tmX;
    nvfp4_status st = encode_codes_map(&tmW, W->codes, W->rows, k, 128, 128);
    if (st != NVFP4_OK) return st;
    st = encode_codes_map(&tmX, A->codes, A->rows, k, mp, 128);
    if (st != NVFP4_OK) return st;
    GemmParams p;
    p.sfa = static_cast<const uint8_t *>(A->scales);
    p.sfb = static_cast<const uint8_t *>(W->scales);
    p.d = static_cast<uint16_t *>(D);
    p.ldd = ldd;
    p.d_vec16 = (aligned16(D) && ldd % 8 == 0) ? 1 : 0;
    p.m = (int32_t)m;
    p.n = (int32_t)n;
    p.k = (int32_t)k;
    p.groups = 0;
    p.slot_offsets = nullptr;
    p.group_rows = nullptr;
    p.ga = A->global;
    p.gw = W->global;
    p.a_row_blocks = 1;
    p.b_row_blocks = (int32_t)ceil_div(W->rows, 128);
    p.n_fastest = 0;
    p.status = reinterpret_cast<uint32_t *>(workspace);
    p.timeout_cycles = g_timeout_cycles;
    p.splits = 1;
    p.partial = nullptr;
    p.out_amax = nullptr;
    const int64_t ntiles = ceil_div(n, 128);
    const int ktiles = (int)ceil_div(k / 64, 4);
    int64_t best_cost = ceil_div(ntiles, sms) * ktiles;
    if (n % 16 == 0 && p.d_vec16) {
        for (int sp = 2; sp <= std::min(kSwapMaxSplits, ktiles); ++sp) {
            const int64_t cost = ceil_div(ntiles * sp, sms) * ceil_div(ktiles, sp) + 1;
            const size_t need = kStatusBytes + (size_t)sp * (size_t)m * (size_t)n * 4;
            if (cost < best_cost && need <= workspace_bytes) {
                best_cost = cost;
                p.splits = sp;
            }
        }
    }
    if (p.splits > 1)
        p.partial = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(ntiles * p.splits, sms));
    st = launched(launch_gemm_swap(tmW, tmX, p, grid, stream));
    if (st != NVFP4_OK || p.splits == 1) return st;
    const int64_t quads = m * (n / 4);
    const int fgrid = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(quads, 256), 4LL * sms));
    return launched(launch_splitk_finalize(p.partial, p.splits, (int)m, (int)n, p.ga, p.gw, p.d,
                                           p.ldd, fgrid, stream));
}

static nvfp4_status gemm_common(int32_t groups, const int32_t *d_slot_offsets,
                                const int32_t *d_group_rows, const nvfp4_tensor *A,
                                const nvfp4_tensor *W, const float *gw, int64_t n, void *D,
                                int64_t ldd, void *workspace, size_t workspace_bytes,
                                void *stream, bool mx = false, uint32_t *out_amax = nullptr) {
    nvfp4_status st = mx ? check_mx_tensor(A) : check_tensor(A);
    if (st != NVFP4_OK) return st;
    st = mx ? check_mx_tensor(W) : check_tensor(W);
    if (st != NVFP4_OK) return st;
    if (A->sf_layout != NVFP4_SF_SWIZZLED_128x4 || W->sf_layout != NVFP4_SF_SWIZZLED_128x4)
        return NVFP4_ERR_INVALID_ARG;
    const int64_t k = A->cols;
    if (W->cols != k || k <= 0 || k % 64 != 0) return NVFP4_ERR_SHAPE;
    if (A->rows > INT32_MAX || W->rows > INT32_MAX || k > INT32_MAX) return NVFP4_ERR_SHAPE;
    if (groups > 0) {
        if (groups > kMaxGroups || d_slot_offsets == nullptr || d_group_rows == nullptr ||
            gw == nullptr)
            return NVFP4_ERR_INVALID_ARG;
        if (n <= 0 || n % 128 != 0 || W->rows != (int64_t)groups * n) return NVFP4_ERR_SHAPE;
        if (A->rows % 128 != 0) return NVFP4_ERR_SHAPE;
    }
    const int64_t m = A->rows;
    if (m == 0 || n == 0) return NVFP4_OK;
    if (D == nullptr) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(D) & 1u) != 0) return NVFP4_ERR_ALIGNMENT;
    if (ldd < n) return NVFP4_ERR_SHAPE;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes);   // more enables split-K
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    st = get_encode();
    if (st != NVFP4_OK) return st;
    const bool pair = !mx && groups == 0 && m >= kPairMinRows && sms >= 2 && g_use_pairs;
    if (!mx && groups == 0 && m <= kSwapMaxRows)
        return gemm_swap(A, W, m, n, k, D, ldd, workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream), sms);
    CUtensorMap tmA, tmB;
    const uint32_t box_bytes = pair ? kPairBoxBytes : kSingleBoxBytes;
    st = encode_codes_map(&tmA, A->codes, A->rows, k, kBM, box_bytes);
    if (st != NVFP4_OK) return st;
    st = encode_codes_map(&tmB, W->codes, W->rows, k, pair ? 128 : kBN, box_bytes);
    if (st != NVFP4_OK) return st;

    GemmParams p;
    p.sfa = static_cast<const uint8_t *>(A->scales);
    p.sfb = static_cast<const uint8_t *>(W->scales);
    p.d = static_cast<uint16_t *>(D);
    p.ldd = ldd;
    p.d_vec16 = (aligned16(D) && ldd % 8 == 0) ? 1 : 0;
    p.m = (int32_t)m;
    p.n = (int32_t)n;
    p.k = (int32_t)k;
    p.groups = groups;
    p.slot_offsets = d_slot_offsets;
    p.group_rows = d_group_rows;
    p.ga = A->global;
    p.gw = gw;
    p.a_row_blocks = (int32_t)ceil_div(A->rows, 128);
    p.b_row_blocks = (int32_t)ceil_div(W->rows, 128);
    // Grouped: N fastest, so the CTAs working at one time hold a few experts'
    // rows and sweep their weights once; M fastest would re-read the whole
    // grouped activation tensor (larger than L2) once per N tile.
    p.n_fastest = groups > 0 ? 1 : (A->rows * (k / 2) > kL2SweepBytes && A->rows > W->rows) ? 1 : 0;
    p.status = reinterpret_cast<uint32_t *>(workspace);
    p.timeout_cycles = g_timeout_cycles;
    p.splits = 1;
    p.partial = nullptr;
    p.out_amax = out_amax;
    // Split-K for dense GEMMs with fewer output tiles than SMs (small M):
    // pick the split count that minimises the stage count of the busiest SM
    // (ties: fewer splits), if the FP32 slices fit in the workspace.
    const int64_t tiles_mn = ceil_div(m, kBM) * ceil_div(n, kBN);
    const int ktiles = (int)ceil_div(k / 64, kKB);     // the kernel's stages per tile
    if (!mx && !pair && groups == 0 && tiles_mn < sms && n % 16 == 0 && p.d_vec16) {
        int best = 1;
        int64_t best_cost = ktiles;                              // one unit per SM
        for (int sp = 2; sp <= std::min(8, ktiles); ++sp) {
            const int64_t cost = ceil_div(tiles_mn * sp, sms) * ceil_div(ktiles, sp);
            const size_t need = kStatusBytes + (size_t)sp * (size_t)m * (size_t)n * 4;
            if (cost < best_cost && need <= workspace_bytes) {
                best = sp;
                best_cost = cost;
            }
        }
        if (best > 1) {
            p.splits = best;
            p.partial = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
        }
    }
    if (pair) {
        const int64_t pair_tiles = ceil_div(m, 256) * ceil_div(n, 256);
        const int clusters = (int)std::max<int64_t>(1, std::min<int64_t>(pair_tiles, sms / 2));
        return launched(launch_gemm_pair(tmA, tmB, p, clusters, static_cast<cudaStream_t>(stream)));
    }
    const int64_t tiles = tiles_mn * p.splits;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, sms));
    st = launched(launch_gemm(tmA, tmB, p, grid, static_cast<cudaStream_t>(stream), mx));
    if (st != NVFP4_OK || p.splits == 1) return st;
    const int64_t quads = m * (n / 4);
    const int fgrid = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(quads, 256), 4LL * sms));
    return launched(launch_splitk_finalize(p.partial, p.splits, (int)m, (int)n, p.ga, p.gw, p.d,
                                           p.ldd, fgrid, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *W, void *D, int64_t ldd,
                        void *workspace, size_t workspace_bytes, void *stream) {
    if (W == nullptr) return NVFP4_ERR_INVALID_ARG;
    return gemm_common(0, nullptr, nullptr, A, W, W->global, W->rows, D, ldd, workspace,
                       workspace_bytes, stream);
}

nvfp4_status nvfp4_gemm_mx(const nvfp4_tensor *A, const nvfp4_tensor *W, void *D, int64_t ldd,
                           void *workspace, size_t workspace_bytes, void *stream) {
    if (W == nullptr) return NVFP4_ERR_INVALID_ARG;
    return gemm_common(0, nullptr, nullptr, A, W, nullptr, W->rows, D, ldd, workspace,
                       workspace_bytes, stream, true);
}

nvfp4_status nvfp4_grouped_gemm(int32_t groups, const int32_t *d_slot_offsets,
                                const int32_t *d_group_rows, const nvfp4_tensor *A,
                                const nvfp4_tensor *W, const float *d_w_globals, int64_t n,
                                void *D, int64_t ldd, void *workspace, size_t workspace_bytes,
                                void *stream) {
    if (groups <= 0) return NVFP4_ERR_INVALID_ARG;
    return gemm_common(groups, d_slot_offsets, d_group_rows, A, W, d_w_globals, n, D, ldd,
                       workspace, workspace_bytes, stream);
}

nvfp4_status nvfp4_grouped_gemm_out_scale(int32_t groups, const int32_t *d_slot_offsets,
                                          const int32_t *d_group_rows, const nvfp4_tensor *A,
                                          const nvfp4_tensor *W, const float *d_w_globals,
                                          int64_t n, void *D, int64_t ldd, float *d_out_global,
                                          void *workspace, size_t workspace_bytes, void *stream) {
    if (groups <= 0 || d_out_global == nullptr) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_out_global) & 3u) != 0) return NVFP4_ERR_ALIGNMENT;
    nvfp4_status st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(workspace);
    uint32_t *amax = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kOutAmaxOffset);
    if (cudaMemsetAsync(amax, 0, sizeof(uint32_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
    st = gemm_common(groups, d_slot_offsets, d_group_rows, A, W, d_w_globals, n, D, ldd, workspace,
                     workspace_bytes, stream, false, amax);
    if (st != NVFP4_OK) return st;
    k_finalize_g<<<1, 256, 0, s>>>(amax, 1, d_out_global, status);
    return launched(cudaGetLastError());
}

nvfp4_status nvfp4_check_status(void *workspace, void *stream) {
    if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v != 0 && cudaMemset(workspace, 0, 4) != cudaSuccess) return NVFP4_ERR_CUDA;
    return static_cast<nvfp4_status>(v);
}

const char *nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_ALIGNMENT: return "pointer or pitch not 16-byte aligned";
        case NVFP4_ERR_SHAPE: return "shape not supported by this call";
        case NVFP4_ERR_NONFINITE: return "input holds Inf or NaN";
        case NVFP4_ERR_RANGE: return "tensor amax too small for an FP32 tensor scale";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
        case NVFP4_ERR_TIMEOUT: return "device pipeline wait timed out";
        case NVFP4_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
        case NVFP4_ERR_CUDA: return "CUDA call failed";
    }
    return "unknown status";
}

int32_t nvfp4_version(void) { return 100; }

int64_t nvfp4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

// Test hook: bound (in SM clock cycles) of every pipeline wait in the GEMM
// kernels; <= 0 restores the default.  Returns the previous bound.
long long nvfp4_set_wait_limit_cycles(long long cycles) {
    long long prev = g_timeout_cycles;
    g_timeout_cycles = cycles > 0 ? cycles : kDefaultTimeoutCycles;
    return prev;
}

// Route dense GEMMs of >= 256 rows to CTA pairs (1) or to the single-CTA
// kernel (0, default: faster at the measured shapes).  Returns the previous
// setting.
int32_t nvfp4_set_gemm_pairs(int32_t enable) {
    const int32_t prev = g_use_pairs ? 1 : 0;
    g_use_pairs = enable != 0;
    return prev;
}

}  // extern "C"
