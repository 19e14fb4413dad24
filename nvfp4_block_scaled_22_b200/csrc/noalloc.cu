// nvfp4_quantize_noalloc: the two-level quantize (the same k_amax + k_encode
// kernels as nvfp4_quantize) with its scratch held by the library instead
// of a caller-provided workspace.
//
// Who needs this: callers that cannot allocate device memory at the point
// they quantize -- code running while a CUDA graph is being captured
// (cudaMalloc cannot be captured), latency-critical paths that cannot take
// cudaMalloc's implicit device synchronisation, and host frameworks whose
// memory pool already owns the whole device and hands out no extra buffers.
//
// The scratch (status word + per-CTA partial maxima) is a fixed-size
// file-scope device array: every GPU that loads the library keeps its copy
// until the process exits.  All calls share it, so two calls whose kernels
// overlap on the GPU (different streams, no ordering between them) race on
// it and must not be issued.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nvfp4.h"
#include "ptx.cuh"

namespace {

// Layout: [0, 256) status word (+ padding), [256, 256 + 4*kNoAllocPartials)
// one partial maximum per amax CTA.  4352 bytes in total.
constexpr int kNoAllocPartials = 1024;
constexpr size_t kNoAllocStatusBytes = 256;
constexpr size_t kNoAllocScratchBytes = kNoAllocStatusBytes + 4 * kNoAllocPartials;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevs = 64;
struct ScratchAddr {
    unsigned long long ctx = 0;   // unique ID of the context the address belongs to
    void *ptr = nullptr;
};
ScratchAddr g_scratch_addr[kMaxDevs];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_once;

// Unique ID of the calling thread's current CUDA context, 0 if there is none
// yet or the driver cannot say.  A context destroyed and created again (for
// instance by cudaDeviceReset) gets a new ID, and its copy of the scratch
// array may live at a new address.
unsigned long long current_context_id() {
    std::call_once(g_ctx_once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current == nullptr || g_ctx_get_id == nullptr || g_ctx_current(&c) != CUDA_SUCCESS ||
        c == nullptr || g_ctx_get_id(c, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array in the current context.  The array's
// name in host code is only a host-side stand-in, so the address is looked
// up with cudaGetSymbolAddress (with the device current) the first time a
// context calls, and cached against that context's ID; a new context
// (after a device reset) looks it up again.
cudaError_t scratch_address(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchAddr &a = g_scratch_addr[dev];
    const unsigned long long id = current_context_id();
    if (id == 0 || a.ptr == nullptr || a.ctx != id) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        a.ptr = p;
        a.ctx = current_context_id();   // the lookup has made the context current
    }
    *out = a.ptr;
    return cudaSuccess;
}

// Report a device-detected error in band and clear the shared status word:
// a non-zero status (non-finite input, amax out of range) turns the output
// tensor scale into NaN, so the caller sees it without a workspace.
__global__ void k_status_to_global(uint32_t *status, float *global) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        if (*status != 0u) *global = __int_as_float(0x7FC00000);
        *status = 0u;
    }
}

inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void *x, int64_t ld, const nvfp4_tensor *out,
                                               int32_t global_supplied, void *stream) {
    using namespace nvfp4;
    if (out == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (out->rows < 0 || out->cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (out->sf_layout != NVFP4_SF_SWIZZLED_128x4 && out->sf_layout != NVFP4_SF_LINEAR)
        return NVFP4_ERR_INVALID_ARG;
    if (out->cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (out->global == nullptr) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out->global) & 3u) != 0) return NVFP4_ERR_ALIGNMENT;
    if (global_supplied != 0 && global_supplied != 1) return NVFP4_ERR_INVALID_ARG;
    if (out->rows > 0 && out->cols > 0) {
        if (x == nullptr || out->codes == nullptr || out->scales == nullptr)
            return NVFP4_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(out->codes) & 15u) ||
            (reinterpret_cast<uintptr_t>(out->scales) & 15u) || ld % 8 != 0)
            return NVFP4_ERR_ALIGNMENT;
        if (ld < out->cols) return NVFP4_ERR_SHAPE;
    }
    int dev = 0, major = 0, minor = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevs) return NVFP4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;

    // The amax pass writes one partial maximum per CTA and runs at most four
    // CTAs per SM (they stride over any number of rows, so the tensor's size
    // never needs more).  A device with more than 256 SMs would need more
    // partial slots than the array holds: refused, not truncated.
    const int amax_ctas =
        (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div64(out->rows, 8), 4LL * sms));
    if (amax_ctas > kNoAllocPartials) return NVFP4_ERR_WORKSPACE;
    const int64_t tasks = encode_tasks(out->rows, out->cols, out->sf_layout);
    if (tasks >= (int64_t)UINT32_MAX - 65536LL * 1024) return NVFP4_ERR_SHAPE;

    void *scratch = nullptr;
    if (scratch_address(dev, &scratch) != cudaSuccess) return NVFP4_ERR_CUDA;
    uint32_t *status = static_cast<uint32_t *>(scratch);
    uint32_t *partials = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(scratch) + kNoAllocStatusBytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    int n_partials = 0;
    if (!global_supplied) {
        k_amax<<<amax_ctas, 256, 0, s>>>(static_cast<const uint16_t *>(x), ld, out->rows, out->cols,
                                         nullptr, out->rows, partials, status);
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
        n_partials = amax_ctas;
    }
    EncodeParams p;
    p.x = static_cast<const uint16_t *>(x);
    p.ld = ld;
    p.rows = out->rows;
    p.cols = out->cols;
    p.gather = nullptr;
    p.src_rows = out->rows;
    p.codes = static_cast<uint8_t *>(out->codes);
    p.scales = static_cast<uint8_t *>(out->scales);
    p.layout = out->sf_layout;
    p.global = out->global;
    p.global_supplied = global_supplied;
    p.partials = partials;
    p.n_partials = n_partials;
    p.status = status;
    const bool narrow = tasks_are_groups(out->cols);
    void (*kernel)(EncodeParams) = narrow ? k_encode_narrow : k_encode;
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>(ceil_div64(tasks, 8 * (narrow ? 4 : 1)), 8LL * sms));
    kernel<<<grid, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) {
        // The amax pass may already have flagged the shared status word:
        // clear it anyway (best effort), or the next clean call would report
        // this call's error.
        k_status_to_global<<<1, 32, 0, s>>>(status, out->global);
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
    }
    k_status_to_global<<<1, 32, 0, s>>>(status, out->global);
    if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}
