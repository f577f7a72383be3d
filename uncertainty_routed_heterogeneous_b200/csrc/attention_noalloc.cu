// attention_noalloc.cu -- heta_attention for callers that cannot allocate.
//
// heta_attention needs device scratch (the work-item counter of the
// persistent kernel and, when the dense rows' key range is split, the halves'
// partial results; without the split only the counter).  Some callers cannot
// provide it: code that must not call cudaMalloc at all (a real-time loop that
// may not block on the allocator, a plug-in host that owns every allocation,
// code running where the allocator is off limits).  heta_attention_noalloc
// runs the same kernel with its scratch in a fixed array that lives in this
// file's device memory.
//
// The array is kStaticScratchBytes (16 MiB) and every GPU that loads the
// library keeps it until the process exits.  The driver commits it when this
// file's module is loaded in a context: with lazy module loading (the CUDA
// default) that is the first call on each device (and again in a new context,
// e.g. after cudaDeviceReset), so that first call should be a warm-up made
// outside any region that must not allocate, and before any stream capture.
// Calls share the array and it keeps the previous call's contents: each call
// clears the counters it needs before its kernel runs, and two calls whose
// kernels overlap on the GPU (different streams, no ordering between them)
// race on it.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "heta_internal.cuh"

namespace heta {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The driver's cuCtxGetCurrent, fetched through the runtime (the library does
// not link libcuda).
PFN_cuCtxGetCurrent_v4000 ctx_get_current_fn()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    });
    return fn;
}

std::mutex g_mu;
struct Cached {
    CUcontext ctx;  // the context the address was looked up in
    void *ptr;      // the array's device address there
};
Cached g_scratch[kMaxDevices];

// Device address of the array in the current device's current context.  In
// host code the array's name is only a stand-in, so the address is looked up
// (with the device current) the first time a device is used and again
// whenever the current context is not the one it was looked up in: after
// cudaDeviceReset the module is loaded anew in a new primary context, and a
// caller may make another context of the same device current.
cudaError_t scratch_on_current_device(void **ptr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    auto get_ctx = ctx_get_current_fn();
    if (!get_ctx) return cudaErrorInvalidDevice;
    CUcontext ctx = nullptr;  // null: no context is current yet
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    Cached &c = g_scratch[dev];
    if (!ctx || !c.ptr || c.ctx != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        // (the lookup made the device's primary context current if none was)
        if (!ctx && (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)) return cudaErrorInvalidDevice;
        c.ctx = ctx;
        c.ptr = p;
    }
    *ptr = c.ptr;
    return cudaSuccess;
}

}  // namespace
}  // namespace heta

extern "C" {

HETA_API heta_status heta_attention_noalloc(const uint16_t *Q, const uint16_t *K,
                                            const uint16_t *V, int B, int H, int d, int Tg,
                                            int Hg, int Wg, int wt, int wh, int ww, float scale,
                                            const int32_t *dense_idx, int k, uint16_t *out,
                                            int32_t *status_dev, void *stream)
{
    size_t need = 0;
    heta_status st =
        heta_attention_workspace_size(B, H, d, Tg, Hg, Wg, wt, wh, ww, k, &need);
    if (st != HETA_OK) return st;
    // When the halves' partials of a split last wave do not fit the array,
    // every dense pair runs over its whole key range instead (the counter
    // alone): slower for that wave, the same result up to rounding order.
    const bool allow_split = need <= heta::kStaticScratchBytes;
    void *scratch = nullptr;
    if (heta::scratch_on_current_device(&scratch) != cudaSuccess) return HETA_ERR_CUDA;
    return static_cast<heta_status>(heta::attention_checked(
        Q, K, V, B, H, d, Tg, Hg, Wg, wt, wh, ww, scale, dense_idx, k, out, scratch,
        heta::kStaticScratchBytes, status_dev, stream, allow_split));
}

}  // extern "C"
