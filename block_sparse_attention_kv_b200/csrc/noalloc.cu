// Allocation-free centroid build + INT4 quantisation.
//
// Some callers cannot allocate device memory at the point where they build
// a layer's centroids: code that runs inside a host framework which owns
// every device allocation through its own pool (an inference server, a
// plugin of another runtime), or code on a path where a cudaMalloc is not
// allowed or would synchronise the device.  absp_build_centroids needs a
// caller-provided workspace; this entry point instead uses a scratch array
// compiled into the library, so the caller only passes the layer (inputs)
// and the centroid buffers (outputs).
//
// The scratch is a file-scope __device__ array of ABSP_NOALLOC_BUILD_WS_BYTES
// bytes.  It lives in the library's module: every GPU on which the module is
// loaded holds it until the process exits.  With lazy module loading (the
// CUDA default) that is from the first call of the entry point on that GPU;
// with eager loading (CUDA_MODULE_LOADING=EAGER) it is from the creation of
// the context on every GPU the process uses, whether or not the entry point
// is ever called.  All calls on one GPU share it and it keeps the last
// call's contents, so each call clears the parts that must start at zero
// (the error word and the per-channel min/max keys), and calls whose work
// overlaps on the GPU (different streams, no ordering between them) race on
// it: the caller must order them.
#include <mutex>

#include "absp_internal.cuh"
#include "absp_trace.h"

namespace {

__device__ __align__(256) uint8_t g_noalloc_build_ws[ABSP_NOALLOC_BUILD_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};
unsigned long long g_ctx_id[kMaxDevices] = {};  // context the address belongs to

// Driver entry points that identify the current context (resolved once).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
struct CtxFns {
    CtxGetCurrentFn current = nullptr;
    CtxGetIdFn id = nullptr;
};
const CtxFns& ctx_fns() {
    static const CtxFns f = [] {
        CtxFns r;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            r.current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            r.id = reinterpret_cast<CtxGetIdFn>(p);
        return r;
    }();
    return f;
}

// Unique id of the calling thread's current context, 0 if none or unknown.
unsigned long long current_ctx_id() {
    const CtxFns& f = ctx_fns();
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (f.current == nullptr || f.id == nullptr || f.current(&c) != CUDA_SUCCESS || c == nullptr)
        return 0;
    return f.id(c, &id) == CUDA_SUCCESS ? id : 0;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress, once per device and context, with that device
// current.  The lookup is repeated when the device's context is not the one
// the cached address belongs to (a cudaDeviceReset destroys the primary
// context, and the array is reloaded at another address in the next one).
cudaError_t noalloc_scratch(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long ctx = current_ctx_id();
    if (g_ws_ptr[dev] == nullptr || ctx == 0 || ctx != g_ctx_id[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_build_ws);
        if (e != cudaSuccess) return e;
        g_ws_ptr[dev] = p;
        // the lookup made the device's context current if none was
        g_ctx_id[dev] = current_ctx_id();
    }
    *out = g_ws_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" absp_status absp_build_quantize_noalloc(const absp_layer_kv* kv,
                                                   const absp_centroids* out,
                                                   int32_t* device_status, void* stream) {
    ABSP_TRACE("absp_build_quantize_noalloc");
    absp::KvDesc d;
    absp_status st = absp::make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if ((st = absp::check_cent(out)) != ABSP_OK) return st;
    if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) % 4) != 0)
        return ABSP_ERR_INVALID_ARG;
    if (absp::build_ws_bytes(d) > static_cast<size_t>(ABSP_NOALLOC_BUILD_WS_BYTES))
        return ABSP_ERR_UNSUPPORTED;
    void* ws = nullptr;
    cudaError_t e = noalloc_scratch(&ws);
    if (e != cudaSuccess) return absp::cuda_status(e);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the error word and detail start at zero; launch_build resets the
    // min/max keys itself
    if ((e = cudaMemsetAsync(ws, 0, 2 * sizeof(int32_t), s)) != cudaSuccess)
        return absp::cuda_status(e);
    const absp::BuildWs w = absp::build_ws_layout(ws, d);
    if ((e = absp::launch_build(d, w, s)) != cudaSuccess) return absp::cuda_status(e);
    if ((e = absp::launch_quantize(d, w, out->codes, out->scale, out->zp, out->format, s)) !=
        cudaSuccess)
        return absp::cuda_status(e);
    if (device_status != nullptr &&
        (e = cudaMemcpyAsync(device_status, ws, 2 * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                             s)) != cudaSuccess)
        return absp::cuda_status(e);
    return ABSP_OK;
}
