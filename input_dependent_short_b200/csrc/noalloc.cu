// Static-filter backward whose scratch memory is built into the library.
//
// The regular dsc_bwd_static takes a caller-allocated workspace for its
// per-tile partial filter gradients.  Some callers cannot provide one: plugin
// or custom-op interfaces that hand an operator only its input and output
// buffers, and services that allocate all device memory at start-up and must
// not call cudaMalloc/cudaFree later (those calls can synchronise the device
// and stall every stream).  dsc_bwd_static_noalloc serves them: its scratch is
// the fixed-size array below, which lives in the library's device image, so
// every GPU that loads the library holds DSC_NOALLOC_SCRATCH_BYTES of it until
// the process exits.  The computation is the regular backward, unchanged.
#include <mutex>

#include "kernels.cuh"

namespace dsc {

constexpr size_t NOALLOC_SCRATCH_FLOATS = DSC_NOALLOC_SCRATCH_BYTES / sizeof(float);

// One array per device.  Host code must not use this name as a pointer: on
// the host it is only a stand-in for the symbol; its device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) float g_noalloc_scratch[NOALLOC_SCRATCH_FLOATS];

// Device address of the array on the current device.  Looked up on the first
// call made with each device current, then cached for the life of the process
// (a cudaDeviceReset after that first call is not supported: the module, and
// the array with it, may be reloaded elsewhere).  A failed CUDA call leaves no
// sticky last-error behind, so the next entry point does not report it as its
// own launch failure.
static float *noalloc_scratch(cudaError_t &err) {
    static std::mutex mu;
    static float *addr[64] = {nullptr};
    int dev = 0;
    err = cudaGetDevice(&dev);
    if (err != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (dev < 0 || dev >= 64) {
        err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (err != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = static_cast<float *>(p);
    }
    return addr[dev];
}

}  // namespace dsc

extern "C" dsc_status dsc_bwd_static_noalloc(const dsc_problem *p, const void *x, const void *ws, const void *dy,
                                             void *dx, float *dws, void *stream) {
    // The same argument checks as dsc_bwd_static, in the same order and with
    // the same status codes, so that a rejected call touches no device state.
    const dsc_status s = dsc::validate(p, false);
    if (s != DSC_OK) return s;
    for (const void *q : {x, ws, dy, (const void *)dx, (const void *)dws})
        if (!q) return DSC_ERR_INVALID_ARG;
    for (const void *q : {x, ws, dy, (const void *)dx, (const void *)dws})
        if (reinterpret_cast<uintptr_t>(q) & 15u) return DSC_ERR_MISALIGNED;
    if (dsc_bwd_static_workspace_bytes(p) > DSC_NOALLOC_SCRATCH_BYTES) return DSC_ERR_UNSUPPORTED;
    cudaError_t err = cudaSuccess;
    float *scratch = dsc::noalloc_scratch(err);
    if (!scratch) return DSC_ERR_CUDA;
    // Every partial the kernels later read is first written by the same call,
    // so the array needs no clearing between calls.
    return dsc_bwd_static(p, x, ws, dy, dx, dws, scratch, DSC_NOALLOC_SCRATCH_BYTES, stream);
}
