// Fused low-rank kernels of the dynamic short convolution (sm_100a).
#include "kernels.cuh"

namespace dsc {

// Device status word of this library on each device: 0 = OK, otherwise the
// dsc_status a kernel recorded when one of its bounded waits expired.
__device__ int g_dsc_status = 0;

int take_device_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    return v;
}

bool lowrank_fused_ok(const dsc_problem &) { return false; }

cudaError_t launch_lr_fwd_fused(const Ctx &, const dsc_problem &, const void *, const void *, const void *, void *) {
    return cudaErrorNotSupported;
}

cudaError_t launch_lr_bwd_fused(const Ctx &, const dsc_problem &, const void *, const void *, const void *,
                                const void *, void *, void *, float *, void *, size_t) {
    return cudaErrorNotSupported;
}

size_t lr_bwd_fused_ws_bytes(const Ctx &, const dsc_problem &) { return 0; }

}  // namespace dsc
