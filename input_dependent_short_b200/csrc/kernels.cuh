// Launch interface between the C entry points (api.cu) and the kernels.
#pragma once

#include <utility>

#include "common.cuh"

namespace dsc {

// Mapping of the time-streaming kernels.  Each thread owns one 16-byte vector
// of channels (V = 8 bf16 or 4 fp32) and walks Tt consecutive tokens of one
// sequence.  A warp covers CW channels starting at wc*CW; lane l owns channels
// wc*CW + l*V .. +V-1 and is active when l < lanes_used and the channel is < D.
// When H is a multiple of V, the L = H/V consecutive lanes of one filter group
// reduce the group's filter gradient with shuffles; when V is a multiple of H a
// lane owns GPT = V/H whole groups.
struct StreamMap {
    int64_t B, T, D, H, G;
    int W;
    int Tt, nTiles, nWc, CW, lanes_used, L, gpt;
    int64_t n_warps;
    int residual;
    int vb;  // bytes of a thread's channel vector (16, or 8 for W >= 5)
};

struct HwArgs {
    StreamMap m;
    const void *x, *w, *dy;
    void *y, *dx, *dw;
    float *partial;  // static filter-gradient partials [B*nTiles][D][W]
};

// Generic per-channel kernels (any D, H, W <= 8); `wmode` selects the filter.
enum { WMODE_HEADWISE = 0, WMODE_STATIC = 1 };

struct GenArgs {
    int64_t B, T, D, H, G;
    int W, Tt, nTiles, residual, wmode;
    const void *x, *w, *dy;
    void *y, *dx, *dw;
    float *partial;
};

// Argument checks shared by the entry points (api.cu): the problem shape and
// dtype, as documented in dsc.h (DSC_ERR_INVALID_ARG or DSC_ERR_UNSUPPORTED).
dsc_status validate(const dsc_problem *p, bool lowrank);

struct Ctx {
    cudaStream_t stream;
    int sms;
};

// conv_stream.cu
bool stream_map(const dsc_problem &p, int V, StreamMap &m);
bool stream_plan(const dsc_problem &p, StreamMap &m);
void finish_map(StreamMap &m, int64_t target_warps);
cudaError_t launch_hw_fwd(const Ctx &c, const dsc_problem &p, HwArgs a);
cudaError_t launch_hw_bwd(const Ctx &c, const dsc_problem &p, HwArgs a);
cudaError_t launch_st_fwd(const Ctx &c, const dsc_problem &p, HwArgs a);
cudaError_t launch_st_bwd(const Ctx &c, const dsc_problem &p, HwArgs a, float *dws);
size_t st_partial_count(const Ctx &c, const dsc_problem &p);

// generic.cu (w may be a fp32 workspace: `w_f32`)
cudaError_t launch_gen_fwd(const Ctx &c, const dsc_problem &p, GenArgs a, bool w_f32);
cudaError_t launch_gen_dx(const Ctx &c, const dsc_problem &p, GenArgs a, bool w_f32);
cudaError_t launch_gen_dw(const Ctx &c, const dsc_problem &p, GenArgs a, bool out_f32);
cudaError_t launch_gen_dws(const Ctx &c, const dsc_problem &p, GenArgs a, float *dws, float *partial, int tile);
cudaError_t launch_lr_filters(const Ctx &c, const dsc_problem &p, const void *z, const void *U, float *wf);
// C[i][j] = sum_k A[i*sai + k*sak] * B[j*sbj + k*sbk], fp32 accumulate.
cudaError_t launch_gemm(const Ctx &c, int M, int N, int K, const void *A, bool a_f32, int64_t sai, int64_t sak,
                        const void *B, bool b_f32, int64_t sbj, int64_t sbk, void *C, bool c_f32, int64_t ldc,
                        bool bf16_io);
cudaError_t launch_reduce_partials(const Ctx &c, const float *partial, int64_t S, int64_t n, float *out);

// lowrank.cu (fused kernels)
bool lowrank_fused_ok(const dsc_problem &p);
cudaError_t launch_lr_fwd_fused(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                                void *y);
cudaError_t launch_lr_bwd_fused(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                                const void *dy, void *dx, void *dz, float *dU, void *ws, size_t ws_bytes);
size_t lr_bwd_fused_ws_bytes(const Ctx &c, const dsc_problem &p);

// lowrank_tc_fwd.cu, lowrank_tc_bwd.cu (tensor-core kernels, bf16)
bool lowrank_tc_ok(const dsc_problem &p);
size_t lr_tc_fwd_ws_bytes(const dsc_problem &p);
cudaError_t launch_lr_fwd_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U, void *y,
                             void *ws, size_t ws_bytes);
int take_tc_status(cudaStream_t stream);
cudaError_t launch_wait_selftest(cudaStream_t stream);
bool lowrank_tc_bwd_ok(const dsc_problem &p, int sms);
size_t lr_tc_bwd_ws_bytes(const dsc_problem &p, int sms);
cudaError_t launch_lr_bwd_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                             const void *dy, void *dx, void *dz, float *dU, void *ws, size_t ws_bytes);

// proj.cu: the first low-rank projection z = h V (h [N, d], V [d, R]) and its
// gradients dh = dz V^T, dV = h^T dz; tensor cores for bf16 with R a multiple
// of 8 up to 64 and d a multiple of 128, the CUDA-core GEMM otherwise.
bool proj_tc_ok(const dsc_problem &p, int64_t d);
size_t proj_dV_part_bytes(const dsc_problem &p, int64_t d, int sms);
cudaError_t launch_proj_z(const Ctx &c, const dsc_problem &p, int64_t d, const void *h, const void *V, void *z);
cudaError_t launch_proj_bwd(const Ctx &c, const dsc_problem &p, int64_t d, const void *h, const void *V, const void *dz,
                            void *dh, float *dV, float *part);
int take_proj_status(cudaStream_t stream);

int resident_blocks(const void *kernel, int threads, size_t smem);

// Records one kernel launch (api.cu keeps the process-wide count).
void count_launch();

// Programmatic dependent launch.  A kernel launched with launch_pdl may be
// scheduled while the previous kernel of the stream is still finishing; it
// runs its prologue, then pdl_wait() blocks until that kernel has completed
// and its writes are visible, so it must come before the first access to
// global memory.  pdl_trigger() lets the next kernel of the stream be
// scheduled the same way (it still waits for this one to complete).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    count_launch();
    return e;
}

// Status word of kernels with bounded waits (lowrank.cu): returns the
// recorded dsc_status of the current device and clears it.
int take_device_status(cudaStream_t stream);

}  // namespace dsc
