/*
 * dsc.h -- C ABI of the B200 (sm_100a) dynamic short convolution library
 * (libdsc.so).
 *
 * The operation (from "Dynamic Short Convolutions Improve Transformers",
 * technical summary, Methodology: "Mechanism", "Parameterisation",
 * "Placement"; and the authors' thread, on static short convolutions):
 *
 *   y[b,t,c] = r*x[b,t,c] + sum_{k=0}^{W-1} w(t)_k[c] * x[b,t-k,c]
 *
 * a causal depthwise convolution of width W whose filter is chosen per token;
 * terms with t-k < 0 are zero and every batch row is an independent sequence.
 * r is the residual flag (the pages place the op as X = X + conv(X)).  The
 * filter of channel c at token t is:
 *   head-wise:  w[b,t,c/H,k]                (one filter per H consecutive
 *                                            channels, w is [B,T,G,W], G=D/H)
 *   low-rank:   sum_r z[b,t,r] * U[r, (c/H)*W + k]
 *               (z [B,T,R], U [R, G*W]; the product is formed on chip and the
 *                full filter tensor is never written to memory)
 *   static:     ws[c,k]                     (ws [D,W], the same at every t)
 *
 * Backward (the gradients of the definition above; the pages' kernels are
 * training kernels but print no formula):
 *   dx[b,s,c]   = r*dy[b,s,c] + sum_{k, s+k<T} w(s+k)_k[c] * dy[b,s+k,c]
 *   dw[b,t,g,k] = sum_{c in group g} dy[b,t,c] * x[b,t-k,c]     (0 if t < k)
 *   dz[b,t,r]   = sum_{g,k} dw[b,t,g,k] * U[r, g*W+k]
 *   dU[r,g*W+k] = sum_{b,t} z[b,t,r] * dw[b,t,g,k]
 *   dws[c,k]    = sum_{b,t} dy[b,t,c] * x[b,t-k,c]
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are caller-owned DEVICE pointers, dense row-major
 *    in the shapes above (last index fastest), base address 16-byte aligned
 *    (else DSC_ERR_MISALIGNED).  Outputs must not alias inputs.
 *  - dtype DSC_BF16: x, w, z, U, ws, dy and the outputs y, dx, dw, dz are
 *    bf16; arithmetic is fp32; dU and dws are fp32.  DSC_F32: everything fp32.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on that stream and returns; it never
 *    synchronises and never allocates device memory.  Scratch memory, where a
 *    call needs it, is passed in by the caller (`workspace`); its size comes
 *    from the matching *_workspace_bytes query, it must stay untouched until
 *    the stream has passed the call, and it may be NULL when the query
 *    returns 0.
 *  - Validation: B,T >= 1; D >= 1; 1 <= W <= 8; H >= 1 with D % H == 0;
 *    low-rank 1 <= R <= 256; non-NULL tensor pointers; else
 *    DSC_ERR_INVALID_ARG.  Nothing is launched when validation fails.
 *  - A failed launch returns DSC_ERR_CUDA (cudaGetLastError() is left set
 *    for the caller to inspect).
 *  - Kernels that wait on on-chip barriers wait a bounded time; on expiry
 *    they record DSC_ERR_TIMEOUT in a device status word and return.
 *    dsc_check() reads and clears it.
 */
#ifndef DSC_H
#define DSC_H

#include <stddef.h>
#include <stdint.h>

#ifndef DSC_API
#define DSC_API __attribute__((visibility("default")))
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSC_OK = 0,
    DSC_ERR_INVALID_ARG = 1,
    DSC_ERR_UNSUPPORTED = 2,
    DSC_ERR_MISALIGNED = 3,
    DSC_ERR_CUDA = 4,
    DSC_ERR_TIMEOUT = 5
} dsc_status;

typedef enum { DSC_F32 = 0, DSC_BF16 = 1 } dsc_dtype;

/* Problem shape.  H: channels per shared filter (G = D/H groups).  R: rank
 * of the low-rank factorisation (ignored by the other variants).  residual:
 * 1 adds x to y and dy to dx, 0 does not. */
typedef struct {
    int64_t B, T, D, W, H, R;
    int32_t dtype;    /* dsc_dtype */
    int32_t residual;
} dsc_problem;

/* Head-wise forward: x [B,T,D], w [B,T,G,W] -> y [B,T,D]. */
DSC_API dsc_status dsc_fwd_headwise(const dsc_problem *p, const void *x, const void *w, void *y, void *stream);

/* Head-wise backward: x, w, dy -> dx [B,T,D], dw [B,T,G,W]. */
DSC_API dsc_status dsc_bwd_headwise(const dsc_problem *p, const void *x, const void *w, const void *dy, void *dx, void *dw,
                            void *stream);

/* Bytes of scratch the low-rank forward / backward need for this problem.
 * Forward: a copy of U with each vector's filter columns in tap order
 * (R*G*W bf16) for the tensor-core kernel with H < 8, 0 for the other fused
 * kernels, the filters w = zU (B*T*G*W fp32) on the unfused path.  Backward:
 * operand images of z and U, partial sums of dU and dz (fused), or w and
 * dw (unfused).  Neither ever holds the filter tensor on the fused paths. */
DSC_API size_t dsc_fwd_lowrank_workspace_bytes(const dsc_problem *p);
DSC_API size_t dsc_bwd_lowrank_workspace_bytes(const dsc_problem *p);

/* Kernel family a low-rank problem runs on, forward (backward = 0),
 * backward (backward = 1) or decode step (backward = 2, p->T = 1), as chosen
 * by the same host-side plan the calls use (on the current device's SM count;
 * 148 without a device).  Launches nothing and touches no device memory.
 * Returns one of:
 *   DSC_LR_TENSOR_CORE  fused, the filter contractions on tcgen05 tensor cores
 *                       (bf16; R a multiple of 8 up to 64, H a divisor of
 *                       64, D a multiple of 32*H, and a plan that fits the
 *                       shared memory and tensor memory);
 *   DSC_LR_FUSED        fused, contractions on CUDA cores (fp32, other shapes);
 *   DSC_LR_UNFUSED      filters (and their gradient) in the caller's workspace;
 * or -1 when the problem is invalid. */
#define DSC_LR_TENSOR_CORE 0
#define DSC_LR_FUSED 1
#define DSC_LR_UNFUSED 2
DSC_API int dsc_lowrank_kernels(const dsc_problem *p, int backward);

/* Low-rank forward: x [B,T,D], z [B,T,R], U [R,G*W] -> y [B,T,D]. */
DSC_API dsc_status dsc_fwd_lowrank(const dsc_problem *p, const void *x, const void *z, const void *U, void *y,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Low-rank backward: x, z, U, dy -> dx [B,T,D], dz [B,T,R], dU [R,G*W] fp32
 * (dU is overwritten, not accumulated into). */
DSC_API dsc_status dsc_bwd_lowrank(const dsc_problem *p, const void *x, const void *z, const void *U, const void *dy,
                           void *dx, void *dz, float *dU, void *workspace, size_t workspace_bytes, void *stream);

/* Static-filter forward: x [B,T,D], ws [D,W] -> y [B,T,D]. */
DSC_API dsc_status dsc_fwd_static(const dsc_problem *p, const void *x, const void *ws, void *y, void *stream);

/* Scratch bytes of the static backward (per-tile partial filter gradients). */
DSC_API size_t dsc_bwd_static_workspace_bytes(const dsc_problem *p);

/* Static-filter backward: x, ws, dy -> dx [B,T,D], dws [D,W] fp32
 * (overwritten).  Deterministic: partial sums are reduced in a fixed order. */
DSC_API dsc_status dsc_bwd_static(const dsc_problem *p, const void *x, const void *ws, const void *dy, void *dx, float *dws,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Size of the scratch array built into the library for
 * dsc_bwd_static_noalloc (16 MiB per device that loads the library). */
#define DSC_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* Static-filter backward that allocates nothing and takes no workspace.
 * The paper has no counterpart: this exists for callers that cannot hand the
 * library scratch memory -- plugin or custom-op interfaces that pass an
 * operator only its inputs and outputs, and services that allocate all device
 * memory at start-up and must not call cudaMalloc/cudaFree afterwards.
 * Same arguments, results (bit for bit) and argument errors as
 * dsc_bwd_static, except:
 *  - its scratch is an array of DSC_NOALLOC_SCRATCH_BYTES inside the library,
 *    one per device, held from library load until process exit; a problem
 *    whose scratch (dsc_bwd_static_workspace_bytes) exceeds that size is
 *    rejected with DSC_ERR_UNSUPPORTED before anything is launched;
 *  - the first call with a given device current looks the array's device
 *    address up (cudaGetSymbolAddress) and keeps it for the life of the
 *    process; make that first call before any stream capture on that device,
 *    and do not reset the device (cudaDeviceReset) after it;
 *  - all calls on a device share the one array: calls whose work overlaps on
 *    the GPU (different streams without ordering between them) race and give
 *    wrong results.  Each call writes every scratch element it reads, so the
 *    array needs no clearing between calls. */
DSC_API dsc_status dsc_bwd_static_noalloc(const dsc_problem *p, const void *x, const void *ws, const void *dy,
                                          void *dx, float *dws, void *stream);

/* ---------------------------------------------------------------- decode ---
 * Inference step: one new token per sequence.  A causal convolution of width
 * W needs only the last W-1 inputs of each sequence, kept in a state
 * [B, W-1, D] (dtype of x) whose row j holds x_{t-W+1+j}, oldest first, with
 * zero rows for positions before the sequence start.  A step computes
 *   y[b,c] = r x[b,c] + w_0 x[b,c] + sum_{k=1}^{W-1} w_k state[b, W-1-k, c]
 * with the new token's filters and then shifts the state in place (rows
 * 1 .. W-2 move down one row, x becomes the last row).  p->T must be 1;
 * x, y are [B, D]; for W = 1 there is no state and `state` may be NULL.
 * Buffers must not overlap.  Steps from a zero state reproduce the training
 * forward token by token (up to rounding order).
 * Errors as for the training calls; T != 1 gives DSC_ERR_INVALID_ARG. */

/* Head-wise decode: w [B, G, W] holds the new token's filters. */
DSC_API dsc_status dsc_decode_headwise(const dsc_problem *p, const void *x, const void *w, void *state, void *y,
                                       void *stream);

/* Static decode: ws [D, W] as in dsc_fwd_static (p->H is not used). */
DSC_API dsc_status dsc_decode_static(const dsc_problem *p, const void *x, const void *ws, void *state, void *y,
                                     void *stream);

/* Scratch of the low-rank decode: 0 when a fused kernel takes the problem,
 * else the new token's filters, B*G*W fp32.  Fused: the tensor-core kernel
 * for bf16 shapes of the training tensor-core map (R a multiple of 8 up to
 * 64, H a divisor of 64, D a multiple of 32*H, tiles fitting shared
 * memory); otherwise the CUDA-core kernel when D is a multiple of the
 * 16-byte vector width, H divides or is divided by it, and U's columns of 8
 * vectors with R rows fit shared memory. */
DSC_API size_t dsc_decode_lowrank_workspace_bytes(const dsc_problem *p);

/* Low-rank decode: z [B, R] and U [R, G*W].  The fused kernels form the new
 * token's filters w = zU on chip (in TMEM by one MMA per tile of 128
 * sequences, or in registers from U columns staged in shared memory); other
 * shapes form them in the workspace first (`workspace` may be NULL when the
 * size above is 0). */
DSC_API dsc_status dsc_decode_lowrank(const dsc_problem *p, const void *x, const void *z, const void *U, void *state,
                                      void *y, void *workspace, size_t workspace_bytes, void *stream);

/* State after a prompt x [B, T, D] (p->T = prompt length): row j of
 * sequence b holds x[b, T-(W-1)+j], zero where that index is negative.  The
 * prompt's outputs come from the training forward (dsc_fwd_*). */
DSC_API dsc_status dsc_decode_state(const dsc_problem *p, const void *x, void *state, void *stream);

/* ------------------------------------------------------ packed documents ---
 * Variable-length batches ("Dynamic Short Convolutions Improve Transformers",
 * technical summary, Methodology, "Mechanism": the convolution is causal
 * within a sequence, so every document starts from zero history).
 * p->B must be 1: the single row of p->T tokens holds n_docs documents,
 * document d spanning tokens [cu_seqlens[d], cu_seqlens[d+1]).
 *  - cu_seqlens: DEVICE array of n_docs + 1 int32 offsets, non-decreasing
 *    from cu_seqlens[0] = 0 to cu_seqlens[n_docs] = T; 4-byte aligned (else
 *    DSC_ERR_MISALIGNED).  A document may be empty (equal consecutive
 *    offsets, as in a padded list of documents): it has no tokens and
 *    changes nothing.  The offsets are read on the device only: values
 *    outside [0, T] are clamped, so a malformed array gives wrong results
 *    but no access out of bounds.
 *  - n_docs >= 1, else DSC_ERR_INVALID_ARG; DSC_ERR_UNSUPPORTED when
 *    n_docs * (W-1) * ceil(D/256) reaches 2^31 (the fix-up grids).
 * Per document the result is the single-sequence op of the calls above:
 *   y[t]  = r x_t + sum_{k, t-k >= start(t)} w(t)_k x_{t-k}
 *   dx[s] = r dy_s + sum_{k, s+k < end(s)} w(s+k)_k dy_{s+k}
 *   dw[t,g,k] (and dws, dz, dU through it) has no term with t-k < start(t);
 * dU and dws sum over every document.  Each call runs the plain kernels on
 * the row, then recomputes the outputs within W-1 tokens of a document
 * boundary (cost O(n_docs * W * D)).  Arguments, layouts and the remaining
 * errors as in the plain calls. */
DSC_API dsc_status dsc_fwd_headwise_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs,
                                           const void *x, const void *w, void *y, void *stream);
DSC_API dsc_status dsc_bwd_headwise_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs,
                                           const void *x, const void *w, const void *dy, void *dx, void *dw,
                                           void *stream);
/* workspace: as for dsc_fwd_lowrank. */
DSC_API dsc_status dsc_fwd_lowrank_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs,
                                          const void *x, const void *z, const void *U, void *y, void *workspace,
                                          size_t workspace_bytes, void *stream);
/* The plain backward's workspace plus 2 * n_docs * (W-1) * G * W fp32 for
 * the dw rows of the tokens next to a document start. */
DSC_API size_t dsc_bwd_lowrank_varlen_workspace_bytes(const dsc_problem *p, int64_t n_docs);
DSC_API dsc_status dsc_bwd_lowrank_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs,
                                          const void *x, const void *z, const void *U, const void *dy, void *dx,
                                          void *dz, float *dU, void *workspace, size_t workspace_bytes,
                                          void *stream);
DSC_API dsc_status dsc_fwd_static_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs,
                                         const void *x, const void *ws, void *y, void *stream);
/* workspace: dsc_bwd_static_workspace_bytes(p). */
DSC_API dsc_status dsc_bwd_static_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs,
                                         const void *x, const void *ws, const void *dy, void *dx, float *dws,
                                         void *workspace, size_t workspace_bytes, void *stream);

/* -------------------------------------------------------- sequence chunks ---
 * Context parallelism: the sequences are split along time and each call
 * handles one chunk, tokens [t0, t0 + T) of every sequence (p->T = chunk
 * length, row b = sequence b).  The convolution reaches W-1 tokens across a
 * chunk edge, so a chunk takes its neighbours' rows (the halos):
 *  - x_prev  [B, W-1, D]: x at positions t0-W+1 .. t0-1 (row j = position
 *    t0-W+1+j, zero rows for positions before the sequence start -- the
 *    decode state's layout); NULL for a sequence's first chunk;
 *  - dy_next [B, W-1, D]: dy at positions t0+T .. t0+T+W-2 (row j = position
 *    t0+T+j, zero rows past the sequence end), with the filters of the same
 *    tokens: head-wise w_next [B, W-1, G, W], low-rank z_next [B, W-1, R]
 *    (static filters are the same everywhere); NULL for the last chunk.
 * Halos are DEVICE pointers in the dtype of x, 16-byte aligned (else
 * DSC_ERR_MISALIGNED); a dy_next without its filters is DSC_ERR_INVALID_ARG.
 * Results: the rows [t0, t0+T) of the op on the whole sequences; dU and dws
 * sum over this chunk's tokens only (sum them over the chunks).
 * edges_only = 0: the whole call.  edges_only = 1: only the outputs within
 * W-1 tokens of the chunk's edges are recomputed (and dU / dws corrected);
 * the output buffers must already hold the plain call's results on the same
 * inputs (dsc_fwd_headwise etc.), so a caller can run the plain call while
 * the halos are still being exchanged.  For W = 1 the halos are ignored. */
DSC_API dsc_status dsc_fwd_headwise_chunk(const dsc_problem *p, const void *x_prev, const void *x, const void *w,
                                          void *y, int edges_only, void *stream);
DSC_API dsc_status dsc_bwd_headwise_chunk(const dsc_problem *p, const void *x_prev, const void *dy_next,
                                          const void *w_next, const void *x, const void *w, const void *dy, void *dx,
                                          void *dw, int edges_only, void *stream);
/* workspace: as for dsc_fwd_lowrank (not used when edges_only = 1). */
DSC_API dsc_status dsc_fwd_lowrank_chunk(const dsc_problem *p, const void *x_prev, const void *x, const void *z,
                                         const void *U, void *y, void *workspace, size_t workspace_bytes,
                                         int edges_only, void *stream);
/* The plain backward's workspace plus 2 * B * (W-1) * G * W fp32. */
DSC_API size_t dsc_bwd_lowrank_chunk_workspace_bytes(const dsc_problem *p);
DSC_API dsc_status dsc_bwd_lowrank_chunk(const dsc_problem *p, const void *x_prev, const void *dy_next,
                                         const void *z_next, const void *x, const void *z, const void *U,
                                         const void *dy, void *dx, void *dz, float *dU, void *workspace,
                                         size_t workspace_bytes, int edges_only, void *stream);
DSC_API dsc_status dsc_fwd_static_chunk(const dsc_problem *p, const void *x_prev, const void *x, const void *ws,
                                        void *y, int edges_only, void *stream);
/* workspace: dsc_bwd_static_workspace_bytes(p) (may be NULL when edges_only = 1). */
DSC_API dsc_status dsc_bwd_static_chunk(const dsc_problem *p, const void *x_prev, const void *dy_next, const void *x,
                                        const void *ws, const void *dy, void *dx, float *dws, void *workspace,
                                        size_t workspace_bytes, int edges_only, void *stream);

/* ------------------------------------------------- first projection z = hV ---
 * The filter generator is a linear map of the current hidden state factorised
 * at rank R ("Dynamic Short Convolutions Improve Transformers", technical
 * summary, Methodology, "Parameterisation" 1): w(t) = h_t V U, with h
 * [B, T, d_model], V [d_model, R] and U [R, G*W].  These calls take h and V
 * and form z = h V themselves (tensor cores for bf16 with R a multiple of 8
 * up to 64 and d_model a multiple of 128, CUDA cores otherwise; fp32
 * accumulation), then run the low-rank convolution on it.  h and V are in
 * the dtype of x; 1 <= d_model <= 2^30 else DSC_ERR_INVALID_ARG. */

/* Workspace of dsc_fwd_lowrank_proj (that of dsc_fwd_lowrank). */
DSC_API size_t dsc_fwd_lowrank_proj_workspace_bytes(const dsc_problem *p, int64_t d_model);

/* Forward: z [B,T,R] = h V (written: the backward takes it), then y as
 * dsc_fwd_lowrank with that z. */
DSC_API dsc_status dsc_fwd_lowrank_proj(const dsc_problem *p, int64_t d_model, const void *x, const void *h,
                                        const void *V, const void *U, void *z, void *y, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* Workspace of dsc_bwd_lowrank_proj: dz, the low-rank backward's workspace
 * and per-token-range partial sums of dV (never NULL). */
DSC_API size_t dsc_bwd_lowrank_proj_workspace_bytes(const dsc_problem *p, int64_t d_model);

/* Backward, from the forward's z: dx [B,T,D], dh [B,T,d_model] = dz V^T (dtype
 * of x), dV [d_model,R] = sum over tokens of h^T dz (fp32) and dU [R,G*W]
 * (fp32), dz being the low-rank backward's gradient of z (kept in the
 * workspace).  dV and dU are overwritten.  dU is reduced in a fixed order;
 * dh and dV follow dz, which on some shapes is summed over channel blocks
 * with atomic fp32 adds, so they can differ in the last bits between runs. */
DSC_API dsc_status dsc_bwd_lowrank_proj(const dsc_problem *p, int64_t d_model, const void *x, const void *h,
                                        const void *V, const void *z, const void *U, const void *dy, void *dx,
                                        void *dh, float *dV, float *dU, void *workspace, size_t workspace_bytes,
                                        void *stream);

/* Synchronise `stream`, then return and clear the device status word of the
 * current device: DSC_OK, DSC_ERR_TIMEOUT, or DSC_ERR_CUDA if the stream
 * reported an error. */
DSC_API dsc_status dsc_check(void *stream);

/* Failure-detection self-test.  Launches one single-thread kernel that waits
 * on an on-chip barrier nothing completes, with the same bounded wait as the
 * tensor-core kernels but a limit of about 10 million cycles (~5 ms).  The
 * wait gives up, records DSC_ERR_TIMEOUT in the device status word and the
 * kernel returns, leaving the context usable; the next dsc_check() on the
 * stream returns DSC_ERR_TIMEOUT and clears the word.  Returns DSC_OK once
 * the kernel is launched, DSC_ERR_CUDA if the launch failed. */
DSC_API dsc_status dsc_selftest_timeout(void *stream);

/* Static description of a status code. */
DSC_API const char *dsc_status_string(dsc_status s);

/* Number of kernels this library has launched in this process so far (all
 * devices, all streams).  Lets a caller count the launches of a region. */
DSC_API uint64_t dsc_launch_count(void);

/* Library version, major*10000 + minor*100 + patch. */
DSC_API int dsc_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DSC_H */
