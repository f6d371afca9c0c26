// Declarations of the sequence-edge fix-ups (edges.cu), kept apart from
// kernels.cuh so that the row-pass kernels' sources do not depend on them.
#pragma once

#include "kernels.cuh"

namespace dsc {

// edges.cu: outputs near sequence edges inside a call -- document starts and
// ends of packed documents, the ends of a time chunk of longer sequences --
// recomputed after the zero-padded pass over the whole row or chunk.
enum { EDGE_HEADWISE = 0, EDGE_LOWRANK = 1, EDGE_STATIC = 2 };

struct EdgeArgs {
    int64_t B, T, D, H, G, R, GW;
    int W, residual, kind;
    int early;          // 1: the call ran the row pass just before (which waited on the stream's earlier
                        // kernels), so the fix-ups may load before they wait; 0: they wait first
    const int32_t *cu;  // packed documents: nseg + 1 offsets into the single row; NULL: chunks (segment b = row b)
    int64_t nseg;
    const void *x_prev;   // chunk: x of the W-1 tokens before the chunk [B, W-1, D] (NULL: none)
    const void *dy_next;  // chunk: dy of the W-1 tokens after it [B, W-1, D] (NULL: none)
    const void *f_next;   // chunk: their filters, head-wise [B, W-1, G, W] or low-rank z [B, W-1, R]
    const void *x, *w, *z, *U, *dy;  // w: head-wise filters, or the static ws [D, W]
    void *y, *dx, *dw, *dz;
    float *dU, *dws;
    float *dwfull, *dwdelta;  // low-rank scratch: [nseg * (W-1)][G*W] each
};

void edge_args(const dsc_problem &p, int kind, EdgeArgs &a);
size_t edge_scratch_bytes(const dsc_problem &p, int kind, int64_t nseg);
cudaError_t launch_edges_fwd(const Ctx &c, const dsc_problem &p, const EdgeArgs &a);
cudaError_t launch_edges_bwd(const Ctx &c, const dsc_problem &p, const EdgeArgs &a);

}  // namespace dsc
