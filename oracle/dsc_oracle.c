/*
 * dsc_oracle.c -- plain fp64 CPU oracle of the dynamic short convolution.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this file's library.  The CUDA library never links,
 * includes or calls it, and it shares no code with the CUDA path.
 *
 * Source of the method: "Dynamic Short Convolutions Improve Transformers"
 * (Sieberling, Runwal, Panda, Kim), as summarised on the gist.science
 * technical-summary pages ("Resumen Tecnico: Las Convoluciones Cortas
 * Dinamicas Mejoran los Transformers" and its French, German and Hindi
 * versions) and in the authors' announcement thread.
 *
 *  - Methodology, "Mechanism": the output of one channel-wise step is
 *    y_t = sum_{k=0}^{W-1} w(t)_k (.) x_{t-k}, the filter w(t) being chosen per
 *    time step.  k is the lag: tap 0 multiplies x_t, tap W-1 multiplies
 *    x_{t-W+1}; positions t-k < 0 contribute zero (the static short conv it
 *    generalises is a causal depthwise conv, authors' thread).
 *  - Methodology, "Placement": the op is used with a residual,
 *    X = X + dynamicShortConv(X); the flag `residual` selects it.
 *  - Methodology, "Parameterisation" 2, head-wise tying: one filter per block
 *    of H consecutive channels, so channel c uses filter group g = floor(c/H)
 *    of G = D/H groups: w has shape [B,T,G,W] (tap fastest).
 *  - Methodology, "Parameterisation" 1, low rank R, with the fused kernel of
 *    "Efficient training implementation": w(t) = z_t U, z of shape [B,T,R],
 *    U of shape [R, G*W] whose column g*W+k holds tap k of group g.
 *  - The static special case: one filter per channel, ws of shape [D,W],
 *    the same for every token.
 *  - Backward (the pages' kernels are training kernels; no formula is
 *    printed, so the gradients of the definition above are written out):
 *      dx[b,s,c]   = r*dy[b,s,c] + sum_{k, s+k<T} w(s+k)_k[c] * dy[b,s+k,c]
 *      dw[b,t,g,k] = sum_{c in group g} dy[b,t,c] * x[b,t-k,c]   (0 if t<k)
 *      dz[b,t,r]   = sum_{g,k} dw[b,t,g,k] * U[r, g*W+k]
 *      dU[r,g*W+k] = sum_{b,t} z[b,t,r] * dw[b,t,g,k]
 *      dws[c,k]    = sum_{b,t} dy[b,t,c] * x[b,t-k,c]
 *
 * Everything is evaluated in fp64 from the exact values of the stored inputs
 * (fp32, bf16 bit patterns or fp64).  The full-tensor functions evaluate the
 * per-element definitions at every index; OpenMP only spreads independent
 * output elements over threads and never reorders a sum.
 */

#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };
enum { ORC_HEADWISE = 0, ORC_LOWRANK = 1, ORC_STATIC = 2 };
enum { ORC_Y = 0, ORC_DX = 1, ORC_DW = 2, ORC_DZ = 3, ORC_DU = 4, ORC_DWS = 5, ORC_W = 6 };

typedef struct {
    int64_t B, T, D, W, H, R;
    int64_t residual;
} orc_problem;

typedef struct {
    const void *p;
    int64_t dt;
} orc_in;

/* Filters of one call: head-wise w [B,T,G,W], static ws [D,W], or low-rank
 * z [B,T,R] and U [R,G*W]. */
typedef struct {
    int64_t kind;
    orc_in w;
    orc_in z;
    orc_in U;
} orc_filter;

/* Exact fp64 value of element i of a stored tensor. */
static double val(orc_in a, int64_t i)
{
    if (a.dt == ORC_F32) return (double)((const float *)a.p)[i];
    if (a.dt == ORC_F64) return ((const double *)a.p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)a.p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int64_t tok(const orc_problem *P, int64_t b, int64_t t) { return b * P->T + t; }

/* Low-rank factorisation: tap k of group g at token (b,t) is z_t . U[:, g*W+k]. */
static double lowrank_tap(const orc_problem *P, const orc_filter *F, int64_t b, int64_t t, int64_t g, int64_t k)
{
    int64_t GW = (P->D / P->H) * P->W;
    double s = 0.0;
    for (int64_t r = 0; r < P->R; ++r)
        s += val(F->z, tok(P, b, t) * P->R + r) * val(F->U, r * GW + g * P->W + k);
    return s;
}

/* Tap k of the filter that channel c uses at token (b,t). */
static double tap(const orc_problem *P, const orc_filter *F, int64_t b, int64_t t, int64_t c, int64_t k)
{
    int64_t G = P->D / P->H;
    int64_t g = c / P->H;
    if (F->kind == ORC_STATIC) return val(F->w, c * P->W + k);
    if (F->kind == ORC_LOWRANK) return lowrank_tap(P, F, b, t, g, k);
    return val(F->w, (tok(P, b, t) * G + g) * P->W + k);
}

static double xval(const orc_problem *P, orc_in x, int64_t b, int64_t t, int64_t c)
{
    return val(x, tok(P, b, t) * P->D + c);
}

/* y[b,t,c] = r*x_t + sum_k w(t)_k x_{t-k}, causal with zero padding. */
static double y_at(const orc_problem *P, const orc_filter *F, orc_in x, int64_t b, int64_t t, int64_t c)
{
    double s = P->residual ? xval(P, x, b, t, c) : 0.0;
    for (int64_t k = 0; k < P->W; ++k)
        if (t - k >= 0) s += tap(P, F, b, t, c, k) * xval(P, x, b, t - k, c);
    return s;
}

/* dx[b,s,c]: x_s enters y_{s+k} through tap k of w(s+k). */
static double dx_at(const orc_problem *P, const orc_filter *F, orc_in dy, int64_t b, int64_t s, int64_t c)
{
    double acc = P->residual ? xval(P, dy, b, s, c) : 0.0;
    for (int64_t k = 0; k < P->W; ++k)
        if (s + k < P->T) acc += tap(P, F, b, s + k, c, k) * xval(P, dy, b, s + k, c);
    return acc;
}

/* dw[b,t,g,k]: sum over the H channels that share filter group g. */
static double dw_at(const orc_problem *P, orc_in x, orc_in dy, int64_t b, int64_t t, int64_t g, int64_t k)
{
    if (t - k < 0) return 0.0;
    double s = 0.0;
    for (int64_t c = g * P->H; c < (g + 1) * P->H; ++c)
        s += xval(P, dy, b, t, c) * xval(P, x, b, t - k, c);
    return s;
}

/* dz[b,t,r] = sum_{g,k} dw[b,t,g,k] U[r, g*W+k]. */
static double dz_at(const orc_problem *P, const orc_filter *F, orc_in x, orc_in dy, int64_t b, int64_t t, int64_t r)
{
    int64_t G = P->D / P->H, GW = G * P->W;
    double s = 0.0;
    for (int64_t g = 0; g < G; ++g)
        for (int64_t k = 0; k < P->W; ++k)
            s += dw_at(P, x, dy, b, t, g, k) * val(F->U, r * GW + g * P->W + k);
    return s;
}

/* dU[r, g*W+k] = sum over every token of z[b,t,r] dw[b,t,g,k]. */
static double dU_at(const orc_problem *P, const orc_filter *F, orc_in x, orc_in dy, int64_t r, int64_t g, int64_t k)
{
    double s = 0.0;
    for (int64_t b = 0; b < P->B; ++b)
        for (int64_t t = 0; t < P->T; ++t)
            s += val(F->z, tok(P, b, t) * P->R + r) * dw_at(P, x, dy, b, t, g, k);
    return s;
}

/* Static filter gradient dws[c,k] = sum over every token of dy_t x_{t-k}. */
static double dws_at(const orc_problem *P, orc_in x, orc_in dy, int64_t c, int64_t k)
{
    double s = 0.0;
    for (int64_t b = 0; b < P->B; ++b)
        for (int64_t t = k; t < P->T; ++t)
            s += xval(P, dy, b, t, c) * xval(P, x, b, t - k, c);
    return s;
}

/* ---------------------------------------------------------------- API --- */

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* w[b,t,g,k] = z_t . U[:, g*W+k] for every token (the oracle may hold it). */
void orc_lowrank_filters(const orc_problem *P, orc_in z, orc_in U, double *w_out)
{
    orc_filter F = {ORC_LOWRANK, {0, 0}, z, U};
    int64_t G = P->D / P->H, NT = P->B * P->T;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < NT; ++n)
        for (int64_t g = 0; g < G; ++g)
            for (int64_t k = 0; k < P->W; ++k)
                w_out[(n * G + g) * P->W + k] = lowrank_tap(P, &F, n / P->T, n % P->T, g, k);
}

/* Forward, head-wise (w [B,T,G,W]) or static (w [D,W]): y [B,T,D] in fp64. */
void orc_forward(const orc_problem *P, int64_t kind, orc_in w, orc_in x, double *y_out)
{
    orc_filter F = {kind, w, {0, 0}, {0, 0}};
    int64_t NT = P->B * P->T;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < NT; ++n)
        for (int64_t c = 0; c < P->D; ++c)
            y_out[n * P->D + c] = y_at(P, &F, x, n / P->T, n % P->T, c);
}

/* Backward, head-wise or static: dx [B,T,D]; dw [B,T,G,W] (head-wise) or
 * dws [D,W] (static), both fp64. */
void orc_backward(const orc_problem *P, int64_t kind, orc_in w, orc_in x, orc_in dy, double *dx_out, double *dw_out)
{
    orc_filter F = {kind, w, {0, 0}, {0, 0}};
    int64_t NT = P->B * P->T, G = P->D / P->H;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < NT; ++n)
        for (int64_t c = 0; c < P->D; ++c)
            dx_out[n * P->D + c] = dx_at(P, &F, dy, n / P->T, n % P->T, c);
    if (kind == ORC_STATIC) {
#pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < P->D; ++c)
            for (int64_t k = 0; k < P->W; ++k)
                dw_out[c * P->W + k] = dws_at(P, x, dy, c, k);
    } else {
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < NT; ++n)
            for (int64_t g = 0; g < G; ++g)
                for (int64_t k = 0; k < P->W; ++k)
                    dw_out[(n * G + g) * P->W + k] = dw_at(P, x, dy, n / P->T, n % P->T, g, k);
    }
}

/* Low-rank filter-side gradients from the head-wise dw of the same call:
 * dz [B,T,R] = dw . U^T per token, dU [R,G*W] = sum over tokens of z^T dw. */
void orc_lowrank_grads(const orc_problem *P, orc_in z, orc_in U, const double *dw, double *dz_out, double *dU_out)
{
    int64_t GW = (P->D / P->H) * P->W, NT = P->B * P->T;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < NT; ++n)
        for (int64_t r = 0; r < P->R; ++r) {
            double s = 0.0;
            for (int64_t j = 0; j < GW; ++j) s += dw[n * GW + j] * val(U, r * GW + j);
            dz_out[n * P->R + r] = s;
        }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < GW; ++j)
        for (int64_t r = 0; r < P->R; ++r) {
            double s = 0.0;
            for (int64_t n = 0; n < NT; ++n) s += val(z, n * P->R + r) * dw[n * GW + j];
            dU_out[r * GW + j] = s;
        }
}

/* Element-by-element evaluation at n sample points, for checks at sizes where
 * whole tensors are too costly.  `idx` holds 4 int64 per point:
 *   ORC_Y, ORC_DX : (b, t, c, -)
 *   ORC_DW, ORC_W : (b, t, g, k)
 *   ORC_DZ        : (b, t, r, -)
 *   ORC_DU        : (r, g, k, -)
 *   ORC_DWS       : (c, k, -, -)                                            */
void orc_sample(const orc_problem *P, const orc_filter *F, orc_in x, orc_in dy, int64_t what, int64_t n,
                const int64_t *idx, double *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t *q = idx + 4 * i;
        double v = 0.0;
        switch (what) {
        case ORC_Y: v = y_at(P, F, x, q[0], q[1], q[2]); break;
        case ORC_DX: v = dx_at(P, F, dy, q[0], q[1], q[2]); break;
        case ORC_DW: v = dw_at(P, x, dy, q[0], q[1], q[2], q[3]); break;
        case ORC_W: v = tap(P, F, q[0], q[1], q[2] * P->H, q[3]); break;
        case ORC_DZ: v = dz_at(P, F, x, dy, q[0], q[1], q[2]); break;
        case ORC_DU: v = dU_at(P, F, x, dy, q[0], q[1], q[2]); break;
        case ORC_DWS: v = dws_at(P, x, dy, q[0], q[1]); break;
        default: v = NAN;
        }
        out[i] = v;
    }
}

/* Decode step: the definition above evaluated at the newest token t of each
 * sequence, with its W-1 predecessors taken from a state [B, W-1, D] whose
 * row j holds x_{t-W+1+j} (zero rows stand for positions before the
 * sequence start).  P->T is 1: the filters of the new token are head-wise
 * w [B,1,G,W], low-rank z [B,1,R] with U [R,G*W], or static ws [D,W].
 *   y[b,c] = r*x[b,c] + w_0 x[b,c] + sum_{k=1}^{W-1} w_k state[b, W-1-k, c]
 * The state after the step holds x_{t-W+2} .. x_t: rows 1 .. W-2 of the old
 * state, then x. */
void orc_decode(const orc_problem *P, const orc_filter *F, orc_in x, orc_in state, double *y_out,
                double *state_out)
{
    const int64_t S = P->W - 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < P->B; ++b)
        for (int64_t c = 0; c < P->D; ++c) {
            const double xt = val(x, b * P->D + c);
            double s = P->residual ? xt : 0.0;
            for (int64_t k = 0; k < P->W; ++k) {
                const double xk = k == 0 ? xt : val(state, (b * S + (S - k)) * P->D + c);
                s += tap(P, F, b, 0, c, k) * xk;
            }
            y_out[b * P->D + c] = s;
            for (int64_t j = 0; j + 1 < S; ++j)
                state_out[(b * S + j) * P->D + c] = val(state, (b * S + j + 1) * P->D + c);
            if (S > 0) state_out[(b * S + S - 1) * P->D + c] = xt;
        }
}

/* Variable-length (packed) sequences: one row of P->T tokens (P->B = 1)
 * holds nseq documents, document d spanning tokens [cu[d], cu[d+1]), with
 * cu[0] = 0 and cu[nseq] = P->T.  A document is a sequence of its own, so
 * the definition's zero padding applies at every document start: tap k of
 * token t contributes only when t-k lies in t's document.  The gradients
 * follow: dx[s] takes tap k of token s+k only when s+k lies in s's document,
 * and dw[t,g,k] (and the static dws) takes dy_t x_{t-k} only when t-k does.
 * Head-wise filters w [1,T,G,W] (low-rank: the materialised w = zU) or
 * static ws [D,W]. */
static int64_t doc_of(const int64_t *cu, int64_t nseq, int64_t t)
{
    int64_t d = 0;
    while (d + 1 < nseq && cu[d + 1] <= t) ++d;
    return d;
}

void orc_forward_varlen(const orc_problem *P, int64_t kind, orc_in w, orc_in x, const int64_t *cu, int64_t nseq,
                        double *y_out)
{
    orc_filter F = {kind, w, {0, 0}, {0, 0}};
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < P->T; ++t) {
        const int64_t start = cu[doc_of(cu, nseq, t)];
        for (int64_t c = 0; c < P->D; ++c) {
            double s = P->residual ? xval(P, x, 0, t, c) : 0.0;
            for (int64_t k = 0; k < P->W; ++k)
                if (t - k >= start) s += tap(P, &F, 0, t, c, k) * xval(P, x, 0, t - k, c);
            y_out[t * P->D + c] = s;
        }
    }
}

void orc_backward_varlen(const orc_problem *P, int64_t kind, orc_in w, orc_in x, orc_in dy, const int64_t *cu,
                         int64_t nseq, double *dx_out, double *dw_out)
{
    orc_filter F = {kind, w, {0, 0}, {0, 0}};
    const int64_t G = P->D / P->H;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < P->T; ++s) {
        const int64_t end = cu[doc_of(cu, nseq, s) + 1];
        for (int64_t c = 0; c < P->D; ++c) {
            double acc = P->residual ? xval(P, dy, 0, s, c) : 0.0;
            for (int64_t k = 0; k < P->W; ++k)
                if (s + k < end) acc += tap(P, &F, 0, s + k, c, k) * xval(P, dy, 0, s + k, c);
            dx_out[s * P->D + c] = acc;
        }
    }
    if (kind == ORC_STATIC) {
#pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < P->D; ++c)
            for (int64_t k = 0; k < P->W; ++k) {
                double acc = 0.0;
                for (int64_t t = 0; t < P->T; ++t)
                    if (t - k >= cu[doc_of(cu, nseq, t)]) acc += xval(P, dy, 0, t, c) * xval(P, x, 0, t - k, c);
                dw_out[c * P->W + k] = acc;
            }
    } else {
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < P->T; ++t) {
            const int64_t start = cu[doc_of(cu, nseq, t)];
            for (int64_t g = 0; g < G; ++g)
                for (int64_t k = 0; k < P->W; ++k) {
                    double acc = 0.0;
                    if (t - k >= start)
                        for (int64_t c = g * P->H; c < (g + 1) * P->H; ++c)
                            acc += xval(P, dy, 0, t, c) * xval(P, x, 0, t - k, c);
                    dw_out[(t * G + g) * P->W + k] = acc;
                }
        }
    }
}

/* A chunk of longer sequences (context parallelism, the sequence split along
 * time over ranks): row b holds tokens [t0, t0+T) of sequence b.  The
 * definition is unchanged; only the values outside the chunk come from its
 * neighbours instead of being zero:
 *   xp  [B, W-1, D]: x at positions t0-W+1 .. t0-1 (row j = position
 *        t0-W+1+j, the decode state's layout), or NULL when t0 = 0;
 *   dyn [B, W-1, D]: dy at positions t0+T .. t0+T+W-2 (row j = t0+T+j), and
 *   wn  [B, W-1, G, W]: the head-wise filters of those tokens (low-rank: the
 *        materialised zU), both NULL for the sequence's last chunk.
 * With a chunk index u relative to t0 (so u < 0 is in xp, u >= T in dyn):
 *   y[b,t,c]   = r*x_t + sum_k w(t)_k x_{t-k}
 *   dx[b,s,c]  = r*dy_s + sum_k w(s+k)_k dy_{s+k}
 *   dw[b,t,g,k] = sum_{c in g} dy_t x_{t-k};  dws[c,k] = sum_{b,t} dy_t x_{t-k}
 * where x, dy and w at indices outside the chunk read the halos (terms with
 * no halo are absent, as in the zero-padded definition). */
typedef struct {
    orc_in xp, dyn, wn;
} orc_halo;

static int x_ext(const orc_problem *P, orc_in x, const orc_halo *h, int64_t b, int64_t u, int64_t c, double *v)
{
    if (u >= 0) {
        *v = xval(P, x, b, u, c);
        return 1;
    }
    if (!h->xp.p) return 0;
    *v = val(h->xp, (b * (P->W - 1) + (u + P->W - 1)) * P->D + c);
    return 1;
}

static int dy_ext(const orc_problem *P, orc_in dy, const orc_halo *h, int64_t b, int64_t u, int64_t c, double *v)
{
    if (u < P->T) {
        *v = xval(P, dy, b, u, c);
        return 1;
    }
    if (!h->dyn.p) return 0;
    *v = val(h->dyn, (b * (P->W - 1) + (u - P->T)) * P->D + c);
    return 1;
}

static double tap_ext(const orc_problem *P, const orc_filter *F, const orc_halo *h, int64_t b, int64_t u, int64_t c,
                      int64_t k)
{
    if (u < P->T || F->kind == ORC_STATIC) return tap(P, F, b, u, c, k);
    const int64_t G = P->D / P->H;
    return val(h->wn, ((b * (P->W - 1) + (u - P->T)) * G + c / P->H) * P->W + k);
}

void orc_forward_chunk(const orc_problem *P, int64_t kind, orc_in w, orc_in x, orc_in xp, double *y_out)
{
    orc_filter F = {kind, w, {0, 0}, {0, 0}};
    orc_halo h = {xp, {0, 0}, {0, 0}};
    int64_t NT = P->B * P->T;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < NT; ++n) {
        const int64_t b = n / P->T, t = n % P->T;
        for (int64_t c = 0; c < P->D; ++c) {
            double s = P->residual ? xval(P, x, b, t, c) : 0.0, xv;
            for (int64_t k = 0; k < P->W; ++k)
                if (x_ext(P, x, &h, b, t - k, c, &xv)) s += tap(P, &F, b, t, c, k) * xv;
            y_out[n * P->D + c] = s;
        }
    }
}

void orc_backward_chunk(const orc_problem *P, int64_t kind, orc_in w, orc_in x, orc_in dy, orc_in xp, orc_in dyn,
                        orc_in wn, double *dx_out, double *dw_out)
{
    orc_filter F = {kind, w, {0, 0}, {0, 0}};
    orc_halo h = {xp, dyn, wn};
    const int64_t NT = P->B * P->T, G = P->D / P->H;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < NT; ++n) {
        const int64_t b = n / P->T, s = n % P->T;
        for (int64_t c = 0; c < P->D; ++c) {
            double acc = P->residual ? xval(P, dy, b, s, c) : 0.0, d;
            for (int64_t k = 0; k < P->W; ++k)
                if (dy_ext(P, dy, &h, b, s + k, c, &d)) acc += tap_ext(P, &F, &h, b, s + k, c, k) * d;
            dx_out[n * P->D + c] = acc;
        }
    }
    if (kind == ORC_STATIC) {
#pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < P->D; ++c)
            for (int64_t k = 0; k < P->W; ++k) {
                double acc = 0.0, xv;
                for (int64_t b = 0; b < P->B; ++b)
                    for (int64_t t = 0; t < P->T; ++t)
                        if (x_ext(P, x, &h, b, t - k, c, &xv)) acc += xval(P, dy, b, t, c) * xv;
                dw_out[c * P->W + k] = acc;
            }
    } else {
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < NT; ++n) {
            const int64_t b = n / P->T, t = n % P->T;
            for (int64_t g = 0; g < G; ++g)
                for (int64_t k = 0; k < P->W; ++k) {
                    double acc = 0.0, xv;
                    for (int64_t c = g * P->H; c < (g + 1) * P->H; ++c)
                        if (x_ext(P, x, &h, b, t - k, c, &xv)) acc += xval(P, dy, b, t, c) * xv;
                    dw_out[(n * G + g) * P->W + k] = acc;
                }
        }
    }
}
