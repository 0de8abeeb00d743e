/*
 * gspn_ref.c -- plain double-precision CPU oracle of the GSPN line scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this file's library.  It shares no code with the
 * CUDA library and is deliberately slow and literal: nested loops over
 * planes, directions, lines and positions, each step in the order the method
 * states it, every value in double.
 *
 * What it computes (cited by page title and section):
 *
 *  a1  Gate normalisation -- "Parallel Sequence Modeling via Generalized
 *      Spatial Propagation Network" (GSPN, CVPR 2025 reading notes), Key
 *      design 1 (stability-context condition): each row of w_i is made
 *      row-stochastic by a sigmoid on its non-zero entries followed by
 *      normalisation of the row.  The non-zero entries are the three taps of
 *      Key design 2 (tridiagonal w_i: upper-left, up, upper-right); a tap
 *      that falls outside the line is not an entry of w_i, so it is dropped
 *      and the row is normalised over the remaining ones.
 *  a2  The linear recurrence h_i = w_i h_{i-1} + lambda_i (.) x_i (Key
 *      design 1), with h_{-1} = 0, run line by line (Key design 2: lines are
 *      sequential, positions within a line are independent).
 *  a3  Four scan directions, top->bottom, bottom->top, left->right and
 *      right->left (Key design 2; Overall framework).
 *  a4  Local variant: the scan axis is cut into g equal groups, each
 *      propagated on its own, i.e. the state restarts at every group start
 *      (Key design 3).
 *  a5  Compact mode: one 3-tap set per pixel and direction shared by all
 *      channels, with per-channel lambda -- "GSPN-2: Efficient Parallel
 *      Sequence Modeling" (OpenReview response), "Justification for
 *      Channel-Agnostic Propagation" (W kron I(C) with per-channel gains).
 *  a6  The directions are merged by an unweighted sum (the plainest reading
 *      of the "merger" of Key design 2).
 *  a7  Backward: the exact gradient of a1..a6, obtained by running the
 *      recurrence's adjoint from the last line back to the first.
 *
 * Coordinates.  For direction d, line i (scan order) and position j (along
 * the line) the image pixel (r, c) is:
 *     T2B (i, j) -> (i, j)          B2T (i, j) -> (H-1-i, j)
 *     L2R (i, j) -> (j, i)          R2L (i, j) -> (j, W-1-i)
 * Tap k in {0,1,2} of position j reads position j+k-1 of the previous line;
 * the logits of line i's taps are stored at line i's own pixels.
 *
 * Layouts (dense, row-major): x, out, dout, dx: [B,C,H,W];
 * lam, dlam: [D,B,C,H,W]; logits, dlogits: [D,B,Cw,3,H,W] with Cw = 1 in
 * compact mode, else C.  The D axis follows the set bits of dir_mask in the
 * order T2B(1), B2T(2), L2R(4), R2L(8).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t B, C, H, W;
    uint32_t dir_mask;
    int32_t groups;
    int32_t shared; /* 1: one tap set per (b, pixel, direction) for all channels */
} ref_desc;

enum { REF_OK = 0, REF_ERR_ARG = 1, REF_ERR_NOMEM = 2 };

static int ndirs(uint32_t m) { return (int)((m & 1) + ((m >> 1) & 1) + ((m >> 2) & 1) + ((m >> 3) & 1)); }

/* direction of D-axis slot `slot` */
static int dir_of_slot(uint32_t mask, int slot) {
    for (int d = 0; d < 4; ++d)
        if (mask & (1u << d)) {
            if (slot == 0) return d;
            --slot;
        }
    return -1;
}

static int64_t scan_len(int d, int64_t H, int64_t W) { return d < 2 ? H : W; }
static int64_t line_len(int d, int64_t H, int64_t W) { return d < 2 ? W : H; }

/* image offset r*W + c of scan coordinate (i, j) in direction d */
static int64_t pix(int d, int64_t H, int64_t W, int64_t i, int64_t j) {
    switch (d) {
    case 0: return i * W + j;             /* T2B */
    case 1: return (H - 1 - i) * W + j;   /* B2T */
    case 2: return j * W + i;             /* L2R */
    default: return j * W + (W - 1 - i);  /* R2L */
    }
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

static int valid_tap(int64_t j, int k, int64_t N) {
    int64_t q = j + k - 1;
    return q >= 0 && q < N;
}

static int check(const ref_desc* dsc) {
    if (!dsc || dsc->B <= 0 || dsc->C <= 0 || dsc->H <= 0 || dsc->W <= 0) return REF_ERR_ARG;
    if ((dsc->dir_mask & 15u) == 0 || (dsc->dir_mask & ~15u)) return REF_ERR_ARG;
    /* g must divide the scan length of every requested direction */
    if (dsc->groups < 1) return REF_ERR_ARG;
    if ((dsc->dir_mask & 3u) && dsc->H % dsc->groups) return REF_ERR_ARG;
    if ((dsc->dir_mask & 12u) && dsc->W % dsc->groups) return REF_ERR_ARG;
    return REF_OK;
}

/* a1: for one direction and one logit plane set lg ([3][H][W]) fill, per
 * scan coordinate (i, j) and tap k, the sigmoid s, the row sum S and the
 * normalised weight w.  Invalid taps get s = w = 0. */
static void gate_weights(const double* lg, int d, int64_t H, int64_t W, double* s, double* S, double* w) {
    const int64_t L = scan_len(d, H, W), N = line_len(d, H, W), HW = H * W;
    for (int64_t i = 0; i < L; ++i)
        for (int64_t j = 0; j < N; ++j) {
            const int64_t p = pix(d, H, W, i, j), t = i * N + j;
            double sum = 0.0;
            for (int k = 0; k < 3; ++k) {
                double v = valid_tap(j, k, N) ? sigmoid(lg[k * HW + p]) : 0.0;
                s[3 * t + k] = v;
                sum += v;
            }
            S[t] = sum;
            for (int k = 0; k < 3; ++k) w[3 * t + k] = s[3 * t + k] / sum;
        }
}

/* a2 + a4: scan one direction of one plane; h receives every line in scan
 * coordinates ([L][N]). */
static void scan_dir(const double* x, const double* lam, const double* w, int d, int64_t H, int64_t W,
                     int64_t groups, double* h) {
    const int64_t L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / groups;
    for (int64_t i = 0; i < L; ++i)
        for (int64_t j = 0; j < N; ++j) {
            const int64_t p = pix(d, H, W, i, j), t = i * N + j;
            double v = lam[p] * x[p];
            if (i % seg != 0)
                for (int k = 0; k < 3; ++k)
                    if (valid_tap(j, k, N)) v += w[3 * t + k] * h[(i - 1) * N + (j + k - 1)];
            h[t] = v;
        }
}

typedef struct {
    double *s, *S, *w, *h, *a, *an;
} scratch;

static int scratch_alloc(scratch* sc, int64_t HW, int64_t maxN) {
    sc->s = malloc(sizeof(double) * 3 * HW);
    sc->S = malloc(sizeof(double) * HW);
    sc->w = malloc(sizeof(double) * 3 * HW);
    sc->h = malloc(sizeof(double) * HW);
    sc->a = malloc(sizeof(double) * maxN);
    sc->an = malloc(sizeof(double) * maxN);
    return sc->s && sc->S && sc->w && sc->h && sc->a && sc->an;
}

static void scratch_free(scratch* sc) {
    free(sc->s); free(sc->S); free(sc->w); free(sc->h); free(sc->a); free(sc->an);
}

/* Forward: out[b,c] = sum over directions of h^(d) (a6). */
int gspn_ref_fwd(const ref_desc* dsc, const double* x, const double* logits, const double* lam, double* out,
                 int nthreads) {
    int rc = check(dsc);
    if (rc) return rc;
    const int64_t B = dsc->B, C = dsc->C, H = dsc->H, W = dsc->W, HW = H * W;
    const int64_t Cw = dsc->shared ? 1 : C;
    const int D = ndirs(dsc->dir_mask);
    const int64_t maxN = H > W ? H : W;
    int failed = 0;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads) reduction(| : failed)
    {
        scratch sc;
        if (!scratch_alloc(&sc, HW, maxN)) failed = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t pl = 0; pl < B * C; ++pl) {
            if (failed) continue;
            const int64_t b = pl / C, c = pl % C, cw = dsc->shared ? 0 : c;
            double* o = out + pl * HW;
            for (int64_t q = 0; q < HW; ++q) o[q] = 0.0;
            for (int slot = 0; slot < D; ++slot) {
                const int d = dir_of_slot(dsc->dir_mask, slot);
                const double* lg = logits + ((slot * B + b) * Cw + cw) * 3 * HW;
                const double* lm = lam + ((slot * B + b) * C + c) * HW;
                gate_weights(lg, d, H, W, sc.s, sc.S, sc.w);
                scan_dir(x + pl * HW, lm, sc.w, d, H, W, dsc->groups, sc.h);
                const int64_t L = scan_len(d, H, W), N = line_len(d, H, W);
                for (int64_t i = 0; i < L; ++i)
                    for (int64_t j = 0; j < N; ++j) o[pix(d, H, W, i, j)] += sc.h[i * N + j];
            }
        }
        scratch_free(&sc);
    }
    return failed ? REF_ERR_NOMEM : REF_OK;
}

/* Backward (a7).  With a_i = dL/dh_i (total) in scan coordinates:
 *   a_i[j] = dout_i[j] + sum_k w_{i+1}[j-k+1][k] * a_{i+1}[j-k+1]
 * where the carry term is absent when line i+1 starts a group (its h does not
 * read h_i) or i is the last line.  Then, per pixel of line i:
 *   dx   += lam * a          (summed over directions)
 *   dlam  = x * a
 *   dw_k  = a * h_{i-1}[j+k-1]  (valid taps, lines that are not group starts)
 *   dlogit_k = s_k (1 - s_k) / S * (dw_k - sum_m w_m dw_m)
 * which is the chain rule through w_k = s_k / S, s_k = sigmoid(logit_k).
 * In compact mode dlogits are summed over channels. */
int gspn_ref_bwd(const ref_desc* dsc, const double* x, const double* logits, const double* lam, const double* dout,
                 double* dx, double* dlogits, double* dlam, int nthreads) {
    int rc = check(dsc);
    if (rc) return rc;
    const int64_t B = dsc->B, C = dsc->C, H = dsc->H, W = dsc->W, HW = H * W;
    const int64_t Cw = dsc->shared ? 1 : C;
    const int D = ndirs(dsc->dir_mask);
    const int64_t maxN = H > W ? H : W;
    const int64_t nlog = (int64_t)D * B * Cw * 3 * HW;
    if (nthreads < 1) nthreads = 1;
    /* compact mode: one private dlogits accumulator per thread, summed after */
    double* priv = NULL;
    if (dsc->shared) {
        priv = calloc((size_t)nthreads * (size_t)nlog, sizeof(double));
        if (!priv) return REF_ERR_NOMEM;
    } else {
        memset(dlogits, 0, sizeof(double) * (size_t)nlog);
    }
    int failed = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : failed)
    {
        scratch sc;
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double* dlg_base = dsc->shared ? priv + (int64_t)tid * nlog : dlogits;
        if (!scratch_alloc(&sc, HW, maxN)) failed = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t pl = 0; pl < B * C; ++pl) {
            if (failed) continue;
            const int64_t b = pl / C, c = pl % C, cw = dsc->shared ? 0 : c;
            const double* xp = x + pl * HW;
            const double* g = dout + pl * HW;
            double* dxp = dx + pl * HW;
            for (int64_t q = 0; q < HW; ++q) dxp[q] = 0.0;
            for (int slot = 0; slot < D; ++slot) {
                const int d = dir_of_slot(dsc->dir_mask, slot);
                const int64_t L = scan_len(d, H, W), N = line_len(d, H, W), seg = L / dsc->groups;
                const double* lg = logits + ((slot * B + b) * Cw + cw) * 3 * HW;
                const double* lm = lam + ((slot * B + b) * C + c) * HW;
                double* dlm = dlam + ((slot * B + b) * C + c) * HW;
                double* dlg = dlg_base + ((slot * B + b) * Cw + cw) * 3 * HW;
                gate_weights(lg, d, H, W, sc.s, sc.S, sc.w);
                scan_dir(xp, lm, sc.w, d, H, W, dsc->groups, sc.h);
                for (int64_t j = 0; j < N; ++j) sc.an[j] = 0.0;
                for (int64_t i = L - 1; i >= 0; --i) {
                    const int carry = (i + 1 < L) && ((i + 1) % seg != 0);
                    for (int64_t j = 0; j < N; ++j) {
                        double v = g[pix(d, H, W, i, j)];
                        if (carry)
                            for (int k = 0; k < 3; ++k) {
                                const int64_t jj = j - k + 1;
                                if (jj >= 0 && jj < N) v += sc.w[3 * ((i + 1) * N + jj) + k] * sc.an[jj];
                            }
                        sc.a[j] = v;
                    }
                    for (int64_t j = 0; j < N; ++j) {
                        const int64_t p = pix(d, H, W, i, j), t = i * N + j;
                        const double a = sc.a[j];
                        dxp[p] += lm[p] * a;
                        dlm[p] = xp[p] * a;
                        if (i % seg == 0) continue; /* group start: taps unused, zero gradient */
                        double dw[3], tw = 0.0;
                        for (int k = 0; k < 3; ++k) {
                            dw[k] = valid_tap(j, k, N) ? a * sc.h[(i - 1) * N + (j + k - 1)] : 0.0;
                            tw += sc.w[3 * t + k] * dw[k];
                        }
                        for (int k = 0; k < 3; ++k) {
                            if (!valid_tap(j, k, N)) continue;
                            const double s = sc.s[3 * t + k];
                            dlg[k * HW + p] += s * (1.0 - s) / sc.S[t] * (dw[k] - tw);
                        }
                    }
                    double* tmp = sc.an; sc.an = sc.a; sc.a = tmp;
                }
            }
        }
        scratch_free(&sc);
    }
    if (dsc->shared) {
        if (!failed) {
            memset(dlogits, 0, sizeof(double) * (size_t)nlog);
            for (int t = 0; t < nthreads; ++t)
                for (int64_t q = 0; q < nlog; ++q) dlogits[q] += priv[(int64_t)t * nlog + q];
        }
        free(priv);
    }
    return failed ? REF_ERR_NOMEM : REF_OK;
}

int gspn_ref_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
