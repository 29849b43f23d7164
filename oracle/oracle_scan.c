/*
 * Reference oracle for the selective diagonal scan -- TEST INFRASTRUCTURE.
 *
 * Plain, slow, sequential fp64 C.  Only the test-suite, the smoke check and
 * the CPU-baseline leg of the benchmark may build, load or call this file;
 * the product path never does.  It shares no code, header or constant with
 * the CUDA library.
 *
 * What it computes (all citations are to the pages the method is taken from):
 *
 *  - the linear-transition recurrence h_t = A_t h_{t-1} + B_t u_t,
 *    y_t = C_t h_t + D u_t  ("When a Diagonal State Is Not Enough",
 *    sungsoo.github.io, Part 01 "Definition", first display; Part 03,
 *    "Selective SSM and masked linear attention" display);
 *  - discretisation by the step dt: the state transition over one step is
 *    exp(dt * A) (robocikowo.com state-space-model glossary, mechanism item 2;
 *    S4D abstract, "On the Parameterization and Initialization of Diagonal
 *    State Space Models"); the write uses B_t scaled by the step (Euler);
 *  - HybridMamba's state: real coordinates with their own decay (Mamba-1
 *    style) followed by complex coordinates stored as real 2x2
 *    decay-rotation blocks (Mamba-3 style), under Mamba-2-style heads that
 *    share one transition across P channels ("Diagonal Equivalence in State
 *    Space Models: New Insights into Retrieval Rank and Selective Scaling",
 *    kongchang.com, "From MIMO to HybridMamba"; sungsoo.github.io Part 04);
 *  - the two-endpoint write of the exponential-trapezoidal discretisation
 *    (sungsoo.github.io Part 05): the write of step t is
 *        dt_t * ( lam_t * W_t + (1 - lam_t) * A_t W_{t-1} ),  W_t = B_t u_t,
 *    i.e. the trapezoid rule on the integral of exp(A (t - s)) B u over one
 *    step, weighting the right endpoint by lam and the left one by 1 - lam
 *    (lam = 1 gives the Euler write of Mamba-1/2);
 *  - SSD-MIMO routing: u_t has R value rows, B_t is N x R and C_t is O x N
 *    (sungsoo.github.io Part 03 "SISO and MIMO", Part 08 item 3).
 *
 * Per (batch b, head h), with H_{-1} = h0 and W_{-1} = w0 (zero if absent):
 *      gamma_t = lam_t dt_t,  beta_t = (1 - lam_t) dt_t
 *      W_t = B_t u_t                               (N x P)
 *      H_t = A_t (H_{t-1} + beta_t W_{t-1}) + gamma_t W_t
 *      y_t = C_t H_t + D_h u_t                     (O x P; D only when O == R)
 *  A_t = diag(exp(dt_t a_n)) on real rows, and on rotation pair j (rows
 *  n_real+2j = re, n_real+2j+1 = im) the block
 *      exp(dt_t a_j) [[cos phi, -sin phi], [sin phi, cos phi]],  phi = dt_t theta_j,
 *  with a = -exp(A_log) (one value per head, or one per real row / pair).
 *  Real static rows (n_static > 0: the first n_static real rows; HybridMamba
 *  mixes real static, real dynamic and complex dynamic rows, sungsoo.github.io
 *  Part 08 item 3): the transition of such a row is exp(a_n) at every step,
 *  independent of dt_t (read: "static" = not selective); its write is that of
 *  every other row.
 *  Exact zero-order hold (zoh = 1; robocikowo.com glossary item 2 names ZOH as
 *  a discretisation of the continuous system): with the input held constant
 *  over the step, the continuous state x' = lam x + b u (lam = a on a real
 *  row, a + i omega on a pair) moves by exactly
 *      x_t = e^{dt lam} x_{t-1} + ((e^{dt lam} - 1) / lam) b u_t,
 *  so the write W_t of mode m is scaled by Z = dt phi1(mu), mu = dt a + i phi
 *  (phi the step's rotation angle), phi1(mu) = (e^mu - 1) / mu, instead of by
 *  dt.  Only with the Euler form (two_endpoint = 0).
 *  Per-token rotation angles (angle_per_token = 1, the data-dependent angles of
 *  Mamba-3's complex state, sungsoo.github.io Part 05): phi = theta_t[j] is an
 *  input per (batch, token, head, pair) instead of dt_t theta_j, and its
 *  gradient is returned per token.
 *
 * Parity pins that do not go through this file (see tests/): the quadratic
 * masked-attention form, a complex128 recurrence, the LTI Vandermonde
 * convolution, linear attention at a -> 0, the Mamba-2 segment-sum form, the
 * retrieval-rank bound and central finite differences of the gradients.
 *
 * Layouts (all contiguous, row-major, fp64):
 *   x  [B][L][H][R][P]     dt, lam [B][L][H]      A_log [H][n_decay]
 *   theta [H][n_pairs]     D [H]
 *   Bm [B][L][G][R][N]  (B_t[n][r] = Bm[b][t][g][r][n])
 *   Cm [B][L][G][O][N]  (C_t[o][n] = Cm[b][t][g][o][n])
 *   y, dy [B][L][H][O][P]  h0, w0, hT, wT [B][H][N][P]
 * Head h reads group g = h / (H / G).
 */
#include <complex.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ORACLE_MUTANT plants one known mistake (tests only: they check that the
 * pins catch each one).  0 = the oracle as specified. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#define MUT(k) (ORACLE_MUTANT == (k))

typedef struct {
    long batch, seqlen, nheads, headdim, ngroups;
    int n_real, n_pairs, rank_in, rank_out;
    int per_coord_decay; /* 0: one decay per head; 1: one per real row / pair */
    int two_endpoint;    /* 0: lam == 1 (Euler write) */
    int angle_per_token; /* 0: phi = dt_t theta[h][j]; 1: phi = theta[b][t][h][j] */
    int n_static;        /* the first n_static real rows decay by exp(a_n) per step */
    int zoh;             /* 1: exact zero-order-hold write (needs two_endpoint = 0, n_static = 0) */
} oracle_desc;

/* ---- index helpers ---------------------------------------------------- */
#define NST(d) ((long)(d)->n_real + 2L * (d)->n_pairs)
#define NDEC(d) ((d)->per_coord_decay ? (long)(d)->n_real + (d)->n_pairs : 1L)

static long ix_x(const oracle_desc *d, long b, long t, long h, long r, long p) {
    return ((((b * d->seqlen + t) * d->nheads + h) * d->rank_in + r) * d->headdim) + p;
}
static long ix_y(const oracle_desc *d, long b, long t, long h, long o, long p) {
    return ((((b * d->seqlen + t) * d->nheads + h) * d->rank_out + o) * d->headdim) + p;
}
static long ix_bl(const oracle_desc *d, long b, long t, long h) {
    return (b * d->seqlen + t) * d->nheads + h;
}
static long ix_B(const oracle_desc *d, long b, long t, long g, long r, long n) {
    return (((b * d->seqlen + t) * d->ngroups + g) * d->rank_in + r) * NST(d) + n;
}
static long ix_C(const oracle_desc *d, long b, long t, long g, long o, long n) {
    return (((b * d->seqlen + t) * d->ngroups + g) * d->rank_out + o) * NST(d) + n;
}
static long ix_st(const oracle_desc *d, long b, long h, long n, long p) {
    return ((b * d->nheads + h) * NST(d) + n) * d->headdim + p;
}
/* decay index of state row n (real row n, or pair j covering rows n_real+2j, +1) */
static long dec_of_row(const oracle_desc *d, long n) {
    if (!d->per_coord_decay) return 0;
    if (n < d->n_real) return n;
    return d->n_real + (n - d->n_real) / 2;
}

/* One step's transition coefficients for head h:
 *   real row n: e[n] = exp(dt * a_n)
 *   pair j:     e[j] = exp(dt * a_j), c[j] = cos(dt * w_j), s[j] = sin(dt * w_j) */
typedef struct { double *er, *ep, *cp, *sp; } step_coef;

static void make_step(const oracle_desc *d, const double *A_log, const double *theta,
                      long b, long t, long h, double dtv, step_coef *sc) {
    long nd = NDEC(d);
    for (long n = 0; n < d->n_real; ++n) {
        double a = -exp(A_log[h * nd + dec_of_row(d, n)]);
        sc->er[n] = (n < d->n_static && !MUT(10)) ? exp(a) : exp(dtv * a);
    }
    for (long j = 0; j < d->n_pairs; ++j) {
        double a = -exp(A_log[h * nd + dec_of_row(d, d->n_real + 2 * j)]);
        double phi = d->angle_per_token
                         ? theta[((b * d->seqlen + t) * d->nheads + h) * d->n_pairs + j]
                         : dtv * theta[h * d->n_pairs + j];
        sc->ep[j] = exp(dtv * a);
        sc->cp[j] = cos(phi);
        sc->sp[j] = sin(phi);
    }
}

/* phi1(mu) = (e^mu - 1) / mu and its derivative, by their Taylor series near 0 */
static double complex zoh_phi1(double complex mu) {
    if (cabs(mu) < 0.05) {
        double complex s = 0.0, term = 1.0;
        for (int k = 0; k < 14; ++k) {   /* mu^k / (k + 1)! */
            s += term;
            term *= mu / (double)(k + 2);
        }
        return s;
    }
    return (cexp(mu) - 1.0) / mu;
}
static double complex zoh_phi1_d(double complex mu) {
    if (cabs(mu) < 0.05) {
        double complex s = 0.0, term = 0.5;   /* (k + 1) mu^k / (k + 2)! */
        for (int k = 0; k < 14; ++k) {
            s += (double)(k + 1) * term;
            term *= mu / (double)(k + 3);
        }
        return s;
    }
    return (cexp(mu) * (mu - 1.0) + 1.0) / (mu * mu);
}

/* ZOH write coefficient Z_m of every mode m (real rows, then pairs) for one step,
 * and the derivatives of Z_m with respect to dt, a_m and the angle (theta_j for
 * static angles, phi_t for per-token ones). */
typedef struct { double complex *z, *z_dt, *z_a, *z_w; } zoh_coef;

static void make_zoh(const oracle_desc *d, const double *A_log, const double *theta, long b,
                     long t, long h, double dtv, zoh_coef *zc) {
    long nd = NDEC(d);
    for (long m = 0; m < d->n_real + d->n_pairs; ++m) {
        long n0 = m < d->n_real ? m : d->n_real + 2 * (m - d->n_real);
        double a = -exp(A_log[h * nd + dec_of_row(d, n0)]);
        double phi = 0.0, w = 0.0;
        if (m >= d->n_real) {
            long j = m - d->n_real;
            if (d->angle_per_token) {
                phi = theta[((b * d->seqlen + t) * d->nheads + h) * d->n_pairs + j];
            } else {
                w = theta[h * d->n_pairs + j];
                phi = dtv * w;
            }
        }
        double complex mu = dtv * a + I * phi;
        double complex f1 = zoh_phi1(mu), f1d = zoh_phi1_d(mu);
        zc->z[m] = dtv * f1;
        zc->z_a[m] = dtv * dtv * f1d;
        if (m >= d->n_real && d->angle_per_token) {
            zc->z_dt[m] = f1 + dtv * a * f1d;   /* phi does not move with dt */
            zc->z_w[m] = I * dtv * f1d;          /* d/dphi_t */
        } else {
            zc->z_dt[m] = MUT(13) ? f1 : cexp(mu);   /* d/ddt of (e^{dt lam} - 1) / lam */
            zc->z_w[m] = I * dtv * dtv * f1d;    /* d/dtheta_j */
        }
    }
}

/* H += gamma W (Euler / two-endpoint) or H += Z (.) W per mode (ZOH) */
static void add_write(const oracle_desc *d, const zoh_coef *zc, double gamma, const double *W,
                      double *H) {
    long P = d->headdim, NP = NST(d) * P;
    if (!d->zoh) {
        for (long i = 0; i < NP; ++i) H[i] += gamma * W[i];
        return;
    }
    for (long n = 0; n < d->n_real; ++n)
        for (long p = 0; p < P; ++p) H[n * P + p] += creal(zc->z[n]) * W[n * P + p];
    for (long j = 0; j < d->n_pairs; ++j) {
        long re = d->n_real + 2 * j, im = re + 1;
        double zr = creal(zc->z[d->n_real + j]), zi = cimag(zc->z[d->n_real + j]);
        for (long p = 0; p < P; ++p) {
            double wr = W[re * P + p], wi = W[im * P + p];
            H[re * P + p] += zr * wr - zi * wi;
            H[im * P + p] += zi * wr + zr * wi;
        }
    }
}

/* out = A_t * in  (in, out: N x P, may not alias) */
static void apply_transition(const oracle_desc *d, const step_coef *sc, const double *in,
                             double *out) {
    long P = d->headdim;
    for (long n = 0; n < d->n_real; ++n)
        for (long p = 0; p < P; ++p) out[n * P + p] = sc->er[n] * in[n * P + p];
    for (long j = 0; j < d->n_pairs; ++j) {
        long re = d->n_real + 2 * j, im = re + 1;
        double e = sc->ep[j], c = sc->cp[j], s = sc->sp[j];
        for (long p = 0; p < P; ++p) {
            double zr = in[re * P + p], zi = in[im * P + p];
            double sg = MUT(2) ? -s : s;
            out[re * P + p] = e * (c * zr - sg * zi);
            out[im * P + p] = e * (sg * zr + c * zi);
        }
    }
}

/* out = A_t^T * in */
static void apply_transition_T(const oracle_desc *d, const step_coef *sc, const double *in,
                               double *out) {
    long P = d->headdim;
    for (long n = 0; n < d->n_real; ++n)
        for (long p = 0; p < P; ++p) out[n * P + p] = sc->er[n] * in[n * P + p];
    for (long j = 0; j < d->n_pairs; ++j) {
        long re = d->n_real + 2 * j, im = re + 1;
        double e = sc->ep[j], c = sc->cp[j], s = sc->sp[j];
        for (long p = 0; p < P; ++p) {
            double gr = in[re * P + p], gi = in[im * P + p];
            double sg = MUT(8) ? -s : s;
            out[re * P + p] = e * (c * gr + sg * gi);
            out[im * P + p] = e * (-sg * gr + c * gi);
        }
    }
}

/* W = B_t u_t  (N x P) */
static void make_write(const oracle_desc *d, const double *x, const double *Bm, long b, long t,
                       long h, long g, double *W) {
    long N = NST(d), P = d->headdim;
    for (long n = 0; n < N; ++n)
        for (long p = 0; p < P; ++p) {
            double acc = 0.0;
            for (long r = 0; r < d->rank_in; ++r)
                acc += Bm[ix_B(d, b, t, g, MUT(4) ? (d->rank_in - 1 - r) : r, n)] *
                       x[ix_x(d, b, t, h, r, p)];
            W[n * P + p] = acc;
        }
}

static void step_weights(const oracle_desc *d, const double *dt, const double *lam, long b,
                         long t, long h, double *gamma, double *beta, double *lamv) {
    double dv = dt[ix_bl(d, b, t, h)];
    double l = d->two_endpoint ? lam[ix_bl(d, b, t, h)] : 1.0;
    *lamv = l;
    *gamma = l * dv;
    *beta = (1.0 - l) * dv;
}

/* Forward for one (b, h).  Hs (optional) receives H_t for t in [0, L). */
static void fwd_unit(const oracle_desc *d, long b, long h, const double *x, const double *dt,
                     const double *A_log, const double *theta, const double *Bm,
                     const double *Cm, const double *D, const double *lam, const double *h0,
                     const double *w0, double *y, double *hT, double *wT, double *work) {
    long N = NST(d), P = d->headdim, NP = N * P;
    long g = h / (d->nheads / d->ngroups);
    double *H = work, *Wp = H + NP, *W = Wp + NP, *Z = W + NP, *tmp = Z + NP;
    double *coef = tmp + NP;
    step_coef sc = {coef, coef + d->n_real, coef + d->n_real + d->n_pairs,
                    coef + d->n_real + 2 * d->n_pairs};
    long nm = d->n_real + d->n_pairs;
    double complex *zbuf = (double complex *)malloc(sizeof(double complex) * (4 * nm + 1));
    zoh_coef zc = {zbuf, zbuf + nm, zbuf + 2 * nm, zbuf + 3 * nm};
    for (long i = 0; i < NP; ++i) {
        H[i] = h0 ? h0[ix_st(d, b, h, 0, 0) + i] : 0.0;
        Wp[i] = w0 ? w0[ix_st(d, b, h, 0, 0) + i] : 0.0;
    }
    for (long t = 0; t < d->seqlen; ++t) {
        double gamma, beta, lv;
        step_weights(d, dt, lam, b, t, h, &gamma, &beta, &lv);
        make_step(d, A_log, theta, b, t, h, dt[ix_bl(d, b, t, h)], &sc);
        if (d->zoh) make_zoh(d, A_log, theta, b, t, h, dt[ix_bl(d, b, t, h)], &zc);
        make_write(d, x, Bm, b, t, h, g, W);
        for (long i = 0; i < NP; ++i) Z[i] = H[i] + (MUT(1) ? 0.0 : beta) * Wp[i];
        apply_transition(d, &sc, Z, tmp);
        memcpy(H, tmp, sizeof(double) * NP);
        add_write(d, &zc, gamma, W, H);
        for (long o = 0; o < d->rank_out; ++o)
            for (long p = 0; p < P; ++p) {
                double acc = 0.0;
                long gc = MUT(3) ? (h % d->ngroups) : g;
                for (long n = 0; n < N; ++n) acc += Cm[ix_C(d, b, t, gc, o, n)] * H[n * P + p];
                if (d->rank_out == d->rank_in && !MUT(9)) acc += D[h] * x[ix_x(d, b, t, h, o, p)];
                y[ix_y(d, b, t, h, o, p)] = acc;
            }
        memcpy(Wp, W, sizeof(double) * NP);
    }
    if (hT) memcpy(hT + ix_st(d, b, h, 0, 0), H, sizeof(double) * NP);
    if (wT) memcpy(wT + ix_st(d, b, h, 0, 0), Wp, sizeof(double) * NP);
    free(zbuf);
}

static long unit_work_doubles(const oracle_desc *d) {
    return 5 * NST(d) * d->headdim + d->n_real + 3 * d->n_pairs + 8;
}

int oracle_scan_fwd(const oracle_desc *d, const double *x, const double *dt, const double *A_log,
                    const double *theta, const double *Bm, const double *Cm, const double *D,
                    const double *lam, const double *h0, const double *w0, double *y,
                    double *hT, double *wT) {
    if (d->nheads % d->ngroups) return -1;
    long units = d->batch * d->nheads;
    long wd = unit_work_doubles(d);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        double *work = (double *)malloc(sizeof(double) * wd);
        if (!work) {
            err = -2;
            continue;
        }
        fwd_unit(d, u / d->nheads, u % d->nheads, x, dt, A_log, theta, Bm, Cm, D, lam, h0, w0,
                 y, hT, wT, work);
        free(work);
    }
    return err;
}

/* ---- backward ---------------------------------------------------------
 * Hand-written reverse mode of fwd_unit.  Walking t = L-1 .. 0 with
 * G = dL/dH_t (accumulated) and Wbar = gradient reaching W_t from step t+1:
 *   G    += C_t^T dy_t;   dC_t = dy_t H_t^T;   dD += <dy_t, u_t>;  du_t = D dy_t
 *   dW_t  = gamma_t G + Wbar;   dgamma_t = <G, W_t>
 *   Gz    = A_t^T G                              (gradient of Z_t = H_{t-1} + beta_t W_{t-1})
 *   dA_t : real row n   g_rho = sum_p G[n,p] (A_t Z)[n,p]
 *          pair j       g_rho = <G_j, (A_t Z)_j>,  g_phi = <G_j, e R'(phi) Z_j>
 *   dbeta_t = <Gz, W_{t-1}>;   Wbar <- beta_t Gz;   G <- Gz  (= dL/dH_{t-1})
 *   ddt_t = sum a g_rho + sum theta g_phi + lam dgamma + (1 - lam) dbeta
 *   dlam_t = dt_t (dgamma - dbeta);  da += dt_t g_rho;  dtheta += dt_t g_phi
 *   dB_t = dW_t u_t^T;  du_t += B_t^T dW_t
 * At the end dh0 = G and dw0 = Wbar; dA_log = da * a (a = -exp(A_log)).
 * Forward states are re-created per segment from checkpoints every SEG steps.
 */
#define SEG 64

static void bwd_unit(const oracle_desc *d, long b, long h, const double *x, const double *dt,
                     const double *A_log, const double *theta, const double *Bm,
                     const double *Cm, const double *D, const double *lam, const double *h0,
                     const double *w0, const double *dy, double *dx, double *ddt,
                     double *dA_unit, double *dth_unit, double *dtheta, double *dB_head,
                     double *dC_head, double *dD_unit, double *dlam, double *dh0, double *dw0) {
    long N = NST(d), P = d->headdim, NP = N * P, L = d->seqlen, nd = NDEC(d);
    long g = h / (d->nheads / d->ngroups);
    long nseg = (L + SEG - 1) / SEG;
    /* checkpoints: H and W_prev at the start of every segment */
    double *ckH = (double *)calloc((size_t)nseg * NP, sizeof(double));
    double *ckW = (double *)calloc((size_t)nseg * NP, sizeof(double));
    double *segH = (double *)calloc((size_t)(SEG + 1) * NP, sizeof(double)); /* H_{t0-1..} */
    double *segW = (double *)calloc((size_t)(SEG + 1) * NP, sizeof(double)); /* W_{t0-1..} */
    double *G = (double *)calloc(NP, sizeof(double));
    double *Gz = (double *)calloc(NP, sizeof(double));
    double *Wbar = (double *)calloc(NP, sizeof(double));
    double *dW = (double *)calloc(NP, sizeof(double));
    double *Z = (double *)calloc(NP, sizeof(double));
    double *AZ = (double *)calloc(NP, sizeof(double));
    double *coef = (double *)calloc(d->n_real + 3 * d->n_pairs + 4, sizeof(double));
    step_coef sc = {coef, coef + d->n_real, coef + d->n_real + d->n_pairs,
                    coef + d->n_real + 2 * d->n_pairs};
    long nm = d->n_real + d->n_pairs;
    double complex *zbuf = (double complex *)calloc(4 * nm + 1, sizeof(double complex));
    zoh_coef zc = {zbuf, zbuf + nm, zbuf + 2 * nm, zbuf + 3 * nm};
    double *zoh_dphi = (double *)calloc(d->n_pairs + 1, sizeof(double));
    double *H = segH, *W = segW;

    /* pass 1: checkpoints */
    for (long i = 0; i < NP; ++i) {
        H[i] = h0 ? h0[ix_st(d, b, h, 0, 0) + i] : 0.0;
        W[i] = w0 ? w0[ix_st(d, b, h, 0, 0) + i] : 0.0;
    }
    for (long t = 0; t < L; ++t) {
        if (t % SEG == 0) {
            memcpy(ckH + (t / SEG) * NP, H, sizeof(double) * NP);
            memcpy(ckW + (t / SEG) * NP, W, sizeof(double) * NP);
        }
        double gamma, beta, lv;
        step_weights(d, dt, lam, b, t, h, &gamma, &beta, &lv);
        make_step(d, A_log, theta, b, t, h, dt[ix_bl(d, b, t, h)], &sc);
        if (d->zoh) make_zoh(d, A_log, theta, b, t, h, dt[ix_bl(d, b, t, h)], &zc);
        for (long i = 0; i < NP; ++i) Z[i] = H[i] + beta * W[i];
        apply_transition(d, &sc, Z, AZ);
        make_write(d, x, Bm, b, t, h, g, W);
        memcpy(H, AZ, sizeof(double) * NP);
        add_write(d, &zc, gamma, W, H);
    }

    /* pass 2: reverse, one segment at a time */
    for (long sidx = nseg - 1; sidx >= 0; --sidx) {
        long t0 = sidx * SEG, t1 = t0 + SEG < L ? t0 + SEG : L;
        /* re-create H_{t}, W_{t} for t in [t0-1, t1): slot k holds index t0-1+k */
        memcpy(segH, ckH + sidx * NP, sizeof(double) * NP);
        memcpy(segW, ckW + sidx * NP, sizeof(double) * NP);
        for (long t = t0; t < t1; ++t) {
            long k = t - t0 + 1;
            double gamma, beta, lv;
            step_weights(d, dt, lam, b, t, h, &gamma, &beta, &lv);
            make_step(d, A_log, theta, b, t, h, dt[ix_bl(d, b, t, h)], &sc);
            if (d->zoh) make_zoh(d, A_log, theta, b, t, h, dt[ix_bl(d, b, t, h)], &zc);
            for (long i = 0; i < NP; ++i) Z[i] = segH[(k - 1) * NP + i] + beta * segW[(k - 1) * NP + i];
            apply_transition(d, &sc, Z, AZ);
            make_write(d, x, Bm, b, t, h, g, segW + k * NP);
            memcpy(segH + k * NP, AZ, sizeof(double) * NP);
            add_write(d, &zc, gamma, segW + k * NP, segH + k * NP);
        }
        for (long t = t1 - 1; t >= t0; --t) {
            long k = t - t0 + 1;
            const double *Ht = segH + k * NP, *Hm = segH + (k - 1) * NP;
            const double *Wt = segW + k * NP, *Wm = segW + (k - 1) * NP;
            double gamma, beta, lv, dtv = dt[ix_bl(d, b, t, h)];
            step_weights(d, dt, lam, b, t, h, &gamma, &beta, &lv);
            make_step(d, A_log, theta, b, t, h, dtv, &sc);
            /* output y_t = C_t H_t + D u_t */
            for (long n = 0; n < N; ++n)
                for (long p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (long o = 0; o < d->rank_out; ++o)
                        acc += Cm[ix_C(d, b, t, g, o, n)] * dy[ix_y(d, b, t, h, o, p)];
                    G[n * P + p] += acc;
                }
            for (long o = 0; o < d->rank_out; ++o)
                for (long n = 0; n < N; ++n) {
                    double acc = 0.0;
                    for (long p = 0; p < P; ++p) acc += dy[ix_y(d, b, t, h, o, p)] * Ht[n * P + p];
                    dC_head[(((b * L + t) * d->nheads + h) * d->rank_out + o) * N + n] = acc;
                }
            for (long r = 0; r < d->rank_in; ++r)
                for (long p = 0; p < P; ++p) {
                    double v = 0.0;
                    if (d->rank_out == d->rank_in) {
                        v = D[h] * dy[ix_y(d, b, t, h, r, p)];
                        *dD_unit += dy[ix_y(d, b, t, h, r, p)] * x[ix_x(d, b, t, h, r, p)];
                    }
                    dx[ix_x(d, b, t, h, r, p)] = v;
                }
            /* H_t = A_t Z_t + gamma W_t */
            double dgamma = 0.0, ddt_zoh = 0.0;
            if (!d->zoh) {
                for (long i = 0; i < NP; ++i) {
                    dW[i] = gamma * G[i] + Wbar[i];
                    dgamma += G[i] * Wt[i];
                }
            } else {
                /* H_t = A_t H_{t-1} + Z (.) W_t: dW = Z^T G, and the gradient of each
                   mode's Z, g = dL/dRe Z + i dL/dIm Z, reaches dt, a and the angle */
                make_zoh(d, A_log, theta, b, t, h, dtv, &zc);
                for (long n = 0; n < d->n_real; ++n) {
                    double z = creal(zc.z[n]), gz = 0.0;
                    for (long p = 0; p < P; ++p) {
                        dW[n * P + p] = z * G[n * P + p] + Wbar[n * P + p];
                        gz += G[n * P + p] * Wt[n * P + p];
                    }
                    ddt_zoh += gz * creal(zc.z_dt[n]);
                    dA_unit[dec_of_row(d, n)] += gz * creal(zc.z_a[n]);
                }
                for (long j = 0; j < d->n_pairs; ++j) {
                    long m = d->n_real + j, re = d->n_real + 2 * j, im = re + 1;
                    double zr = creal(zc.z[m]), zi = cimag(zc.z[m]), gr = 0.0, gi = 0.0;
                    for (long p = 0; p < P; ++p) {
                        double Gr = G[re * P + p], Gi = G[im * P + p];
                        double wr = Wt[re * P + p], wi = Wt[im * P + p];
                        double zt = MUT(14) ? -zi : zi;   /* the mutant applies Z, not Z^T */
                        dW[re * P + p] = zr * Gr + zt * Gi + Wbar[re * P + p];
                        dW[im * P + p] = -zt * Gr + zr * Gi + Wbar[im * P + p];
                        gr += Gr * wr + Gi * wi;
                        gi += -Gr * wi + Gi * wr;
                    }
                    ddt_zoh += gr * creal(zc.z_dt[m]) + gi * cimag(zc.z_dt[m]);
                    dA_unit[dec_of_row(d, re)] += gr * creal(zc.z_a[m]) + gi * cimag(zc.z_a[m]);
                    double gw = gr * creal(zc.z_w[m]) + gi * cimag(zc.z_w[m]);
                    if (d->angle_per_token)
                        zoh_dphi[j] = gw;
                    else
                        dth_unit[j] += gw;
                }
            }
            for (long i = 0; i < NP; ++i) Z[i] = Hm[i] + beta * Wm[i];
            apply_transition(d, &sc, Z, AZ);
            apply_transition_T(d, &sc, G, Gz);
            double ddt_acc = 0.0;
            for (long n = 0; n < d->n_real; ++n) {
                double grho = 0.0;
                for (long p = 0; p < P; ++p) grho += G[n * P + p] * AZ[n * P + p];
                double a = -exp(A_log[h * nd + dec_of_row(d, n)]);
                if (n < d->n_static) {
                    /* static row: log-transition a_n, independent of the step */
                    dA_unit[dec_of_row(d, n)] += (MUT(11) ? dtv : 1.0) * grho;
                } else {
                    ddt_acc += a * grho;
                    dA_unit[dec_of_row(d, n)] += dtv * grho;
                }
            }
            for (long j = 0; j < d->n_pairs; ++j) {
                long re = d->n_real + 2 * j, im = re + 1;
                double e = sc.ep[j], c = sc.cp[j], s = sc.sp[j];
                double grho = 0.0, gphi = 0.0;
                for (long p = 0; p < P; ++p) {
                    double zr = Z[re * P + p], zi = Z[im * P + p];
                    double gr = G[re * P + p], gi = G[im * P + p];
                    grho += gr * AZ[re * P + p] + gi * AZ[im * P + p];
                    /* d/dphi of e R(phi) z = e [[-s, -c], [c, -s]] z */
                    gphi += gr * e * (-s * zr - c * zi) + gi * e * (c * zr - s * zi);
                }
                long di = dec_of_row(d, re);
                double a = -exp(A_log[h * nd + di]);
                ddt_acc += a * grho;
                dA_unit[di] += dtv * grho;
                if (d->angle_per_token) {
                    /* phi is an input of its own: its gradient, per token */
                    dtheta[((b * L + t) * d->nheads + h) * d->n_pairs + j] =
                        (MUT(12) ? -gphi : gphi) + (d->zoh ? zoh_dphi[j] : 0.0);
                } else {
                    double w = theta[h * d->n_pairs + j];
                    ddt_acc += w * gphi;
                    dth_unit[j] += (MUT(5) ? -dtv : dtv) * gphi;
                }
            }
            double dbeta = 0.0;
            for (long i = 0; i < NP; ++i) dbeta += Gz[i] * (MUT(6) ? Wt[i] : Wm[i]);
            ddt_acc += (MUT(7) ? 0.0 : lv * dgamma) + (1.0 - lv) * dbeta + ddt_zoh;
            ddt[ix_bl(d, b, t, h)] = ddt_acc;
            if (dlam) dlam[ix_bl(d, b, t, h)] = d->two_endpoint ? dtv * (dgamma - dbeta) : 0.0;
            /* W_t = B_t u_t */
            for (long r = 0; r < d->rank_in; ++r) {
                for (long n = 0; n < N; ++n) {
                    double acc = 0.0;
                    for (long p = 0; p < P; ++p) acc += dW[n * P + p] * x[ix_x(d, b, t, h, r, p)];
                    dB_head[(((b * L + t) * d->nheads + h) * d->rank_in + r) * N + n] = acc;
                }
                for (long p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (long n = 0; n < N; ++n) acc += Bm[ix_B(d, b, t, g, r, n)] * dW[n * P + p];
                    dx[ix_x(d, b, t, h, r, p)] += acc;
                }
            }
            for (long i = 0; i < NP; ++i) {
                Wbar[i] = beta * Gz[i];
                G[i] = Gz[i];
            }
        }
    }
    if (dh0) memcpy(dh0 + ix_st(d, b, h, 0, 0), G, sizeof(double) * NP);
    if (dw0) memcpy(dw0 + ix_st(d, b, h, 0, 0), Wbar, sizeof(double) * NP);
    free(ckH); free(ckW); free(segH); free(segW); free(G); free(Gz); free(Wbar);
    free(dW); free(Z); free(AZ); free(coef); free(zbuf); free(zoh_dphi);
}

int oracle_scan_bwd(const oracle_desc *d, const double *x, const double *dt, const double *A_log,
                    const double *theta, const double *Bm, const double *Cm, const double *D,
                    const double *lam, const double *h0, const double *w0, const double *dy,
                    double *dx, double *ddt, double *dA_log, double *dtheta, double *dBm,
                    double *dCm, double *dD, double *dlam, double *dh0, double *dw0) {
    if (d->nheads % d->ngroups) return -1;
    long Bt = d->batch, H = d->nheads, L = d->seqlen, N = NST(d), nd = NDEC(d);
    long R = d->rank_in, O = d->rank_out, G = d->ngroups, hpg = H / G;
    long units = Bt * H;
    double *dA_u = (double *)calloc((size_t)units * nd, sizeof(double));
    double *dth_u = (double *)calloc((size_t)units * (d->n_pairs + 1), sizeof(double));
    double *dD_u = (double *)calloc((size_t)units, sizeof(double));
    double *dBh = (double *)calloc((size_t)Bt * L * H * R * N, sizeof(double));
    double *dCh = (double *)calloc((size_t)Bt * L * H * O * N, sizeof(double));
    if (!dA_u || !dth_u || !dD_u || !dBh || !dCh) {
        free(dA_u); free(dth_u); free(dD_u); free(dBh); free(dCh);
        return -2;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        bwd_unit(d, u / H, u % H, x, dt, A_log, theta, Bm, Cm, D, lam, h0, w0, dy, dx, ddt,
                 dA_u + u * nd, dth_u + u * (d->n_pairs + 1), dtheta, dBh, dCh, dD_u + u, dlam,
                 dh0, dw0);
    }
    /* reductions in a fixed order: over batch for the per-head parameters,
       over the heads of a group for the shared B and C */
    for (long h = 0; h < H; ++h) {
        for (long k = 0; k < nd; ++k) {
            double acc = 0.0;
            for (long b = 0; b < Bt; ++b) acc += dA_u[(b * H + h) * nd + k];
            dA_log[h * nd + k] = acc * (-exp(A_log[h * nd + k]));
        }
        for (long j = 0; j < d->n_pairs && !d->angle_per_token; ++j) {
            double acc = 0.0;
            for (long b = 0; b < Bt; ++b) acc += dth_u[(b * H + h) * (d->n_pairs + 1) + j];
            dtheta[h * d->n_pairs + j] = acc;
        }
        double acc = 0.0;
        for (long b = 0; b < Bt; ++b) acc += dD_u[b * H + h];
        dD[h] = acc;
    }
    for (long b = 0; b < Bt; ++b)
        for (long t = 0; t < L; ++t)
            for (long gi = 0; gi < G; ++gi) {
                for (long r = 0; r < R; ++r)
                    for (long n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (long hh = gi * hpg; hh < (gi + 1) * hpg; ++hh)
                            acc += dBh[(((b * L + t) * H + hh) * R + r) * N + n];
                        dBm[ix_B(d, b, t, gi, r, n)] = acc;
                    }
                for (long o = 0; o < O; ++o)
                    for (long n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (long hh = gi * hpg; hh < (gi + 1) * hpg; ++hh)
                            acc += dCh[(((b * L + t) * H + hh) * O + o) * N + n];
                        dCm[ix_C(d, b, t, gi, o, n)] = acc;
                    }
            }
    free(dA_u); free(dth_u); free(dD_u); free(dBh); free(dCh);
    return 0;
}
