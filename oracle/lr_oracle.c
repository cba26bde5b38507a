/*
 * lr_oracle.c -- plain, sequential, fp64 CPU oracle for the fused linear-recurrence scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file:
 * only the tests, the package smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or helper with the CUDA library; the two meet only at the seeded input
 * generators, which hold none of the method's arithmetic.
 *
 * What it computes (all in double precision, one plain loop over time per independent unit, the
 * whole state trajectory kept in memory for the backward pass):
 *
 *   The recurrence  h_t = a_t (.) h_{t-1} + b_t,  y_t = readout(h_t),  h_{-1} = 0,
 *   run over the whole sequence -- "mlx-recurrence" (Apple Developer Forums thread 840535),
 *   opening paragraphs; the same recurrence written as h_t = abar_t h_{t-1} + bbar_t in the
 *   K-Search / mlx-mamba blog post (techtrendfeed repost), paragraph after Table 1.
 *
 *   Four kinds, as listed under "Current kernels" in the mlx-recurrence post:
 *     rglru_scan   real diagonal, state [B, D]
 *     rotlru_scan  complex diagonal with a magnitude gate and a per-step rotation of
 *                  interleaved channel pairs, state [B, D]
 *     ssd_scan     head-wise selective scan, state [B, H, Dh, N]
 *     gla_scan     scalar forget gate and outer-product write, state [B, H, Dh, Dh]
 *   plus the time-varying S6 selective scan with ZOH or bilinear discretisation from
 *   "lrnnx: A library for Linear RNNs" (ai.info summary), Key Contributions 2 and 3.
 *
 * Readings taken where the pages are silent (each one is listed in the design notes):
 *   - initial state is zero; the readout uses h_t after the step-t update;
 *   - rglru / rotlru read out the state itself (y_t = h_t);
 *   - rotlru: lambda_t = mag_k * g_t[k] * exp(i theta_k), one fixed angle per pair;
 *   - ZOH is the exact zero-order hold: abar = exp(dt A), beta = (exp(dt A) - 1) / A;
 *     bilinear is Tustin: abar = (1 + dt A/2) / (1 - dt A/2), beta = dt / (1 - dt A/2);
 *   - S6 readout: y = (sum_n C_t[n] h_t[n] + D x_t) * silu(z_t); SSD the same per (p) with
 *     B, C shared by the heads of a group and an optional z gate; GLA: o_t = S_t^T q_t.
 *
 * Checkpoints: every *_fwd may also return the state after k*S steps for k = 0..ceil(L/S)-1
 * (slot 0 is the initial state) -- the segment checkpoints of the mlx-recurrence post's
 * "segment checkpointing with recomputation during the backward pass".
 *
 * Initial and final state (decode and continuation): every *_fwd takes an optional initial state
 * h0 (NULL = zero) and optionally returns the state after the last step in hL, both in the kind's
 * state layout (rglru, rotlru [B, D]; S6 [B, D, N]; SSD [B, H, P, N]; GLA [B, H, K, V]).  Running
 * L1 steps and then L2 steps from the returned state is the same recurrence as L1 + L2 steps.
 *
 * Layouts are row-major, last index contiguous, token-major:
 *   per-token tensors [B, L, ...]; parameters as documented per function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_DISC_NONE = 0, ORC_DISC_ZOH = 1, ORC_DISC_BILINEAR = 2, ORC_DISC_DIRAC = 3, ORC_DISC_ZOH_EULER = 4 };

static int g_threads = 0;

/* Number of OpenMP threads the oracle uses (0 = OpenMP's default). */
void orc_set_threads(int n) { g_threads = n; }

int orc_get_threads(void)
{
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

#ifdef _OPENMP
#define ORC_NT (g_threads > 0 ? g_threads : omp_get_max_threads())
#endif

static double sigm(double z) { return 1.0 / (1.0 + exp(-z)); }

static void *xcalloc(size_t n, size_t sz)
{
    void *p = calloc(n ? n : 1, sz);
    if (!p) abort();
    return p;
}

/* ------------------------------------------------------------------------------------------ */
/* Discretisation (lrnnx summary, Key Contributions 2-3, which name ZOH, bilinear, dirac and    */
/* asynchronous discretisation without defining them):                                         */
/*   ZOH        abar = e^{dt A}, beta = (e^{dt A} - 1) / A   (exact zero-order hold)           */
/*   bilinear   abar = (1 + dt A/2) / (1 - dt A/2), beta = dt / (1 - dt A/2)   (Tustin)         */
/*   dirac      abar = e^{dt A}, beta = 1   (the input an impulse at the sample: it enters the  */
/*              state undamped)                                                                */
/*   ZOH-Euler  abar = e^{dt A}, beta = dt  (zero-order hold for A, Euler for B: the form the   */
/*              selective-scan kernels the lrnnx kernels derive from use)                       */
/* ------------------------------------------------------------------------------------------ */

/* abar and beta for one (dt, A) pair.  beta multiplies B*x in the state update. */
static void discretise(int disc, double dt, double A, double *abar, double *beta)
{
    if (disc == ORC_DISC_ZOH) {
        double u = dt * A;
        *abar = exp(u);
        *beta = (A != 0.0) ? expm1(u) / A : dt;        /* limit A -> 0: beta -> dt */
    } else if (disc == ORC_DISC_DIRAC) {
        *abar = exp(dt * A);
        *beta = 1.0;
    } else if (disc == ORC_DISC_ZOH_EULER) {
        *abar = exp(dt * A);
        *beta = dt;
    } else {                                             /* bilinear (Tustin)        */
        double v = 1.0 - 0.5 * dt * A;
        *abar = (1.0 + 0.5 * dt * A) / v;
        *beta = dt / v;
    }
}

/* Partial derivatives of abar and beta with respect to dt and A. */
static void discretise_grad(int disc, double dt, double A, double *da_ddt, double *da_dA,
                            double *db_ddt, double *db_dA)
{
    if (disc == ORC_DISC_ZOH) {
        double ab = exp(dt * A);
        double be = (A != 0.0) ? expm1(dt * A) / A : dt;
        *da_ddt = A * ab;
        *da_dA = dt * ab;
        *db_ddt = ab;
        *db_dA = (A != 0.0) ? (dt * ab - be) / A : 0.5 * dt * dt;
    } else if (disc == ORC_DISC_DIRAC || disc == ORC_DISC_ZOH_EULER) {
        double ab = exp(dt * A);
        *da_ddt = A * ab;
        *da_dA = dt * ab;
        *db_ddt = disc == ORC_DISC_ZOH_EULER ? 1.0 : 0.0;
        *db_dA = 0.0;
    } else {
        double v = 1.0 - 0.5 * dt * A;
        double v2 = v * v;
        *da_ddt = A / v2;
        *da_dA = dt / v2;
        *db_ddt = 1.0 / v + 0.5 * dt * A / v2;
        *db_dA = 0.5 * dt * dt / v2;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* rglru_scan: real diagonal recurrence, state [B, D] (mlx-recurrence post, "Current kernels"). */
/*   h_t = a_t h_{t-1} + b_t,   y_t = h_t.   a, b, y: [B, L, D].                               */
/* ------------------------------------------------------------------------------------------ */

void orc_rglru_fwd(int64_t B, int64_t L, int64_t D, const double *a, const double *b, double *y,
                   int64_t S, double *ck, const double *h0, double *hL)
{
#pragma omp parallel for collapse(2) schedule(static) num_threads(ORC_NT)
    for (int64_t bi = 0; bi < B; ++bi)
        for (int64_t d = 0; d < D; ++d) {
            double h = h0 ? h0[bi * D + d] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                if (ck && S > 0 && t % S == 0) ck[((t / S) * B + bi) * D + d] = h;
                int64_t i = (bi * L + t) * D + d;
                h = a[i] * h + b[i];
                y[i] = h;
            }
            if (hL) hL[bi * D + d] = h;
        }
}

/* Backward by the adjoint recurrence G_t = dy_t + a_{t+1} G_{t+1}:
 *   db_t = G_t,  da_t = G_t h_{t-1}. */
void orc_rglru_bwd(int64_t B, int64_t L, int64_t D, const double *a, const double *b,
                   const double *dy, double *da, double *db)
{
#pragma omp parallel num_threads(ORC_NT)
    {
        double *hs = (double *)xcalloc((size_t)L, sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t d = 0; d < D; ++d) {
                double h = 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    int64_t i = (bi * L + t) * D + d;
                    h = a[i] * h + b[i];
                    hs[t] = h;
                }
                double Gn = 0.0, an = 0.0;          /* G_{t+1}, a_{t+1} */
                for (int64_t t = L - 1; t >= 0; --t) {
                    int64_t i = (bi * L + t) * D + d;
                    double G = dy[i] + an * Gn;
                    db[i] = G;
                    da[i] = G * (t > 0 ? hs[t - 1] : 0.0);
                    Gn = G;
                    an = a[i];
                }
            }
        free(hs);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* rotlru_scan: complex diagonal, magnitude gate, per-step rotation of interleaved channel     */
/* pairs (mlx-recurrence post, "Current kernels").                                             */
/*   pair k = channels (2k, 2k+1) = (re, im);  m_t = mag_k g_t[k];                             */
/*   lambda_t = m_t (cos theta_k + i sin theta_k);  h_t = lambda_t h_{t-1} + b_t;  y_t = h_t.  */
/*   b, y: [B, L, D] interleaved; g: [B, L, D/2]; mag, theta: [D/2].                           */
/* ------------------------------------------------------------------------------------------ */

void orc_rotlru_fwd(int64_t B, int64_t L, int64_t D, const double *b, const double *g,
                    const double *mag, const double *theta, double *y, int64_t S, double *ck,
                    const double *h0, double *hL)
{
    int64_t K = D / 2;
#pragma omp parallel for collapse(2) schedule(static) num_threads(ORC_NT)
    for (int64_t bi = 0; bi < B; ++bi)
        for (int64_t k = 0; k < K; ++k) {
            double c = cos(theta[k]), s = sin(theta[k]);
            double hr = h0 ? h0[bi * D + 2 * k] : 0.0, hi = h0 ? h0[bi * D + 2 * k + 1] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                if (ck && S > 0 && t % S == 0) {
                    ck[((t / S) * B + bi) * D + 2 * k] = hr;
                    ck[((t / S) * B + bi) * D + 2 * k + 1] = hi;
                }
                double m = mag[k] * g[(bi * L + t) * K + k];
                double lr = m * c, li = m * s;
                int64_t i = (bi * L + t) * D + 2 * k;
                double nr = lr * hr - li * hi + b[i];
                double ni = lr * hi + li * hr + b[i + 1];
                hr = nr;
                hi = ni;
                y[i] = hr;
                y[i + 1] = hi;
            }
            if (hL) {
                hL[bi * D + 2 * k] = hr;
                hL[bi * D + 2 * k + 1] = hi;
            }
        }
}

/* Backward with the complex cotangent G = dl/dRe + i dl/dIm:
 *   G_t = dy_t + conj(lambda_{t+1}) G_{t+1},  db_t = G_t,
 *   dlambda_t = G_t conj(h_{t-1}),  dl/dm_t = Re(dlambda_t e^{-i theta}),
 *   dg_t = mag dl/dm_t,  dmag = sum_{b,t} g_t dl/dm_t,  dtheta = sum_{b,t} m_t Im(dlambda_t e^{-i theta}). */
void orc_rotlru_bwd(int64_t B, int64_t L, int64_t D, const double *b, const double *g,
                    const double *mag, const double *theta, const double *dy, double *db,
                    double *dg, double *dmag, double *dtheta)
{
    int64_t K = D / 2;
#pragma omp parallel num_threads(ORC_NT)
    {
        double *hs = (double *)xcalloc((size_t)(2 * L), sizeof(double));
#pragma omp for schedule(static)
        for (int64_t k = 0; k < K; ++k) {
            double c = cos(theta[k]), s = sin(theta[k]);
            double sum_mag = 0.0, sum_th = 0.0;
            for (int64_t bi = 0; bi < B; ++bi) {
                double hr = 0.0, hi = 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    double m = mag[k] * g[(bi * L + t) * K + k];
                    int64_t i = (bi * L + t) * D + 2 * k;
                    double nr = m * c * hr - m * s * hi + b[i];
                    double ni = m * c * hi + m * s * hr + b[i + 1];
                    hr = nr;
                    hi = ni;
                    hs[2 * t] = hr;
                    hs[2 * t + 1] = hi;
                }
                double Gr_n = 0.0, Gi_n = 0.0, lr_n = 0.0, li_n = 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {
                    int64_t i = (bi * L + t) * D + 2 * k;
                    /* conj(lambda_{t+1}) * G_{t+1} */
                    double Gr = dy[i] + (lr_n * Gr_n + li_n * Gi_n);
                    double Gi = dy[i + 1] + (lr_n * Gi_n - li_n * Gr_n);
                    db[i] = Gr;
                    db[i + 1] = Gi;
                    double pr = t > 0 ? hs[2 * (t - 1)] : 0.0;
                    double pi = t > 0 ? hs[2 * (t - 1) + 1] : 0.0;
                    /* dlambda = G * conj(h_{t-1}) */
                    double dlr = Gr * pr + Gi * pi;
                    double dli = Gi * pr - Gr * pi;
                    double dm = dlr * c + dli * s;
                    double gt = g[(bi * L + t) * K + k];
                    double m = mag[k] * gt;
                    dg[(bi * L + t) * K + k] = mag[k] * dm;
                    sum_mag += gt * dm;
                    sum_th += m * (dli * c - dlr * s);
                    Gr_n = Gr;
                    Gi_n = Gi;
                    lr_n = m * c;
                    li_n = m * s;
                }
            }
            dmag[k] = sum_mag;
            dtheta[k] = sum_th;
        }
        free(hs);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* S6: time-varying selective scan (lrnnx summary, Key Contributions 3; Methodology).          */
/*   per (b, d, n): abar, beta = discretise(dt_t[b,t,d], A[d,n]);                              */
/*   h_t[n] = abar h_{t-1}[n] + beta B_t[n] x_t;   s_t = sum_n C_t[n] h_t[n] + D_d x_t;          */
/*   y_t = s_t * silu(z_t)   (y_t = s_t when z is NULL).                                       */
/*   x, dt, z, y: [B, L, D];  A: [D, N];  Bm, Cm: [B, L, N];  Dskip: [D] (NULL = no skip).     */
/*   checkpoints ck: [nseg, B, D, N].                                                          */
/* ------------------------------------------------------------------------------------------ */

void orc_s6_fwd(int64_t B, int64_t L, int64_t D, int64_t N, int disc, const double *x,
                const double *dt, const double *A, const double *Bm, const double *Cm,
                const double *Dskip, const double *z, double *y, int64_t S, double *ck,
                const double *h0, double *hL)
{
#pragma omp parallel num_threads(ORC_NT)
    {
        double *h = (double *)xcalloc((size_t)N, sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t d = 0; d < D; ++d) {
                for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[(bi * D + d) * N + n] : 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    if (ck && S > 0 && t % S == 0)
                        for (int64_t n = 0; n < N; ++n)
                            ck[(((t / S) * B + bi) * D + d) * N + n] = h[n];
                    int64_t i = (bi * L + t) * D + d;
                    double xv = x[i], s = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        double ab, be;
                        discretise(disc, dt[i], A[d * N + n], &ab, &be);
                        h[n] = ab * h[n] + be * Bm[(bi * L + t) * N + n] * xv;
                        s += Cm[(bi * L + t) * N + n] * h[n];
                    }
                    if (Dskip) s += Dskip[d] * xv;
                    y[i] = z ? s * z[i] * sigm(z[i]) : s;
                }
                if (hL)
                    for (int64_t n = 0; n < N; ++n) hL[(bi * D + d) * N + n] = h[n];
            }
        free(h);
    }
}

/* Backward (adjoint G_t[n] = ds_t C_t[n] + abar_{t+1} G_{t+1}[n], ds = dy * silu(z)):
 *   dC_t[n] = sum_d ds_t h_t[n];   dB_t[n] = sum_d G_t beta x_t;
 *   dx_t = ds_t D + sum_n G_t beta B_t[n];   dD = sum_{b,t} ds_t x_t;
 *   dabar = G_t h_{t-1}, dbeta = G_t B_t[n] x_t, chained through the discretisation into
 *   d(dt)_t = sum_n (...)  and  dA[d,n] = sum_{b,t} (...);
 *   dz = dy s sigma(z) (1 + z (1 - sigma(z))).
 * dA, dBm, dCm, dDskip are written (not accumulated).  Any of dz, dDskip may be NULL. */
void orc_s6_bwd(int64_t B, int64_t L, int64_t D, int64_t N, int disc, const double *x,
                const double *dt, const double *A, const double *Bm, const double *Cm,
                const double *Dskip, const double *z, const double *dy, double *dx, double *ddt,
                double *dA, double *dBm, double *dCm, double *dDskip, double *dz)
{
    double *dA_part = (double *)xcalloc((size_t)(B * D * N), sizeof(double));
    double *dD_part = (double *)xcalloc((size_t)(B * D), sizeof(double));
    memset(dBm, 0, sizeof(double) * (size_t)(B * L * N));
    memset(dCm, 0, sizeof(double) * (size_t)(B * L * N));
#pragma omp parallel num_threads(ORC_NT)
    {
        double *hs = (double *)xcalloc((size_t)(L * N), sizeof(double));
        double *G = (double *)xcalloc((size_t)N, sizeof(double));
        double *an = (double *)xcalloc((size_t)N, sizeof(double));
#pragma omp for schedule(static)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t d = 0; d < D; ++d) {
                /* forward, keeping the whole trajectory */
                for (int64_t t = 0; t < L; ++t) {
                    int64_t i = (bi * L + t) * D + d;
                    for (int64_t n = 0; n < N; ++n) {
                        double ab, be;
                        discretise(disc, dt[i], A[d * N + n], &ab, &be);
                        double hp = t > 0 ? hs[(t - 1) * N + n] : 0.0;
                        hs[t * N + n] = ab * hp + be * Bm[(bi * L + t) * N + n] * x[i];
                    }
                }
                for (int64_t n = 0; n < N; ++n) { G[n] = 0.0; an[n] = 0.0; }
                double sumD = 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {
                    int64_t i = (bi * L + t) * D + d;
                    double xv = x[i];
                    double s = 0.0;
                    for (int64_t n = 0; n < N; ++n) s += Cm[(bi * L + t) * N + n] * hs[t * N + n];
                    if (Dskip) s += Dskip[d] * xv;
                    double ds = dy[i];
                    if (z) {
                        double sg = sigm(z[i]);
                        ds = dy[i] * z[i] * sg;
                        if (dz) dz[i] = dy[i] * s * sg * (1.0 + z[i] * (1.0 - sg));
                    }
                    double dxv = Dskip ? ds * Dskip[d] : 0.0;
                    sumD += ds * xv;
                    double ddt_t = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        double ab, be, a_dt, a_A, b_dt, b_A;
                        double An = A[d * N + n];
                        discretise(disc, dt[i], An, &ab, &be);
                        discretise_grad(disc, dt[i], An, &a_dt, &a_A, &b_dt, &b_A);
                        double Bv = Bm[(bi * L + t) * N + n], Cv = Cm[(bi * L + t) * N + n];
                        double Gt = ds * Cv + an[n] * G[n];
                        double hp = t > 0 ? hs[(t - 1) * N + n] : 0.0;
                        dCm[(bi * L + t) * N + n] += ds * hs[t * N + n];
                        dBm[(bi * L + t) * N + n] += Gt * be * xv;
                        dxv += Gt * be * Bv;
                        double dab = Gt * hp;
                        double dbe = Gt * Bv * xv;
                        ddt_t += dab * a_dt + dbe * b_dt;
                        dA_part[(bi * D + d) * N + n] += dab * a_A + dbe * b_A;
                        G[n] = Gt;
                        an[n] = ab;
                    }
                    dx[i] = dxv;
                    ddt[i] = ddt_t;
                }
                dD_part[bi * D + d] = sumD;
            }
        free(hs);
        free(G);
        free(an);
    }
    for (int64_t d = 0; d < D; ++d) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t bi = 0; bi < B; ++bi) acc += dA_part[(bi * D + d) * N + n];
            dA[d * N + n] = acc;
        }
        if (dDskip) {
            double acc = 0.0;
            for (int64_t bi = 0; bi < B; ++bi) acc += dD_part[bi * D + d];
            dDskip[d] = acc;
        }
    }
    free(dA_part);
    free(dD_part);
}

/* ------------------------------------------------------------------------------------------ */
/* SSD: head-wise selective scan, state [B, H, P, N] (mlx-recurrence post, "ssd_scan").        */
/*   per (b, h): abar_t, beta_t = discretise(dt[b,t,h], A[h])  (scalars per step and head);    */
/*   h_t[p,n] = abar_t h_{t-1}[p,n] + beta_t x_t[p] B_t[n];                                    */
/*   y_t[p] = sum_n C_t[n] h_t[p,n] + D_h x_t[p]   (times silu(z_t[p]) when z is given).        */
/*   x, z, y: [B, L, H, P];  dt: [B, L, H];  A, Dskip: [H];  Bm, Cm: [B, L, G, N], head h      */
/*   reads group h / (H / G).  checkpoints ck: [nseg, B, H, P, N].                             */
/* ------------------------------------------------------------------------------------------ */

void orc_ssd_fwd(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t Gn, int disc,
                 const double *x, const double *dt, const double *A, const double *Bm,
                 const double *Cm, const double *Dskip, const double *z, double *y, int64_t S,
                 double *ck, const double *h0, double *hL)
{
    int64_t hpg = H / Gn;
#pragma omp parallel num_threads(ORC_NT)
    {
        double *h = (double *)xcalloc((size_t)(P * N), sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t hh = 0; hh < H; ++hh) {
                int64_t gi = hh / hpg;
                if (h0)
                    memcpy(h, h0 + (bi * H + hh) * P * N, sizeof(double) * (size_t)(P * N));
                else
                    memset(h, 0, sizeof(double) * (size_t)(P * N));
                for (int64_t t = 0; t < L; ++t) {
                    if (ck && S > 0 && t % S == 0)
                        memcpy(ck + (((t / S) * B + bi) * H + hh) * P * N, h,
                               sizeof(double) * (size_t)(P * N));
                    double ab, be;
                    discretise(disc, dt[(bi * L + t) * H + hh], A[hh], &ab, &be);
                    const double *xt = x + ((bi * L + t) * H + hh) * P;
                    const double *Bt = Bm + ((bi * L + t) * Gn + gi) * N;
                    const double *Ct = Cm + ((bi * L + t) * Gn + gi) * N;
                    for (int64_t p = 0; p < P; ++p) {
                        double s = 0.0;
                        for (int64_t n = 0; n < N; ++n) {
                            h[p * N + n] = ab * h[p * N + n] + be * xt[p] * Bt[n];
                            s += Ct[n] * h[p * N + n];
                        }
                        if (Dskip) s += Dskip[hh] * xt[p];
                        int64_t i = ((bi * L + t) * H + hh) * P + p;
                        y[i] = z ? s * z[i] * sigm(z[i]) : s;
                    }
                }
                if (hL) memcpy(hL + (bi * H + hh) * P * N, h, sizeof(double) * (size_t)(P * N));
            }
        free(h);
    }
}

/* Backward (adjoint G_t[p,n] = ds_t[p] C_t[n] + abar_{t+1} G_{t+1}[p,n]):
 *   dC_t[n] = sum_{heads in group, p} ds_t[p] h_t[p,n];  dB_t[n] = sum_{heads, p} G beta x_t[p];
 *   dx_t[p] = ds_t[p] D + sum_n G beta B_t[n];  dabar_t = sum G h_{t-1};  dbeta_t = sum G x B;
 *   d(dt)_t and dA_h through the discretisation;  dD_h = sum_{b,t,p} ds x. */
void orc_ssd_bwd(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t Gn, int disc,
                 const double *x, const double *dt, const double *A, const double *Bm,
                 const double *Cm, const double *Dskip, const double *z, const double *dy,
                 double *dx, double *ddt, double *dA, double *dBm, double *dCm, double *dDskip,
                 double *dz)
{
    int64_t hpg = H / Gn;
    int64_t U = B * H;
    double *dB_part = (double *)xcalloc((size_t)(U * L * N), sizeof(double));
    double *dC_part = (double *)xcalloc((size_t)(U * L * N), sizeof(double));
    double *dA_part = (double *)xcalloc((size_t)U, sizeof(double));
    double *dD_part = (double *)xcalloc((size_t)U, sizeof(double));
#pragma omp parallel num_threads(ORC_NT)
    {
        double *hs = (double *)xcalloc((size_t)(L * P * N), sizeof(double));
        double *G = (double *)xcalloc((size_t)(P * N), sizeof(double));
        double *ds = (double *)xcalloc((size_t)P, sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < U; ++u) {
            int64_t bi = u / H, hh = u % H, gi = hh / hpg;
            for (int64_t t = 0; t < L; ++t) {
                double ab, be;
                discretise(disc, dt[(bi * L + t) * H + hh], A[hh], &ab, &be);
                const double *xt = x + ((bi * L + t) * H + hh) * P;
                const double *Bt = Bm + ((bi * L + t) * Gn + gi) * N;
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) {
                        double hp = t > 0 ? hs[((t - 1) * P + p) * N + n] : 0.0;
                        hs[(t * P + p) * N + n] = ab * hp + be * xt[p] * Bt[n];
                    }
            }
            memset(G, 0, sizeof(double) * (size_t)(P * N));
            double a_next = 0.0, sumA = 0.0, sumD = 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                double dtv = dt[(bi * L + t) * H + hh];
                double ab, be, a_dt, a_A, b_dt, b_A;
                discretise(disc, dtv, A[hh], &ab, &be);
                discretise_grad(disc, dtv, A[hh], &a_dt, &a_A, &b_dt, &b_A);
                const double *xt = x + ((bi * L + t) * H + hh) * P;
                const double *Bt = Bm + ((bi * L + t) * Gn + gi) * N;
                const double *Ct = Cm + ((bi * L + t) * Gn + gi) * N;
                for (int64_t p = 0; p < P; ++p) {
                    int64_t i = ((bi * L + t) * H + hh) * P + p;
                    double s = 0.0;
                    for (int64_t n = 0; n < N; ++n) s += Ct[n] * hs[(t * P + p) * N + n];
                    if (Dskip) s += Dskip[hh] * xt[p];
                    ds[p] = dy[i];
                    if (z) {
                        double sg = sigm(z[i]);
                        ds[p] = dy[i] * z[i] * sg;
                        if (dz) dz[i] = dy[i] * s * sg * (1.0 + z[i] * (1.0 - sg));
                    }
                    sumD += ds[p] * xt[p];
                }
                double dab = 0.0, dbe = 0.0;
                for (int64_t p = 0; p < P; ++p) {
                    double dxv = Dskip ? ds[p] * Dskip[hh] : 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        double Gt = ds[p] * Ct[n] + a_next * G[p * N + n];
                        double hp = t > 0 ? hs[((t - 1) * P + p) * N + n] : 0.0;
                        dC_part[(u * L + t) * N + n] += ds[p] * hs[(t * P + p) * N + n];
                        dB_part[(u * L + t) * N + n] += Gt * be * xt[p];
                        dxv += Gt * be * Bt[n];
                        dab += Gt * hp;
                        dbe += Gt * xt[p] * Bt[n];
                        G[p * N + n] = Gt;
                    }
                    dx[((bi * L + t) * H + hh) * P + p] = dxv;
                }
                ddt[(bi * L + t) * H + hh] = dab * a_dt + dbe * b_dt;
                sumA += dab * a_A + dbe * b_A;
                a_next = ab;
            }
            dA_part[u] = sumA;
            dD_part[u] = sumD;
        }
        free(hs);
        free(G);
        free(ds);
    }
    for (int64_t bi = 0; bi < B; ++bi)
        for (int64_t t = 0; t < L; ++t)
            for (int64_t gi = 0; gi < Gn; ++gi)
                for (int64_t n = 0; n < N; ++n) {
                    double sb = 0.0, sc = 0.0;
                    for (int64_t hh = gi * hpg; hh < (gi + 1) * hpg; ++hh) {
                        int64_t u = bi * H + hh;
                        sb += dB_part[(u * L + t) * N + n];
                        sc += dC_part[(u * L + t) * N + n];
                    }
                    dBm[((bi * L + t) * Gn + gi) * N + n] = sb;
                    dCm[((bi * L + t) * Gn + gi) * N + n] = sc;
                }
    for (int64_t hh = 0; hh < H; ++hh) {
        double sa = 0.0, sd = 0.0;
        for (int64_t bi = 0; bi < B; ++bi) {
            sa += dA_part[bi * H + hh];
            sd += dD_part[bi * H + hh];
        }
        dA[hh] = sa;
        if (dDskip) dDskip[hh] = sd;
    }
    free(dB_part);
    free(dC_part);
    free(dA_part);
    free(dD_part);
}

/* ------------------------------------------------------------------------------------------ */
/* GLA: scalar forget gate and outer-product write, state [B, H, K, V]                        */
/* (mlx-recurrence post, "gla_scan").                                                          */
/*   S_t = g_t S_{t-1} + k_t v_t^T;   o_t = S_t^T q_t.                                          */
/*   q, k: [B, L, H, K];  v, o: [B, L, H, V];  g: [B, L, H];  checkpoints ck: [nseg,B,H,K,V].   */
/* ------------------------------------------------------------------------------------------ */

void orc_gla_fwd(int64_t B, int64_t L, int64_t H, int64_t K, int64_t V, const double *q,
                 const double *k, const double *v, const double *g, double *o, int64_t S,
                 double *ck, const double *h0, double *hL)
{
#pragma omp parallel num_threads(ORC_NT)
    {
        double *St = (double *)xcalloc((size_t)(K * V), sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t hh = 0; hh < H; ++hh) {
                if (h0)
                    memcpy(St, h0 + (bi * H + hh) * K * V, sizeof(double) * (size_t)(K * V));
                else
                    memset(St, 0, sizeof(double) * (size_t)(K * V));
                for (int64_t t = 0; t < L; ++t) {
                    if (ck && S > 0 && t % S == 0)
                        memcpy(ck + (((t / S) * B + bi) * H + hh) * K * V, St,
                               sizeof(double) * (size_t)(K * V));
                    double gt = g[(bi * L + t) * H + hh];
                    const double *qt = q + ((bi * L + t) * H + hh) * K;
                    const double *kt = k + ((bi * L + t) * H + hh) * K;
                    const double *vt = v + ((bi * L + t) * H + hh) * V;
                    for (int64_t i = 0; i < K; ++i)
                        for (int64_t j = 0; j < V; ++j)
                            St[i * V + j] = gt * St[i * V + j] + kt[i] * vt[j];
                    double *ot = o + ((bi * L + t) * H + hh) * V;
                    for (int64_t j = 0; j < V; ++j) {
                        double s = 0.0;
                        for (int64_t i = 0; i < K; ++i) s += St[i * V + j] * qt[i];
                        ot[j] = s;
                    }
                }
                if (hL) memcpy(hL + (bi * H + hh) * K * V, St, sizeof(double) * (size_t)(K * V));
            }
        free(St);
    }
}

/* Backward (adjoint G_t = q_t do_t^T + g_{t+1} G_{t+1}):
 *   dq_t = S_t do_t;  dk_t = G_t v_t;  dv_t = G_t^T k_t;  dg_t = <G_t, S_{t-1}>_F. */
void orc_gla_bwd(int64_t B, int64_t L, int64_t H, int64_t K, int64_t V, const double *q,
                 const double *k, const double *v, const double *g, const double *dout,
                 double *dq, double *dk, double *dv, double *dg)
{
#pragma omp parallel num_threads(ORC_NT)
    {
        double *Ss = (double *)xcalloc((size_t)(L * K * V), sizeof(double));
        double *G = (double *)xcalloc((size_t)(K * V), sizeof(double));
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int64_t bi = 0; bi < B; ++bi)
            for (int64_t hh = 0; hh < H; ++hh) {
                for (int64_t t = 0; t < L; ++t) {
                    double gt = g[(bi * L + t) * H + hh];
                    const double *kt = k + ((bi * L + t) * H + hh) * K;
                    const double *vt = v + ((bi * L + t) * H + hh) * V;
                    for (int64_t i = 0; i < K; ++i)
                        for (int64_t j = 0; j < V; ++j) {
                            double prev = t > 0 ? Ss[((t - 1) * K + i) * V + j] : 0.0;
                            Ss[(t * K + i) * V + j] = gt * prev + kt[i] * vt[j];
                        }
                }
                memset(G, 0, sizeof(double) * (size_t)(K * V));
                double g_next = 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {
                    const double *qt = q + ((bi * L + t) * H + hh) * K;
                    const double *kt = k + ((bi * L + t) * H + hh) * K;
                    const double *vt = v + ((bi * L + t) * H + hh) * V;
                    const double *dot = dout + ((bi * L + t) * H + hh) * V;
                    double sg = 0.0;
                    for (int64_t i = 0; i < K; ++i)
                        for (int64_t j = 0; j < V; ++j) {
                            double Gt = qt[i] * dot[j] + g_next * G[i * V + j];
                            double prev = t > 0 ? Ss[((t - 1) * K + i) * V + j] : 0.0;
                            sg += Gt * prev;
                            G[i * V + j] = Gt;
                        }
                    dg[(bi * L + t) * H + hh] = sg;
                    double *dqt = dq + ((bi * L + t) * H + hh) * K;
                    double *dkt = dk + ((bi * L + t) * H + hh) * K;
                    double *dvt = dv + ((bi * L + t) * H + hh) * V;
                    for (int64_t i = 0; i < K; ++i) {
                        double sq = 0.0, sk = 0.0;
                        for (int64_t j = 0; j < V; ++j) {
                            sq += Ss[(t * K + i) * V + j] * dot[j];
                            sk += G[i * V + j] * vt[j];
                        }
                        dqt[i] = sq;
                        dkt[i] = sk;
                    }
                    for (int64_t j = 0; j < V; ++j) {
                        double sv = 0.0;
                        for (int64_t i = 0; i < K; ++i) sv += G[i * V + j] * kt[i];
                        dvt[j] = sv;
                    }
                    g_next = g[(bi * L + t) * H + hh];
                }
            }
        free(Ss);
        free(G);
    }
}
