/*
 * oracle.c -- plain sequential fp64 reference of the selective scan (S6) used by
 * Vision Mamba (bidirectional scan) and VMamba (four-direction cross-scan).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code with the CUDA library.
 *
 * What it computes is written straight from the equations of the page
 * "Vision Mamba Guide: Efficient Bidirectional SSM & VMamba" (aifetchly-blog):
 *   - ZOH discretisation, section "Discretization via Zero-Order Hold (ZOH)":
 *       Abar = exp(Delta*A),  Bbar ~= Delta*B  (the approximate form, the default),
 *       or on request the exact form Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B,
 *       which for a diagonal A is expm1(Delta A_n) / A_n * B_n per state;
 *   - recurrence and readout, same section and section "Continuous-Time State
 *     Space Equations":  h_t = Abar h_{t-1} + Bbar x_t,  y_t = C h_t + D x_t;
 *   - selectivity, section "The Selective State Space (S6) Mechanism":
 *       Delta_t = softplus(...) (here softplus(delta_raw + delta_bias));
 *   - bidirectional pathways and the gated fusion, section "2. The Bidirectional
 *     Mamba Block": forward pass over tokens 1..N+1, backward pass from N+1 down to
 *     1, Y = y^f * silu(z) + y^b * silu(z) (the output projection is not part of it);
 *   - the four traversal orders and the merge, sections "1. Cross-Scan Traversal
 *     (CS-Traverse)" and "3. Cross-Merge Reversal (CS-Merge)".
 *
 * Readings where the page is silent (the same list is kept with the design notes):
 *   softplus(x) = log1p(exp(x)), taken as x itself for x > 20;  h starts at 0 for
 *   every direction;  the D*u skip is added once per direction;  per-direction B/C
 *   of the cross-scan are stored in grid order (direction k reads them at the grid
 *   position it visits);  silu(z) = z / (1 + exp(-z)).
 *
 * Everything is double precision and strictly sequential along each scan; the
 * only parallelism is over independent (batch, channel) pairs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MAX_STATE 256

/* "Delta_t = Softplus(Linear_Delta(x_t))" -- S6 mechanism section. */
static double softplus(double x) { return x > 20.0 ? x : log1p(exp(x)); }

/* sigma(z) in the gated fusion is the SiLU activation (Bidirectional Mamba Block). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * The four CS-Traverse orders on an H x W grid whose positions are numbered
 * p = h*W + w (row-major, "Top-Left (0,0)" first).  Writes order[t] = grid
 * position visited at scan step t, for t = 0..H*W-1.
 *   k = 0  Scan 1, rows from (0,0) to (H-1,W-1)
 *   k = 1  Scan 2, the reverse of scan 1
 *   k = 2  Scan 3, columns from (0,0) down to (H-1,W-1): step t = w*H + h
 *   k = 3  Scan 4, the reverse of scan 3
 * Returns 0, or -1 for a bad direction index.
 */
int oracle_cross_order(int k, int H, int W, int64_t *order)
{
    int64_t L = (int64_t)H * W;
    for (int64_t t = 0; t < L; ++t) {
        int64_t s = (k == 1 || k == 3) ? (L - 1 - t) : t;
        int64_t p;
        if (k == 0 || k == 1) {
            p = s;
        } else if (k == 2 || k == 3) {
            int64_t h = s % H, w = s / H;
            p = h * W + w;
        } else {
            return -1;
        }
        order[t] = p;
    }
    return 0;
}

/*
 * One S6 direction over every (batch, channel) sequence.
 *   u, delta : [batch, L, Di]          input and Delta (raw or final, see below)
 *   B, C     : [batch, L, N]           indexed by token position
 *   A        : [Di, N], D, bias : [Di]
 *   order    : [L] positions in visiting order (a permutation of 0..L-1)
 *   y        : [batch, L, Di]          y[b, order[t], d] receives the readout of step t;
 *                                      added to the existing value if accumulate != 0
 *   delta_is_raw != 0 : Delta = softplus(delta + bias[d]); otherwise Delta = delta
 *                       as given and bias is ignored.
 *   zoh != 0 : exact zero-order-hold Bbar (see bbar below); otherwise Bbar = Delta B.
 * Returns 0, or -1 on bad sizes.
 */
/*
 * Bbar of one state.  Section "Discretization via Zero-Order Hold (ZOH)" gives
 * Bbar = (Delta A)^-1 (exp(Delta A) - I) . Delta B and its first-order form Delta B.
 * With A diagonal the matrix inverse is a division per state, so the exact form is
 * (exp(Delta A_n) - 1) / A_n * B_n, evaluated with expm1 so that small Delta A_n
 * loses nothing to cancellation; at A_n = 0 it is its limit Delta B_n.
 */
static double bbar(double dt, double An, double Bn, int zoh)
{
    if (!zoh || An == 0.0) return dt * Bn;
    return expm1(dt * An) / An * Bn;
}

/*
 * Derivatives of one state's hold gain e(Delta, A_n) = Bbar_n / B_n (e = Delta for the
 * first-order form; e = (exp(Delta A_n) - 1) / A_n for the exact hold, Delta at A_n = 0):
 *   de/dDelta = 1, or exp(Delta A_n);
 *   de/dA_n   = 0, or (z e^z - (e^z - 1)) / A_n^2 = Delta^2 S(z) with z = Delta A_n and
 *               S(z) = sum_{k >= 1} k z^(k-1) / (k+1)!  (= 1/2 + z/3 + z^2/8 + ...),
 * which follows from differentiating e = Delta sum_{k >= 0} z^k / (k+1)! term by term.
 * S is summed as that series (18 terms, Horner) for |z| < 1/2, where the closed form
 * loses digits to cancellation, and in closed form elsewhere; at A_n = 0 it is 1/2.
 */
static double hold_gain_ddt(double dt, double An, int zoh)
{
    return zoh ? exp(dt * An) : 1.0;
}

static double hold_gain_dA(double dt, double An, int zoh)
{
    if (!zoh) return 0.0;
    double zz = dt * An;
    if (fabs(zz) < 0.5) {
        double c[19], f = 1.0;                 /* c[k] = k / (k+1)! */
        for (int k = 1; k <= 18; ++k) {
            f *= (double)(k + 1);
            c[k] = (double)k / f;
        }
        double sum = c[18];
        for (int k = 17; k >= 1; --k) sum = sum * zz + c[k];
        return dt * dt * sum;
    }
    return (zz * exp(zz) - expm1(zz)) / (An * An);
}

int oracle_s6_direction(const double *u, const double *delta, const double *B, const double *C,
                        const double *A, const double *D, const double *bias,
                        const int64_t *order, double *y,
                        int batch, int L, int Di, int N, int delta_is_raw, int accumulate, int zoh)
{
    if (batch < 0 || L < 0 || Di < 0 || N < 1 || N > ORACLE_MAX_STATE) return -1;
    int64_t pairs = (int64_t)batch * Di;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t bd = 0; bd < pairs; ++bd) {
        int64_t b = bd / Di, d = bd % Di;
        double h[ORACLE_MAX_STATE];
        for (int n = 0; n < N; ++n) h[n] = 0.0;                 /* h_0 = 0 */
        for (int64_t t = 0; t < L; ++t) {
            int64_t p = order[t];
            int64_t ix = (b * L + p) * Di + d;                    /* [b, p, d] */
            const double *Bt = B + (b * L + p) * N;               /* [b, p, :] */
            const double *Ct = C + (b * L + p) * N;
            double dt = delta_is_raw ? softplus(delta[ix] + bias[d]) : delta[ix];
            double x = u[ix];
            double yt = 0.0;
            for (int n = 0; n < N; ++n) {
                double Abar = exp(dt * A[d * N + n]);             /* Abar = exp(Delta A) */
                double Bbar = bbar(dt, A[d * N + n], Bt[n], zoh); /* Bbar (~= Delta B)   */
                h[n] = Abar * h[n] + Bbar * x;                    /* h_t = Abar h + Bbar x */
                yt += Ct[n] * h[n];                               /* C h_t               */
            }
            yt += D[d] * x;                                       /* + D x_t             */
            if (accumulate) y[ix] += yt; else y[ix] = yt;
        }
    }
    return 0;
}

/*
 * The smoothing in front of each pathway of the Vim block (page "Vision Mamba Guide",
 * section "2. The Bidirectional Mamba Block" figure: "Linear Projection -> 1D Conv ->
 * SiLU"; its PyTorch block: a depthwise Conv1d with kernel 3 and padding 1 per
 * pathway, the backward one applied to the reversed sequence):
 *   u_f[t] = silu(cb_f + w_f[0] x[t-1] + w_f[1] x[t] + w_f[2] x[t+1])
 *   u_b[t] = silu(cb_b + w_b[0] x[t+1] + w_b[1] x[t] + w_b[2] x[t-1])
 * with x = 0 outside 0..L-1 (u_b is the convolution of the reversed sequence, read
 * back at original positions).  x, u: [batch, L, Di]; w: [Di][3]; cb: [Di].
 */
int oracle_conv_silu(const double *x, const double *w, const double *cb, double *u,
                     int batch, int L, int Di, int reversed)
{
    if (batch < 0 || L < 0 || Di < 0) return -1;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t t = 0; t < L; ++t)
            for (int64_t d = 0; d < Di; ++d) {
                double acc = cb[d];
                for (int k = 0; k < 3; ++k) {
                    int64_t s = reversed ? t + 1 - k : t + k - 1;   /* tap k reads x[s] */
                    if (s >= 0 && s < L) acc += w[d * 3 + k] * x[(b * L + s) * Di + d];
                }
                u[(b * L + t) * Di + d] = silu(acc);
            }
    return 0;
}

/* y <- y * silu(z), elementwise over n values (skipped when z is NULL). */
static void apply_gate(double *y, const double *z, int64_t n)
{
    if (!z) return;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) y[i] *= silu(z[i]);
}

/*
 * Vim bidirectional S6 with gated fusion.
 *   u, delta, z : [batch, L, Di];  z may be NULL (no gate)
 *   B, C        : [batch, L, N]; the backward direction reads B + bc_dir_stride and
 *                 C + bc_dir_stride (0 = both directions share B and C)
 *   A [2, Di, N], D [2, Di], bias [2, Di]: index 0 = forward, 1 = backward
 *   y           : [batch, L, Di] = (y^f + y^b) * silu(z)
 *   delta_is_raw, zoh: as in oracle_s6_direction
 */
int oracle_vim_bidir(const double *u, const double *delta, const double *z,
                     const double *B, const double *C, int64_t bc_dir_stride,
                     const double *A, const double *D, const double *bias,
                     double *y, int batch, int L, int Di, int N, int delta_is_raw, int zoh)
{
    if (L < 0) return -1;
    int64_t *order = (int64_t *)calloc((size_t)(L > 0 ? L : 1), sizeof(int64_t));
    if (!order) return -1;
    int rc = 0;
    for (int64_t t = 0; t < L; ++t) order[t] = t;                 /* forward: 1 .. N+1 */
    rc |= oracle_s6_direction(u, delta, B, C, A, D, bias, order, y,
                              batch, L, Di, N, delta_is_raw, 0, zoh);
    for (int64_t t = 0; t < L; ++t) order[t] = L - 1 - t;         /* backward: N+1 .. 1 */
    rc |= oracle_s6_direction(u, delta, B + bc_dir_stride, C + bc_dir_stride,
                              A + (int64_t)Di * N, D + Di, bias + Di, order, y,
                              batch, L, Di, N, delta_is_raw, 1, zoh);
    free(order);
    if (rc) return -1;
    apply_gate(y, z, (int64_t)batch * L * Di);
    return 0;
}

/*
 * The Vim block's scan with its convolution front: each pathway runs on its own
 * smoothed input, u_f = oracle_conv_silu(x, w[0], cb[0], forward) and u_b =
 * oracle_conv_silu(x, w[1], cb[1], reversed); the rest is oracle_vim_bidir.
 *   conv_w [2][Di][3], conv_b [2][Di]; other arguments as in oracle_vim_bidir.
 */
int oracle_vim_bidir_conv(const double *x, const double *conv_w, const double *conv_b,
                          const double *delta, const double *z,
                          const double *B, const double *C, int64_t bc_dir_stride,
                          const double *A, const double *D, const double *bias,
                          double *y, int batch, int L, int Di, int N, int delta_is_raw, int zoh)
{
    if (batch < 0 || L < 0 || Di < 0) return -1;
    size_t n = (size_t)batch * (size_t)L * (size_t)Di;
    double *uf = (double *)calloc(n > 0 ? n : 1, sizeof(double));
    double *ub = (double *)calloc(n > 0 ? n : 1, sizeof(double));
    int64_t *order = (int64_t *)calloc((size_t)(L > 0 ? L : 1), sizeof(int64_t));
    int rc = (!uf || !ub || !order) ? -1 : 0;
    if (!rc) rc |= oracle_conv_silu(x, conv_w, conv_b, uf, batch, L, Di, 0);
    if (!rc) rc |= oracle_conv_silu(x, conv_w + (int64_t)Di * 3, conv_b + Di, ub, batch, L, Di, 1);
    if (!rc) {
        for (int64_t t = 0; t < L; ++t) order[t] = t;
        rc |= oracle_s6_direction(uf, delta, B, C, A, D, bias, order, y, batch, L, Di, N, delta_is_raw, 0, zoh);
        for (int64_t t = 0; t < L; ++t) order[t] = L - 1 - t;
        rc |= oracle_s6_direction(ub, delta, B + bc_dir_stride, C + bc_dir_stride, A + (int64_t)Di * N,
                                  D + Di, bias + Di, order, y, batch, L, Di, N, delta_is_raw, 1, zoh);
    }
    free(uf); free(ub); free(order);
    if (rc) return -1;
    apply_gate(y, z, (int64_t)batch * L * Di);
    return 0;
}

/*
 * VMamba SS2D: four independent S6 over the CS-Traverse orders, CS-Merge by sum.
 *   u, delta, z : [batch, H, W, Ci] (grid positions p = h*W + w);  z may be NULL
 *   B, C        : [4, batch, H*W, N], grid order (direction k reads B[k, b, p, :])
 *   A [4, Ci, N], D [4, Ci], bias [4, Ci]
 *   y           : [batch, H, W, Ci] = (y_1 + y_2 + y_3 + y_4) * silu(z)
 */
int oracle_cross_scan4(const double *u, const double *delta, const double *z,
                       const double *B, const double *C,
                       const double *A, const double *D, const double *bias,
                       double *y, int batch, int H, int W, int Ci, int N, int delta_is_raw, int zoh)
{
    if (H < 0 || W < 0) return -1;
    int64_t L = (int64_t)H * W;
    int64_t *order = (int64_t *)calloc((size_t)(L > 0 ? L : 1), sizeof(int64_t));
    if (!order) return -1;
    int rc = 0;
    int64_t bc = (int64_t)batch * L * N;
    for (int k = 0; k < 4; ++k) {
        rc |= oracle_cross_order(k, H, W, order);
        rc |= oracle_s6_direction(u, delta, B + k * bc, C + k * bc,
                                  A + (int64_t)k * Ci * N, D + (int64_t)k * Ci,
                                  bias + (int64_t)k * Ci, order, y,
                                  batch, (int)L, Ci, N, delta_is_raw, k > 0, zoh);
    }
    free(order);
    if (rc) return -1;
    apply_gate(y, z, (int64_t)batch * L * Ci);
    return 0;
}

/*
 * CS-Merge alone: ys [4, batch, H*W, Ci], each direction's outputs in its own
 * scan order (row t of direction k belongs to grid position order_k[t]).
 *   y [batch, H, W, Ci] = (sum_k ys_k mapped back to (h, w)) * silu(z)
 */
int oracle_cross_merge4(const double *ys, const double *z, double *y,
                        int batch, int H, int W, int Ci)
{
    if (H < 0 || W < 0 || batch < 0 || Ci < 0) return -1;
    int64_t L = (int64_t)H * W;
    int64_t *order = (int64_t *)calloc((size_t)(L > 0 ? L : 1), sizeof(int64_t));
    if (!order) return -1;
    int64_t total = (int64_t)batch * L * Ci;
    for (int64_t i = 0; i < total; ++i) y[i] = 0.0;
    for (int k = 0; k < 4; ++k) {
        if (oracle_cross_order(k, H, W, order)) { free(order); return -1; }
        const double *yk = ys + (int64_t)k * total;
        for (int64_t b = 0; b < batch; ++b)
            for (int64_t t = 0; t < L; ++t) {
                int64_t p = order[t];
                for (int64_t c = 0; c < Ci; ++c)
                    y[(b * L + p) * Ci + c] += yk[(b * L + t) * Ci + c];
            }
    }
    free(order);
    apply_gate(y, z, total);
    return 0;
}

/* ------------------------------------------------------------------------------
 * Reverse-mode derivatives (training through the scan).  The pages motivate the
 * scan by efficient training on GPUs; the derivative of the forward map above is
 * taken here by the chain rule, step by step in reverse visiting order, for a
 * scalar loss  ell = sum dy[b,t,d] * y[b,t,d].  Only the first-order Bbar = Delta B
 * is covered.
 * ------------------------------------------------------------------------------ */

/* d softplus(x) / dx with the same cut as softplus(): 1/(1 + e^-x), and 1 above 20. */
static double softplus_grad(double x) { return x > 20.0 ? 1.0 : 1.0 / (1.0 + exp(-x)); }

/* d silu(z) / dz = s (1 + z (1 - s)), s = 1/(1 + e^-z). */
static double silu_grad(double z)
{
    double s = 1.0 / (1.0 + exp(-z));
    return s * (1.0 + z * (1.0 - s));
}

/*
 * Derivative of one S6 direction (oracle_s6_direction; the first-order Bbar, or the
 * exact hold when zoh != 0).
 *   dy       : [batch, L, Di], the loss's derivative with respect to y
 *   du, ddelta : [batch, L, Di]   (ddelta is w.r.t. the raw delta when delta_is_raw,
 *                                  else w.r.t. Delta itself)
 *   dB, dC   : [batch, L, N];  dA : [Di, N];  dD, dbias : [Di]  (dbias only when raw)
 * Every output is ADDED to (so that directions sharing an input accumulate).
 * For each (b, d) the forward pass is run first, keeping h_t for every step; then
 * the adjoint g of h runs backwards: g <- g + C_t dy_t is dl/dh_t, from which
 *   dl/dC_t = dy_t h_t,  dl/dD += dy_t u_t,  dl/du_t += D dy_t + sum_n g_n Delta_t B_tn,
 *   dl/dAbar_n = g_n h_{t-1,n}  ->  dl/dDelta += that * Abar_n * A_n,
 *                                   dl/dA_n   += that * Abar_n * Delta_t,
 *   dl/dDelta += sum_n g_n B_tn u_t,  dl/dB_tn += g_n Delta_t u_t,
 * and g <- g * Abar is dl/dh_{t-1}.  With the exact hold, Bbar_n = e_n B_n with the
 * gain e_n = (exp(Delta A_n) - 1) / A_n in place of Delta: Delta_t becomes e_n in
 * dl/du and dl/dB, the Delta term gains the factor de_n/dDelta = exp(Delta A_n), and
 * dl/dA_n gains g_n B_tn u_t de_n/dA_n (hold_gain_dA).
 */
int oracle_s6_direction_bwd(const double *u, const double *delta, const double *B, const double *C,
                            const double *A, const double *D, const double *bias,
                            const int64_t *order, const double *dy,
                            double *du, double *ddelta, double *dB, double *dC,
                            double *dA, double *dD, double *dbias,
                            int batch, int L, int Di, int N, int delta_is_raw, int zoh)
{
    if (batch < 0 || L < 0 || Di < 0 || N < 1 || N > ORACLE_MAX_STATE) return -1;
    int rc = 0;
    #pragma omp parallel
    {
        double *hs = (double *)malloc(((size_t)(L > 0 ? L : 1)) * (size_t)N * sizeof(double));
        double *dts = (double *)malloc(((size_t)(L > 0 ? L : 1)) * sizeof(double));
        double *dA_loc = (double *)calloc((size_t)Di * N, sizeof(double));
        double *dD_loc = (double *)calloc((size_t)(Di > 0 ? Di : 1), sizeof(double));
        double *db_loc = (double *)calloc((size_t)(Di > 0 ? Di : 1), sizeof(double));
        int ok = hs && dts && dA_loc && dD_loc && db_loc;
        if (!ok) {
            #pragma omp atomic write
            rc = -1;
        }
        /* batch items in parallel: dB and dC rows belong to one batch item */
        #pragma omp for schedule(dynamic, 1)
        for (int64_t b = 0; b < batch; ++b) {
            if (!ok) continue;
            for (int64_t d = 0; d < Di; ++d) {
                const double *Ad = A + d * N;
                double h[ORACLE_MAX_STATE], g[ORACLE_MAX_STATE];
                for (int n = 0; n < N; ++n) h[n] = 0.0;
                for (int64_t t = 0; t < L; ++t) {                 /* forward, keeping h_t */
                    int64_t p = order[t];
                    int64_t ix = (b * L + p) * Di + d;
                    const double *Bt = B + (b * L + p) * N;
                    double dt = delta_is_raw ? softplus(delta[ix] + bias[d]) : delta[ix];
                    dts[t] = dt;
                    for (int n = 0; n < N; ++n) {
                        h[n] = exp(dt * Ad[n]) * h[n] + bbar(dt, Ad[n], Bt[n], zoh) * u[ix];
                        hs[t * N + n] = h[n];
                    }
                }
                for (int n = 0; n < N; ++n) g[n] = 0.0;
                for (int64_t t = L - 1; t >= 0; --t) {            /* adjoint, in reverse */
                    int64_t p = order[t];
                    int64_t ix = (b * L + p) * Di + d;
                    const double *Bt = B + (b * L + p) * N, *Ct = C + (b * L + p) * N;
                    double *dBt = dB + (b * L + p) * N, *dCt = dC + (b * L + p) * N;
                    double dt = dts[t], x = u[ix], e = dy[ix];
                    double dDelta = 0.0, dx = D[d] * e;
                    dD_loc[d] += e * x;
                    for (int n = 0; n < N; ++n) {
                        g[n] += Ct[n] * e;                        /* dl/dh_t            */
                        dCt[n] += e * hs[t * N + n];
                        double Abar = exp(dt * Ad[n]);
                        double hprev = t > 0 ? hs[(t - 1) * N + n] : 0.0;
                        double dAbar = g[n] * hprev;
                        double gain = bbar(dt, Ad[n], 1.0, zoh);  /* Bbar_n / B_n       */
                        dDelta += dAbar * Abar * Ad[n] + g[n] * Bt[n] * x * hold_gain_ddt(dt, Ad[n], zoh);
                        dA_loc[d * N + n] += dAbar * Abar * dt;
                        if (zoh) dA_loc[d * N + n] += g[n] * Bt[n] * x * hold_gain_dA(dt, Ad[n], zoh);
                        dBt[n] += g[n] * gain * x;
                        dx += g[n] * gain * Bt[n];
                        g[n] *= Abar;                             /* dl/dh_{t-1} part   */
                    }
                    du[ix] += dx;
                    if (delta_is_raw) {
                        double s = softplus_grad(delta[ix] + bias[d]);
                        ddelta[ix] += dDelta * s;
                        db_loc[d] += dDelta * s;
                    } else {
                        ddelta[ix] += dDelta;
                    }
                }
            }
        }
        #pragma omp critical
        {
            if (ok) {
                for (int64_t i = 0; i < (int64_t)Di * N; ++i) dA[i] += dA_loc[i];
                for (int64_t d = 0; d < Di; ++d) {
                    dD[d] += dD_loc[d];
                    if (delta_is_raw) dbias[d] += db_loc[d];
                }
            }
        }
        free(hs); free(dts); free(dA_loc); free(dD_loc); free(db_loc);
    }
    return rc;
}

/*
 * Derivative of oracle_vim_bidir (first-order Bbar, or the exact hold when zoh != 0)
 * for ell = sum dout * y.
 *   dout : [batch, L, Di].  Outputs (overwritten):
 *   du, ddelta, dz : [batch, L, Di]  (dz untouched when z is NULL; ddelta w.r.t. the
 *                    raw delta when delta_is_raw)
 *   dB, dC : shaped like B and C (with bc_dir_stride > 0 the backward direction's part
 *            starts bc_dir_stride elements in; with 0 both directions add into one)
 *   dA [2, Di, N], dD [2, Di], dbias [2, Di]
 * With y = (y^f + y^b) silu(z):  dl/dz = dout (y^f + y^b) silu'(z) and each direction
 * sees dl/dy^k = dout silu(z).
 */
int oracle_vim_bidir_bwd(const double *u, const double *delta, const double *z,
                         const double *B, const double *C, int64_t bc_dir_stride,
                         const double *A, const double *D, const double *bias, const double *dout,
                         double *du, double *ddelta, double *dz, double *dB, double *dC,
                         double *dA, double *dD, double *dbias,
                         int batch, int L, int Di, int N, int delta_is_raw, int zoh)
{
    if (batch < 0 || L < 0 || Di < 0 || N < 1 || bc_dir_stride < 0) return -1;
    int64_t n_act = (int64_t)batch * L * Di, n_bc = (int64_t)batch * L * N;
    int64_t n_bc_all = bc_dir_stride > 0 ? bc_dir_stride + n_bc : n_bc;
    double *dy = (double *)malloc((size_t)(n_act > 0 ? n_act : 1) * sizeof(double));
    int64_t *order = (int64_t *)malloc((size_t)(L > 0 ? L : 1) * sizeof(int64_t));
    if (!dy || !order) { free(dy); free(order); return -1; }
    for (int64_t i = 0; i < n_act; ++i) { du[i] = 0.0; ddelta[i] = 0.0; }
    for (int64_t i = 0; i < n_bc_all; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    for (int64_t i = 0; i < 2 * (int64_t)Di * N; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < 2 * (int64_t)Di; ++i) { dD[i] = 0.0; dbias[i] = 0.0; }
    int rc = 0;
    if (z) {
        /* the ungated sum y^f + y^b, for dl/dz */
        double *ys = (double *)malloc((size_t)(n_act > 0 ? n_act : 1) * sizeof(double));
        if (!ys) { free(dy); free(order); return -1; }
        rc |= oracle_vim_bidir(u, delta, NULL, B, C, bc_dir_stride, A, D, bias, ys,
                               batch, L, Di, N, delta_is_raw, zoh);
        for (int64_t i = 0; i < n_act; ++i) {
            dz[i] = dout[i] * ys[i] * silu_grad(z[i]);
            dy[i] = dout[i] * silu(z[i]);
        }
        free(ys);
    } else {
        for (int64_t i = 0; i < n_act; ++i) dy[i] = dout[i];
    }
    for (int64_t t = 0; t < L; ++t) order[t] = t;
    rc |= oracle_s6_direction_bwd(u, delta, B, C, A, D, bias, order, dy, du, ddelta, dB, dC,
                                  dA, dD, dbias, batch, L, Di, N, delta_is_raw, zoh);
    for (int64_t t = 0; t < L; ++t) order[t] = L - 1 - t;
    rc |= oracle_s6_direction_bwd(u, delta, B + bc_dir_stride, C + bc_dir_stride,
                                  A + (int64_t)Di * N, D + Di, bias + Di, order, dy, du, ddelta,
                                  dB + bc_dir_stride, dC + bc_dir_stride,
                                  dA + (int64_t)Di * N, dD + Di, dbias + Di,
                                  batch, L, Di, N, delta_is_raw, zoh);
    free(dy); free(order);
    return rc ? -1 : 0;
}

/*
 * Derivative of oracle_vim_bidir_conv (the scan with each pathway's convolution front)
 * for ell = sum dout * y.  Outputs (overwritten):
 *   dx : [batch, L, Di];  dconv_w [2][Di][3];  dconv_b [2][Di];
 *   ddelta, dz, dB, dC, dA, dD, dbias : as in oracle_vim_bidir_bwd.
 * The chain rule through u_k = silu(pre_k): each direction's dl/du_k comes from
 * oracle_s6_direction_bwd on its own u_k; with dpre_k = dl/du_k * silu'(pre_k) and tap
 * j of pathway k reading x[s_kj(t)] (s = t + j - 1 forward, t + 1 - j backward):
 *   dl/dx[s_kj(t)] += w_k[j] dpre_k[t],  dl/dw_k[j] += dpre_k[t] x[s_kj(t)],
 *   dl/dcb_k += dpre_k[t]   (taps that fall outside 0..L-1 read the zero padding).
 */
int oracle_vim_bidir_conv_bwd(const double *x, const double *conv_w, const double *conv_b,
                              const double *delta, const double *z, const double *B, const double *C,
                              int64_t bc_dir_stride, const double *A, const double *D, const double *bias,
                              const double *dout, double *dx, double *dconv_w, double *dconv_b,
                              double *ddelta, double *dz, double *dB, double *dC,
                              double *dA, double *dD, double *dbias,
                              int batch, int L, int Di, int N, int delta_is_raw, int zoh)
{
    if (batch < 0 || L < 0 || Di < 0 || N < 1 || bc_dir_stride < 0) return -1;
    int64_t n_act = (int64_t)batch * L * Di, n_bc = (int64_t)batch * L * N;
    int64_t n_bc_all = bc_dir_stride > 0 ? bc_dir_stride + n_bc : n_bc;
    size_t na = (size_t)(n_act > 0 ? n_act : 1);
    double *u[2], *du[2], *dy = (double *)malloc(na * sizeof(double));
    int64_t *order = (int64_t *)malloc((size_t)(L > 0 ? L : 1) * sizeof(int64_t));
    u[0] = (double *)calloc(na, sizeof(double)); u[1] = (double *)calloc(na, sizeof(double));
    du[0] = (double *)calloc(na, sizeof(double)); du[1] = (double *)calloc(na, sizeof(double));
    int rc = (!dy || !order || !u[0] || !u[1] || !du[0] || !du[1]) ? -1 : 0;
    if (!rc) {
        rc |= oracle_conv_silu(x, conv_w, conv_b, u[0], batch, L, Di, 0);
        rc |= oracle_conv_silu(x, conv_w + (int64_t)Di * 3, conv_b + Di, u[1], batch, L, Di, 1);
    }
    if (!rc) {
        for (int64_t i = 0; i < n_act; ++i) { dx[i] = 0.0; ddelta[i] = 0.0; }
        for (int64_t i = 0; i < n_bc_all; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
        for (int64_t i = 0; i < 2 * (int64_t)Di * N; ++i) dA[i] = 0.0;
        for (int64_t i = 0; i < 2 * (int64_t)Di; ++i) { dD[i] = 0.0; dbias[i] = 0.0; dconv_b[i] = 0.0; }
        for (int64_t i = 0; i < 6 * (int64_t)Di; ++i) dconv_w[i] = 0.0;
        if (z) {
            double *ys = (double *)malloc(na * sizeof(double));
            if (!ys) rc = -1;
            else {
                rc |= oracle_vim_bidir_conv(x, conv_w, conv_b, delta, NULL, B, C, bc_dir_stride, A, D, bias, ys,
                                            batch, L, Di, N, delta_is_raw, zoh);
                for (int64_t i = 0; i < n_act; ++i) {
                    dz[i] = dout[i] * ys[i] * silu_grad(z[i]);
                    dy[i] = dout[i] * silu(z[i]);
                }
                free(ys);
            }
        } else {
            for (int64_t i = 0; i < n_act; ++i) dy[i] = dout[i];
        }
    }
    if (!rc) {
        for (int64_t t = 0; t < L; ++t) order[t] = t;
        rc |= oracle_s6_direction_bwd(u[0], delta, B, C, A, D, bias, order, dy, du[0], ddelta, dB, dC,
                                      dA, dD, dbias, batch, L, Di, N, delta_is_raw, zoh);
        for (int64_t t = 0; t < L; ++t) order[t] = L - 1 - t;
        rc |= oracle_s6_direction_bwd(u[1], delta, B + bc_dir_stride, C + bc_dir_stride,
                                      A + (int64_t)Di * N, D + Di, bias + Di, order, dy, du[1], ddelta,
                                      dB + bc_dir_stride, dC + bc_dir_stride,
                                      dA + (int64_t)Di * N, dD + Di, dbias + Di,
                                      batch, L, Di, N, delta_is_raw, zoh);
    }
    if (!rc) {
        for (int k = 0; k < 2; ++k) {
            const double *w = conv_w + (int64_t)k * Di * 3, *cb = conv_b + (int64_t)k * Di;
            double *dw = dconv_w + (int64_t)k * Di * 3, *dcb = dconv_b + (int64_t)k * Di;
            for (int64_t b = 0; b < batch; ++b)
                for (int64_t t = 0; t < L; ++t)
                    for (int64_t d = 0; d < Di; ++d) {
                        double pre = cb[d];
                        for (int j = 0; j < 3; ++j) {
                            int64_t s = k ? t + 1 - j : t + j - 1;
                            if (s >= 0 && s < L) pre += w[d * 3 + j] * x[(b * L + s) * Di + d];
                        }
                        double dpre = du[k][(b * L + t) * Di + d] * silu_grad(pre);
                        dcb[d] += dpre;
                        for (int j = 0; j < 3; ++j) {
                            int64_t s = k ? t + 1 - j : t + j - 1;
                            if (s < 0 || s >= L) continue;
                            dx[(b * L + s) * Di + d] += w[d * 3 + j] * dpre;
                            dw[d * 3 + j] += dpre * x[(b * L + s) * Di + d];
                        }
                    }
        }
    }
    free(dy); free(order); free(u[0]); free(u[1]); free(du[0]); free(du[1]);
    return rc ? -1 : 0;
}

/*
 * The input projections of the S6 module (page "Vision Mamba Guide", the PyTorch
 * SimpleSelectiveSSM under "The Selective State Space (S6) Mechanism": x_proj is a
 * linear map without bias from d_model to 2N + 1 columns, read as B (columns 0..N-1),
 * C (columns N..2N-1) and the one-column step input (column 2N); dt_proj maps that
 * column back to d_model with a bias, and softplus gives Delta):
 *   P[m, j] = sum_d u[m, d] Wx[d, j]          m < M, j < NO
 * u: [M, Di], Wx: [Di, NO], P: [M, NO].
 */
int oracle_xproj(const double *u, const double *Wx, double *P, int64_t M, int Di, int NO)
{
    if (M < 0 || Di < 0 || NO < 1) return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < NO; ++j) {
            double acc = 0.0;
            for (int d = 0; d < Di; ++d) acc += u[m * Di + d] * Wx[(int64_t)d * NO + j];
            P[m * NO + j] = acc;
        }
    return 0;
}

/*
 * Derivative of the Vim block scan with its projections (the composition the Python
 * side's vim_block_scan evaluates: per pathway k, u_k = silu(conv_k(x)) (conv_w given)
 * or x, P_k = u_k Wx[k], B_k = P_k[:, 0:N], C_k = P_k[:, N:2N], s_k = P_k[:, 2N],
 * delta_raw_k[t, d] = s_k[t] Wdt[k][d], y = (S6_f + S6_b) silu(z)), first-order Bbar, for
 * ell = sum dout * y.  By the chain rule through each step:
 *   dl/dP_k = [dl/dB_k | dl/dC_k | dl/ds_k],  dl/ds_k[t] = sum_d dl/ddelta_raw_k[t, d] Wdt[k][d],
 *   dl/dWdt[k][d] = sum_t dl/ddelta_raw_k[t, d] s_k[t],
 *   dl/du_k += dl/dP_k Wx[k]^T,  dl/dWx[k] = u_k^T dl/dP_k,
 * and then through the convolution front as in oracle_vim_bidir_conv_bwd (without it,
 * dl/dx = dl/du_f + dl/du_b).
 *   x, z, dout : [batch, L, Di] (z may be NULL);  Wx [2][Di][2N+1];  Wdt, bias, D [2][Di];
 *   A [2][Di][N];  conv_w [2][Di][3], conv_b [2][Di] or both NULL.
 *   Outputs (overwritten): dx [batch, L, Di]; dz (untouched when z is NULL); dWx
 *   [2][Di][2N+1]; dWdt, dbias, dD [2][Di]; dA [2][Di][N]; dconv_w, dconv_b (when
 *   conv_w is given).
 */
int oracle_vim_block_scan_bwd(const double *x, const double *conv_w, const double *conv_b, const double *Wx,
                              const double *Wdt, const double *A, const double *D, const double *bias,
                              const double *z, const double *dout, double *dx, double *dz, double *dWx,
                              double *dWdt, double *dbias, double *dD, double *dA, double *dconv_w,
                              double *dconv_b, int batch, int L, int Di, int N)
{
    if (batch < 0 || L < 0 || Di < 0 || N < 1 || (!conv_w != !conv_b)) return -1;
    const int NO = 2 * N + 1;
    const int64_t M = (int64_t)batch * L, n_act = M * Di;
    size_t na = (size_t)(n_act > 0 ? n_act : 1), nm = (size_t)(M > 0 ? M : 1);
    double *u[2], *du[2], *P[2], *Bk[2], *Ck[2], *dr[2], *ddr[2], *dB[2], *dC[2];
    double *dy = (double *)malloc(na * sizeof(double)), *ys = (double *)calloc(na, sizeof(double));
    int64_t *order = (int64_t *)malloc((size_t)(L > 0 ? L : 1) * sizeof(int64_t));
    int rc = (!dy || !ys || !order) ? -1 : 0;
    for (int k = 0; k < 2; ++k) {
        u[k] = (double *)calloc(na, sizeof(double)); du[k] = (double *)calloc(na, sizeof(double));
        P[k] = (double *)calloc(nm * NO, sizeof(double));
        Bk[k] = (double *)calloc(nm * N, sizeof(double)); Ck[k] = (double *)calloc(nm * N, sizeof(double));
        dr[k] = (double *)calloc(na, sizeof(double)); ddr[k] = (double *)calloc(na, sizeof(double));
        dB[k] = (double *)calloc(nm * N, sizeof(double)); dC[k] = (double *)calloc(nm * N, sizeof(double));
        if (!u[k] || !du[k] || !P[k] || !Bk[k] || !Ck[k] || !dr[k] || !ddr[k] || !dB[k] || !dC[k]) rc = -1;
    }
    /* the forward steps of each pathway */
    for (int k = 0; k < 2 && !rc; ++k) {
        if (conv_w) rc |= oracle_conv_silu(x, conv_w + (int64_t)k * Di * 3, conv_b + (int64_t)k * Di, u[k],
                                           batch, L, Di, k);
        else for (int64_t i = 0; i < n_act; ++i) u[k][i] = x[i];
        rc |= oracle_xproj(u[k], Wx + (int64_t)k * Di * NO, P[k], M, Di, NO);
        for (int64_t m = 0; m < M; ++m) {
            for (int n = 0; n < N; ++n) {
                Bk[k][m * N + n] = P[k][m * NO + n];
                Ck[k][m * N + n] = P[k][m * NO + N + n];
            }
            for (int64_t d = 0; d < Di; ++d) dr[k][m * Di + d] = P[k][m * NO + 2 * N] * Wdt[(int64_t)k * Di + d];
        }
        for (int64_t t = 0; t < L; ++t) order[t] = k ? L - 1 - t : t;
        rc |= oracle_s6_direction(u[k], dr[k], Bk[k], Ck[k], A + (int64_t)k * Di * N, D + (int64_t)k * Di,
                                  bias + (int64_t)k * Di, order, ys, batch, L, Di, N, 1, k, 0);
    }
    if (!rc) {
        for (int64_t i = 0; i < n_act; ++i) {
            if (z) { dz[i] = dout[i] * ys[i] * silu_grad(z[i]); dy[i] = dout[i] * silu(z[i]); }
            else dy[i] = dout[i];
            dx[i] = 0.0;
        }
        for (int64_t i = 0; i < 2 * (int64_t)Di * N; ++i) dA[i] = 0.0;
        for (int64_t i = 0; i < 2 * (int64_t)Di; ++i) { dD[i] = 0.0; dbias[i] = 0.0; dWdt[i] = 0.0; }
        for (int64_t i = 0; i < 2 * (int64_t)Di * NO; ++i) dWx[i] = 0.0;
        if (conv_w) {
            for (int64_t i = 0; i < 6 * (int64_t)Di; ++i) dconv_w[i] = 0.0;
            for (int64_t i = 0; i < 2 * (int64_t)Di; ++i) dconv_b[i] = 0.0;
        }
    }
    /* the scan's derivative per pathway, then the projections' */
    for (int k = 0; k < 2 && !rc; ++k) {
        for (int64_t t = 0; t < L; ++t) order[t] = k ? L - 1 - t : t;
        rc |= oracle_s6_direction_bwd(u[k], dr[k], Bk[k], Ck[k], A + (int64_t)k * Di * N, D + (int64_t)k * Di,
                                      bias + (int64_t)k * Di, order, dy, du[k], ddr[k], dB[k], dC[k],
                                      dA + (int64_t)k * Di * N, dD + (int64_t)k * Di, dbias + (int64_t)k * Di,
                                      batch, L, Di, N, 1, 0);
        const double *W = Wx + (int64_t)k * Di * NO, *wdt = Wdt + (int64_t)k * Di;
        double *dW = dWx + (int64_t)k * Di * NO, *dwdt = dWdt + (int64_t)k * Di;
        for (int64_t m = 0; m < M && !rc; ++m) {
            double dP[2 * ORACLE_MAX_STATE + 1];
            double s = P[k][m * NO + 2 * N], ds = 0.0;
            for (int64_t d = 0; d < Di; ++d) {
                ds += ddr[k][m * Di + d] * wdt[d];
                dwdt[d] += ddr[k][m * Di + d] * s;
            }
            for (int n = 0; n < N; ++n) { dP[n] = dB[k][m * N + n]; dP[N + n] = dC[k][m * N + n]; }
            dP[2 * N] = ds;
            for (int64_t d = 0; d < Di; ++d) {
                double acc = 0.0;
                for (int j = 0; j < NO; ++j) {
                    acc += dP[j] * W[d * NO + j];
                    dW[d * NO + j] += u[k][m * Di + d] * dP[j];
                }
                du[k][m * Di + d] += acc;
            }
        }
    }
    /* through the convolution front (or the identity) to x */
    if (!rc && conv_w) {
        for (int k = 0; k < 2; ++k) {
            const double *w = conv_w + (int64_t)k * Di * 3, *cb = conv_b + (int64_t)k * Di;
            double *dw = dconv_w + (int64_t)k * Di * 3, *dcb = dconv_b + (int64_t)k * Di;
            for (int64_t b = 0; b < batch; ++b)
                for (int64_t t = 0; t < L; ++t)
                    for (int64_t d = 0; d < Di; ++d) {
                        double pre = cb[d];
                        for (int j = 0; j < 3; ++j) {
                            int64_t sx = k ? t + 1 - j : t + j - 1;
                            if (sx >= 0 && sx < L) pre += w[d * 3 + j] * x[(b * L + sx) * Di + d];
                        }
                        double dpre = du[k][(b * L + t) * Di + d] * silu_grad(pre);
                        dcb[d] += dpre;
                        for (int j = 0; j < 3; ++j) {
                            int64_t sx = k ? t + 1 - j : t + j - 1;
                            if (sx < 0 || sx >= L) continue;
                            dx[(b * L + sx) * Di + d] += w[d * 3 + j] * dpre;
                            dw[d * 3 + j] += dpre * x[(b * L + sx) * Di + d];
                        }
                    }
        }
    } else if (!rc) {
        for (int64_t i = 0; i < n_act; ++i) dx[i] = du[0][i] + du[1][i];
    }
    free(dy); free(ys); free(order);
    for (int k = 0; k < 2; ++k) {
        free(u[k]); free(du[k]); free(P[k]); free(Bk[k]); free(Ck[k]); free(dr[k]); free(ddr[k]); free(dB[k]);
        free(dC[k]);
    }
    return rc ? -1 : 0;
}

/*
 * Derivative of oracle_cross_scan4 (first-order Bbar, or the exact hold when zoh != 0)
 * for ell = sum dout * y, with
 * y = (sum_k y_k) * silu(z): dl/dz = dout (sum_k y_k) silu'(z), and each of the four
 * CS-Traverse directions sees dl/dy_k = dout silu(z) at the grid positions it visits.
 *   dout : [batch, H*W, Ci].  Outputs (overwritten): du, ddelta, dz [batch, H*W, Ci]
 *   (dz untouched when z is NULL); dB, dC [4, batch, H*W, N] (grid order, per
 *   direction); dA [4, Ci, N]; dD, dbias [4, Ci].
 */
int oracle_cross_scan4_bwd(const double *u, const double *delta, const double *z,
                           const double *B, const double *C,
                           const double *A, const double *D, const double *bias, const double *dout,
                           double *du, double *ddelta, double *dz, double *dB, double *dC,
                           double *dA, double *dD, double *dbias,
                           int batch, int H, int W, int Ci, int N, int delta_is_raw, int zoh)
{
    if (H < 0 || W < 0 || batch < 0 || Ci < 0 || N < 1) return -1;
    int64_t L = (int64_t)H * W;
    int64_t n_act = (int64_t)batch * L * Ci, bc = (int64_t)batch * L * N;
    double *dy = (double *)malloc((size_t)(n_act > 0 ? n_act : 1) * sizeof(double));
    int64_t *order = (int64_t *)malloc((size_t)(L > 0 ? L : 1) * sizeof(int64_t));
    if (!dy || !order) { free(dy); free(order); return -1; }
    for (int64_t i = 0; i < n_act; ++i) { du[i] = 0.0; ddelta[i] = 0.0; }
    for (int64_t i = 0; i < 4 * bc; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    for (int64_t i = 0; i < 4 * (int64_t)Ci * N; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < 4 * (int64_t)Ci; ++i) { dD[i] = 0.0; dbias[i] = 0.0; }
    int rc = 0;
    if (z) {
        double *ys = (double *)malloc((size_t)(n_act > 0 ? n_act : 1) * sizeof(double));
        if (!ys) { free(dy); free(order); return -1; }
        rc |= oracle_cross_scan4(u, delta, NULL, B, C, A, D, bias, ys, batch, H, W, Ci, N, delta_is_raw, zoh);
        for (int64_t i = 0; i < n_act; ++i) {
            dz[i] = dout[i] * ys[i] * silu_grad(z[i]);
            dy[i] = dout[i] * silu(z[i]);
        }
        free(ys);
    } else {
        for (int64_t i = 0; i < n_act; ++i) dy[i] = dout[i];
    }
    for (int k = 0; k < 4; ++k) {
        rc |= oracle_cross_order(k, H, W, order);
        rc |= oracle_s6_direction_bwd(u, delta, B + k * bc, C + k * bc, A + (int64_t)k * Ci * N,
                                      D + (int64_t)k * Ci, bias + (int64_t)k * Ci, order, dy, du, ddelta,
                                      dB + k * bc, dC + k * bc, dA + (int64_t)k * Ci * N, dD + (int64_t)k * Ci,
                                      dbias + (int64_t)k * Ci, batch, (int)L, Ci, N, delta_is_raw, zoh);
    }
    free(dy); free(order);
    return rc ? -1 : 0;
}
