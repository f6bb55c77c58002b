/*
 * esa_oracle.c -- plain, sequential, double-precision CPU oracle for the
 * Entangled State Attention (ESA) gated linear recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the yardstick the CUDA path is
 * measured against.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header, table or helper
 * with the GPU library, and the GPU library never calls it.
 *
 * What it computes (all arithmetic in double, one (b, h) head at a time,
 * one time step after another, no blocking or reordering):
 *
 *   gate      A_t = sigma(a_t)                    for both modes
 *   write     B_t = v_t                           direct mode
 *             B_t = (1 - A_t) * v_t               controlled mode
 *   state     E_t = A_t * E_{t-1} + B_t,  E_0 = E_init (zeros when absent)
 *   readout   r_t = 1 / sqrt(mean_d E_t^2 + 1e-6) over the D channels of a head
 *             y_t = q_t * E_t * r_t
 *
 * Sources:
 *   - The recurrence E_t = A_t (.) E_{t-1} + B_t: "Entangled State Attention
 *     v2.1" (entangled_state_attention-2.1.0 PKG-INFO), opening section; and
 *     "Entangled State Attention" (mlbricks-web.pages.dev/esa), "Core
 *     recurrence" panel of the Architecture section.
 *   - Direct mode A_t = sigma(x W_A), V_t = x W_V, E_t = A_t E_{t-1} + V_t and
 *     controlled mode E_t = g_t E_{t-1} + (1 - g_t) V_t with g_t = sigma(x W_g):
 *     "entangled-state-attention 0.1.0" (PyPI), section "Core idea".  The
 *     projections x W are outside this path: a, v, q are their outputs, and
 *     a is the pre-sigmoid gate logit in both modes.
 *   - Readout y_t = W_O(q_t (.) Norm(E_t)): same page, "Core idea", Readout.
 *     The page leaves Norm open; it is read here as a per-head RMS over the
 *     head dimension D with eps = 1e-6 inside the square root and no learned
 *     scale.  W_O is outside this path, so y is the value before W_O.
 *   - State shape [B, H, D], prompt length not a dimension of it:
 *     mlbricks-web.pages.dev/esa, "Generation / memory", "State shape".
 *   - The backward pass is not printed on any page; training through the
 *     layer (loss.backward() in "Entangled State Attention v2.1", section 9
 *     "Continue training a loaded model") implies it.  It is
 *     derived here by the chain rule from the forward definition above:
 *       n = E r,  dq = dy n,  dn = dy q,
 *       ghat_t = r (dn - n * mean_d(dn n))          (gradient into E_t via y_t)
 *       G_t = ghat_t + A_{t+1} G_{t+1},  G_T = ghat_T + dE_final
 *       dB_t = G_t,  dA_t = G_t E_{t-1},  dE_init = A_1 G_1
 *       direct:      dv = G,        da = G E_{t-1} A (1 - A)
 *       controlled:  dv = G (1-A),  da = G (E_{t-1} - v) A (1 - A)
 *
 * Layout: a, v, q, y, dy, da, dv, dq are contiguous [B, T, H, D]; E_init,
 * E_final, dE_final, dE_init and the step state E are contiguous [B, H, D].
 * The caller rounds inputs to the I/O dtype first and widens them to double,
 * so this code sees exactly the values the GPU sees.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>

#define ESA_ORACLE_EPS 1e-6

enum { ORACLE_DIRECT = 0, ORACLE_CONTROLLED = 1 };

/* Logistic sigmoid, evaluated so that exp never overflows. */
static double oracle_sigmoid(double x)
{
    if (x >= 0.0) {
        return 1.0 / (1.0 + exp(-x));
    }
    double e = exp(x);
    return e / (1.0 + e);
}

/* Offset of element (b, t, h, d) in a contiguous [B, T, H, D] array. */
static size_t at_bthd(long b, long t, long h, long d, long T, long H, long D)
{
    return (((size_t)b * (size_t)T + (size_t)t) * (size_t)H + (size_t)h) * (size_t)D + (size_t)d;
}

/* Offset of element (b, h, d) in a contiguous [B, H, D] array. */
static size_t at_bhd(long b, long h, long d, long H, long D)
{
    return ((size_t)b * (size_t)H + (size_t)h) * (size_t)D + (size_t)d;
}

static int oracle_check(long B, long T, long H, long D, int mode)
{
    if (B < 0 || T < 0 || H < 0 || D < 0) return -1;
    if (mode != ORACLE_DIRECT && mode != ORACLE_CONTROLLED) return -1;
    return 0;
}

/*
 * One head's readout at one time step: given the state e[0..D) and the
 * query q (stride 1), write y = q * e * r and return r.
 */
static double oracle_readout(const double *e, const double *q, double *y, long D)
{
    double sumsq = 0.0;
    for (long d = 0; d < D; ++d) sumsq += e[d] * e[d];
    double r = 1.0 / sqrt(sumsq / (double)D + ESA_ORACLE_EPS);
    for (long d = 0; d < D; ++d) y[d] = q[d] * e[d] * r;
    return r;
}

/*
 * Forward scan.  y may be NULL (not stored); E_final may be NULL; E_init may
 * be NULL (zeros); E_all, when not NULL, receives every E_t as [B, T, H, D].
 * Returns 0, or -1 on a bad argument.
 */
int esa_oracle_scan_fwd(const double *a, const double *v, const double *q,
                        double *y, double *E_final,
                        long B, long T, long H, long D, int mode,
                        const double *E_init, double *E_all)
{
    if (oracle_check(B, T, H, D, mode)) return -1;
    double *e = (double *)malloc(sizeof(double) * (size_t)(D > 0 ? D : 1));
    double *ybuf = (double *)malloc(sizeof(double) * (size_t)(D > 0 ? D : 1));
    if (!e || !ybuf) { free(e); free(ybuf); return -2; }

    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            for (long d = 0; d < D; ++d)
                e[d] = E_init ? E_init[at_bhd(b, h, d, H, D)] : 0.0;
            for (long t = 0; t < T; ++t) {
                for (long d = 0; d < D; ++d) {
                    size_t i = at_bthd(b, t, h, d, T, H, D);
                    double A = oracle_sigmoid(a[i]);
                    double Bt = (mode == ORACLE_DIRECT) ? v[i] : (1.0 - A) * v[i];
                    e[d] = A * e[d] + Bt;
                    if (E_all) E_all[i] = e[d];
                }
                size_t row = at_bthd(b, t, h, 0, T, H, D);
                oracle_readout(e, q + row, ybuf, D);
                if (y)
                    for (long d = 0; d < D; ++d) y[row + d] = ybuf[d];
            }
            if (E_final)
                for (long d = 0; d < D; ++d) E_final[at_bhd(b, h, d, H, D)] = e[d];
        }
    }
    free(e);
    free(ybuf);
    return 0;
}

/*
 * Backward scan.  Inputs are the forward's a, v, q, E_init (NULL = zeros)
 * and the upstream gradients dy and dE_final (NULL = zeros).  Outputs da, dv,
 * dq ([B, T, H, D]) and dE_init ([B, H, D], may be NULL).  The forward states
 * of one head are recomputed and kept (T * D doubles) before the reverse loop.
 */
int esa_oracle_scan_bwd(const double *a, const double *v, const double *q,
                        const double *dy, const double *dE_final,
                        double *da, double *dv, double *dq, double *dE_init,
                        long B, long T, long H, long D, int mode,
                        const double *E_init)
{
    if (oracle_check(B, T, H, D, mode)) return -1;
    size_t nd = (size_t)(D > 0 ? D : 1);
    size_t ntd = (size_t)(T > 0 ? T : 1) * nd;
    double *Es = (double *)malloc(sizeof(double) * ntd);    /* E_t, t = 1..T */
    double *As = (double *)malloc(sizeof(double) * ntd);    /* A_t */
    double *gh = (double *)malloc(sizeof(double) * nd);     /* ghat_t */
    double *hin = (double *)malloc(sizeof(double) * nd);    /* gradient into E_t from t+1 */
    double *e0 = (double *)malloc(sizeof(double) * nd);     /* E_0 */
    if (!Es || !As || !gh || !hin || !e0) {
        free(Es); free(As); free(gh); free(hin); free(e0);
        return -2;
    }

    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            /* Forward replay of this head, keeping every state. */
            for (long d = 0; d < D; ++d)
                e0[d] = E_init ? E_init[at_bhd(b, h, d, H, D)] : 0.0;
            for (long t = 0; t < T; ++t) {
                for (long d = 0; d < D; ++d) {
                    size_t i = at_bthd(b, t, h, d, T, H, D);
                    double A = oracle_sigmoid(a[i]);
                    double Bt = (mode == ORACLE_DIRECT) ? v[i] : (1.0 - A) * v[i];
                    double prev = (t == 0) ? e0[d] : Es[(size_t)(t - 1) * nd + (size_t)d];
                    As[(size_t)t * nd + (size_t)d] = A;
                    Es[(size_t)t * nd + (size_t)d] = A * prev + Bt;
                }
            }
            /* Reverse loop over time. */
            for (long d = 0; d < D; ++d)
                hin[d] = dE_final ? dE_final[at_bhd(b, h, d, H, D)] : 0.0;
            for (long t = T - 1; t >= 0; --t) {
                const double *Et = Es + (size_t)t * nd;
                size_t row = at_bthd(b, t, h, 0, T, H, D);
                /* Readout backward: y = q * E * r, r = (mean E^2 + eps)^-1/2. */
                double sumsq = 0.0;
                for (long d = 0; d < D; ++d) sumsq += Et[d] * Et[d];
                double r = 1.0 / sqrt(sumsq / (double)D + ESA_ORACLE_EPS);
                double dot = 0.0;   /* sum_d dn_d * n_d */
                for (long d = 0; d < D; ++d) {
                    double n = Et[d] * r;
                    double dn = dy[row + d] * q[row + d];
                    dq[row + d] = dy[row + d] * n;
                    dot += dn * n;
                }
                for (long d = 0; d < D; ++d) {
                    double n = Et[d] * r;
                    double dn = dy[row + d] * q[row + d];
                    gh[d] = r * (dn - n * dot / (double)D);
                }
                /* Recurrence backward. */
                for (long d = 0; d < D; ++d) {
                    double A = As[(size_t)t * nd + (size_t)d];
                    double prev = (t == 0) ? e0[d] : Es[(size_t)(t - 1) * nd + (size_t)d];
                    double G = gh[d] + hin[d];
                    double dA;
                    if (mode == ORACLE_DIRECT) {
                        dv[row + d] = G;
                        dA = G * prev;
                    } else {
                        dv[row + d] = G * (1.0 - A);
                        dA = G * (prev - v[row + d]);
                    }
                    da[row + d] = dA * A * (1.0 - A);
                    hin[d] = A * G;
                }
            }
            if (dE_init)
                for (long d = 0; d < D; ++d) dE_init[at_bhd(b, h, d, H, D)] = hin[d];
        }
    }
    free(Es); free(As); free(gh); free(hin); free(e0);
    return 0;
}

/*
 * One-token recurrent update (decode): E <- A E + B in place, then the
 * readout of the new state.  a_t, v_t, q_t, y_t and E are [B, H, D].
 * "Entangled State Attention v2.1", ESA-Lightning low-level interface
 * (lightning_step), and mlbricks-web.pages.dev/esa, Architecture step 05
 * "One-token update".
 */
int esa_oracle_step(const double *a_t, const double *v_t, const double *q_t,
                    double *E, double *y_t, long B, long H, long D, int mode)
{
    if (oracle_check(B, 1, H, D, mode)) return -1;
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            size_t row = at_bhd(b, h, 0, H, D);
            for (long d = 0; d < D; ++d) {
                double A = oracle_sigmoid(a_t[row + d]);
                double Bt = (mode == ORACLE_DIRECT) ? v_t[row + d] : (1.0 - A) * v_t[row + d];
                E[row + d] = A * E[row + d] + Bt;
            }
            oracle_readout(E + row, q_t + row, y_t + row, D);
        }
    }
    return 0;
}
