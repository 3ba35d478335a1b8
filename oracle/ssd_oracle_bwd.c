/*
 * ssd_oracle_bwd.c -- plain, slow, fp64 CPU oracle for the gradient of the
 * selective state-space scan.  TEST INFRASTRUCTURE ONLY, like ssd_oracle.c:
 * nothing in the product path may link, load or call it.
 *
 * The forward is the recurrence of "5.3 Tensor Parallelism support and
 * large-cluster training", section 2.1, with A_t = a_t I (section 3.1), read as
 * in ssd_oracle.c:
 *   z_t = dt_t + dt_bias_h,  d_t = softplus(z_t),  a_t = exp(d_t A_h),
 *   h_t = a_t h_{t-1} + d_t B_t x_t^T,  y_t = C_t^T h_t + D_h x_t,
 * per (sequence, head), h_{-1} = init_state (or 0), final_state = h_last.  The
 * pages train these models (the backward pass is part of the training step they
 * describe) but print no gradient formulas; this file is the plain adjoint of
 * the forward above, derived by the chain rule.  For the scalar objective
 *   J = sum_t <dy_t, y_t> + <dfinal, final_state>
 * the adjoint state g_t = dJ/dh_t runs backwards in time:
 *   g_last = dfinal + C_last dy_last^T,   g_t = C_t dy_t^T + a_{t+1} g_{t+1},
 * and each input's gradient is read off the step that used it:
 *   dC_t = h_t dy_t                       dx_t = D dy_t + d_t g_t^T B_t
 *   dB_t = d_t g_t x_t                    dD  += <dy_t, x_t>
 *   dJ/da_t = <g_t, h_{t-1}>              dJ/dd_t = dJ/da_t a_t A + B_t^T g_t x_t
 *   dA  += dJ/da_t a_t d_t                dz_t = dJ/dd_t sigmoid(z_t)
 *   ddt_t = dz_t, ddt_bias += dz_t        dinit = a_first g_first
 * with B and C gradients summed over the heads of a group, and everything
 * restarted per packed sequence (the reset of section 4.3).
 *
 * Literal loops in double precision: the forward states are stored, then one
 * reverse sweep per (sequence, head).  Pinned in tests/test_oracle_bwd.py by
 * finite differences of the forward oracle, by automatic differentiation of a
 * separately written forward, by closed forms and by planted mistakes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

double oracle_softplus(double z); /* ssd_oracle.c */

static double sigmoid(double z) {
    if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
    const double e = exp(z);
    return e / (1.0 + e);
}

/*
 * Layouts as oracle_ssd_scan (row-major, double):
 *   x, dx (b, L, H, P); dt, ddt (b, L, H); B, C, dB, dC (b, L, G, N);
 *   dt_bias, A, D (H) (dt_bias, D may be NULL); init_state, dinit (S, H, N, P)
 *   (init_state may be NULL: zero); seq_idx int32 (L) with b == 1, or NULL;
 *   dy (b, L, H, P); dfinal (S, H, N, P) or NULL (zero);
 *   ddt_bias, dA, dD (H).  Every output is overwritten.
 * Returns 0, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_ssd_scan_bwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                        int64_t dstate, int64_t ngroups, int64_t nseqs,
                        const double *x, const double *dt, const double *dt_bias,
                        const double *A, const double *B, const double *C, const double *D,
                        const double *init_state, const int32_t *seq_idx,
                        const double *dy, const double *dfinal,
                        double *dx, double *ddt, double *ddt_bias, double *dA, double *dB,
                        double *dC, double *dD, double *dinit) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        nheads % ngroups != 0)
        return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen;
    const int64_t S = seq_idx ? nseqs : batch;
    if (seq_idx && batch != 1) return -1;
    if (!A || !dy || (batch * L > 0 && (!x || !dt || !B || !C))) return -1;
    if (!dx || !ddt || !ddt_bias || !dA || !dB || !dC || !dD || !dinit) return -1;

    memset(dx, 0, sizeof(double) * batch * L * H * P);
    memset(ddt, 0, sizeof(double) * batch * L * H);
    memset(ddt_bias, 0, sizeof(double) * H);
    memset(dA, 0, sizeof(double) * H);
    memset(dB, 0, sizeof(double) * batch * L * G * N);
    memset(dC, 0, sizeof(double) * batch * L * G * N);
    memset(dD, 0, sizeof(double) * H);
    memset(dinit, 0, sizeof(double) * S * H * N * P);

    double *hs = (double *)malloc(sizeof(double) * (L + 1) * N * P); /* h_{t0-1} .. h_{t1-1} */
    double *g = (double *)malloc(sizeof(double) * N * P);
    if (!hs || !g) { free(hs); free(g); return -2; }

    for (int64_t s = 0; s < S; ++s) {
        int64_t row, t0, t1;
        if (seq_idx) {
            row = 0;
            t0 = 0;
            while (t0 < L && seq_idx[t0] != s) t0++;
            t1 = t0;
            while (t1 < L && seq_idx[t1] == s) t1++;
        } else {
            row = s; t0 = 0; t1 = L;
        }
        for (int64_t h = 0; h < H; ++h) {
            const int64_t grp = h / (H / G);
            const double bias = dt_bias ? dt_bias[h] : 0.0;
            const double Ah = A[h];
            const double Dh = D ? D[h] : 0.0;
            /* forward, keeping every state: hs[k] = h_{t0 + k - 1} */
            if (init_state) memcpy(hs, init_state + (s * H + h) * N * P, sizeof(double) * N * P);
            else memset(hs, 0, sizeof(double) * N * P);
            for (int64_t t = t0; t < t1; ++t) {
                const int64_t tok = row * L + t;
                const double d = oracle_softplus(dt[tok * H + h] + bias);
                const double a = exp(d * Ah);
                const double *xt = x + (tok * H + h) * P;
                const double *Bt = B + (tok * G + grp) * N;
                const double *prev = hs + (t - t0) * N * P;
                double *cur = hs + (t - t0 + 1) * N * P;
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p)
                        cur[n * P + p] = a * prev[n * P + p] + d * Bt[n] * xt[p];
            }
            /* reverse sweep: g = dJ/dh_t, starting from dfinal */
            if (dfinal) memcpy(g, dfinal + (s * H + h) * N * P, sizeof(double) * N * P);
            else memset(g, 0, sizeof(double) * N * P);
            for (int64_t t = t1 - 1; t >= t0; --t) {
                const int64_t tok = row * L + t;
                const double z = dt[tok * H + h] + bias;
                const double d = oracle_softplus(z);
                const double a = exp(d * Ah);
                const double *xt = x + (tok * H + h) * P;
                const double *Bt = B + (tok * G + grp) * N;
                const double *Ct = C + (tok * G + grp) * N;
                const double *dyt = dy + (tok * H + h) * P;
                const double *prev = hs + (t - t0) * N * P;
                const double *cur = hs + (t - t0 + 1) * N * P;
                double *dxt = dx + (tok * H + h) * P;
                double *dBt = dB + (tok * G + grp) * N;
                double *dCt = dC + (tok * G + grp) * N;
                /* g_t = C_t dy_t^T + a_{t+1} g_{t+1} (g holds the carried part, or dfinal) */
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p) g[n * P + p] += Ct[n] * dyt[p];
                /* y_t = C_t^T h_t + D x_t */
                for (int64_t n = 0; n < N; ++n) {
                    double acc = 0.0;
                    for (int64_t p = 0; p < P; ++p) acc += cur[n * P + p] * dyt[p];
                    dCt[n] += acc;
                }
                for (int64_t p = 0; p < P; ++p) {
                    dD[h] += dyt[p] * xt[p];
                    dxt[p] += Dh * dyt[p];
                }
                /* h_t = a_t h_{t-1} + d_t B_t x_t^T */
                double da = 0.0, dd_input = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double gx = 0.0;
                    for (int64_t p = 0; p < P; ++p) {
                        da += g[n * P + p] * prev[n * P + p];
                        gx += g[n * P + p] * xt[p];
                    }
                    dBt[n] += d * gx;
                    dd_input += Bt[n] * gx;
                }
                for (int64_t p = 0; p < P; ++p) {
                    double gb = 0.0;
                    for (int64_t n = 0; n < N; ++n) gb += g[n * P + p] * Bt[n];
                    dxt[p] += d * gb;
                }
                const double dd = da * a * Ah + dd_input;
                dA[h] += da * a * d;
                const double dz = dd * sigmoid(z);
                ddt[tok * H + h] += dz;
                ddt_bias[h] += dz;
                /* carry: dJ/dh_{t-1} gets a_t g_t */
                for (int64_t e = 0; e < N * P; ++e) g[e] *= a;
            }
            /* g now holds dJ/dh_{t0-1} = dJ/d init_state */
            double *di = dinit + (s * H + h) * N * P;
            for (int64_t e = 0; e < N * P; ++e) di[e] = g[e];
        }
    }
    free(hs);
    free(g);
    return 0;
}
