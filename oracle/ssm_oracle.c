/*
 * ssm_oracle.c -- float64 CPU oracle for the selective state space (S6) scan.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this code. It shares no source, header,
 * table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes is the plain definition, written out as a sequential loop
 * over time for every channel, in double precision:
 *
 *   continuous model  h'(t) = A h(t) + B x(t),  y(t) = C h(t) + D x(t)
 *       [SSM glossary (yapayzekasozluk.tr), "Temel Matematiksel Cerceve"]
 *   selection         Delta_t = softplus(dt_raw_t + dt_bias), B_t, C_t per token,
 *                     A fixed and acting through Delta
 *       [Mamba summary (azimuth.plus), the selectivity paragraph]
 *   discretisation    zero-order hold: Abar = exp(Delta * A); Bbar = Delta * B
 *       (the pages name ZOH but print no Bbar formula; Delta * B is the reading
 *        used for the scan. The exact-ZOH Bbar = (exp(Delta A) - 1) / A * B is
 *        selectable because it is the form under which Theorem 1 holds exactly.)
 *   recurrence        h_t = Abar_t (.) h_{t-1} + Bbar_t x_t
 *       [Mamba summary, hardware-aware algorithm paragraph (parallel scan)]
 *   readout           y_t = C_t . h_t + D x_t  (after the update of h_t)
 *   gate              y_t <- y_t * silu(z_t),  silu(z) = z * sigma(z)
 *       [Mamba summary, block-architecture paragraph (gate branch: SiLU, multiply)]
 *   recurrent decode  one token: the same update with the state carried in place
 *       [SSM blog (shakilmahmud.com), section 3 "dual form": recurrence at O(1)]
 *   short convolution (optional, oracle_scan_conv_f64) the block's main branch runs
 *                     a short causal convolution (kernel width 4) and SiLU before the
 *                     selective SSM; the SSM's input, in Bbar x and in D x, is then
 *                     u_t = silu(conv_b + sum_{k=0..3} conv_w[d,k] x_{t-3+k}), one
 *                     filter per channel, x_tau for tau < 0 taken from conv_x0 (the
 *                     three tokens before the sequence, oldest first) or 0
 *       [Mamba summary, block-architecture paragraph: projection, 1-D convolution of
 *        kernel size 4, SiLU, selective SSM]
 *
 * Inputs are read in their storage type (float32, or bfloat16 given as raw
 * 16-bit patterns) and widened exactly to double, so a comparison measures the
 * error of the computation under test, not the quantisation of its inputs.
 *
 * Layouts (all row-major, contiguous):
 *   x, dt, z : [Bsz, L, Dm]     B, C : [Bsz, L, N]
 *   A : [Dm, N]   Dskip, dt_bias : [Dm]   h0, h_last : [Bsz, Dm, N]
 *   conv_w : [Dm, 4]   conv_b : [Dm]   conv_x0 : [Bsz, 3, Dm] (storage type of x)
 *   y (double) : [Bsz, L, Dm]
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DELTA_SOFTPLUS 1u /* Delta = softplus(dt + dt_bias); else Delta = dt + dt_bias */
#define ORACLE_EXACT_ZOH 2u      /* Bbar = (exp(Delta A) - 1) / A * B instead of Delta * B */
#define ORACLE_CONV_K 4          /* width of the short causal convolution */

/* Widen element i of a float32 (dtype 0) or bfloat16 (dtype 1) array to double. */
static double widen(const void *p, int dtype, int64_t i) {
    if (dtype == 0) return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* softplus(v) = log(1 + exp(v)), evaluated without overflow. */
static double softplus(double v) {
    return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v));
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

typedef struct {
    int64_t Bsz, L, Dm, N;
    int dtype;
    unsigned flags;
    const void *x, *dt, *z, *Bm, *Cm;
    const float *A, *Dskip, *dt_bias, *h0;
    double *y, *h_last;
    const double *h0_f64; /* optional double initial state (used by the decode oracle) */
    int64_t ch_begin, ch_end; /* channel range [begin, end) over b * Dm + d */
    const float *conv_w, *conv_b; /* optional short convolution: [Dm, 4] taps, [Dm] bias */
    const void *conv_x0;          /* [Bsz, 3, Dm] tokens before t = 0, or NULL for zeros */
} scan_job;

/* Raw input token x_tau of channel (b, d); tau in [-3, 0) reads conv_x0, else 0. */
static double raw_token(const scan_job *J, int64_t b, int64_t tau, int64_t d) {
    if (tau >= 0) return widen(J->x, J->dtype, (b * J->L + tau) * J->Dm + d);
    if (J->conv_x0) return widen(J->conv_x0, J->dtype, (b * (ORACLE_CONV_K - 1) + (tau + ORACLE_CONV_K - 1)) * J->Dm + d);
    return 0.0;
}

/* The SSM's input at step t after the block's causal convolution and SiLU:
   v = conv_b[d] + sum_k conv_w[d,k] x_{t-3+k} (tap 3 meets the current token), u = v sigma(v). */
static double conv_silu(const scan_job *J, int64_t b, int64_t t, int64_t d) {
    double v = J->conv_b ? (double)J->conv_b[d] : 0.0;
    for (int k = 0; k < ORACLE_CONV_K; k++)
        v += (double)J->conv_w[d * ORACLE_CONV_K + k] * raw_token(J, b, t - (ORACLE_CONV_K - 1) + k, d);
    return v * sigmoid(v);
}

/* One channel (b, d): the whole sequence, in time order. */
static void scan_channel(const scan_job *J, int64_t b, int64_t d, double *h) {
    const int64_t L = J->L, Dm = J->Dm, N = J->N;
    for (int64_t n = 0; n < N; n++) {
        int64_t hi = (b * Dm + d) * N + n;
        h[n] = J->h0_f64 ? J->h0_f64[hi] : (J->h0 ? (double)J->h0[hi] : 0.0);
    }
    const double bias = J->dt_bias ? (double)J->dt_bias[d] : 0.0;
    const double dskip = J->Dskip ? (double)J->Dskip[d] : 0.0;
    for (int64_t t = 0; t < L; t++) {
        const int64_t i = (b * L + t) * Dm + d;        /* token element (b, t, d) */
        const int64_t bc = (b * L + t) * N;            /* row of B_t and C_t      */
        const double v = widen(J->dt, J->dtype, i) + bias;
        const double delta = (J->flags & ORACLE_DELTA_SOFTPLUS) ? softplus(v) : v;
        const double xv = J->conv_w ? conv_silu(J, b, t, d) : widen(J->x, J->dtype, i);
        double y = 0.0;
        for (int64_t n = 0; n < N; n++) {
            const double a = (double)J->A[d * N + n];
            const double abar = exp(delta * a);
            double bbar;
            if (J->flags & ORACLE_EXACT_ZOH)
                bbar = (a != 0.0 ? expm1(delta * a) / a : delta) * widen(J->Bm, J->dtype, bc + n);
            else
                bbar = delta * widen(J->Bm, J->dtype, bc + n);
            h[n] = abar * h[n] + bbar * xv;
            y += widen(J->Cm, J->dtype, bc + n) * h[n];
        }
        y += dskip * xv;
        if (J->z) {
            const double zv = widen(J->z, J->dtype, i);
            y *= zv * sigmoid(zv);
        }
        J->y[i] = y;
    }
    if (J->h_last)
        for (int64_t n = 0; n < N; n++) J->h_last[(b * Dm + d) * N + n] = h[n];
}

static void *scan_worker(void *arg) {
    const scan_job *J = (const scan_job *)arg;
    double h[256];
    for (int64_t c = J->ch_begin; c < J->ch_end; c++) scan_channel(J, c / J->Dm, c % J->Dm, h);
    return NULL;
}

/* Run `base` over all its channels, split over `nthreads` POSIX threads
   (nthreads <= 1 runs on the calling thread). */
static void run_jobs(const scan_job *base, int nthreads) {
    const int64_t nch = base->ch_end - base->ch_begin;
    if (nthreads <= 1 || nch < 2) {
        scan_worker((void *)base);
        return;
    }
    if (nthreads > 512) nthreads = 512;
    if (nthreads > nch) nthreads = (int)nch;
    pthread_t tid[512];
    scan_job jobs[512];
    for (int k = 0; k < nthreads; k++) {
        jobs[k] = *base;
        jobs[k].ch_begin = base->ch_begin + nch * k / nthreads;
        jobs[k].ch_end = base->ch_begin + nch * (k + 1) / nthreads;
        if (pthread_create(&tid[k], NULL, scan_worker, &jobs[k]) != 0) {
            scan_worker(&jobs[k]); /* run inline if a thread cannot be started */
            tid[k] = 0;
        }
    }
    for (int k = 0; k < nthreads; k++)
        if (tid[k]) pthread_join(tid[k], NULL);
}

/*
 * Full-sequence scan. Returns 0 on success, -1 on invalid arguments.
 * Channels (b, d) are independent and are split over `nthreads` POSIX threads
 * (nthreads <= 1 runs on the calling thread). Each channel is one plain loop.
 */
int oracle_scan_f64(int64_t Bsz, int64_t L, int64_t Dm, int64_t N, int dtype, unsigned flags,
                    const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                    const float *A, const float *Dskip, const float *dt_bias, const float *h0,
                    double *y, double *h_last, int nthreads) {
    if (Bsz < 0 || L < 0 || Dm < 0 || N < 1 || N > 256 || (dtype != 0 && dtype != 1)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !y) return -1;
    scan_job base = {Bsz, L, Dm, N, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, h0,
                     y, h_last, NULL, 0, Bsz * Dm, NULL, NULL, NULL};
    run_jobs(&base, nthreads);
    return 0;
}

/*
 * The scan behind the block's short causal convolution and SiLU: as oracle_scan_f64,
 * with the SSM's input u_t = silu(conv_b + sum_k conv_w[d,k] x_{t-3+k}) (conv_w
 * [Dm, 4] required; conv_b [Dm] or NULL; conv_x0 [Bsz, 3, Dm] in x's storage type, or
 * NULL for zero tokens before t = 0).
 */
int oracle_scan_conv_f64(int64_t Bsz, int64_t L, int64_t Dm, int64_t N, int dtype, unsigned flags,
                         const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                         const float *A, const float *Dskip, const float *dt_bias, const float *h0,
                         const float *conv_w, const float *conv_b, const void *conv_x0,
                         double *y, double *h_last, int nthreads) {
    if (Bsz < 0 || L < 0 || Dm < 0 || N < 1 || N > 256 || (dtype != 0 && dtype != 1)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !y || !conv_w) return -1;
    scan_job base = {Bsz, L, Dm, N, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, h0,
                     y, h_last, NULL, 0, Bsz * Dm, conv_w, conv_b, conv_x0};
    run_jobs(&base, nthreads);
    return 0;
}

/*
 * One recurrent decode step for every (b, d): a scan of length 1 whose state is
 * read from and written back to `h` (double, [Bsz, Dm, N]). x, dt, z : [Bsz, Dm];
 * B, C : [Bsz, N]; y (double) : [Bsz, Dm]. Returns 0, or -1 on invalid arguments.
 */
int oracle_step_f64(int64_t Bsz, int64_t Dm, int64_t N, int dtype, unsigned flags,
                    const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                    const float *A, const float *Dskip, const float *dt_bias,
                    double *h, double *y, int nthreads) {
    if (Bsz < 0 || Dm < 0 || N < 1 || N > 256 || (dtype != 0 && dtype != 1)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !h || !y) return -1;
    /* A step is the scan with L = 1, started from h and writing its end state to h. */
    scan_job base = {Bsz, 1, Dm, N, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, NULL,
                     y, h, h, 0, Bsz * Dm, NULL, NULL, NULL};
    run_jobs(&base, nthreads);
    return 0;
}

/*
 * One decode step behind the block's short convolution: oracle_step_f64 with the SSM's
 * input u = silu(conv_b + sum_k conv_w[d,k] x_{t-3+k}), the three previous tokens read
 * from conv_state ([Bsz, 3, Dm], x's storage type, oldest first). The state itself is
 * left as it is (the caller shifts in the new token).
 */
int oracle_step_conv_f64(int64_t Bsz, int64_t Dm, int64_t N, int dtype, unsigned flags,
                         const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                         const float *A, const float *Dskip, const float *dt_bias,
                         const float *conv_w, const float *conv_b, const void *conv_state,
                         double *h, double *y, int nthreads) {
    if (Bsz < 0 || Dm < 0 || N < 1 || N > 256 || (dtype != 0 && dtype != 1)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !h || !y || !conv_w || !conv_state) return -1;
    scan_job base = {Bsz, 1, Dm, N, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, NULL,
                     y, h, h, 0, Bsz * Dm, conv_w, conv_b, conv_state};
    run_jobs(&base, nthreads);
    return 0;
}

/*
 * Weight of the input under the exact zero-order hold and its two derivatives, for one
 * state: w = (exp(Delta a) - 1) / a (w = Delta for a = 0), dw/dDelta = exp(Delta a), and
 * dw/da = Delta^2 f(Delta a) with f(s) = (s e^s - e^s + 1) / s^2. Near s = 0 the closed
 * form of f cancels, so there f is its Taylor series, the sum over k >= 0 of
 * (k + 1) s^k / (k + 2)! (differentiate w = Delta sum_k s^k / (k + 1)! term by term).
 */
static void zoh_weight(double delta, double a, double *w, double *dw_ddelta, double *dw_da) {
    const double s = delta * a;
    *dw_ddelta = exp(s);
    *w = a != 0.0 ? expm1(s) / a : delta;
    double f;
    if (fabs(s) < 0.25) {
        double term = 0.5, sum = 0.0; /* term_k = (k + 1) s^k / (k + 2)! */
        for (int k = 0; k < 24; k++) {
            sum += term;
            term *= s * (double)(k + 2) / ((double)(k + 1) * (double)(k + 3));
        }
        f = sum;
    } else {
        f = (s * exp(s) - expm1(s)) / (s * s);
    }
    *dw_da = delta * delta * f;
}

/*
 * Backward of the scan: the gradients of a loss with respect to every input, given
 * dL/dy (dy, storage type of the tokens) and optionally dL/dh_L (dh_last, double, or
 * NULL for 0). The pages print no backward formulas; the plain definition is the
 * derivative of the forward above, and this is reverse-mode differentiation of it,
 * written step by step. The Mamba summary's hardware-aware paragraph (recomputation)
 * says the backward recomputes the states instead of storing them; here, on the CPU,
 * each channel's forward states are simply kept for its reverse sweep.
 *
 * Per channel (b, d), with v_t = dt_t + bias, Delta_t = softplus(v_t) (or v_t),
 * Abar_tn = exp(Delta_t A_n), the SSM input u_t (x_t, or the short convolution's output),
 * the input weight w_tn = Delta_t (or, with ORACLE_EXACT_ZOH, (Abar_tn - 1) / A_n),
 * q_t = C_t . h_t + D u_t and y_t = q_t silu(z_t) (or q_t):
 *   dq_t = dy_t silu(z_t);  dz_t = dy_t q_t silu'(z_t)
 *   g_t  = dL/dh_t = dq_t C_t + Abar_{t+1} g_{t+1},  g_L = dq_L C_L + dh_last
 *   du_t = dq_t D + sum_n g_tn w_tn B_tn
 *   dDelta_t = sum_n g_tn (A_n Abar_tn h_{t-1,n} + dw_tn/dDelta B_tn u_t);  ddt_t = dDelta_t sigma(v_t)
 *   dA_n += g_tn (Delta_t Abar_tn h_{t-1,n} + dw_tn/dA_n B_tn u_t)
 *   dB_tn += g_tn w_tn u_t;  dC_tn += dq_t h_tn;  dD += dq_t u_t;  dbias += ddt_t;  dh0 = Abar_1 g_1
 * (dw/dDelta = 1 and dw/dA = 0 for w = Delta.) Without the convolution dx_t = du_t. With it,
 * u_t = silu(p_t), p_t = conv_b + sum_k conv_w[k] x_{t-3+k}, and dp_t = du_t silu'(p_t):
 *   dx_tau += conv_w[k] dp_t (tau = t-3+k; tau < 0 goes to dconv_x0[tau + 3])
 *   dconv_w[k] += dp_t x_{t-3+k};  dconv_b += dp_t
 * dB, dC ([Bsz, L, N]) sum over the channels of a sequence; dA ([Dm, N]), dD, dbias, dconv_w
 * and dconv_b over sequences and time. Single-threaded. Returns 0, or -1 on invalid arguments.
 */
int oracle_scan_bwd_conv_f64(int64_t Bsz, int64_t L, int64_t Dm, int64_t N, int dtype, unsigned flags,
                             const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                             const float *A, const float *Dskip, const float *dt_bias, const float *h0,
                             const float *conv_w, const float *conv_b, const void *conv_x0,
                             const void *dy, const double *dh_last, double *dx, double *ddt, double *dz,
                             double *dB, double *dC, double *dA, double *dD, double *dbias, double *dh0,
                             double *dconv_w, double *dconv_b, double *dconv_x0) {
    if (Bsz < 0 || L < 0 || Dm < 0 || N < 1 || N > 256 || (dtype != 0 && dtype != 1)) return -1;
    if (flags & ~(ORACLE_DELTA_SOFTPLUS | ORACLE_EXACT_ZOH)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !dy || !dx || !ddt || !dB || !dC || !dA || !dD || !dbias) return -1;
    if (z && !dz) return -1;
    if (!conv_w && (conv_b || conv_x0)) return -1;
    if (conv_w && (!dconv_w || !dconv_b || !dconv_x0)) return -1;
    const int softplus_on = (flags & ORACLE_DELTA_SOFTPLUS) != 0;
    const int zoh = (flags & ORACLE_EXACT_ZOH) != 0;
    memset(dx, 0, sizeof(double) * (size_t)(Bsz * L * Dm));
    memset(dB, 0, sizeof(double) * (size_t)(Bsz * L * N));
    memset(dC, 0, sizeof(double) * (size_t)(Bsz * L * N));
    memset(dA, 0, sizeof(double) * (size_t)(Dm * N));
    memset(dD, 0, sizeof(double) * (size_t)Dm);
    memset(dbias, 0, sizeof(double) * (size_t)Dm);
    if (conv_w) {
        memset(dconv_w, 0, sizeof(double) * (size_t)(Dm * ORACLE_CONV_K));
        memset(dconv_b, 0, sizeof(double) * (size_t)Dm);
        memset(dconv_x0, 0, sizeof(double) * (size_t)(Bsz * (ORACLE_CONV_K - 1) * Dm));
    }
    /* the convolution's inputs, read through the forward's own helpers */
    scan_job cj = {Bsz, L, Dm, N, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, h0,
                   NULL, NULL, NULL, 0, 0, conv_w, conv_b, conv_x0};
    /* forward states of one channel: hs[t * N + n] = h_{t-1,n} for t = 0..L (hs[0] = h0) */
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *delta = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *u = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *g = (double *)malloc(sizeof(double) * (size_t)N);
    if (!hs || !delta || !u || !g) {
        free(hs);
        free(delta);
        free(u);
        free(g);
        return -1;
    }
    for (int64_t b = 0; b < Bsz; b++) {
        for (int64_t d = 0; d < Dm; d++) {
            const double bias = dt_bias ? (double)dt_bias[d] : 0.0;
            const double dsk = Dskip ? (double)Dskip[d] : 0.0;
            for (int64_t n = 0; n < N; n++) hs[n] = h0 ? (double)h0[(b * Dm + d) * N + n] : 0.0;
            /* forward, keeping every state */
            for (int64_t t = 0; t < L; t++) {
                const int64_t i = (b * L + t) * Dm + d, bc = (b * L + t) * N;
                const double v = widen(dt, dtype, i) + bias;
                delta[t] = softplus_on ? softplus(v) : v;
                u[t] = conv_w ? conv_silu(&cj, b, t, d) : widen(x, dtype, i);
                for (int64_t n = 0; n < N; n++) {
                    const double a = (double)A[d * N + n];
                    double w = delta[t], wd, wa;
                    if (zoh) zoh_weight(delta[t], a, &w, &wd, &wa);
                    hs[(t + 1) * N + n] = exp(delta[t] * a) * hs[t * N + n] + w * widen(Bm, dtype, bc + n) * u[t];
                }
            }
            /* reverse */
            for (int64_t n = 0; n < N; n++) g[n] = dh_last ? dh_last[(b * Dm + d) * N + n] : 0.0;
            for (int64_t t = L - 1; t >= 0; t--) {
                const int64_t i = (b * L + t) * Dm + d, bc = (b * L + t) * N;
                const double xv = u[t];
                double q = dsk * xv;
                for (int64_t n = 0; n < N; n++) q += widen(Cm, dtype, bc + n) * hs[(t + 1) * N + n];
                double dq = widen(dy, dtype, i);
                if (z) {
                    const double zv = widen(z, dtype, i), sg = sigmoid(zv);
                    dz[i] = dq * q * sg * (1.0 + zv * (1.0 - sg));
                    dq *= zv * sg;
                }
                double dxv = dq * dsk, ddel = 0.0;
                dD[d] += dq * xv;
                for (int64_t n = 0; n < N; n++) {
                    const double a = (double)A[d * N + n], abar = exp(delta[t] * a);
                    const double bn = widen(Bm, dtype, bc + n), hp = hs[t * N + n];
                    double w = delta[t], w_dd = 1.0, w_da = 0.0;
                    if (zoh) zoh_weight(delta[t], a, &w, &w_dd, &w_da);
                    g[n] += dq * widen(Cm, dtype, bc + n);
                    dC[bc + n] += dq * hs[(t + 1) * N + n];
                    dxv += g[n] * w * bn;
                    ddel += g[n] * (a * abar * hp + w_dd * bn * xv);
                    dA[d * N + n] += g[n] * (delta[t] * abar * hp + w_da * bn * xv);
                    dB[bc + n] += g[n] * w * xv;
                    g[n] *= abar; /* now dL/dh_{t-1} through h_t */
                }
                const double v = widen(dt, dtype, i) + bias;
                ddt[i] = softplus_on ? ddel * sigmoid(v) : ddel;
                dbias[d] += ddt[i];
                if (conv_w) {
                    /* dx through the convolution: p_t from the taps, u = silu(p) */
                    double p = conv_b ? (double)conv_b[d] : 0.0;
                    for (int k = 0; k < ORACLE_CONV_K; k++)
                        p += (double)conv_w[d * ORACLE_CONV_K + k] * raw_token(&cj, b, t - (ORACLE_CONV_K - 1) + k, d);
                    const double sp = sigmoid(p), dp = dxv * sp * (1.0 + p * (1.0 - sp));
                    dconv_b[d] += dp;
                    for (int k = 0; k < ORACLE_CONV_K; k++) {
                        const int64_t tau = t - (ORACLE_CONV_K - 1) + k;
                        dconv_w[d * ORACLE_CONV_K + k] += dp * raw_token(&cj, b, tau, d);
                        const double dtok = dp * (double)conv_w[d * ORACLE_CONV_K + k];
                        if (tau >= 0)
                            dx[(b * L + tau) * Dm + d] += dtok;
                        else
                            dconv_x0[(b * (ORACLE_CONV_K - 1) + (tau + ORACLE_CONV_K - 1)) * Dm + d] += dtok;
                    }
                } else {
                    dx[i] = dxv;
                }
            }
            if (dh0)
                for (int64_t n = 0; n < N; n++) dh0[(b * Dm + d) * N + n] = g[n];
        }
    }
    free(hs);
    free(delta);
    free(u);
    free(g);
    return 0;
}

/* The backward without the short convolution (see oracle_scan_bwd_conv_f64). */
int oracle_scan_bwd_f64(int64_t Bsz, int64_t L, int64_t Dm, int64_t N, int dtype, unsigned flags,
                        const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                        const float *A, const float *Dskip, const float *dt_bias, const float *h0,
                        const void *dy, const double *dh_last, double *dx, double *ddt, double *dz,
                        double *dB, double *dC, double *dA, double *dD, double *dbias, double *dh0) {
    return oracle_scan_bwd_conv_f64(Bsz, L, Dm, N, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, h0, NULL,
                                    NULL, NULL, dy, dh_last, dx, ddt, dz, dB, dC, dA, dD, dbias, dh0, NULL, NULL,
                                    NULL);
}
