/*
 * axon_ssm_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * A plain, slow, single-threaded fp64 CPU statement of the selective-scan (S6)
 * layer core (a second build of this file with -fopenmp runs independent
 * channels on several host cores, with each channel's arithmetic unchanged) described on the page "Axon-SSM: Selective State Space Model for
 * Apple Silicon" (bit-axon docs).  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library; neither includes the other.
 *
 * What it computes, per batch row b and channel e, in the pages' order:
 *   1. xpad = conv_cache[b,:,e] (or zeros) followed by x[b,:,e]
 *      ("Autoregressive decoding": conv_cache holds the last K-1 inputs).
 *   2. for t = 0..L-1
 *        xc  = conv_b[e] + sum_k conv_w[e,k] * xpad[t+k]      (causal depthwise
 *              conv1d, cross-correlation orientation: tap K-1 meets x_t)
 *        u   = SiLU(xc)                                         ("Gating", SiLU)
 *        dt  = clip(softplus(dt_raw + dt_bias[e]), 1e-4, 100)   ("Selective
 *              mechanism": epsilon = 1e-4, dt_max = 100.0)
 *        A_n = -exp(A_log[e,n])                                 ("Diagonal state
 *              matrix")
 *        abar_n = exp(dt * A_n);  bbar_n = dt * B[b,t,n]        (first-order
 *              discretisation used by Axon-SSM; ZOH alternative behind a flag)
 *        h_n = abar_n * h_n + bbar_n * u                        (recurrence)
 *        y_ssm = sum_n C[b,t,n] * h_n + D[e] * u
 *        y   = y_ssm * SiLU(z)                                  (output gate)
 *   3. final h -> ssm_state_out (B,E,N); last K-1 entries of xpad -> conv_cache_out.
 *
 * Layouts (row-major, last index fastest): x,z,dt_raw,y (B,L,E); Bm,Cm (B,L,N);
 * conv_w (E,K); conv_b,dt_bias,D (E); A_log (E,N); conv_cache (B,K-1,E);
 * ssm_state (B,E,N).  NULL conv_cache_in / ssm_state_in mean zeros.
 * conv_cache_out / ssm_state_out may be the same arrays as the inputs.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_DT_MIN 1e-4   /* epsilon of the dt clip ("Selective mechanism") */
#define ORACLE_DT_MAX 100.0  /* dt_max of the dt clip */

/* softplus(v) = log(1 + exp(v)), evaluated without overflow. */
static double softplus(double v)
{
    if (v > 0.0) return v + log1p(exp(-v));
    return log1p(exp(v));
}

double oracle_silu(double v) { return v / (1.0 + exp(-v)); }

/* dt = clip(softplus(v), 1e-4, 100), bounds inclusive. */
double oracle_dt(double v)
{
    double sp = softplus(v);
    if (sp < ORACLE_DT_MIN) sp = ORACLE_DT_MIN;
    if (sp > ORACLE_DT_MAX) sp = ORACLE_DT_MAX;
    return sp;
}

/*
 * Scan core only (no conv, no gate): the recurrence h_t = abar*h_{t-1} + bbar*u_t,
 * y_t = C_t . h_t + D*u_t for one channel, with per-step dt.  This is the toy
 * `selective_scan(u, delta, A, B, C)` of the wiki page "Selective State Space
 * Models (Mamba)" extended by the D skip.  zoh = 0: bbar = dt*B (Axon-SSM);
 * zoh = 1: bbar = (exp(dt*A) - 1)/A * B (exact zero-order hold, diagonal form).
 *   u, dt: (L);  A: (N) (the diagonal itself, negative);  Bm, Cm: (L,N);
 *   h: (N) initial state in, final state out;  y: (L).
 */
void oracle_scan_core(int L, int N, const double *u, const double *dt,
                      const double *A, const double *Bm, const double *Cm,
                      double D, int zoh, double *h, double *y)
{
    for (int t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
            double abar = exp(dt[t] * A[n]);
            double bbar = zoh ? expm1(dt[t] * A[n]) / A[n] * Bm[(size_t)t * N + n]
                              : dt[t] * Bm[(size_t)t * N + n];
            h[n] = abar * h[n] + bbar * u[t];
            acc += Cm[(size_t)t * N + n] * h[n];
        }
        y[t] = acc + D * u[t];
    }
}

/*
 * Steps 1-3 above for one (b, e) channel.  Scratch: xpad holds L + K - 1
 * values, h and A hold N.  Channels share nothing, so the caller may run them
 * in any order (or at the same time) on the same arrays.
 */
static void oracle_channel(int b, int e, int L, int E, int N, int K,
                           const double *x, const double *z, const double *dt_raw,
                           const double *Bm, const double *Cm,
                           const double *conv_w, const double *conv_b,
                           const double *dt_bias, const double *A_log, const double *D,
                           const double *conv_cache_in, const double *ssm_state_in,
                           double *y, double *conv_cache_out, double *ssm_state_out,
                           int zoh, double *xpad, double *h, double *A)
{
    const int KM1 = K - 1;
    /* 1. padded input stream for this channel */
    for (int j = 0; j < KM1; ++j)
        xpad[j] = conv_cache_in ? conv_cache_in[((size_t)b * KM1 + j) * E + e] : 0.0;
    for (int t = 0; t < L; ++t)
        xpad[KM1 + t] = x[((size_t)b * L + t) * E + e];
    for (int n = 0; n < N; ++n) {
        h[n] = ssm_state_in ? ssm_state_in[((size_t)b * E + e) * N + n] : 0.0;
        A[n] = -exp(A_log[(size_t)e * N + n]);
    }
    /* 2. the per-step update */
    for (int t = 0; t < L; ++t) {
        size_t idx = ((size_t)b * L + t) * E + e;
        double xc = conv_b[e];
        for (int k = 0; k < K; ++k) xc += conv_w[(size_t)e * K + k] * xpad[t + k];
        double u = oracle_silu(xc);
        double dt = oracle_dt(dt_raw[idx] + dt_bias[e]);
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
            size_t bn = ((size_t)b * L + t) * N + n;
            double abar = exp(dt * A[n]);
            double bbar = zoh ? expm1(dt * A[n]) / A[n] * Bm[bn] : dt * Bm[bn];
            h[n] = abar * h[n] + bbar * u;
            acc += Cm[bn] * h[n];
        }
        double y_ssm = acc + D[e] * u;
        y[idx] = y_ssm * oracle_silu(z[idx]);
    }
    /* 3. final caches (written after all reads, so in == out is fine) */
    for (int j = 0; j < KM1; ++j)
        conv_cache_out[((size_t)b * KM1 + j) * E + e] = xpad[L + j];
    for (int n = 0; n < N; ++n)
        ssm_state_out[((size_t)b * E + e) * N + n] = h[n];
}

/*
 * The layer core over a whole sequence (prefill).  Returns 0 on success,
 * -1 on bad sizes or a failed temporary allocation.
 *
 * The default build is one plain loop over the channels.  A second build of
 * this same file with -fopenmp hands the channels to the host's cores (the
 * pragma below is ignored otherwise); each channel's arithmetic is the same
 * either way, so both builds give identical bits.
 */
int oracle_ssm_scan_fwd(int B, int L, int E, int N, int K,
                        const double *x, const double *z, const double *dt_raw,
                        const double *Bm, const double *Cm,
                        const double *conv_w, const double *conv_b,
                        const double *dt_bias, const double *A_log, const double *D,
                        const double *conv_cache_in, const double *ssm_state_in,
                        double *y, double *conv_cache_out, double *ssm_state_out,
                        int zoh)
{
    if (B < 0 || L < 0 || E < 0 || N <= 0 || K <= 0) return -1;
    int failed = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 4) reduction(| : failed)
    for (int b = 0; b < B; ++b) {
        for (int e = 0; e < E; ++e) {
            double *xpad = (double *)malloc(sizeof(double) * ((size_t)L + K - 1));
            double *h = (double *)malloc(sizeof(double) * (size_t)N);
            double *A = (double *)malloc(sizeof(double) * (size_t)N);
            if (xpad && h && A)
                oracle_channel(b, e, L, E, N, K, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias,
                               A_log, D, conv_cache_in, ssm_state_in, y, conv_cache_out,
                               ssm_state_out, zoh, xpad, h, A);
            else
                failed = 1;
            free(xpad); free(h); free(A);
        }
    }
    return failed ? -1 : 0;
}

/* Host threads the channel loop uses: 1 in the default build. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One cached decode step (the prefill with L = 1), caches updated in place:
 *   x, z, dt_raw, y: (B,E);  Bm, Cm: (B,N);  conv_cache (B,K-1,E);  ssm_state (B,E,N).
 */
int oracle_ssm_step(int B, int E, int N, int K,
                    const double *x, const double *z, const double *dt_raw,
                    const double *Bm, const double *Cm,
                    const double *conv_w, const double *conv_b,
                    const double *dt_bias, const double *A_log, const double *D,
                    double *conv_cache, double *ssm_state, double *y, int zoh)
{
    return oracle_ssm_scan_fwd(B, 1, E, N, K, x, z, dt_raw, Bm, Cm, conv_w, conv_b,
                               dt_bias, A_log, D, conv_cache, ssm_state,
                               y, conv_cache, ssm_state, zoh);
}

/*
 * The conv + SiLU stage alone (steps 1-2 above without the recurrence):
 * u[b,t,e] = SiLU(conv_b[e] + sum_k conv_w[e,k] * x[b, t+k-(K-1), e]), with
 * times before 0 read from conv_cache_in (or zeros).  In the full layer this
 * u is the input of the projection f_proj that produces dt, B and C (Axon-SSM
 * page, "Selective mechanism": the projection starts from the conv output).
 */
int oracle_conv_silu(int B, int L, int E, int K, const double *x, const double *conv_w,
                     const double *conv_b, const double *conv_cache_in, double *u)
{
    if (B < 0 || L < 0 || E < 0 || K <= 0) return -1;
    const int KM1 = K - 1;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < L; ++t)
            for (int e = 0; e < E; ++e) {
                double acc = conv_b[e];
                for (int k = 0; k < K; ++k) {
                    const int s = t + k - KM1;          /* input time met by tap k */
                    double xv = 0.0;
                    if (s >= 0)
                        xv = x[((size_t)b * L + s) * E + e];
                    else if (conv_cache_in)
                        xv = conv_cache_in[((size_t)b * KM1 + (KM1 + s)) * E + e];
                    acc += conv_w[(size_t)e * K + k] * xv;
                }
                u[((size_t)b * L + t) * E + e] = oracle_silu(acc);
            }
    return 0;
}

/*
 * The Mamba-2 (SSD) layer core, one scalar decay per head (wiki page
 * "Selective State Space Models (Mamba)", section "Mamba-2 block (SSD)":
 * d_state 128, headdim 64; the SSD article: a structured SSM whose state is
 * carried token to token).  Per batch row b and head h, state S (P x N):
 *   dt  = clip(softplus(dt_raw[b,t,h] + dt_bias[h]), 1e-4, 100)
 *   a   = exp(dt * A_h),  A_h = -exp(A_log[h])
 *   S[p][n] = a * S[p][n] + dt * x[b,t,h,p] * B[b,t,n]
 *   y[b,t,h,p] = sum_n S[p][n] * C[b,t,n] + D[h] * x[b,t,h,p]
 * Layouts: x, y (B,L,H,P); dt_raw (B,L,H); B, C (B,L,N) shared by all heads;
 * dt_bias, A_log, D (H); h0, h_out (B,H,P,N), h0 may be NULL (zeros).
 */
int oracle_ssd_scan(int B, int L, int H, int P, int N, const double *x, const double *dt_raw,
                    const double *dt_bias, const double *A_log, const double *Bm, const double *Cm,
                    const double *D, const double *h0, double *y, double *h_out)
{
    if (B < 0 || L < 0 || H < 0 || P <= 0 || N <= 0) return -1;
    double *S = (double *)malloc(sizeof(double) * (size_t)P * N);
    if (!S) return -1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const double A = -exp(A_log[h]);
            for (int i = 0; i < P * N; ++i) S[i] = h0 ? h0[((size_t)b * H + h) * P * N + i] : 0.0;
            for (int t = 0; t < L; ++t) {
                const double dt = oracle_dt(dt_raw[((size_t)b * L + t) * H + h] + dt_bias[h]);
                const double a = exp(dt * A);
                const double *xv = x + (((size_t)b * L + t) * H + h) * P;
                const double *Bt = Bm + ((size_t)b * L + t) * N;
                const double *Ct = Cm + ((size_t)b * L + t) * N;
                double *yv = y + (((size_t)b * L + t) * H + h) * P;
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) {
                        double *s = S + (size_t)p * N + n;
                        *s = a * *s + dt * xv[p] * Bt[n];
                        acc += *s * Ct[n];
                    }
                    yv[p] = acc + D[h] * xv[p];
                }
            }
            for (int i = 0; i < P * N; ++i) h_out[((size_t)b * H + h) * P * N + i] = S[i];
        }
    free(S);
    return 0;
}
