/*
 * Selective-scan forward ORACLE: plain, slow, float64, sequential in time.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the bench's CPU
 * baseline leg use it. It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes follows the recurrence spelled out on the page
 *   "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 *   (www.abhik.ai/papers/mamba), section "Original paper, equations and
 *   runnable CPU code", row "2. Retain, write and read each channel's state":
 *       a[t,c,n] = exp(delta[t,c] * A[c,n])
 *       h[t,c,n] = a[t,c,n] * h[t-1,c,n] + delta[t,c] * B[t,n] * x[t,c]
 *       y[t,c]   = sum_n C[t,n] * h[t,c,n] + D[c] * x[t,c]
 *   read AFTER the state update, with an optional incoming state; and row
 *   "1. Produce coefficients from the locally mixed input":
 *       delta = softplus(raw + b_delta),  A = -exp(A_log)
 *   and row "5. Put the selective operator inside the complete mixer":
 *       the scan result (D*x already included) is multiplied by SiLU(z).
 * The same loop, without D, is the sequential reference on the page
 *   "mamba, from scratch | khushi keswani", section "the scan".
 *
 * Readings taken where the pages leave a step open:
 *   - softplus is PyTorch's default F.softplus (beta 1, threshold 20: the
 *     identity above 20), the function the page's coefficient code calls;
 *   - the delta bias is added per channel before softplus; with the softplus
 *     flag off, delta = raw + bias as given;
 *   - D == NULL means no direct path (the page's d=None), z == NULL means no
 *     gate, h0 == NULL means a zero incoming state;
 *   - the write term is evaluated as (delta * B) * x, the page's order;
 *   - with write_zoh set, the write is the exact zero-order-hold input map
 *     instead: Bbar = (delta A)^-1 (exp(delta A) - 1) delta B, which for a
 *     diagonal A is expm1(delta A) / A * B per state ("Mamba: Linear-Time
 *     Sequence Modeling with Selective State Spaces", nadeemcite summary,
 *     section "Core Idea"; the abhik page's "There is a discretization detail
 *     worth keeping explicit"), and delta * B when A = 0 (its limit);
 *   - the readout sums n in ascending order.
 *
 * Layouts (all contiguous, row-major, float64):
 *   x, delta, z, y : [batch, seqlen, dim]        (dim = expanded channels E)
 *   B, C           : [batch, seqlen, dstate]     (shared by every channel)
 *   A_log          : [dim, dstate]
 *   D, delta_bias  : [dim]
 *   h0, h_last     : [batch, dim, dstate]
 *   states         : [batch, seqlen, dim, dstate]  (optional: every state)
 *
 * Parallelism: independent (batch, channel) pairs are spread over OpenMP
 * threads; each pair's loop over time stays strictly sequential.
 *
 * Further entry points, each with its own citation below: the decode step
 * (ssm_oracle_step), the scan with the causal convolution in front
 * (ssm_oracle_scan_conv) and the backward pass (ssm_oracle_scan_bwd).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* PyTorch F.softplus with its defaults (beta = 1, threshold = 20). */
static double softplus_default(double v)
{
    if (v > 20.0)
        return v;
    return log1p(exp(v));
}

/* SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* Step size for one (b, t, c): raw + bias, then softplus if enabled. */
double ssm_oracle_step_size(double raw, double bias, int delta_softplus)
{
    double v = raw + bias;
    return delta_softplus ? softplus_default(v) : v;
}

/* Retention a = exp(delta * A) with A = -exp(A_log). */
double ssm_oracle_retention(double step, double a_log)
{
    double A = -exp(a_log);
    return exp(step * A);
}

/*
 * Returns 0 on success, -1 on a bad argument (NULL required pointer or a
 * non-positive size). The output y must not alias any input.
 */
int ssm_oracle_scan_ex(int64_t batch, int64_t seqlen, int64_t dim,
                       int64_t dstate, const double *x, const double *delta,
                       const double *A_log, const double *B, const double *C,
                       const double *D, const double *z,
                       const double *delta_bias, int delta_softplus,
                       int write_zoh, const double *h0, double *y,
                       double *h_last, double *states, int nthreads);

/* Exact zero-order-hold input factor expm1(step A) / A (step when A = 0). */
static double zoh_factor(double step, double A)
{
    if (A == 0.0)
        return step;
    return expm1(step * A) / A;
}

int ssm_oracle_scan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                    const double *x, const double *delta, const double *A_log,
                    const double *B, const double *C, const double *D,
                    const double *z, const double *delta_bias,
                    int delta_softplus, const double *h0,
                    double *y, double *h_last, double *states, int nthreads)
{
    return ssm_oracle_scan_ex(batch, seqlen, dim, dstate, x, delta, A_log, B,
                              C, D, z, delta_bias, delta_softplus, 0, h0, y,
                              h_last, states, nthreads);
}

int ssm_oracle_scan_ex(int64_t batch, int64_t seqlen, int64_t dim,
                       int64_t dstate, const double *x, const double *delta,
                       const double *A_log, const double *B, const double *C,
                       const double *D, const double *z,
                       const double *delta_bias, int delta_softplus,
                       int write_zoh, const double *h0, double *y,
                       double *h_last, double *states, int nthreads)
{
    if (!x || !delta || !A_log || !B || !C || !y)
        return -1;
    if (batch <= 0 || seqlen <= 0 || dim <= 0 || dstate <= 0)
        return -1;

    const int64_t pairs = batch * dim;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#else
    (void)nthreads;
#endif
    for (int64_t p = 0; p < pairs; ++p) {
        const int64_t b = p / dim;
        const int64_t c = p % dim;
        double *A = (double *)malloc((size_t)dstate * sizeof(double));
        double *h = (double *)malloc((size_t)dstate * sizeof(double));
        for (int64_t n = 0; n < dstate; ++n) {
            A[n] = -exp(A_log[c * dstate + n]);
            h[n] = h0 ? h0[(b * dim + c) * dstate + n] : 0.0;
        }
        const double bias = delta_bias ? delta_bias[c] : 0.0;
        for (int64_t t = 0; t < seqlen; ++t) {
            const int64_t i = (b * seqlen + t) * dim + c;   /* [b, t, c] */
            const int64_t r = (b * seqlen + t) * dstate;    /* row of B, C */
            const double v = delta[i] + bias;
            const double step = delta_softplus ? softplus_default(v) : v;
            const double xv = x[i];
            for (int64_t n = 0; n < dstate; ++n) {
                const double retention = exp(step * A[n]);
                const double write =
                    (write_zoh ? zoh_factor(step, A[n]) : step) * B[r + n] * xv;
                h[n] = retention * h[n] + write;
            }
            if (states) {
                double *s = states + ((b * seqlen + t) * dim + c) * dstate;
                for (int64_t n = 0; n < dstate; ++n)
                    s[n] = h[n];
            }
            double out = 0.0;
            for (int64_t n = 0; n < dstate; ++n)
                out += C[r + n] * h[n];
            if (D)
                out += D[c] * xv;
            if (z)
                out *= silu(z[i]);
            y[i] = out;
        }
        if (h_last)
            for (int64_t n = 0; n < dstate; ++n)
                h_last[(b * dim + c) * dstate + n] = h[n];
        free(A);
        free(h);
    }
    return 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int ssm_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One decode step for a batch of sequences, float64 ("Mamba: Linear-Time
 * Sequence Modeling with Selective State Spaces", www.abhik.ai/papers/mamba,
 * section "Original paper, equations and runnable CPU code", row "6. Carry
 * both buffers to the next token", and row "4. Add causal local context
 * before selecting coefficients"):
 *   conv_state <- shift left by one, append x_new     (K samples, the last
 *                                                      one is the newest)
 *   x  = SiLU(sum_k conv_state[k] * w[c, k] + conv_bias[c])
 *   delta = softplus(raw + delta_bias)  (or raw + bias), A = -exp(A_log)
 *   state <- exp(delta A) * state + delta * B * x  (or the zero-order-hold
 *            write, as in ssm_oracle_scan_ex)
 *   y  = sum_n C[n] * state[n] + D[c] * x, then y *= SiLU(z)
 * With conv_state == NULL the convolution is skipped and x = x_new.
 * Layouts: x_new, delta, z, y: [batch, dim]; conv_state: [batch, dim, K];
 * conv_weight: [dim, K]; conv_bias, D, delta_bias: [dim]; B, C: [batch,
 * dstate]; A_log: [dim, dstate]; state: [batch, dim, dstate]. conv_state and
 * state are updated in place. Returns 0, or -1 on a bad argument.
 */
int ssm_oracle_step(int64_t batch, int64_t dim, int64_t dstate, int64_t width,
                    const double *x_new, double *conv_state,
                    const double *conv_weight, const double *conv_bias,
                    const double *delta, const double *delta_bias,
                    int delta_softplus, int write_zoh, const double *A_log,
                    const double *B, const double *C, const double *D,
                    const double *z, double *state, double *y)
{
    if (!x_new || !delta || !A_log || !B || !C || !state || !y)
        return -1;
    if (batch <= 0 || dim <= 0 || dstate <= 0)
        return -1;
    if (conv_state && (!conv_weight || width <= 0))
        return -1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t c = 0; c < dim; ++c) {
            const int64_t i = b * dim + c;
            double xv = x_new[i];
            if (conv_state) {
                double *buf = conv_state + i * width;
                for (int64_t k = 0; k + 1 < width; ++k)
                    buf[k] = buf[k + 1];
                buf[width - 1] = x_new[i];
                double acc = conv_bias ? conv_bias[c] : 0.0;
                for (int64_t k = 0; k < width; ++k)
                    acc += buf[k] * conv_weight[c * width + k];
                xv = silu(acc);
            }
            const double v = delta[i] + (delta_bias ? delta_bias[c] : 0.0);
            const double step = delta_softplus ? softplus_default(v) : v;
            double out = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                const double A = -exp(A_log[c * dstate + n]);
                const double retention = exp(step * A);
                const double write =
                    (write_zoh ? zoh_factor(step, A) : step) * B[b * dstate + n]
                    * xv;
                double *h = state + i * dstate + n;
                *h = retention * *h + write;
                out += C[b * dstate + n] * *h;
            }
            if (D)
                out += D[c] * xv;
            if (z)
                out *= silu(z[i]);
            y[i] = out;
        }
    }
    return 0;
}

/*
 * The scan with the causal depthwise convolution in front ("Mamba:
 * Linear-Time Sequence Modeling with Selective State Spaces",
 * www.abhik.ai/papers/mamba, section "Original paper, equations and runnable
 * CPU code", row "4. Add causal local context before selecting
 * coefficients" and row "5. Put the selective operator inside the complete
 * mixer"):
 *   x[t, c] = SiLU(conv_bias[c] + sum_{k<K} w[c, k] * v[t - K + 1 + k, c])
 * with zeros before the start (left padding), then ssm_oracle_scan_ex on x
 * (D x and the gate use this x). v: [batch, seqlen, dim]; w: [dim, K].
 */
int ssm_oracle_scan_conv(int64_t batch, int64_t seqlen, int64_t dim,
                         int64_t dstate, int64_t width, const double *v,
                         const double *conv_weight, const double *conv_bias,
                         const double *delta, const double *A_log,
                         const double *B, const double *C, const double *D,
                         const double *z, const double *delta_bias,
                         int delta_softplus, int write_zoh, const double *h0,
                         double *y, double *h_last, int nthreads)
{
    if (!v || !conv_weight || width <= 0 || batch <= 0 || seqlen <= 0 ||
        dim <= 0)
        return -1;
    const int64_t n = batch * seqlen * dim;
    double *x = (double *)malloc((size_t)n * sizeof(double));
    if (!x)
        return -1;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t t = 0; t < seqlen; ++t)
            for (int64_t c = 0; c < dim; ++c) {
                double acc = conv_bias ? conv_bias[c] : 0.0;
                for (int64_t k = 0; k < width; ++k) {
                    const int64_t s = t - width + 1 + k;
                    if (s >= 0)
                        acc += conv_weight[c * width + k] *
                               v[(b * seqlen + s) * dim + c];
                }
                x[(b * seqlen + t) * dim + c] = silu(acc);
            }
    const int rc = ssm_oracle_scan_ex(batch, seqlen, dim, dstate, x, delta,
                                      A_log, B, C, D, z, delta_bias,
                                      delta_softplus, write_zoh, h0, y, h_last,
                                      NULL, nthreads);
    free(x);
    return rc;
}

/*
 * Backward pass of ssm_oracle_scan_ex: the gradients of
 *   loss = sum dy_out * y_out + sum dh_last * h_last
 * with respect to every input, by reverse-mode differentiation of the same
 * recurrence ("Mamba: Linear-Time Sequence Modeling with Selective State
 * Spaces", www.abhik.ai/papers/mamba, rows "1. Produce coefficients from the
 * locally mixed input", "2. Retain, write and read each channel's state" and
 * "5. Put the selective operator inside the complete mixer"; the pages
 * describe training through the scan by recomputing the states on the way
 * back instead of storing them, section "Compose the updates instead of
 * waiting for every state").
 *
 * Per (b, e), with s = step size, a_n = exp(s A_n), w_n the write, the
 * adjoint lam_n = d loss / d h_t[n] runs backwards in time:
 *   g = dy_out[t]; dy = g SiLU(z) (g without a gate);
 *   dz = g (C.h + D x) SiLU'(z);
 *   lam_n += dy C[n];  dC[n] += dy h_t[n];  dD += dy x;  dx += dy D;
 *   dw_n = lam_n;  da_n = lam_n h_{t-1}[n];
 *   write s B x:          ds += sum lam B x;  dB += lam s x;  dx += sum lam s B;
 *   write expm1(sA)/A B x (f = expm1(sA)/A, df/ds = a, df/dA = (s a - f)/A):
 *                         ds += sum lam B x a; dB += lam f x; dx += sum lam f B;
 *                         dA += lam B x (s a - f) / A;
 *   retention:            ds += sum da a A;  dA += da a s;
 *   lam_n <- lam_n a_n    (on to h_{t-1});
 *   draw = ds sigmoid(raw + bias) (ds without softplus); dbias += draw;
 * and at the start dh0 = lam. Finally dA_log = dA A (A = -exp(A_log)).
 * The states h_t are recomputed forward per channel first.
 *
 * Outputs (all written; dB, dC, dA_log, dD, ddelta_bias are sums):
 *   dx, ddelta, dz [batch, seqlen, dim]; dB, dC [batch, seqlen, dstate];
 *   dA_log [dim, dstate]; dD, ddelta_bias [dim]; dh0 [batch, dim, dstate].
 * dz may be NULL when z is; dD when D is; ddelta_bias when delta_bias is;
 * dh0 may be NULL. dh_last may be NULL (zero).
 */
int ssm_oracle_scan_bwd(int64_t batch, int64_t seqlen, int64_t dim,
                        int64_t dstate, const double *x, const double *delta,
                        const double *A_log, const double *B, const double *C,
                        const double *D, const double *z,
                        const double *delta_bias, int delta_softplus,
                        int write_zoh, const double *h0, const double *dy_out,
                        const double *dh_last, double *dx, double *ddelta,
                        double *dA_log, double *dB, double *dC, double *dD,
                        double *dz, double *ddelta_bias, double *dh0,
                        int nthreads)
{
    if (!x || !delta || !A_log || !B || !C || !dy_out || !dx || !ddelta ||
        !dA_log || !dB || !dC)
        return -1;
    if ((z && !dz) || (D && !dD) || (delta_bias && !ddelta_bias))
        return -1;
    if (batch <= 0 || seqlen <= 0 || dim <= 0 || dstate <= 0)
        return -1;
    const int64_t L = seqlen, E = dim, N = dstate;
    memset(dB, 0, (size_t)(batch * L * N) * sizeof(double));
    memset(dC, 0, (size_t)(batch * L * N) * sizeof(double));
    memset(dA_log, 0, (size_t)(E * N) * sizeof(double));
    if (dD)
        memset(dD, 0, (size_t)E * sizeof(double));
    if (ddelta_bias)
        memset(ddelta_bias, 0, (size_t)E * sizeof(double));
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#else
    (void)nthreads;
#endif
    int fail = 0;
    for (int64_t b = 0; b < batch; ++b) {
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
        {
            /* private sums over channels of dB and dC for this batch row */
            double *pB = (double *)calloc((size_t)(L * N), sizeof(double));
            double *pC = (double *)calloc((size_t)(L * N), sizeof(double));
            double *hs = (double *)malloc((size_t)((L + 1) * N) * sizeof(double));
            double *A = (double *)malloc((size_t)N * sizeof(double));
            double *dA = (double *)malloc((size_t)N * sizeof(double));
            double *lam = (double *)malloc((size_t)N * sizeof(double));
            if (!pB || !pC || !hs || !A || !dA || !lam) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                fail = 1;
            } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
                for (int64_t c = 0; c < E; ++c) {
                    const double bias = delta_bias ? delta_bias[c] : 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        A[n] = -exp(A_log[c * N + n]);
                        dA[n] = 0.0;
                        hs[n] = h0 ? h0[(b * E + c) * N + n] : 0.0;
                    }
                    /* forward: hs[(t + 1) N + n] = h_t[n] */
                    for (int64_t t = 0; t < L; ++t) {
                        const int64_t i = (b * L + t) * E + c;
                        const int64_t r = (b * L + t) * N;
                        const double v = delta[i] + bias;
                        const double s = delta_softplus ? softplus_default(v) : v;
                        for (int64_t n = 0; n < N; ++n) {
                            const double f =
                                write_zoh ? zoh_factor(s, A[n]) : s;
                            hs[(t + 1) * N + n] = exp(s * A[n]) * hs[t * N + n] +
                                                  f * B[r + n] * x[i];
                        }
                    }
                    for (int64_t n = 0; n < N; ++n)
                        lam[n] = dh_last ? dh_last[(b * E + c) * N + n] : 0.0;
                    double sum_dD = 0.0, sum_dbias = 0.0;
                    for (int64_t t = L - 1; t >= 0; --t) {
                        const int64_t i = (b * L + t) * E + c;
                        const int64_t r = (b * L + t) * N;
                        const double v = delta[i] + bias;
                        const double s = delta_softplus ? softplus_default(v) : v;
                        const double xv = x[i];
                        const double *h = hs + (t + 1) * N;
                        const double *hp = hs + t * N;
                        const double g = dy_out[i];
                        double dy = g;
                        if (z) {
                            double pre = D ? D[c] * xv : 0.0;
                            for (int64_t n = 0; n < N; ++n)
                                pre += C[r + n] * h[n];
                            const double sg = 1.0 / (1.0 + exp(-z[i]));
                            dy = g * z[i] * sg;
                            dz[i] = g * pre * sg * (1.0 + z[i] * (1.0 - sg));
                        }
                        double dxv = D ? dy * D[c] : 0.0;
                        if (D)
                            sum_dD += dy * xv;
                        double ds = 0.0;
                        for (int64_t n = 0; n < N; ++n) {
                            pC[t * N + n] += dy * h[n];
                            lam[n] += dy * C[r + n];
                            const double a = exp(s * A[n]);
                            const double da = lam[n] * hp[n];
                            if (write_zoh) {
                                const double f = zoh_factor(s, A[n]);
                                ds += lam[n] * B[r + n] * xv * a;
                                pB[t * N + n] += lam[n] * f * xv;
                                dxv += lam[n] * f * B[r + n];
                                dA[n] += lam[n] * B[r + n] * xv *
                                         (s * a - f) / A[n];
                            } else {
                                ds += lam[n] * B[r + n] * xv;
                                pB[t * N + n] += lam[n] * s * xv;
                                dxv += lam[n] * s * B[r + n];
                            }
                            ds += da * a * A[n];
                            dA[n] += da * a * s;
                            lam[n] *= a;
                        }
                        const double draw =
                            delta_softplus ? ds / (1.0 + exp(-v)) : ds;
                        ddelta[i] = draw;
                        sum_dbias += draw;
                        dx[i] = dxv;
                    }
                    if (dh0)
                        for (int64_t n = 0; n < N; ++n)
                            dh0[(b * E + c) * N + n] = lam[n];
                    /* channel c is this thread's alone within batch row b */
                    for (int64_t n = 0; n < N; ++n)
                        dA_log[c * N + n] += dA[n] * A[n];
                    if (dD)
                        dD[c] += sum_dD;
                    if (ddelta_bias)
                        ddelta_bias[c] += sum_dbias;
                }
#ifdef _OPENMP
#pragma omp critical
#endif
                {
                    for (int64_t k = 0; k < L * N; ++k) {
                        dB[b * L * N + k] += pB[k];
                        dC[b * L * N + k] += pC[k];
                    }
                }
            }
            free(pB);
            free(pC);
            free(hs);
            free(A);
            free(dA);
            free(lam);
        }
    }
    return fail ? -1 : 0;
}
