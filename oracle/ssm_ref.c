/*
 * ssm_ref.c -- float64 CPU oracle for the selective state-space scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the package smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or table with the CUDA library.
 *
 * What it computes is the plain definition, one channel at a time, strictly
 * sequential in time and in double precision:
 *
 *   v_t      = delta[b,d,t] + delta_bias[d]
 *   dt_t     = softplus(v_t) = log(1 + e^v_t)        (or v_t when softplus == 0)
 *   Abar     = exp(dt_t * A[d,n])                     zero-order hold of A
 *   Bbar x   = dt_t * B[b,n,t] * x[b,d,t]             Euler step for the input
 *   h_t[n]   = Abar * h_{t-1}[n] + Bbar x             h_{-1} = h0 (or 0)
 *   y_t      = sum_n C[b,n,t] * h_t[n] + D[d] * x[b,d,t]
 *   out_t    = y_t * silu(z[b,d,t]),   silu(z) = z / (1 + e^-z)
 *   h_last   = h_{L-1}
 *
 * Sources (web pages on the Mamba selective SSM):
 *  - "A Secret Weapon For mamba paper" and "Rumored Buzz on mamba paper": the
 *    selection mechanism makes the SSM parameters (dt, B, C) functions of the
 *    input; the recurrent mode processes one timestep at a time.
 *  - "Mamba3" post (tginsight), section on the new discretisation scheme:
 *    Mamba-1/2 discretise with a combination of zero-order hold and Euler;
 *    here ZOH is applied to A and Euler to the B x term.
 *  - Gu & Dao, "Mamba: Linear-Time Sequence Modeling with Selective State
 *    Spaces", Appendix D "Hardware-aware Algorithm For Selective SSMs",
 *    paragraph "Speed": a long sequence may be split into chunks and the scan
 *    continued from the carried state; h0 / h_last are that carried state.
 *  - "Rumored Buzz on mamba paper": the state is kept in higher precision
 *    because SSMs are sensitive to their recurrent dynamics (float64 here).
 *  The pages do not print the softplus parameterisation of dt, the D skip or
 *  the silu gate; the oracle takes the standard Mamba reading of them.
 *
 * Storage (all contiguous, channel-major):
 *   x, delta, z, out : [batch][dim][seqlen]      (activation dtype)
 *   B, C             : [batch][dstate][seqlen]   (activation dtype)
 *   A                : [dim][dstate] float32;  D, delta_bias : [dim] float32
 *   h0, h_last       : [batch][dim][dstate] float32 in, float64 out
 * Activation dtype 0 = float32, 1 = bfloat16 (raw 16-bit patterns).  Every
 * stored value is widened exactly to double before use.
 *
 * Optional pointers (NULL allowed): delta_bias (0), D (no skip), z (no gate),
 * h0 (zero state), h_last (not written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define REF_MAX_DSTATE 256

/* exact widening of one stored activation to double */
static double load_act(const void *p, int64_t i, int dtype)
{
    if (dtype == 1) {
        uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* softplus(v) = log(1 + e^v), written in the overflow-free exact form
 * max(v, 0) + log1p(e^-|v|) */
static double softplus_ref(double v)
{
    return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v)));
}

static double silu_ref(double z)
{
    return z / (1.0 + exp(-z));
}

typedef struct {
    const void *x, *delta;
    const float *delta_bias;
    int softplus;
    const float *A;
    const void *B, *C;
    const float *D;
    const void *z;
    const float *h0;
    int dtype;
    int64_t batch, seqlen, dim, dstate;
} ref_args;

/* The recurrence for one channel (b, d) over all t.  out_row gets seqlen
 * values (stride 1); hl gets dstate values (may be NULL).  xrow, when not
 * NULL, holds the channel's x values in double precision (the output of the
 * causal convolution in front of the scan) and replaces the stored x. */
static void scan_channel_x(const ref_args *a, int64_t b, int64_t d, const double *xrow, double *out_row,
                           double *hl)
{
    const int64_t L = a->seqlen, N = a->dstate, Dm = a->dim;
    double h[REF_MAX_DSTATE];
    const int64_t chan = b * Dm + d;
    for (int64_t n = 0; n < N; n++)
        h[n] = a->h0 ? (double)a->h0[chan * N + n] : 0.0;

    for (int64_t t = 0; t < L; t++) {
        double v = load_act(a->delta, chan * L + t, a->dtype);
        if (a->delta_bias)
            v += (double)a->delta_bias[d];
        const double dt = a->softplus ? softplus_ref(v) : v;
        const double xt = xrow ? xrow[t] : load_act(a->x, chan * L + t, a->dtype);

        for (int64_t n = 0; n < N; n++) {
            const double abar = exp(dt * (double)a->A[d * N + n]);
            const double bt = load_act(a->B, (b * N + n) * L + t, a->dtype);
            h[n] = abar * h[n] + dt * bt * xt;
        }
        double y = 0.0;
        for (int64_t n = 0; n < N; n++)
            y += load_act(a->C, (b * N + n) * L + t, a->dtype) * h[n];
        if (a->D)
            y += (double)a->D[d] * xt;
        if (a->z)
            y *= silu_ref(load_act(a->z, chan * L + t, a->dtype));
        out_row[t] = y;
    }
    if (hl)
        for (int64_t n = 0; n < N; n++)
            hl[n] = h[n];
}

static void scan_channel(const ref_args *a, int64_t b, int64_t d, double *out_row, double *hl)
{
    scan_channel_x(a, b, d, NULL, out_row, hl);
}

static int check_dims(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate)
{
    if (batch <= 0 || seqlen <= 0 || dim <= 0 || dstate <= 0 || dstate > REF_MAX_DSTATE)
        return 1;
    return 0;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Whole forward scan.  out: [batch][dim][seqlen] double; h_last:
 * [batch][dim][dstate] double or NULL.  Returns 0, or 1 on bad sizes. */
int ssm_ref_fwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                const float *A, const void *B, const void *C, const float *D,
                const void *z, const float *h0, int dtype,
                int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                double *out, double *h_last, int nthreads)
{
    if (check_dims(batch, seqlen, dim, dstate) || !x || !delta || !A || !B || !C || !out)
        return 1;
    const ref_args a = {x, delta, delta_bias, softplus, A, B, C, D, z, h0, dtype,
                        batch, seqlen, dim, dstate};
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < nchan; c++)
        scan_channel(&a, c / dim, c % dim, out + c * seqlen, h_last ? h_last + c * dstate : NULL);
    return 0;
}

/* The same scan for a list of channels only (flat index b*dim + d).
 * out_sel: [nsel][seqlen]; hl_sel: [nsel][dstate] or NULL. */
int ssm_ref_fwd_channels(const void *x, const void *delta, const float *delta_bias, int softplus,
                         const float *A, const void *B, const void *C, const float *D,
                         const void *z, const float *h0, int dtype,
                         int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                         const int64_t *chan, int64_t nsel,
                         double *out_sel, double *hl_sel, int nthreads)
{
    if (check_dims(batch, seqlen, dim, dstate) || !x || !delta || !A || !B || !C || !out_sel ||
        !chan || nsel < 0)
        return 1;
    for (int64_t i = 0; i < nsel; i++)
        if (chan[i] < 0 || chan[i] >= batch * dim)
            return 1;
    const ref_args a = {x, delta, delta_bias, softplus, A, B, C, D, z, h0, dtype,
                        batch, seqlen, dim, dstate};
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nsel; i++)
        scan_channel(&a, chan[i] / dim, chan[i] % dim, out_sel + i * seqlen,
                     hl_sel ? hl_sel + i * dstate : NULL);
    return 0;
}

/* One recurrent (decode) step for every channel: the same body as one t of
 * the scan, with h read from and written back to `state` ([batch][dim][dstate]
 * double).  Token tensors are x, delta, z: [batch][dim]; B, C: [batch][dstate].
 * out: [batch][dim] double. */
int ssm_ref_step(double *state, const void *x, const void *delta, const float *delta_bias,
                 int softplus, const float *A, const void *B, const void *C, const float *D,
                 const void *z, int dtype, int64_t batch, int64_t dim, int64_t dstate,
                 double *out, int nthreads)
{
    if (check_dims(batch, 1, dim, dstate) || !state || !x || !delta || !A || !B || !C || !out)
        return 1;
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < nchan; c++) {
        const int64_t b = c / dim, d = c % dim;
        double *h = state + c * dstate;
        double v = load_act(delta, c, dtype);
        if (delta_bias)
            v += (double)delta_bias[d];
        const double dt = softplus ? softplus_ref(v) : v;
        const double xt = load_act(x, c, dtype);
        double y = 0.0;
        for (int64_t n = 0; n < dstate; n++) {
            const double abar = exp(dt * (double)A[d * dstate + n]);
            h[n] = abar * h[n] + dt * load_act(B, b * dstate + n, dtype) * xt;
        }
        for (int64_t n = 0; n < dstate; n++)
            y += load_act(C, b * dstate + n, dtype) * h[n];
        if (D)
            y += (double)D[d] * xt;
        if (z)
            y *= silu_ref(load_act(z, c, dtype));
        out[c] = y;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Short causal convolution in front of the scan.
 *
 * Gu & Dao, "Mamba", Appendix D "Hardware-aware Algorithm For Selective
 * SSMs", paragraph "Memory": the block runs input projection, convolution,
 * activation, scan, output projection; "A Secret Weapon For mamba paper"
 * names the causal_conv1d kernels; "Rumored Buzz on mamba paper": the
 * inference cache holds the convolution state beside the SSM state.  The
 * pages print no formula; the plain reading is a depthwise causal convolution
 * of width K over each channel's sequence followed by silu:
 *
 *   xc[b,d,t] = silu( sum_{k=0}^{K-1} w[d,k] * xin(b,d,t-K+1+k) + bias[d] )
 *
 * (w[d,K-1] multiplies the current input), where xin(b,d,s) = x[b,d,s] for
 * s >= 0 and conv_state[b,d,K-1+s] for -(K-1) <= s < 0: the K-1 inputs that
 * came before this call (zero when conv_state is NULL).  After the call the
 * state holds xin(b,d,L-K+1 .. L-1), the last K-1 inputs.
 *
 * Storage: w [dim][K] float32, bias [dim] float32 (NULL = 0), conv_state
 * [batch][dim][K-1] in the activation dtype for the input (its values are
 * raw inputs), double for the output.
 */
#define REF_MAX_CONV 64

/* xin(b,d,s) of one channel, for -(K-1) <= s < L */
static double conv_input(const void *x, const void *conv_state, int dtype, int64_t chan, int64_t L,
                         int64_t K, int64_t s)
{
    if (s >= 0)
        return load_act(x, chan * L + s, dtype);
    if (!conv_state)
        return 0.0;
    return load_act(conv_state, chan * (K - 1) + (K - 1 + s), dtype);
}

/* The convolution of one channel: xc[0..L) (with silu when `silu`), and the
 * channel's new state (K-1 values) into state_out when not NULL. */
static void conv_channel(const void *x, const float *w, const float *bias, int64_t K,
                         const void *conv_state, int silu, int dtype, int64_t chan, int64_t d,
                         int64_t L, double *xc, double *state_out)
{
    for (int64_t t = 0; t < L; t++) {
        double acc = bias ? (double)bias[d] : 0.0;
        for (int64_t k = 0; k < K; k++)
            acc += (double)w[d * K + k] * conv_input(x, conv_state, dtype, chan, L, K, t - K + 1 + k);
        xc[t] = silu ? silu_ref(acc) : acc;
    }
    if (state_out)
        for (int64_t j = 0; j < K - 1; j++)
            state_out[j] = conv_input(x, conv_state, dtype, chan, L, K, L - (K - 1) + j);
}

/* The convolution alone.  xc: [batch][dim][seqlen] double; state_out:
 * [batch][dim][K-1] double or NULL.  Returns 0, or 1 on bad sizes. */
int ssm_ref_conv1d(const void *x, const float *w, const float *bias, int64_t K, const void *conv_state,
                   int silu, int dtype, int64_t batch, int64_t seqlen, int64_t dim, double *xc,
                   double *state_out, int nthreads)
{
    if (check_dims(batch, seqlen, dim, 1) || K < 1 || K > REF_MAX_CONV || !x || !w || !xc)
        return 1;
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < nchan; c++)
        conv_channel(x, w, bias, K, conv_state, silu, dtype, c, c % dim, seqlen, xc + c * seqlen,
                     state_out ? state_out + c * (K - 1) : NULL);
    return 0;
}

/* Convolution + silu, then the scan on its output (the fused block path):
 * the same outputs as ssm_ref_fwd with x replaced by xc, plus the new
 * convolution state.  out: [batch][dim][seqlen]; h_last: [batch][dim][dstate]
 * or NULL; state_out: [batch][dim][K-1] or NULL (all double). */
int ssm_ref_conv_fwd(const void *x, const float *w, const float *cbias, int64_t K, const void *conv_state,
                     const void *delta, const float *delta_bias, int softplus, const float *A,
                     const void *B, const void *C, const float *D, const void *z, const float *h0,
                     int dtype, int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                     double *out, double *h_last, double *state_out, int nthreads)
{
    if (check_dims(batch, seqlen, dim, dstate) || K < 1 || K > REF_MAX_CONV || !x || !w || !delta ||
        !A || !B || !C || !out)
        return 1;
    const ref_args a = {x, delta, delta_bias, softplus, A, B, C, D, z, h0, dtype,
                        batch, seqlen, dim, dstate};
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < nchan; c++) {
        double *xc = (double *)malloc((size_t)seqlen * sizeof(double));
        if (!xc) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        conv_channel(x, w, cbias, K, conv_state, 1, dtype, c, c % dim, seqlen, xc,
                     state_out ? state_out + c * (K - 1) : NULL);
        scan_channel_x(&a, c / dim, c % dim, xc, out + c * seqlen, h_last ? h_last + c * dstate : NULL);
        free(xc);
    }
    return bad ? 2 : 0;
}

/* One decode step of the fused block: the convolution window is the channel's
 * K-1 stored inputs followed by this token's x; xc = silu(window . w + bias);
 * the state shifts by one input; then the SSM step of ssm_ref_step with x = xc.
 * conv_state: [batch][dim][K-1] double, read and written; state:
 * [batch][dim][dstate] double, read and written; out: [batch][dim] double. */
int ssm_ref_conv_step(double *conv_state, double *state, const void *x, const float *w,
                      const float *cbias, int64_t K, const void *delta, const float *delta_bias,
                      int softplus, const float *A, const void *B, const void *C, const float *D,
                      const void *z, int dtype, int64_t batch, int64_t dim, int64_t dstate,
                      double *out, int nthreads)
{
    if (check_dims(batch, 1, dim, dstate) || K < 1 || K > REF_MAX_CONV || !conv_state || !state ||
        !x || !w || !delta || !A || !B || !C || !out)
        return 1;
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < nchan; c++) {
        const int64_t b = c / dim, d = c % dim;
        double *cs = conv_state + c * (K - 1);
        const double xt_raw = load_act(x, c, dtype);
        double acc = cbias ? (double)cbias[d] : 0.0;
        for (int64_t k = 0; k < K - 1; k++)
            acc += (double)w[d * K + k] * cs[k];
        acc += (double)w[d * K + K - 1] * xt_raw;
        for (int64_t k = 0; k + 1 < K - 1; k++)
            cs[k] = cs[k + 1];
        if (K > 1)
            cs[K - 2] = xt_raw;
        const double xt = silu_ref(acc);

        double *h = state + c * dstate;
        double v = load_act(delta, c, dtype);
        if (delta_bias)
            v += (double)delta_bias[d];
        const double dt = softplus ? softplus_ref(v) : v;
        double y = 0.0;
        for (int64_t n = 0; n < dstate; n++) {
            const double abar = exp(dt * (double)A[d * dstate + n]);
            h[n] = abar * h[n] + dt * load_act(B, b * dstate + n, dtype) * xt;
        }
        for (int64_t n = 0; n < dstate; n++)
            y += load_act(C, b * dstate + n, dtype) * h[n];
        if (D)
            y += (double)D[d] * xt;
        if (z)
            y *= silu_ref(load_act(z, c, dtype));
        out[c] = y;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Exponential-trapezoidal discretisation (Mamba-3).
 *
 * The "Mamba3" posts (tginsight), section on the new discretisation scheme:
 * Mamba-1/2 combine zero-order hold and Euler; Mamba-3 approximates the
 * integral of the state update with both ends of the interval, mixed by a
 * data-dependent coefficient lambda, which is a second-order rule.  The pages
 * print no formula; the plain reading of that description, for
 * h'(s) = A h(s) + B(s) x(s) over a step of length dt, is
 *
 *   h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1} + gamma_t B_t x_t
 *   alpha_t = exp(dt_t A),  beta_t = (1 - lambda_t) dt_t alpha_t,  gamma_t = lambda_t dt_t
 *
 * (the integrand exp((t - s) A) B(s) x(s) taken at the interval's start,
 * weight 1 - lambda, and at its end, weight lambda).  lambda = 1 is the
 * Euler input step of Mamba-1; lambda = 1/2 is the trapezoidal rule.  The
 * input before t = 0 is x_prev[b,d] B_prev[b,:] (zero when either is NULL),
 * which lets a sequence be split into calls.
 *
 * Storage: lam [batch][dim][seqlen] activation dtype; x_prev [batch][dim] and
 * B_prev [batch][dstate] activation dtype; everything else as ssm_ref_fwd.
 */
static void trap_channel(const ref_args *a, const void *lam, const void *x_prev, const void *B_prev,
                         int64_t b, int64_t d, double *out_row, double *hl)
{
    const int64_t L = a->seqlen, N = a->dstate, Dm = a->dim;
    double h[REF_MAX_DSTATE], vprev[REF_MAX_DSTATE];
    const int64_t chan = b * Dm + d;
    const double xp = (x_prev && B_prev) ? load_act(x_prev, chan, a->dtype) : 0.0;
    for (int64_t n = 0; n < N; n++) {
        h[n] = a->h0 ? (double)a->h0[chan * N + n] : 0.0;
        vprev[n] = (x_prev && B_prev) ? load_act(B_prev, b * N + n, a->dtype) * xp : 0.0;
    }
    for (int64_t t = 0; t < L; t++) {
        double v = load_act(a->delta, chan * L + t, a->dtype);
        if (a->delta_bias)
            v += (double)a->delta_bias[d];
        const double dt = a->softplus ? softplus_ref(v) : v;
        const double lt = load_act(lam, chan * L + t, a->dtype);
        const double xt = load_act(a->x, chan * L + t, a->dtype);
        for (int64_t n = 0; n < N; n++) {
            const double alpha = exp(dt * (double)a->A[d * N + n]);
            const double beta = (1.0 - lt) * dt * alpha;
            const double gamma = lt * dt;
            const double vt = load_act(a->B, (b * N + n) * L + t, a->dtype) * xt;
            h[n] = alpha * h[n] + beta * vprev[n] + gamma * vt;
            vprev[n] = vt;
        }
        double y = 0.0;
        for (int64_t n = 0; n < N; n++)
            y += load_act(a->C, (b * N + n) * L + t, a->dtype) * h[n];
        if (a->D)
            y += (double)a->D[d] * xt;
        if (a->z)
            y *= silu_ref(load_act(a->z, chan * L + t, a->dtype));
        out_row[t] = y;
    }
    if (hl)
        for (int64_t n = 0; n < N; n++)
            hl[n] = h[n];
}

int ssm_ref_trap_fwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                     const void *lam, const float *A, const void *B, const void *C, const float *D,
                     const void *z, const float *h0, const void *x_prev, const void *B_prev, int dtype,
                     int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                     double *out, double *h_last, int nthreads)
{
    if (check_dims(batch, seqlen, dim, dstate) || !x || !delta || !lam || !A || !B || !C || !out)
        return 1;
    const ref_args a = {x, delta, delta_bias, softplus, A, B, C, D, z, h0, dtype,
                        batch, seqlen, dim, dstate};
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < nchan; c++)
        trap_channel(&a, lam, x_prev, B_prev, c / dim, c % dim, out + c * seqlen,
                     h_last ? h_last + c * dstate : NULL);
    return 0;
}

/* One recurrent step of the trapezoidal rule: the token's x, B, lambda and
 * the previous token's x_prev [batch][dim] and B_prev [batch][dstate] (NULL:
 * no previous input).  state: [batch][dim][dstate] double, read and written. */
int ssm_ref_trap_step(double *state, const void *x, const void *delta, const float *delta_bias,
                      int softplus, const void *lam, const float *A, const void *B, const void *C,
                      const float *D, const void *z, const void *x_prev, const void *B_prev, int dtype,
                      int64_t batch, int64_t dim, int64_t dstate, double *out, int nthreads)
{
    if (check_dims(batch, 1, dim, dstate) || !state || !x || !delta || !lam || !A || !B || !C || !out)
        return 1;
    set_threads(nthreads);
    const int64_t nchan = batch * dim;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < nchan; c++) {
        double hl[REF_MAX_DSTATE];
        const int64_t b = c / dim, d = c % dim;
        double *h = state + c * dstate;
        double vprev[REF_MAX_DSTATE];
        const double xp = (x_prev && B_prev) ? load_act(x_prev, c, dtype) : 0.0;
        for (int64_t n = 0; n < dstate; n++)
            vprev[n] = (x_prev && B_prev) ? load_act(B_prev, b * dstate + n, dtype) * xp : 0.0;
        double v = load_act(delta, c, dtype);
        if (delta_bias)
            v += (double)delta_bias[d];
        const double dt = softplus ? softplus_ref(v) : v;
        const double lt = load_act(lam, c, dtype);
        const double xt = load_act(x, c, dtype);
        for (int64_t n = 0; n < dstate; n++) {
            const double alpha = exp(dt * (double)A[d * dstate + n]);
            const double vt = load_act(B, b * dstate + n, dtype) * xt;
            hl[n] = alpha * h[n] + (1.0 - lt) * dt * alpha * vprev[n] + lt * dt * vt;
        }
        double y = 0.0;
        for (int64_t n = 0; n < dstate; n++) {
            h[n] = hl[n];
            y += load_act(C, b * dstate + n, dtype) * h[n];
        }
        if (D)
            y += (double)D[d] * xt;
        if (z)
            y *= silu_ref(load_act(z, c, dtype));
        out[c] = y;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Backward pass of the scan (reverse-mode derivatives of ssm_ref_fwd).
 *
 * Gu & Dao, "Mamba", Appendix D "Hardware-aware Algorithm For Selective
 * SSMs", paragraph "Memory": the backward pass does not store the
 * intermediate states but recomputes them.  What it computes is fixed by the
 * forward definition: given dout = dL/dout and dh_last = dL/dh_last (NULL =
 * 0), the derivatives of L with respect to every input.  Written out for one
 * channel, with dy_t = dout_t silu(z_t) and the adjoint
 * g_t = dL/dh_t = C_t dy_t + Abar_{t+1} g_{t+1} (g_{L-1} = C_{L-1} dy_{L-1} + dh_last):
 *
 *   dz_t      = dout_t y_t silu'(z_t),  silu'(z) = s (1 + z (1 - s)), s = sigmoid(z)
 *   dD        = sum_t dy_t x_t
 *   dC[n,t]   = sum_d dy_t h_t[n]
 *   dB[n,t]   = sum_d g_t[n] dt_t x_t
 *   dx_t      = D dy_t + sum_n g_t[n] dt_t B[n,t]
 *   ddt_t     = sum_n g_t[n] (A[n] Abar_t[n] h_{t-1}[n] + B[n,t] x_t)
 *   dA[n]     = sum_{b,t} g_t[n] dt_t Abar_t[n] h_{t-1}[n]
 *   ddelta_t  = ddt_t sigmoid(v_t) (softplus) or ddt_t;   dbias = sum_{b,t} ddelta_t
 *   dh0       = Abar_0 g_0
 *
 * Outputs (all double): dx, ddelta, dz [batch][dim][seqlen] (dz only when z
 * is given), dB, dC [batch][dstate][seqlen], dA [dim][dstate], dD, dbias
 * [dim], dh0 [batch][dim][dstate].  Any output pointer may be NULL.
 */
static double sigmoid_ref(double v)
{
    return 1.0 / (1.0 + exp(-v));
}

static void bwd_channel(const ref_args *a, int64_t b, int64_t d, const void *dout, const float *dh_last,
                        double *hs, double *dx, double *ddelta, double *dz, double *dB, double *dC,
                        double *dA, double *dD, double *dbias, double *dh0)
{
    const int64_t L = a->seqlen, N = a->dstate, Dm = a->dim;
    const int64_t chan = b * Dm + d;
    /* forward, keeping every state: hs[(t + 1) * N + n] = h_t[n], hs[n] = h_{-1}[n] */
    for (int64_t n = 0; n < N; n++)
        hs[n] = a->h0 ? (double)a->h0[chan * N + n] : 0.0;
    for (int64_t t = 0; t < L; t++) {
        double v = load_act(a->delta, chan * L + t, a->dtype);
        if (a->delta_bias)
            v += (double)a->delta_bias[d];
        const double dt = a->softplus ? softplus_ref(v) : v;
        const double xt = load_act(a->x, chan * L + t, a->dtype);
        for (int64_t n = 0; n < N; n++) {
            const double abar = exp(dt * (double)a->A[d * N + n]);
            hs[(t + 1) * N + n] = abar * hs[t * N + n] + dt * load_act(a->B, (b * N + n) * L + t, a->dtype) * xt;
        }
    }
    double g[REF_MAX_DSTATE], gnext_decayed[REF_MAX_DSTATE];
    for (int64_t n = 0; n < N; n++)
        gnext_decayed[n] = dh_last ? (double)dh_last[chan * N + n] : 0.0;
    double dDacc = 0.0, dbacc = 0.0;
    for (int64_t t = L - 1; t >= 0; t--) {
        double v = load_act(a->delta, chan * L + t, a->dtype);
        if (a->delta_bias)
            v += (double)a->delta_bias[d];
        const double dt = a->softplus ? softplus_ref(v) : v;
        const double xt = load_act(a->x, chan * L + t, a->dtype);
        const double *ht = hs + (t + 1) * N, *hp = hs + t * N;
        double y = 0.0;
        for (int64_t n = 0; n < N; n++)
            y += load_act(a->C, (b * N + n) * L + t, a->dtype) * ht[n];
        if (a->D)
            y += (double)a->D[d] * xt;
        const double go = load_act(dout, chan * L + t, a->dtype);
        double dy = go;
        if (a->z) {
            const double zt = load_act(a->z, chan * L + t, a->dtype);
            const double s = sigmoid_ref(zt);
            dy = go * zt * s;
            if (dz)
                dz[chan * L + t] = go * y * s * (1.0 + zt * (1.0 - s));
        }
        double dxt = a->D ? (double)a->D[d] * dy : 0.0;
        dDacc += dy * xt;
        double ddt = 0.0;
        for (int64_t n = 0; n < N; n++) {
            const double Cn = load_act(a->C, (b * N + n) * L + t, a->dtype);
            const double Bn = load_act(a->B, (b * N + n) * L + t, a->dtype);
            const double An = (double)a->A[d * N + n];
            const double abar = exp(dt * An);
            g[n] = Cn * dy + gnext_decayed[n];
            if (dC)
                dC[(b * N + n) * L + t] += dy * ht[n];
            if (dB)
                dB[(b * N + n) * L + t] += g[n] * dt * xt;
            dxt += g[n] * dt * Bn;
            ddt += g[n] * (An * abar * hp[n] + Bn * xt);
            if (dA)
                dA[d * N + n] += g[n] * dt * abar * hp[n];
            gnext_decayed[n] = abar * g[n];
        }
        const double ddel = a->softplus ? ddt * sigmoid_ref(v) : ddt;
        dbacc += ddel;
        if (dx)
            dx[chan * L + t] = dxt;
        if (ddelta)
            ddelta[chan * L + t] = ddel;
    }
    if (dh0)
        for (int64_t n = 0; n < N; n++)
            dh0[chan * N + n] = gnext_decayed[n];
    if (dD)
        dD[d] += dDacc;
    if (dbias)
        dbias[d] += dbacc;
}

/* The backward pass over every channel (OpenMP over channels).  The sums
 * over channels (dB, dC, dA, dD, dbias) are taken per thread and then added
 * thread by thread, in double precision.  Returns 0, 1 on bad sizes, 2 when
 * out of memory. */
int ssm_ref_bwd(const void *x, const void *delta, const float *delta_bias, int softplus,
                const float *A, const void *B, const void *C, const float *D,
                const void *z, const float *h0, const void *dout, const float *dh_last, int dtype,
                int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                double *dx, double *ddelta, double *dz, double *dB, double *dC,
                double *dA, double *dD, double *dbias, double *dh0, int nthreads)
{
    if (check_dims(batch, seqlen, dim, dstate) || !x || !delta || !A || !B || !C || !dout)
        return 1;
    const ref_args a = {x, delta, delta_bias, softplus, A, B, C, D, z, h0, dtype,
                        batch, seqlen, dim, dstate};
    const size_t nbc = (size_t)(batch * dstate * seqlen), na = (size_t)(dim * dstate), nd = (size_t)dim;
    const size_t part = 2 * nbc + na + 2 * nd;  /* one thread's dB, dC, dA, dD, dbias */
    set_threads(nthreads);
    int nt = 1;
#ifdef _OPENMP
    nt = omp_get_max_threads();
#endif
    double *acc = (double *)calloc((size_t)nt * part, sizeof(double));
    if (!acc)
        return 2;
    int bad = 0;
#pragma omp parallel
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double *mine = acc + (size_t)tid * part;
        double *hs = (double *)malloc((size_t)(seqlen + 1) * (size_t)dstate * sizeof(double));
        if (!hs) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t c = 0; c < batch * dim; c++)
                bwd_channel(&a, c / dim, c % dim, dout, dh_last, hs, dx, ddelta, dz, mine, mine + nbc,
                            mine + 2 * nbc, mine + 2 * nbc + na, mine + 2 * nbc + na + nd, dh0);
            free(hs);
        }
    }
    if (!bad) {
        double *outs[5] = {dB, dC, dA, dD, dbias};
        const size_t offs[5] = {0, nbc, 2 * nbc, 2 * nbc + na, 2 * nbc + na + nd};
        const size_t lens[5] = {nbc, nbc, na, nd, nd};
        for (int k = 0; k < 5; k++) {
            if (!outs[k])
                continue;
            for (size_t i = 0; i < lens[k]; i++) {
                double sum = 0.0;
                for (int th = 0; th < nt; th++)
                    sum += acc[(size_t)th * part + offs[k] + i];
                outs[k][i] = sum;
            }
        }
    }
    free(acc);
    return bad ? 2 : 0;
}

/* ---------------------------------------------------------------------------
 * Mamba-2 state space duality (SSD): scalar-times-identity state transition.
 *
 * "A Secret Weapon For mamba paper" (the Mamba-2 abstract: SSMs and attention
 * are connected through structured semiseparable matrices) and the "Mamba3"
 * posts (Mamba-2 reduced the state transition matrix to a scalar times the
 * identity).  The pages print no formula; the plain reading, per batch b and
 * head h with head dimension P and state dimension N, is
 *
 *   dt_t   = softplus(dt[b,t,h] + dt_bias[h])          (dt + dt_bias without softplus)
 *   a_t    = exp(dt_t A[h])                            one scalar per (b, t, h)
 *   H_t    = a_t H_{t-1} + (dt_t x_t) B_t^T            H: P x N, H_{-1} = h0 (or 0)
 *   y_t    = H_t C_t + D[h] x_t                        (y_t[p] = sum_n H_t[p,n] C_t[n] + D x_t[p])
 *
 * with B_t, C_t shared by the heads of a group (G groups, H / G heads each).
 * Storage (time-major, as Mamba-2 layers hold it): x, y [batch][L][H][P];
 * dt [batch][L][H]; B, C [batch][L][G][N] (activation dtype, dt too);
 * A, dt_bias, D [H] float32; h0, h_last [batch][H][P][N] (float32 in, double out).
 */
int ssm_ref_ssd_fwd(const void *x, const void *dt, const float *dt_bias, int softplus, const float *A,
                    const void *B, const void *C, const float *D, const float *h0, int dtype,
                    int64_t batch, int64_t seqlen, int64_t heads, int64_t hdim, int64_t groups, int64_t dstate,
                    double *y, double *h_last, int nthreads)
{
    if (batch <= 0 || seqlen <= 0 || heads <= 0 || hdim <= 0 || groups <= 0 || dstate <= 0 ||
        heads % groups != 0 || !x || !dt || !A || !B || !C || !y)
        return 1;
    set_threads(nthreads);
    const int64_t L = seqlen, Hh = heads, P = hdim, G = groups, N = dstate;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < batch * Hh; bh++) {
        const int64_t b = bh / Hh, h = bh % Hh, g = h / (Hh / G);
        double *S = (double *)malloc((size_t)(P * N) * sizeof(double));
        if (!S) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        for (int64_t i = 0; i < P * N; i++)
            S[i] = h0 ? (double)h0[(b * Hh + h) * P * N + i] : 0.0;
        for (int64_t t = 0; t < L; t++) {
            double v = load_act(dt, (b * L + t) * Hh + h, dtype);
            if (dt_bias)
                v += (double)dt_bias[h];
            const double dtt = softplus ? softplus_ref(v) : v;
            const double at = exp(dtt * (double)A[h]);
            for (int64_t p = 0; p < P; p++) {
                const double xp = load_act(x, ((b * L + t) * Hh + h) * P + p, dtype);
                double yp = 0.0;
                for (int64_t n = 0; n < N; n++) {
                    const double Bn = load_act(B, ((b * L + t) * G + g) * N + n, dtype);
                    const double Cn = load_act(C, ((b * L + t) * G + g) * N + n, dtype);
                    S[p * N + n] = at * S[p * N + n] + dtt * xp * Bn;
                    yp += S[p * N + n] * Cn;
                }
                if (D)
                    yp += (double)D[h] * xp;
                y[((b * L + t) * Hh + h) * P + p] = yp;
            }
        }
        if (h_last)
            for (int64_t i = 0; i < P * N; i++)
                h_last[(b * Hh + h) * P * N + i] = S[i];
        free(S);
    }
    return bad ? 2 : 0;
}
