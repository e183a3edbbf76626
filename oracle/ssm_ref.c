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
 * values (stride 1); hl gets dstate values (may be NULL). */
static void scan_channel(const ref_args *a, int64_t b, int64_t d, double *out_row, double *hl)
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
        const double xt = load_act(a->x, chan * L + t, a->dtype);

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
