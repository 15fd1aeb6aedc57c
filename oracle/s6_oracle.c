/*
 * s6_oracle.c -- plain fp64 CPU oracle for the selective scan (S6) forward and
 * its single-token state update.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, obviously correct
 * definition that the CUDA library is checked against. Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may build, load or call it;
 * the product path never does. It shares no code, header, table or constant
 * with the CUDA library.
 *
 * What it computes, for every row (b, d) independently, sequentially in t:
 *
 *   delta = delta_raw[b,d,t] + delta_bias[d]          (bias added before softplus)
 *   delta = softplus(delta) = log(1 + exp(delta))      if delta_softplus
 *   for n:  h[n] = exp(delta * A[d,n]) * h[n] + (delta * B[b,n,t]) * u[b,d,t]
 *   y      = sum_n C[b,n,t] * h[n]  +  D[d] * u[b,d,t]
 *   y      = y * z * sigmoid(z)                        if z is given
 *
 * starting from h = 0 (or a given initial state), and returns y for every t
 * and the state h after the last step.
 *
 * Passages followed:
 *  - "Notas sobre Mamba", section "O mecanismo de seleção (S6)": the selection
 *    equations (B_t, C_t input dependent; delta = softplus(Linear(x) + bias));
 *    A diagonal with A = -exp(A_log); the time-varying recurrence
 *    h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t^T h_t; and the worked single
 *    step (Abar = exp(delta*A), Bbar = delta*B).
 *  - "Notas sobre Mamba", section "Preliminares: o modelo de espaço de
 *    estados": the first-order rule Bbar_t = delta_t * B_t used by the
 *    implementation instead of the full ZOH Bbar.
 *  - "Notas sobre Mamba", section "Recorrência trapezoidal": the same update
 *    written h_t = exp(delta_t A) h_{t-1} + delta_t B_t x_t (exponential-Euler).
 *  - "Mamba-2 e State Space Duality (SSD)", section "Como o Mamba-1 alcançou
 *    complexidade linear": y_t = C_t h_t + D x_t, and the order of one decode
 *    step (update h, then read y from the updated h).
 *  - "Notas sobre Mamba", section "O bloco Mamba": the SSM output is
 *    multiplied by SiLU of the gate branch z.
 *
 * Readings where the pages are silent:
 *  - the initial state is zero unless one is given;
 *  - D*x is added before the gate, so it is gated too;
 *  - softplus(v) is taken as v itself for v > 20 (the values are equal to
 *    within 2e-9 there);
 *  - y_t is read from h_t after it has absorbed x_t (no one-step delay).
 *
 * Inputs are decoded from exactly the values the GPU receives: float32, or
 * bfloat16 bit patterns widened to float32 (bits << 16), then to double.
 *
 * The convolution prologue (s6_oracle_conv_scan, s6_oracle_conv_state_update)
 * follows "Notas sobre Mamba", section "O bloco Mamba": on the x branch, a
 * short depthwise convolution and a SiLU come before the selective SSM, and
 * "Mamba-2 e State Space Duality (SSD)" configures its width as d_conv = 4.
 * The pages print no formula; the reading taken is the causal depthwise
 * convolution of width K along t, one filter per channel d, with zero input
 * before t = 0:
 *
 *   u[b,d,t] = silu( bias[d] + sum_{k=0}^{K-1} w[d,k] * x[b,d,t-(K-1)+k] )
 *
 * (w[d,K-1] weighs the current input). The decode form keeps the last K
 * inputs of every row (oldest first) as its convolution state.
 *
 * The exponential-trapezoidal scan (s6_oracle_trap_scan) follows "Notas sobre
 * Mamba", section "Recorrência trapezoidal" (Mamba-3):
 *   h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1} + gamma_t B_t x_t,
 *   alpha_t = exp(delta_t A), beta_t = (1 - lambda_t) delta_t alpha_t,
 *   gamma_t = lambda_t delta_t,  lambda_t = sigmoid(lambda_raw_t),
 * with B_{-1} x_{-1} = 0 (the section's code starts its previous-input term
 * at zero) and the same readout, skip and gate as the scan.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

static double load_value(const void *p, int dtype, int64_t i)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double softplus(double v)
{
    return v > 20.0 ? v : log1p(exp(v));
}

static double silu(double v)
{
    return v / (1.0 + exp(-v));
}

/*
 * One row (b, d): run the recurrence over t = 0..seqlen-1.
 * h (dstate doubles) holds the initial state on entry and the final state on
 * exit; y receives seqlen doubles.
 */
static void scan_row(int64_t b, int64_t d, int64_t dim, int64_t dstate, int64_t seqlen,
                     int dtype, const void *u, const double *u_row, const void *delta,
                     const float *A, const void *B, const void *C, const float *D, const void *z,
                     const float *delta_bias, int delta_softplus, double *h, double *y)
{
    const int64_t row = b * dim + d;                 /* row of (batch, dim, L) */
    for (int64_t t = 0; t < seqlen; ++t) {
        const int64_t i = row * seqlen + t;
        /* the SSM input: the given u, or the row's convolution output */
        const double x = u_row ? u_row[t] : load_value(u, dtype, i);
        double dt = load_value(delta, dtype, i);
        if (delta_bias)
            dt += (double)delta_bias[d];
        if (delta_softplus)
            dt = softplus(dt);
        double acc = 0.0;
        for (int64_t n = 0; n < dstate; ++n) {
            const int64_t j = (b * dstate + n) * seqlen + t;   /* (batch, N, L) */
            const double a = (double)A[d * dstate + n];
            const double Bbar = dt * load_value(B, dtype, j);
            h[n] = exp(dt * a) * h[n] + Bbar * x;
            acc += load_value(C, dtype, j) * h[n];
        }
        if (D)
            acc += (double)D[d] * x;
        if (z)
            acc *= silu(load_value(z, dtype, i));
        y[t] = acc;
    }
}

/*
 * Selective scan forward over the rows listed in `rows` (each an index
 * b*dim + d), or over all batch*dim rows in order when rows == NULL.
 *
 *   u, delta, z : (batch, dim, seqlen), contiguous, dtype `dtype`; z may be NULL
 *   B, C        : (batch, dstate, seqlen), contiguous, dtype `dtype`
 *   A           : (dim, dstate) float32;  D, delta_bias: (dim) float32 or NULL
 *   h0          : (n_rows, dstate) doubles or NULL (zero initial state)
 *   y_out       : (n_rows, seqlen) doubles;  h_out: (n_rows, dstate) doubles
 *
 * Returns 0, or -1 on a bad argument.
 */
int s6_oracle_scan(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                   const void *u, const void *delta, const float *A, const void *B,
                   const void *C, const float *D, const void *z, const float *delta_bias,
                   int delta_softplus, const int64_t *rows, int64_t n_rows,
                   const double *h0, double *y_out, double *h_out, int nthreads)
{
    if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0)
        return -1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16)
        return -1;
    if (!rows)
        n_rows = batch * dim;
    if (n_rows > 0 && (!u || !delta || !A || !B || !C || !y_out || !h_out))
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= batch * dim)
            return -1;
    }
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        const int64_t b = row / dim, d = row % dim;
        double *h = h_out + r * dstate;
        for (int64_t n = 0; n < dstate; ++n)
            h[n] = h0 ? h0[r * dstate + n] : 0.0;
        scan_row(b, d, dim, dstate, seqlen, dtype, u, NULL, delta, A, B, C, D, z, delta_bias,
                 delta_softplus, h, y_out + r * seqlen);
    }
    return 0;
}

/*
 * Single-token state update: the scan body for one time step, on the state
 * `state` (batch*dim rows of dstate doubles, updated in place).
 *
 *   x, delta, z : (batch, dim), dtype `dtype`; z may be NULL
 *   B, C        : (batch, dstate), dtype `dtype`
 *   y_out       : (batch, dim) doubles
 *
 * Only the rows listed in `rows` (indices b*dim + d) are updated when rows is
 * not NULL; `state` and `y_out` are then (n_rows, dstate) and (n_rows).
 */
int s6_oracle_state_update(int64_t batch, int64_t dim, int64_t dstate, int dtype,
                           double *state, const void *x, const void *delta, const float *A,
                           const void *B, const void *C, const float *D, const void *z,
                           const float *delta_bias, int delta_softplus,
                           const int64_t *rows, int64_t n_rows, double *y_out, int nthreads)
{
    if (batch < 0 || dim < 0 || dstate < 0)
        return -1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16)
        return -1;
    if (!rows)
        n_rows = batch * dim;
    if (n_rows > 0 && (!state || !x || !delta || !A || !B || !C || !y_out))
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= batch * dim)
            return -1;
    }
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        const int64_t b = row / dim, d = row % dim;
        /* With seqlen = 1 the (batch, dim, L) and (batch, N, L) layouts of the
         * scan are the (batch, dim) and (batch, N) layouts of one token. */
        scan_row(b, d, dim, dstate, 1, dtype, x, NULL, delta, A, B, C, D, z, delta_bias,
                 delta_softplus, state + r * dstate, y_out + r);
    }
    return 0;
}

/*
 * The convolution output of one row: u_row[t] = act(bias + sum_k w[k] *
 * x[t-(K-1)+k]) with x = 0 before t = 0; act = SiLU when `conv_silu`.
 */
static void conv_row(int64_t row, int64_t seqlen, int dtype, const void *x, const float *w,
                     double bias, int width, int conv_silu, double *u_row)
{
    for (int64_t t = 0; t < seqlen; ++t) {
        double acc = bias;
        for (int k = 0; k < width; ++k) {
            const int64_t s = t - (width - 1) + k;
            if (s >= 0)
                acc += (double)w[k] * load_value(x, dtype, row * seqlen + s);
        }
        u_row[t] = conv_silu ? silu(acc) : acc;
    }
}

/*
 * Convolution prologue + selective scan: x (batch, dim, seqlen) of dtype
 * `dtype` is convolved per channel with conv_w (dim, width) float32 and
 * conv_b (dim) float32 or NULL, optionally passed through SiLU, and the result
 * is the scan's input u. Everything else as s6_oracle_scan. u_out, when not
 * NULL, receives the convolution output (n_rows, seqlen) doubles.
 */
int s6_oracle_conv_scan(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                        const void *x, const float *conv_w, const float *conv_b, int width,
                        int conv_silu, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const int64_t *rows, int64_t n_rows,
                        const double *h0, double *y_out, double *h_out, double *u_out,
                        int nthreads)
{
    if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0 || width < 1)
        return -1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16)
        return -1;
    if (!rows)
        n_rows = batch * dim;
    if (n_rows > 0 && (!x || !conv_w || !delta || !A || !B || !C || !y_out || !h_out))
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= batch * dim)
            return -1;
    }
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        const int64_t b = row / dim, d = row % dim;
        double *u_row = u_out ? u_out + r * seqlen : (double *)malloc((size_t)(seqlen > 0 ? seqlen : 1) * sizeof(double));
        if (!u_row) {
            failed = 1;
            continue;
        }
        conv_row(row, seqlen, dtype, x, conv_w + d * width, conv_b ? (double)conv_b[d] : 0.0, width,
                 conv_silu, u_row);
        double *h = h_out + r * dstate;
        for (int64_t n = 0; n < dstate; ++n)
            h[n] = h0 ? h0[r * dstate + n] : 0.0;
        scan_row(b, d, dim, dstate, seqlen, dtype, NULL, u_row, delta, A, B, C, D, z, delta_bias,
                 delta_softplus, h, y_out + r * seqlen);
        if (!u_out)
            free(u_row);
    }
    return failed ? -1 : 0;
}

/*
 * Single-token decode step with the convolution prologue. conv_state holds,
 * per row, the last `width` convolution inputs (oldest first) as doubles; the
 * step drops the oldest, appends x, computes u = act(bias + sum_k w[k] *
 * conv_state[k]) and then runs s6_oracle_state_update's body with u as input.
 * conv_state is (n_rows, width), state (n_rows, dstate), y_out (n_rows).
 */
int s6_oracle_conv_state_update(int64_t batch, int64_t dim, int64_t dstate, int dtype,
                                double *state, double *conv_state, const void *x,
                                const float *conv_w, const float *conv_b, int width,
                                int conv_silu, const void *delta, const float *A,
                                const void *B, const void *C, const float *D, const void *z,
                                const float *delta_bias, int delta_softplus,
                                const int64_t *rows, int64_t n_rows, double *y_out, int nthreads)
{
    if (batch < 0 || dim < 0 || dstate < 0 || width < 1)
        return -1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16)
        return -1;
    if (!rows)
        n_rows = batch * dim;
    if (n_rows > 0 && (!state || !conv_state || !x || !conv_w || !delta || !A || !B || !C || !y_out))
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= batch * dim)
            return -1;
    }
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        const int64_t b = row / dim, d = row % dim;
        double *cs = conv_state + r * width;
        for (int k = 0; k + 1 < width; ++k)
            cs[k] = cs[k + 1];
        cs[width - 1] = load_value(x, dtype, row);
        double acc = conv_b ? (double)conv_b[d] : 0.0;
        for (int k = 0; k < width; ++k)
            acc += (double)conv_w[d * width + k] * cs[k];
        const double u = conv_silu ? silu(acc) : acc;
        scan_row(b, d, dim, dstate, 1, dtype, NULL, &u, delta, A, B, C, D, z, delta_bias,
                 delta_softplus, state + r * dstate, y_out + r);
    }
    return 0;
}

static double sigmoid(double v)
{
    return 1.0 / (1.0 + exp(-v));
}

/*
 * Exponential-trapezoidal selective scan: as s6_oracle_scan, plus lambda_raw
 * (batch, dim, seqlen) of dtype `dtype`, the pre-activation of the per-token
 * mixing gate lambda = sigmoid(lambda_raw).
 */
int s6_oracle_trap_scan(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                        const void *u, const void *delta, const void *lambda_raw, const float *A,
                        const void *B, const void *C, const float *D, const void *z,
                        const float *delta_bias, int delta_softplus, const int64_t *rows, int64_t n_rows,
                        const double *h0, double *y_out, double *h_out, int nthreads)
{
    if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0)
        return -1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16)
        return -1;
    if (!rows)
        n_rows = batch * dim;
    if (n_rows > 0 && (!u || !delta || !lambda_raw || !A || !B || !C || !y_out || !h_out))
        return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= batch * dim)
            return -1;
    }
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t row = rows ? rows[r] : r;
        const int64_t b = row / dim, d = row % dim;
        double *h = h_out + r * dstate;
        double *v_prev = (double *)calloc((size_t)(dstate > 0 ? dstate : 1), sizeof(double));
        if (!v_prev) {
            failed = 1;
            continue;
        }
        for (int64_t n = 0; n < dstate; ++n)
            h[n] = h0 ? h0[r * dstate + n] : 0.0;
        for (int64_t t = 0; t < seqlen; ++t) {
            const int64_t i = row * seqlen + t;
            const double x = load_value(u, dtype, i);
            double dt = load_value(delta, dtype, i);
            if (delta_bias)
                dt += (double)delta_bias[d];
            if (delta_softplus)
                dt = softplus(dt);
            const double lam = sigmoid(load_value(lambda_raw, dtype, i));
            double acc = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                const int64_t j = (b * dstate + n) * seqlen + t;
                const double alpha = exp(dt * (double)A[d * dstate + n]);
                const double beta = (1.0 - lam) * dt * alpha;
                const double gamma = lam * dt;
                const double v = load_value(B, dtype, j) * x;     /* B_t x_t */
                h[n] = alpha * h[n] + beta * v_prev[n] + gamma * v;
                v_prev[n] = v;
                acc += load_value(C, dtype, j) * h[n];
            }
            if (D)
                acc += (double)D[d] * x;
            if (z)
                acc *= silu(load_value(z, dtype, i));
            y_out[r * seqlen + t] = acc;
        }
        free(v_prev);
    }
    return failed ? -1 : 0;
}

int s6_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
