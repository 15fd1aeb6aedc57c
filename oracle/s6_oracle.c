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

/* ORACLE_F64 (double inputs) exists for the finite-difference pins of the
 * backward pass; the GPU never sees it. */
enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };

static double load_value(const void *p, int dtype, int64_t i)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)p)[i];
    if (dtype == ORACLE_F64)
        return ((const double *)p)[i];
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
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16 && dtype != ORACLE_F64)
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

/* ---- Backward pass --------------------------------------------------------
 * Gradients of the scan by reverse-mode differentiation of the forward
 * definition (the backward half of "A varredura paralela ciente do hardware",
 * which recomputes the states instead of storing them; here the fp64
 * reference simply keeps them). With s_t = sum_n C h + D u (before the gate),
 * y_t = s_t silu(z_t) and a_tn = exp(delta_t A_n):
 *   ds_t  = dy_t silu(z_t);  dz_t = dy_t s_t silu'(z_t)
 *   g_tn  = ds_t C_tn + a_{t+1,n} g_{t+1,n}   (g_{L-1} also receives dhT)
 *   dC_tn += ds_t h_tn;  dB_tn += g_tn delta_t u_t;  dD += ds_t u_t
 *   du_t  = sum_n g_tn delta_t B_tn + ds_t D
 *   ddelta_t = sum_n g_tn (B_tn u_t + h_{t-1,n} a_tn A_n)  (times sigmoid(raw) under softplus)
 *   dA_n  += g_tn h_{t-1,n} a_tn delta_t;  dh0_n = a_0n g_0n
 * All arrays are doubles, contiguous: u, delta, z, dy (batch, dim, L); B, C
 * (batch, N, L); A (dim, N); D, delta_bias (dim); h0, dhT, dh0 (batch, dim, N).
 */
static void scan_row_d(int64_t L, int64_t N, const double *u, const double *dr, const double *A_row,
                       const double *Bb, const double *Cb, double D, const double *z, double bias,
                       int softplus_on, double *h, double *y, double *s_pre, double *H, double *Ad,
                       double *dts)
{
    for (int64_t t = 0; t < L; ++t) {
        double dt = dr[t] + bias;
        if (softplus_on)
            dt = softplus(dt);
        if (dts)
            dts[t] = dt;
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double a = exp(dt * A_row[n]);
            h[n] = a * h[n] + dt * Bb[n * L + t] * u[t];
            acc += Cb[n * L + t] * h[n];
            if (H)
                H[t * N + n] = h[n];
            if (Ad)
                Ad[t * N + n] = a;
        }
        acc += D * u[t];
        if (s_pre)
            s_pre[t] = acc;
        y[t] = z ? acc * silu(z[t]) : acc;
    }
}

/* All-double forward: y (batch, dim, L) and the final state (batch, dim, N). */
int s6_oracle_scan_d(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, const double *u,
                     const double *delta, const double *A, const double *B, const double *C,
                     const double *D, const double *z, const double *delta_bias, int delta_softplus,
                     const double *h0, double *y_out, double *h_out)
{
    if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0 || !u || !delta || !A || !B || !C || !y_out || !h_out)
        return -1;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            double *h = h_out + row * dstate;
            for (int64_t n = 0; n < dstate; ++n)
                h[n] = h0 ? h0[row * dstate + n] : 0.0;
            scan_row_d(seqlen, dstate, u + row * seqlen, delta + row * seqlen, A + d * dstate,
                       B + b * dstate * seqlen, C + b * dstate * seqlen, D ? D[d] : 0.0,
                       z ? z + row * seqlen : NULL, delta_bias ? delta_bias[d] : 0.0, delta_softplus, h,
                       y_out + row * seqlen, NULL, NULL, NULL, NULL);
        }
    return 0;
}

int s6_oracle_scan_bwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, const double *u,
                       const double *delta, const double *A, const double *B, const double *C,
                       const double *D, const double *z, const double *delta_bias, int delta_softplus,
                       const double *h0, const double *dy, const double *dhT, double *du, double *ddelta,
                       double *dz, double *dA, double *dB, double *dC, double *dD, double *ddelta_bias,
                       double *dh0)
{
    if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0 || !u || !delta || !A || !B || !C || !dy || !du ||
        !ddelta || !dA || !dB || !dC || !dD || !ddelta_bias || !dh0 || (z && !dz))
        return -1;
    const int64_t L = seqlen, N = dstate;
    memset(dA, 0, (size_t)(dim * N) * sizeof(double));
    memset(dB, 0, (size_t)(batch * N * L) * sizeof(double));
    memset(dC, 0, (size_t)(batch * N * L) * sizeof(double));
    memset(dD, 0, (size_t)dim * sizeof(double));
    memset(ddelta_bias, 0, (size_t)dim * sizeof(double));
    double *H = (double *)malloc((size_t)(L * N + 1) * sizeof(double));
    double *Ad = (double *)malloc((size_t)(L * N + 1) * sizeof(double));
    double *sp = (double *)malloc((size_t)(L + 1) * sizeof(double));
    double *dts = (double *)malloc((size_t)(L + 1) * sizeof(double));
    double *yy = (double *)malloc((size_t)(L + 1) * sizeof(double));
    double *h = (double *)malloc((size_t)(N + 1) * sizeof(double));
    double *g = (double *)malloc((size_t)(N + 1) * sizeof(double));
    if (!H || !Ad || !sp || !dts || !yy || !h || !g) {
        free(H); free(Ad); free(sp); free(dts); free(yy); free(h); free(g);
        return -1;
    }
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            const double *ur = u + row * L, *dr = delta + row * L, *zr = z ? z + row * L : NULL;
            const double *Bb = B + b * N * L, *Cb = C + b * N * L, *Ar = A + d * N;
            const double Dd = D ? D[d] : 0.0, bias = delta_bias ? delta_bias[d] : 0.0;
            for (int64_t n = 0; n < N; ++n)
                h[n] = h0 ? h0[row * N + n] : 0.0;
            scan_row_d(L, N, ur, dr, Ar, Bb, Cb, Dd, zr, bias, delta_softplus, h, yy, sp, H, Ad, dts);
            for (int64_t n = 0; n < N; ++n)
                g[n] = dhT ? dhT[row * N + n] : 0.0;     /* a_{t+1} g_{t+1} carried down */
            for (int64_t t = L - 1; t >= 0; --t) {
                double ds = dy[row * L + t];
                if (zr) {
                    const double zz = zr[t], sg = 1.0 / (1.0 + exp(-zz));
                    dz[row * L + t] = ds * sp[t] * sg * (1.0 + zz * (1.0 - sg));
                    ds *= zz * sg;
                }
                const double dt = dts[t];
                double du_t = ds * Dd, ddt = 0.0;
                dD[d] += ds * ur[t];
                for (int64_t n = 0; n < N; ++n) {
                    const double hprev = t > 0 ? H[(t - 1) * N + n] : (h0 ? h0[row * N + n] : 0.0);
                    const double a = Ad[t * N + n];
                    const double gn = g[n] + ds * Cb[n * L + t];
                    dC[(b * N + n) * L + t] += ds * H[t * N + n];
                    dB[(b * N + n) * L + t] += gn * dt * ur[t];
                    du_t += gn * dt * Bb[n * L + t];
                    ddt += gn * (Bb[n * L + t] * ur[t] + hprev * a * Ar[n]);
                    dA[d * N + n] += gn * hprev * a * dt;
                    g[n] = a * gn;
                }
                du[row * L + t] = du_t;
                if (delta_softplus)
                    ddt *= 1.0 / (1.0 + exp(-(dr[t] + bias)));
                ddelta[row * L + t] = ddt;
                ddelta_bias[d] += ddt;
            }
            for (int64_t n = 0; n < N; ++n)
                dh0[row * N + n] = g[n];
        }
    free(H); free(Ad); free(sp); free(dts); free(yy); free(h); free(g);
    return 0;
}

int s6_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
