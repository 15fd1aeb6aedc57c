/*
 * ssd_oracle.c -- plain fp64 CPU oracle for the Mamba-2 state space model
 * with a scalar decay per head (the structured state space duality, SSD),
 * computed in its recurrent form.
 *
 * TEST INFRASTRUCTURE ONLY. Like s6_oracle.c, this is the slow definition
 * the CUDA library is checked against; only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may build, load or call it. It shares no
 * code, header, table or constant with the CUDA library.
 *
 * What it computes, for every batch b and head h independently, sequentially
 * in t, on a state H of headdim x dstate values (P x N):
 *
 *   delta = dt[b,t,h] + dt_bias[h]                  (bias before softplus)
 *   delta = softplus(delta)                          if dt_softplus
 *   a     = exp(delta * A[h])                        (the scalar decay a_t)
 *   H     = a * H + (delta * x[b,t,h,:]) B[b,t,g,:]^T      (outer product)
 *   y[b,t,h,:] = H C[b,t,g,:] + D[h] * x[b,t,h,:]
 *   y[b,t,h,:] = y * silu(z[b,t,h,:])                if z is given
 *
 * with g = h / (nheads / ngroups) the group whose B and C the head reads.
 *
 * Passages followed:
 *  - "Notas sobre Mamba", section "A forma dual: atenção mascarada": the
 *    transition restricted to a scalar times the identity, Abar_t = a_t I,
 *    and the recurrent form of the printed check (state of P x N values,
 *    updated by a decay and an outer product of X_t and B_t, read out
 *    against C_t), which this file follows step for step with the page's
 *    X_t taken as the discretised input delta_t x_t.
 *  - "Notas sobre Mamba", section "Preliminares: o modelo de espaço de
 *    estados": the first-order rule Bbar = delta B, which gives that
 *    discretised input, and Abar = exp(delta A).
 *  - "Mamba-2 e State Space Duality (SSD)", section "A teoria do State Space
 *    Duality (SSD) no Mamba-2": the decay between positions j < i is
 *    exp(sum_{k=j+1}^{i} delta_k a_k), i.e. a_t = exp(delta_t A) per head.
 *  - "Mamba-2 e State Space Duality (SSD)", section "Implementando Mamba-2 em
 *    pipelines de inferência": heads of headdim channels (headdim = 64), a
 *    state of d_state = 128 per channel, and the block's D skip and SiLU gate
 *    carried over from the Mamba block.
 *
 * Readings where the pages are silent: B and C are shared by the heads of a
 * group (one group unless told otherwise); D and dt_bias are per head; the
 * skip D x is added before the gate, as in the selective scan; the initial
 * state is zero unless one is given.
 *
 * ssd_oracle_rec_d is the recurrent form in the page's own parametrisation
 * (a_t, B, C, X given directly, one head), used to pin this file against the
 * quadratic form that the page prints beside it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { SSD_F32 = 0, SSD_BF16 = 1 };

static double ssd_load(const void *p, int dtype, int64_t i)
{
    if (dtype == SSD_F32)
        return (double)((const float *)p)[i];
    const uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16u;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Recurrent form of one head, in the page's parametrisation:
 *   H = a[t] H + X[t] B[t]^T,  Y[t] = H C[t]
 * a (L), B and C (L, N), X and Y (L, P), all row-major doubles; H (P, N)
 * holds the initial state on entry (zeros for the page's check) and the
 * final state on exit.
 */
int ssd_oracle_rec_d(int64_t L, int64_t P, int64_t N, const double *a, const double *B,
                     const double *C, const double *X, double *H, double *Y)
{
    if (L < 0 || P < 0 || N < 0 || (L > 0 && (!a || !B || !C || !X || !Y)) || (P * N > 0 && !H))
        return -1;
    for (int64_t t = 0; t < L; ++t) {
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double *hpn = &H[p * N + n];
                *hpn = a[t] * *hpn + X[t * P + p] * B[t * N + n];
                acc += *hpn * C[t * N + n];
            }
            Y[t * P + p] = acc;
        }
    }
    return 0;
}

/*
 * The SSD layer forward over the (batch, head) pairs listed in `pairs` (each
 * b*nheads + h), or over all of them in order when pairs == NULL.
 *
 *   x, z, y : (batch, seqlen, nheads, headdim), dtype `dtype`; z may be NULL
 *   dt      : (batch, seqlen, nheads), dtype `dtype`
 *   B, C    : (batch, seqlen, ngroups, dstate), dtype `dtype`
 *   A       : (nheads) float32;  D, dt_bias: (nheads) float32 or NULL
 *   h0      : (n_pairs, headdim, dstate) doubles or NULL (zero initial state)
 *   y_out   : (n_pairs, seqlen, headdim) doubles
 *   h_out   : (n_pairs, headdim, dstate) doubles
 *
 * Returns 0, or -1 on a bad argument.
 */
int ssd_oracle_scan(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t ngroups,
                    int64_t dstate, int dtype, const void *x, const void *dt, const float *A,
                    const void *B, const void *C, const float *D, const void *z, const float *dt_bias,
                    int dt_softplus, const int64_t *pairs, int64_t n_pairs, const double *h0,
                    double *y_out, double *h_out, int nthreads)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || ngroups <= 0 || dstate <= 0)
        return -1;
    if (nheads % ngroups != 0 || (dtype != SSD_F32 && dtype != SSD_BF16))
        return -1;
    if (!pairs)
        n_pairs = batch * nheads;
    if (n_pairs > 0 && (!x || !dt || !A || !B || !C || !y_out || !h_out))
        return -1;
    for (int64_t r = 0; r < n_pairs; ++r) {
        const int64_t pr = pairs ? pairs[r] : r;
        if (pr < 0 || pr >= batch * nheads)
            return -1;
    }
    const int64_t P = headdim, N = dstate, heads_per_group = nheads / ngroups;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < n_pairs; ++r) {
        const int64_t pr = pairs ? pairs[r] : r;
        const int64_t b = pr / nheads, h = pr % nheads, g = h / heads_per_group;
        double *H = h_out + r * P * N;
        for (int64_t i = 0; i < P * N; ++i)
            H[i] = h0 ? h0[r * P * N + i] : 0.0;
        double *y = y_out + r * seqlen * P;
        for (int64_t t = 0; t < seqlen; ++t) {
            double delta = ssd_load(dt, dtype, (b * seqlen + t) * nheads + h);
            if (dt_bias)
                delta += (double)dt_bias[h];
            if (dt_softplus)
                delta = delta > 20.0 ? delta : log1p(exp(delta));
            const double a = exp(delta * (double)A[h]);
            const int64_t xrow = ((b * seqlen + t) * nheads + h) * P;
            const int64_t brow = ((b * seqlen + t) * ngroups + g) * N;
            for (int64_t p = 0; p < P; ++p) {
                const double xv = ssd_load(x, dtype, xrow + p);
                const double xbar = delta * xv;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double *hpn = &H[p * N + n];
                    *hpn = a * *hpn + xbar * ssd_load(B, dtype, brow + n);
                    acc += *hpn * ssd_load(C, dtype, brow + n);
                }
                if (D)
                    acc += (double)D[h] * xv;
                if (z) {
                    const double zv = ssd_load(z, dtype, xrow + p);
                    acc *= zv / (1.0 + exp(-zv));
                }
                y[t * P + p] = acc;
            }
        }
    }
    return 0;
}
