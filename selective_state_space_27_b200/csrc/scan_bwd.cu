// Selective scan (S6) backward for sm_100a: gradients of the scan for the
// loss sum(y dy) + sum(h_T dh_T) with respect to u, delta_raw, z, A, B, C, D,
// delta_bias and the initial state.
//
// The states are recomputed, not stored ("Notas sobre Mamba", section "A
// varredura paralela ciente do hardware": the backward pass recomputes the
// intermediate states instead of reading them from HBM). With
// s_t = sum_n C h + D u, y_t = s_t silu(z_t), a_tn = exp(delta_t A_n):
//   ds_t = dy_t silu(z_t),  dz_t = dy_t s_t silu'(z_t)
//   g_tn = ds_t C_tn + a_{t+1,n} g_{t+1,n}      (g_{L-1} also receives dh_T)
//   dC_tn += ds_t h_tn, dB_tn += g_tn delta_t u_t      (summed over d)
//   du_t = sum_n g_tn delta_t B_tn + ds_t D
//   ddelta_t = sum_n g_tn (B_tn u_t + h_{t-1,n} a_tn A_n)  (* sigmoid(raw) under softplus)
//   dA_n += g_tn h_{t-1,n} a_tn delta_t, dD += ds_t u_t, dh_0 = a_0 g_0.
//
// Design. A CTA owns 16 rows of one batch entry and runs one thread per
// (row, state) chain (256 threads). Phase F walks the sequence forward in
// chunks of 16 steps and writes each chunk's end state to a workspace (one
// float per chain and chunk: 1/16 of the expanded state). Phase B walks the
// chunks backward: it recomputes the chunk's 16 states from the previous
// checkpoint into registers and runs the adjoint recurrence through them.
// Per-(row, t) sums over the 16 states use half-warp shuffles; the B and C
// gradients are summed over the CTA's rows in shared memory and added to
// global memory with atomics, as are the A, D and delta_bias gradients (sums
// over the batch). The caller's reduction outputs are zeroed first.
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kRows = 16;       // rows per CTA
constexpr int kN = 16;          // states per row (smaller dstate is zero-padded)
constexpr int kT = 16;          // steps per chunk
constexpr int kBwdThreads = kRows * kN;

template <typename T>
__device__ __forceinline__ float ldv(const void *p, int64_t i) {
    return to_f32<T>(static_cast<const T *>(p)[i]);
}

// Sum over the 16 lanes of a half-warp (the 16 states of a row).
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_kernel(const ScanParams p, const BwdParams q) {
    __shared__ float dts[kRows][kT + 1], dus[kRows][kT + 1], uus[kRows][kT + 1], dss[kRows][kT + 1];
    __shared__ float Bs[kT][kN + 1], Cs[kT][kN + 1];
    __shared__ float pB[kT][kRows][kN + 1], pC[kT][kRows][kN + 1];
    __shared__ float rdu[kRows][kT + 1], rdd[kRows][kT + 1];

    const int tid = threadIdx.x;
    const int r = tid / kN, n = tid % kN;          // chain (row, state); also item (row, step n)
    const int64_t b = blockIdx.y;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * kRows + r;
    const bool ok = d < p.dim;
    const int64_t dc = ok ? d : p.dim - 1;
    const int dstate = static_cast<int>(p.dstate);
    const bool live = n < dstate;
    const int64_t L = p.seqlen;
    const int64_t nchunks = (L + kT - 1) / kT;
    const int64_t row = b * p.dim + dc;
    const float Areal = live ? __ldg(p.A + dc * dstate + n) : 0.f;
    const float A2 = Areal * kLog2e;
    const float bias = p.delta_bias ? __ldg(p.delta_bias + dc) : 0.f;
    const float Dd = p.D ? __ldg(p.D + dc) : 0.f;
    float *ckpt = q.ckpt + row * nchunks * kN + n;

    // Stage chunk c: per (row, step) delta, delta u and u; per (step, state) B (and C).
    auto stage = [&](int64_t c, bool with_c) {
        const int64_t t = c * kT + n;                 // item (row r, step n)
        const bool in = ok && t < L;
        float u = 0.f, dt = 0.f;
        if (in) {
            u = ldv<T>(p.u, b * p.u_sb + dc * p.u_sd + t);
            float v = ldv<T>(p.delta, b * p.dl_sb + dc * p.dl_sd + t) + bias;
            dt = p.softplus ? softplus(v) : v;
        }
        dts[r][n] = dt;                                // steps past the end: delta = 0 (identity)
        dus[r][n] = dt * u;
        uus[r][n] = u;
        const int tt = tid / kN, nn = tid % kN;        // (step, state) of the B/C tile
        const int64_t ts = c * kT + tt;
        const bool bin = nn < dstate && ts < L;
        Bs[tt][nn] = bin ? ldv<T>(p.B, b * p.B_sb + nn * p.B_sn + ts) : 0.f;
        if (with_c) Cs[tt][nn] = bin ? ldv<T>(p.C, b * p.C_sb + nn * p.C_sn + ts) : 0.f;
    };

    // ---- Phase F: checkpoints at the end of every chunk but the last ----
    const float h_init = (live && p.h0) ? p.h0[row * dstate + n] : 0.f;
    float h = h_init;
    for (int64_t c = 0; c + 1 < nchunks; ++c) {
        stage(c, false);
        __syncthreads();
#pragma unroll
        for (int t = 0; t < kT; ++t) h = fmaf(ex2_approx(dts[r][t] * A2), h, dus[r][t] * Bs[t][n]);
        if (ok) ckpt[c * kN] = h;   // rows past the end share a clamped index: no checkpoints
        __syncthreads();
    }

    // ---- Phase B ----
    float G = (live && ok && q.dhT) ? q.dhT[row * dstate + n] : 0.f;   // a_{t+1} g_{t+1}, carried down
    float dA_acc = 0.f, dD_acc = 0.f, dbias_acc = 0.f;
    for (int64_t c = nchunks - 1; c >= 0; --c) {
        stage(c, true);
        // dy and z of item (row r, step n)
        const int64_t ti = c * kT + n;
        const bool in = ok && ti < L;
        const float dyv = in ? ldv<T>(q.dy, b * q.dy_sb + dc * q.dy_sd + ti) : 0.f;
        const float zv = (in && p.z) ? ldv<T>(p.z, b * p.z_sb + dc * p.z_sd + ti) : 0.f;
        __syncthreads();

        // recompute the chunk's states from the previous checkpoint
        const float hs = (c > 0 && ok) ? ckpt[(c - 1) * kN] : h_init;
        float H[kT], Av[kT];
        {
            float hh = hs;
#pragma unroll
            for (int t = 0; t < kT; ++t) {
                Av[t] = ex2_approx(dts[r][t] * A2);
                hh = fmaf(Av[t], hh, dus[r][t] * Bs[t][n]);
                H[t] = hh;
            }
        }
        // ds, dz of item (row r, step n); s_t needs the row's sum over states
        float s_mine = 0.f;
#pragma unroll
        for (int t = 0; t < kT; ++t) {
            const float st = half_warp_sum(Cs[t][n] * H[t]);
            if (t == n) s_mine = st + Dd * uus[r][t];
        }
        float dsv = dyv;
        if (p.z) {
            const float sg = __fdividef(1.f, 1.f + ex2_approx(-zv * kLog2e));
            if (in && q.dz)
                static_cast<T *>(q.dz)[b * q.dz_sb + dc * q.dz_sd + ti] =
                    from_f32<T>(dyv * s_mine * sg * (1.f + zv * (1.f - sg)));
            dsv = dyv * zv * sg;
        }
        dss[r][n] = dsv;
        dD_acc = fmaf(dsv, uus[r][n], dD_acc);
        __syncthreads();

        // adjoint recurrence through the chunk
#pragma unroll
        for (int t = kT - 1; t >= 0; --t) {
            const float ds = dss[r][t], dt = dts[r][t], Bv = Bs[t][n];
            const float hprev = t > 0 ? H[t - 1] : hs;
            const float gn = fmaf(ds, Cs[t][n], G);
            pC[t][r][n] = ds * H[t];
            pB[t][r][n] = gn * dus[r][t];
            const float du_p = half_warp_sum(gn * dt * Bv);
            const float dd_p = half_warp_sum(gn * fmaf(Bv, uus[r][t], hprev * Av[t] * Areal));
            if (n == t) {
                rdu[r][t] = du_p;
                rdd[r][t] = dd_p;
            }
            dA_acc = fmaf(gn * hprev, Av[t] * dt, dA_acc);
            G = Av[t] * gn;
        }
        __syncthreads();

        // item (row r, step n): du, ddelta; B/C gradients of (step, state) = (tid / 16, tid % 16)
        if (in) {
            const float du = fmaf(dss[r][n], Dd, rdu[r][n]);
            float dd = rdd[r][n];
            if (p.softplus) {
                const float v = ldv<T>(p.delta, b * p.dl_sb + dc * p.dl_sd + ti) + bias;
                dd *= __fdividef(1.f, 1.f + ex2_approx(-v * kLog2e));
            }
            static_cast<T *>(q.du)[b * q.du_sb + dc * q.du_sd + ti] = from_f32<T>(du);
            static_cast<T *>(q.ddelta)[b * q.dd_sb + dc * q.dd_sd + ti] = from_f32<T>(dd);
            dbias_acc += dd;
        }
        {
            const int tt = tid / kN, nn = tid % kN;
            const int64_t ts = c * kT + tt;
            if (nn < dstate && ts < L) {
                float sb = 0.f, sc = 0.f;
#pragma unroll
                for (int rr = 0; rr < kRows; ++rr) {
                    sb += pB[tt][rr][nn];
                    sc += pC[tt][rr][nn];
                }
                atomicAdd(q.dB + (b * dstate + nn) * L + ts, sb);
                atomicAdd(q.dC + (b * dstate + nn) * L + ts, sc);
            }
        }
        __syncthreads();
    }

    if (ok && live) {
        if (q.dh0) q.dh0[row * dstate + n] = G;
        atomicAdd(q.dA + dc * dstate + n, dA_acc);
    }
    // per-row sums over the 16 step-slots of the row's threads
    const float dD_row = half_warp_sum(dD_acc);
    const float db_row = half_warp_sum(dbias_acc);
    if (ok && n == 0) {
        if (q.dD) atomicAdd(q.dD + dc, dD_row);
        if (q.dbias) atomicAdd(q.dbias + dc, db_row);
    }
}

}  // namespace

size_t bwd_workspace_bytes(const ScanParams &p) {
    const int64_t nchunks = (p.seqlen + kT - 1) / kT;
    return static_cast<size_t>(p.batch * p.dim) * static_cast<size_t>(nchunks) * kN * sizeof(float);
}

cudaError_t launch_bwd(const ScanParams &p, const BwdParams &q, int in_dtype, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((p.dim + kRows - 1) / kRows), static_cast<unsigned>(p.batch));
    if (in_dtype == 0)
        bwd_kernel<float><<<grid, kBwdThreads, 0, stream>>>(p, q);
    else
        bwd_kernel<__nv_bfloat16><<<grid, kBwdThreads, 0, stream>>>(p, q);
    return cudaGetLastError();
}

}  // namespace ms
