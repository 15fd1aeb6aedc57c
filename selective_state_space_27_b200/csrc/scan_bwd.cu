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
// Per-(row, t) sums over the 16 states go through [row][step][state] tiles
// in shared memory (written by the chain threads, summed by one thread per
// (row, step) with four vector loads; both access patterns are free of bank
// conflicts); the B and C
// gradients are summed over the CTA's rows the same way and added to global
// memory with atomics, as are the A, D and delta_bias gradients (sums over
// the batch). The caller's reduction outputs are zeroed first.
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

// Dynamic shared memory of a CTA, in floats. The per-row step tiles have rows
// of 20 floats (16-byte aligned) so that a chain thread reads four steps of its
// row with one vector load.
constexpr int kTS = kT + 4;
constexpr int kRT = kRows * kTS;                 // a [row][step] tile
constexpr int kTN = kT * (kN + 1);               // a [step][state] tile
// [step][row][state] tiles summed over the rows by one thread per (step, state):
// rows 16 floats apart, steps 272, so that the two rows a warp writes and the
// two steps a warp sums fall on disjoint banks
constexpr int kBR = kN, kBT = kRows * kN + 16;
constexpr int kRNT = kT * kBT;
// [row][step][state] tiles summed over the states by one thread per (row, step):
// steps 20 floats apart, rows 336 (both write and read patterns conflict free)
constexpr int kQS = kN + 4, kQR = kT * kQS + 16;
constexpr int kRTN = kRows * kQR;
constexpr int kBwdSmemFloats = 4 * kRT + 2 * kTN + 2 * kRNT + 2 * kRTN;
static_assert(kRTN <= 2 * kRNT, "the readout tile aliases the B and C gradient tiles");

template <typename T>
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_kernel(const ScanParams p, const BwdParams q) {
    extern __shared__ __align__(16) float smf[];
    auto dts = reinterpret_cast<float (*)[kTS]>(smf);
    auto dus = reinterpret_cast<float (*)[kTS]>(smf + kRT);
    auto uus = reinterpret_cast<float (*)[kTS]>(smf + 2 * kRT);
    auto dss = reinterpret_cast<float (*)[kTS]>(smf + 3 * kRT);
    auto Bs = reinterpret_cast<float (*)[kN + 1]>(smf + 4 * kRT);
    auto Cs = reinterpret_cast<float (*)[kN + 1]>(smf + 4 * kRT + kTN);
    float *tiles = smf + 4 * kRT + 2 * kTN;
    float *pB = tiles;                                                          // [step][row][state]
    float *pC = tiles + kRNT;
    auto trs = [](int step, int row, int state) { return step * kBT + row * kBR + state; };
    float *pS = tiles;                                                          // [row][step][state], before pB
    float *pDU = tiles + 2 * kRNT;
    float *pDD = tiles + 2 * kRNT + kRTN;
    auto rts = [](int row, int step, int state) { return row * kQR + step * kQS + state; };
    // sum over the 16 states of (row, step) in a [row][step][state] tile
    auto state_sum = [&](const float *tile, int row, int step) {
        const float4 *v = reinterpret_cast<const float4 *>(tile + rts(row, step, 0));
        const float4 a = v[0], b4 = v[1], c4 = v[2], d4 = v[3];
        return ((a.x + a.y) + (a.z + a.w)) + ((b4.x + b4.y) + (b4.z + b4.w)) + ((c4.x + c4.y) + (c4.z + c4.w)) +
               ((d4.x + d4.y) + (d4.z + d4.w));
    };

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

    // The raw values one thread contributes to chunk c's tiles: item (row r,
    // step n) -- u, delta_raw, dy, z -- and (step, state) (tid / 16, tid % 16)
    // of the B and C tiles. Loaded one chunk ahead of use, so the global
    // latency hides behind the current chunk's work.
    struct RawVals { float u, dl, dy, z, bv, cv; };
    auto load_raw = [&](int64_t c, bool grads) {
        RawVals v{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const int64_t t = c * kT + n;
        if (ok && t < L) {
            v.u = ldv<T>(p.u, b * p.u_sb + dc * p.u_sd + t);
            v.dl = ldv<T>(p.delta, b * p.dl_sb + dc * p.dl_sd + t);
            if (grads) {
                v.dy = ldv<T>(q.dy, b * q.dy_sb + dc * q.dy_sd + t);
                if (p.z) v.z = ldv<T>(p.z, b * p.z_sb + dc * p.z_sd + t);
            }
        }
        const int tt = tid / kN, nn = tid % kN;
        const int64_t ts = c * kT + tt;
        if (nn < dstate && ts < L) {
            v.bv = ldv<T>(p.B, b * p.B_sb + nn * p.B_sn + ts);
            if (grads) v.cv = ldv<T>(p.C, b * p.C_sb + nn * p.C_sn + ts);
        }
        return v;
    };
    // Stage chunk c's tiles from its raw values: per (row, step) delta, delta u
    // and u (steps past the end: delta = 0, the identity); per (step, state) B, C.
    auto stage = [&](int64_t c, const RawVals &v) {
        const bool in = ok && c * kT + n < L;
        const float dt = in ? (p.softplus ? softplus(v.dl + bias) : v.dl + bias) : 0.f;
        dts[r][n] = dt;
        dus[r][n] = dt * v.u;
        uus[r][n] = v.u;
        Bs[tid / kN][tid % kN] = v.bv;
        Cs[tid / kN][tid % kN] = v.cv;
    };

    // ---- Phase F: checkpoints at the end of every chunk but the last ----
    const float h_init = (live && p.h0) ? p.h0[row * dstate + n] : 0.f;
    float h = h_init;
    RawVals nxt = nchunks > 1 ? load_raw(0, false) : RawVals{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t c = 0; c + 1 < nchunks; ++c) {
        const RawVals cur = nxt;
        stage(c, cur);
        if (c + 2 < nchunks) nxt = load_raw(c + 1, false);
        __syncthreads();
#pragma unroll
        for (int t4 = 0; t4 < kT; t4 += 4) {
            const float4 dt4 = *reinterpret_cast<const float4 *>(&dts[r][t4]);
            const float4 du4 = *reinterpret_cast<const float4 *>(&dus[r][t4]);
            const float dtv[4] = {dt4.x, dt4.y, dt4.z, dt4.w}, duv[4] = {du4.x, du4.y, du4.z, du4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) h = fmaf(ex2_approx(dtv[e] * A2), h, duv[e] * Bs[t4 + e][n]);
        }
        if (ok) ckpt[c * kN] = h;   // rows past the end share a clamped index: no checkpoints
        __syncthreads();
    }

    // ---- Phase B ----
    float G = (live && ok && q.dhT) ? q.dhT[row * dstate + n] : 0.f;   // a_{t+1} g_{t+1}, carried down
    float dA_acc = 0.f, dD_acc = 0.f, dbias_acc = 0.f;
    nxt = load_raw(nchunks - 1, true);
    for (int64_t c = nchunks - 1; c >= 0; --c) {
        const RawVals cur = nxt;
        stage(c, cur);
        if (c > 0) nxt = load_raw(c - 1, true);
        // dy and z of item (row r, step n)
        const int64_t ti = c * kT + n;
        const bool in = ok && ti < L;
        const float dyv = cur.dy, zv = cur.z;
        __syncthreads();

        // recompute the chunk's states from the previous checkpoint
        const float hs = (c > 0 && ok) ? ckpt[(c - 1) * kN] : h_init;
        float H[kT], Av[kT];
        {
            float hh = hs;
#pragma unroll
            for (int t4 = 0; t4 < kT; t4 += 4) {
                const float4 dt4 = *reinterpret_cast<const float4 *>(&dts[r][t4]);
                const float4 du4 = *reinterpret_cast<const float4 *>(&dus[r][t4]);
                const float dtv[4] = {dt4.x, dt4.y, dt4.z, dt4.w}, duv[4] = {du4.x, du4.y, du4.z, du4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    Av[t4 + e] = ex2_approx(dtv[e] * A2);
                    hh = fmaf(Av[t4 + e], hh, duv[e] * Bs[t4 + e][n]);
                    H[t4 + e] = hh;
                }
            }
        }
        // ds, dz of item (row r, step n); s_t sums C h over the row's states
#pragma unroll
        for (int t = 0; t < kT; ++t) pS[rts(r, t, n)] = Cs[t][n] * H[t];
        __syncthreads();
        const float s_mine = Dd * uus[r][n] + state_sum(pS, r, n);
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
        for (int t4 = kT - 4; t4 >= 0; t4 -= 4) {
            const float4 ds4 = *reinterpret_cast<const float4 *>(&dss[r][t4]);
            const float4 dt4 = *reinterpret_cast<const float4 *>(&dts[r][t4]);
            const float4 du4 = *reinterpret_cast<const float4 *>(&dus[r][t4]);
            const float4 uu4 = *reinterpret_cast<const float4 *>(&uus[r][t4]);
            const float dsv4[4] = {ds4.x, ds4.y, ds4.z, ds4.w}, dtv4[4] = {dt4.x, dt4.y, dt4.z, dt4.w};
            const float duv4[4] = {du4.x, du4.y, du4.z, du4.w}, uuv4[4] = {uu4.x, uu4.y, uu4.z, uu4.w};
#pragma unroll
            for (int e = 3; e >= 0; --e) {
                const int t = t4 + e;
                const float ds = dsv4[e], dt = dtv4[e], Bv = Bs[t][n];
                const float hprev = t > 0 ? H[t - 1] : hs;
                const float gn = fmaf(ds, Cs[t][n], G);
                pC[trs(t, r, n)] = ds * H[t];
                pB[trs(t, r, n)] = gn * duv4[e];
                pDU[rts(r, t, n)] = gn * dt * Bv;
                pDD[rts(r, t, n)] = gn * fmaf(Bv, uuv4[e], hprev * Av[t] * Areal);
                dA_acc = fmaf(gn * hprev, Av[t] * dt, dA_acc);
                G = Av[t] * gn;
            }
        }
        __syncthreads();

        // item (row r, step n): du, ddelta; B/C gradients of (step, state) = (tid / 16, tid % 16)
        if (in) {
            const float du = dss[r][n] * Dd + state_sum(pDU, r, n);
            float dd = state_sum(pDD, r, n);
            if (p.softplus) dd *= __fdividef(1.f, 1.f + ex2_approx(-(cur.dl + bias) * kLog2e));
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
                    sb += pB[trs(tt, rr, nn)];
                    sc += pC[trs(tt, rr, nn)];
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
    const int smem = kBwdSmemFloats * static_cast<int>(sizeof(float));
    const void *k = in_dtype == 0 ? reinterpret_cast<const void *>(bwd_kernel<float>)
                                  : reinterpret_cast<const void *>(bwd_kernel<__nv_bfloat16>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    void *args[] = {const_cast<ScanParams *>(&p), const_cast<BwdParams *>(&q)};
    e = cudaLaunchKernel(k, grid, dim3(kBwdThreads), args, static_cast<size_t>(smem), stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ms
