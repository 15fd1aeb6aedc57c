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
//   du_t = delta_t sum_n g_tn B_tn + ds_t D
//   ddelta_t = u_t sum_n g_tn B_tn + sum_n g_tn h_{t-1,n} a_tn A_n  (* sigmoid(raw) under softplus)
//   dA_n += g_tn h_{t-1,n} a_tn delta_t, dD += ds_t u_t, dh_0 = a_0 g_0.
//
// Design. The lanes hold the state as the forward's sequential kernel does:
// LPR lanes per channel row (4 or 8), each with 16 / LPR of its 16 states,
// 32 / LPR rows per warp, one warp per CTA. Phase F runs the
// recurrence forward and leaves the state at the end of every chunk of 8
// steps in a workspace (one float per chain and chunk). Phase B walks the
// chunks backward: it recomputes the chunk's 8 states and decays from the
// previous checkpoint into registers, then runs the adjoint recurrence
// through them. Every sum is a register reduction inside the warp:
//   - per (row, step) sums over the states (s_t, sum g B, sum g h a A) are
//     summed over the row's LPR lanes in a transposed shuffle reduction, so
//     that lane q ends with the totals of steps q, q + LPR, ..., the steps
//     whose scalar work (gate, softplus derivative, stores) it does;
//   - per (step, state) sums over the rows (the B and C gradients) are summed
//     over the warp's rows the same way, leaving each lane one (tensor,
//     state) total per step, which it adds to global memory in one vector
//     reduction (red.global.add.v4.f32) per 4 steps.
// The warps are independent: each stages its own rows' per-chunk inputs
// (delta, delta u, u, ds per row and step) and its own copy of the chunk's B
// and C ([step][state]) in shared memory, read as broadcasts, and only
// synchronises with itself. The checkpoint a chunk starts from is loaded one
// chunk ahead. The A, D and delta_bias gradients are register sums added once
// per row. The caller's reduction outputs are zeroed first.
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kN = 16;                 // states per row (smaller dstate is zero-padded)
constexpr int kW = 1;                  // warps per CTA (independent; one-warp CTAs balance best)
constexpr int kT = 8;                  // steps per chunk (checkpoint interval)
constexpr int kBwdThreads = kW * 32;
constexpr int kBCL = kT * kN / 32;     // B (and C) entries a lane stages per chunk
static_assert(kT * kN % 32 == 0 && 32 % kT == 0, "whole B/C entries per lane");

// Shared memory of a warp, in floats. Per row: delta, delta u, u and ds of
// the chunk's steps at offsets 0, 8, 16, 24, rows 36 floats apart so that the
// rows fall on distinct bank groups; then the B and C tiles, [step][state]
// with steps 20 floats apart (the staging stores, eight steps of one state
// per quarter-warp, hit distinct banks; the reads are broadcasts).
constexpr int kF_DT = 0, kF_DU = kT, kF_U = 2 * kT, kF_DS = 3 * kT;
constexpr int kXR = 4 * kT + 4;
constexpr int kBS = kN + 4;
constexpr int kBC = kT * kBS;

template <int LPR> struct BwdShape {
    static constexpr int NPL = kN / LPR;        // states per lane
    static constexpr int NP = NPL / 2;          // ... as float2 pairs
    static constexpr int RW = 32 / LPR;         // rows per warp
    static constexpr int ROWS = kW * RW;        // rows per CTA
    static constexpr int IPL = kT / LPR;        // steps a lane finishes per chunk
    static constexpr int WARP_FLOATS = RW * kXR + 2 * kBC;
    static constexpr int SMEM_FLOATS = kW * WARP_FLOATS;
    static constexpr int MINB = LPR == 4 ? 10 : 16;   // resident CTAs: the register budget per thread
    static_assert(LPR == 4 || LPR == 8, "4 or 8 lanes per row");
    static_assert(2 * NPL == RW, "the row reduction leaves one value per lane");
};

// Transposed sum over the row's K lanes (the low lane bits, K a power of 2)
// of v[0..K-1], partial sums of K consecutive steps: lane q returns the total
// of step q. Each round a lane keeps half of its values, adds the partner's
// copy of that half and passes on the other half.
// With STRIDE > 1 the same over the lanes q STRIDE (the rows of a warp).
template <int K, int STRIDE>
__device__ __forceinline__ float transposed_sum(float (&v)[K], int q) {
#pragma unroll
    for (int half = K / 2; half >= 1; half /= 2) {
        const bool hi = q & half;
#pragma unroll
        for (int e = 0; e < half; ++e) {
            const float keep = hi ? v[e + half] : v[e];
            const float send = hi ? v[e] : v[e + half];
            v[e] = keep + __shfl_xor_sync(0xffffffffu, send, half * STRIDE);
        }
    }
    return v[0];
}

// Fire-and-forget vector reduction into global memory (16-byte aligned dst):
// no value comes back, so nothing waits on the round trip.
__device__ __forceinline__ void red_add4(float *dst, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float sigmoid(float x) { return __fdividef(1.f, 1.f + ex2_approx(-x * kLog2e)); }

// The lane's NPL entries of step t of a [step][state] tile, as pairs.
template <int NP>
__device__ __forceinline__ void ld_pairs(const float *src, float2 (&o)[NP]) {
    if constexpr (NP == 2) {
        const float4 w = *reinterpret_cast<const float4 *>(src);
        o[0] = f2(w.x, w.y);
        o[1] = f2(w.z, w.w);
    } else {
        o[0] = *reinterpret_cast<const float2 *>(src);
    }
}

template <typename T, int LPR>
__global__ void __launch_bounds__(kBwdThreads, BwdShape<LPR>::MINB) bwd_kernel(const ScanParams p, const BwdParams g) {
    using S = BwdShape<LPR>;
    constexpr int NPL = S::NPL, NP = S::NP, RW = S::RW, IPL = S::IPL;
    extern __shared__ __align__(16) float smf[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int q = lane % LPR, rw = lane / LPR;
    float *xt = smf + warp * S::WARP_FLOATS;
    float *bt = xt + RW * kXR;
    float *ct = bt + kBC;
    const int64_t b = blockIdx.y;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * S::ROWS + warp * RW;   // the warp's first row
    const int64_t d = row0 + rw;
    const bool ok = d < p.dim;
    const bool warp_live = row0 < p.dim;
    const int64_t dc = ok ? d : p.dim - 1;
    const int dstate = static_cast<int>(p.dstate);
    const int L = static_cast<int>(p.seqlen);   // at most 2^30 (checked by the caller)
    const int nchunks = (L + kT - 1) / kT;
    const int64_t row = b * p.dim + dc;
    float *xr = xt + rw * kXR;
    // the row's sequences, indexed by step
    const T *u_row = static_cast<const T *>(p.u) + b * p.u_sb + dc * p.u_sd;
    const T *dl_row = static_cast<const T *>(p.delta) + b * p.dl_sb + dc * p.dl_sd;
    const T *dy_row = static_cast<const T *>(g.dy) + b * g.dy_sb + dc * g.dy_sd;
    const T *z_row = p.z ? static_cast<const T *>(p.z) + b * p.z_sb + dc * p.z_sd : u_row;
    T *du_row = static_cast<T *>(g.du) + b * g.du_sb + dc * g.du_sd;
    T *dd_row = static_cast<T *>(g.ddelta) + b * g.dd_sb + dc * g.dd_sd;
    T *dz_row = g.dz ? static_cast<T *>(g.dz) + b * g.dz_sb + dc * g.dz_sd : du_row;
    // the lane's B / C tile entries j: state lane / 8 + 4 j, step lane % 8 of the chunk
    const T *b_lane = static_cast<const T *>(p.B) + b * p.B_sb + (lane / kT) * p.B_sn + lane % kT;
    const T *c_lane = static_cast<const T *>(p.C) + b * p.C_sb + (lane / kT) * p.C_sn + lane % kT;
    const int64_t b_jstride = (32 / kT) * p.B_sn, c_jstride = (32 / kT) * p.C_sn;

    // the lane's states n = NPL q .. NPL q + NPL - 1: A (and A log2 e), padded with 0
    float Ar[NPL];
    float2 ap[NP];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int n = NPL * q + i;
        Ar[i] = n < dstate ? __ldg(p.A + dc * dstate + n) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < NP; ++j) ap[j] = f2(Ar[2 * j] * kLog2e, Ar[2 * j + 1] * kLog2e);
    const float bias = p.delta_bias ? __ldg(p.delta_bias + dc) : 0.f;
    const float Dd = p.D ? __ldg(p.D + dc) : 0.f;
    // checkpoint c (the state at the end of chunk c) of the lane's states
    float *ck = g.ckpt + row * nchunks * kN + NPL * q;
    auto ck_store = [&](int c, const float2 (&h)[NP]) {
        if constexpr (NP == 2)
            *reinterpret_cast<float4 *>(ck + c * kN) = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
        else
            *reinterpret_cast<float2 *>(ck + c * kN) = h[0];
    };

    // The raw values one lane contributes to chunk c: its row's steps
    // q + LPR k (u, delta_raw and, in phase B, dy and z) and entries
    // lane + 32 j of its warp's B and C tiles (state e / 8, step e % 8: eight
    // lanes read eight consecutive steps of one state). Loaded a chunk ahead.
    struct Raw {
        float u[IPL], dl[IPL], dy[IPL], z[IPL], bv[kBCL], cv[kBCL];
    };
    // (bounds are checked only in the ragged last chunk)
    auto load_raw = [&](int c, bool grads) {
        Raw v;
        const int t0 = c * kT;
        const bool full = t0 + kT <= L;
#pragma unroll
        for (int k = 0; k < IPL; ++k) {
            v.u[k] = v.dl[k] = v.dy[k] = v.z[k] = 0.f;
            const int t = t0 + q + LPR * k;
            if (ok && (full || t < L)) {
                v.u[k] = to_f32<T>(u_row[t]);
                v.dl[k] = to_f32<T>(dl_row[t]);
                if (grads) {
                    v.dy[k] = to_f32<T>(dy_row[t]);
                    if (p.z) v.z[k] = to_f32<T>(z_row[t]);
                }
            }
        }
        const bool tin = full || t0 + lane % kT < L;
#pragma unroll
        for (int j = 0; j < kBCL; ++j) {
            v.bv[j] = v.cv[j] = 0.f;
            if (tin && lane / kT + (32 / kT) * j < dstate) {
                v.bv[j] = to_f32<T>(b_lane[j * b_jstride + t0]);
                if (grads) v.cv[j] = to_f32<T>(c_lane[j * c_jstride + t0]);
            }
        }
        return v;
    };
    // Stage chunk c: delta, delta u and u of the lane's steps (steps past the
    // end: delta = 0, the identity), its B and C entries.
    auto stage = [&](int c, const Raw &v) {
#pragma unroll
        for (int k = 0; k < IPL; ++k) {
            const int t = q + LPR * k;
            const bool in = ok && c * kT + t < L;
            const float x = v.dl[k] + bias;
            const float dt = in ? (p.softplus ? softplus(x) : x) : 0.f;
            xr[kF_DT + t] = dt;
            xr[kF_DU + t] = dt * v.u[k];
            xr[kF_U + t] = v.u[k];
        }
#pragma unroll
        for (int j = 0; j < kBCL; ++j) {
            const int e = lane + 32 * j, nn = e / kT, tt = e % kT;
            bt[tt * kBS + nn] = v.bv[j];
            ct[tt * kBS + nn] = v.cv[j];
        }
    };
    // eight steps of a per-row field
    auto row8 = [&](int f, float (&o)[kT]) {
        const float4 a = *reinterpret_cast<const float4 *>(xr + f);
        const float4 c4 = *reinterpret_cast<const float4 *>(xr + f + 4);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = c4.x; o[5] = c4.y; o[6] = c4.z; o[7] = c4.w;
    };

    // ---- Phase F: the state at the end of every chunk but the last ----
    float2 h_init[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        float h2[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = NPL * q + 2 * j + e;
            if (p.h0 && ok && n < dstate) h2[e] = __ldg(p.h0 + row * dstate + n);
        }
        h_init[j] = f2(h2[0], h2[1]);
    }
    if (!g.ckpt_ready) {   // (skipped when the forward left the checkpoints)
        float2 hp[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) hp[j] = h_init[j];
        Raw nxt;
        if (nchunks > 1) nxt = load_raw(0, false);
        for (int c = 0; c + 1 < nchunks; ++c) {
            const Raw cur = nxt;
            stage(c, cur);
            if (c + 2 < nchunks) nxt = load_raw(c + 1, false);
            __syncwarp();
            float dtv[kT], duv[kT];
            row8(kF_DT, dtv);
            row8(kF_DU, duv);
#pragma unroll
            for (int t = 0; t < kT; ++t) {
                float2 Bp[NP];
                ld_pairs<NP>(bt + t * kBS + NPL * q, Bp);
                const float2 dt2 = f2(dtv[t], dtv[t]), du2 = f2(duv[t], duv[t]);
#pragma unroll
                for (int j = 0; j < NP; ++j) hp[j] = fma2(ex2x2(mul2(dt2, ap[j])), hp[j], mul2(du2, Bp[j]));
            }
            if (ok) ck_store(c, hp);
            __syncwarp();
        }
    }

    // ---- Phase B ----
    float2 G[NP];   // a_{t+1} g_{t+1}, carried down
    float2 dA[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        float g2[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = NPL * q + 2 * j + e;
            if (ok && g.dhT && n < dstate) g2[e] = g.dhT[row * dstate + n];
        }
        G[j] = f2(g2[0], g2[1]);
        dA[j] = f2(0.f, 0.f);
    }
    float dD_acc = 0.f, dbias_acc = 0.f;
    const bool vec_atomic =
        ((reinterpret_cast<uintptr_t>(g.dB) | reinterpret_cast<uintptr_t>(g.dC)) & 15u) == 0 && (L & 3) == 0;
    // the state chunk c starts from: its predecessor's checkpoint (rows past
    // the end have none and carry zeros), or the initial state
    auto start_state = [&](int c, float2 (&h)[NP]) {
        if (c > 0 && ok) {
            ld_pairs<NP>(ck + (c - 1) * kN, h);
        } else {
#pragma unroll
            for (int j = 0; j < NP; ++j) h[j] = h_init[j];
        }
    };
    Raw nxt = load_raw(nchunks - 1, true);
    float2 hnext[NP];
    start_state(nchunks - 1, hnext);
    for (int c = nchunks - 1; c >= 0; --c) {
        const Raw cur = nxt;
        float2 hs[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) hs[j] = hnext[j];
        stage(c, cur);
        if (c > 0) {
            nxt = load_raw(c - 1, true);
            start_state(c - 1, hnext);
        }
        __syncwarp();

        float dtv[kT], duv[kT];
        row8(kF_DT, dtv);
        row8(kF_DU, duv);
        // recompute the chunk's states and decays from the previous checkpoint
        float2 H[kT][NP], Av[kT][NP];
        float s_own[IPL];   // C h summed over the row's states, the lane's steps
        {
            float2 hh[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) hh[j] = hs[j];
#pragma unroll
            for (int t0 = 0; t0 < kT; t0 += LPR) {
                float ps[LPR];
#pragma unroll
                for (int e = 0; e < LPR; ++e) {
                    const int t = t0 + e;
                    float2 Bp[NP], Cp[NP];
                    ld_pairs<NP>(bt + t * kBS + NPL * q, Bp);
                    ld_pairs<NP>(ct + t * kBS + NPL * q, Cp);
                    const float2 dt2 = f2(dtv[t], dtv[t]), du2 = f2(duv[t], duv[t]);
                    float2 sc = f2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        Av[t][j] = ex2x2(mul2(dt2, ap[j]));
                        hh[j] = fma2(Av[t][j], hh[j], mul2(du2, Bp[j]));
                        H[t][j] = hh[j];
                        sc = fma2(Cp[j], hh[j], sc);
                    }
                    ps[e] = sc.x + sc.y;
                }
                s_own[t0 / LPR] = transposed_sum<LPR, 1>(ps, q);
            }
        }
        // the lane's steps: ds (to the tile), dz, the D gradient
#pragma unroll
        for (int k = 0; k < IPL; ++k) {
            const int t = q + LPR * k;
            const int ti = c * kT + t;
            const bool in = ok && ti < L;
            const float u = cur.u[k], dy = cur.dy[k];
            float ds = dy;
            if (p.z) {
                const float zv = cur.z[k];
                const float sg = sigmoid(zv);
                if (in && g.dz) {
                    const float s = s_own[k] + Dd * u;
                    dz_row[ti] = from_f32<T>(dy * s * sg * (1.f + zv * (1.f - sg)));
                }
                ds = dy * zv * sg;
            }
            xr[kF_DS + t] = ds;   // 0 past the end (dy = 0 there)
            dD_acc = fmaf(ds, u, dD_acc);
        }
        __syncwarp();
        float dsv[kT];
        row8(kF_DS, dsv);

        // adjoint recurrence through the chunk, last step first
        float red[kT];   // the warp's rows summed: value rw (tensor rw / NPL, state NPL q + rw % NPL) per step
#pragma unroll
        for (int t0 = kT - LPR; t0 >= 0; t0 -= LPR) {
            float s1[LPR], s2[LPR];   // per step: sum of g B, sum of g h_{t-1} a A over the lane's states
#pragma unroll
            for (int e = LPR - 1; e >= 0; --e) {
                const int t = t0 + e;
                float2 Bp[NP], Cp[NP];
                ld_pairs<NP>(bt + t * kBS + NPL * q, Bp);
                ld_pairs<NP>(ct + t * kBS + NPL * q, Cp);
                const float2 ds2 = f2(dsv[t], dsv[t]), du2 = f2(duv[t], duv[t]), dt2 = f2(dtv[t], dtv[t]);
                float v[2 * NPL];   // B gradient partials of the lane's states, then C gradient partials
                float2 a1 = f2(0.f, 0.f), a2 = f2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const float2 gn = fma2(ds2, Cp[j], G[j]);
                    const float2 gB = mul2(gn, du2);
                    const float2 gC = mul2(ds2, H[t][j]);
                    v[2 * j] = gB.x;
                    v[2 * j + 1] = gB.y;
                    v[NPL + 2 * j] = gC.x;
                    v[NPL + 2 * j + 1] = gC.y;
                    a1 = fma2(gn, Bp[j], a1);
                    const float2 hprev = t > 0 ? H[t - 1][j] : hs[j];
                    const float2 gx = mul2(gn, mul2(hprev, Av[t][j]));
                    a2 = fma2(gx, f2(Ar[2 * j], Ar[2 * j + 1]), a2);
                    dA[j] = fma2(gx, dt2, dA[j]);
                    G[j] = mul2(Av[t][j], gn);
                }
                s1[e] = a1.x + a1.y;
                s2[e] = a2.x + a2.y;
                red[t] = transposed_sum<RW, LPR>(v, rw);
            }
            // the lane's step t0 + q: du, ddelta
            const float S1 = transposed_sum<LPR, 1>(s1, q);
            const float S2 = transposed_sum<LPR, 1>(s2, q);
            const int k = t0 / LPR;
            const int t = t0 + q;
            const int ti = c * kT + t;
            if (ok && ti < L) {
                const float u = cur.u[k];
                const float du = fmaf(xr[kF_DT + t], S1, xr[kF_DS + t] * Dd);
                float dd = fmaf(u, S1, S2);
                if (p.softplus) dd *= sigmoid(cur.dl[k] + bias);
                du_row[ti] = from_f32<T>(du);
                dd_row[ti] = from_f32<T>(dd);
                dbias_acc += dd;
            }
        }
        // the lane's (tensor, state) of the B and C gradients, steps c kT .. c kT + 7
        const int n = NPL * q + rw % NPL;
        if (warp_live && n < dstate) {
            const int ts = c * kT;
            float *dst = (rw < NPL ? g.dB : g.dC) + (b * dstate + n) * L + ts;
            if (vec_atomic && ts + kT <= L) {
#pragma unroll
                for (int t4 = 0; t4 < kT; t4 += 4)
                    red_add4(dst + t4, red[t4], red[t4 + 1], red[t4 + 2], red[t4 + 3]);
            } else {
#pragma unroll
                for (int t = 0; t < kT; ++t)
                    if (ts + t < L) atomicAdd(dst + t, red[t]);
            }
        }
        __syncwarp();   // the tiles are read: the next chunk may stage
    }

    if (ok) {
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int n = NPL * q + i;
            if (n < dstate) {
                const float gi = (i & 1) ? G[i / 2].y : G[i / 2].x;
                if (g.dh0) g.dh0[row * dstate + n] = gi;
                atomicAdd(g.dA + dc * dstate + n, (i & 1) ? dA[i / 2].y : dA[i / 2].x);
            }
        }
    }
    // per-row sums over the row's lanes
#pragma unroll
    for (int m = 1; m < LPR; m *= 2) {
        dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m);
        dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, m);
    }
    if (ok && q == 0) {
        if (g.dD) atomicAdd(g.dD + dc, dD_acc);
        if (g.dbias) atomicAdd(g.dbias + dc, dbias_acc);
    }
}

#ifndef MS_BWD_LANES
#define MS_BWD_LANES 4
#endif

template <int LPR>
cudaError_t launch_lpr(const ScanParams &p, const BwdParams &q, int in_dtype, cudaStream_t stream) {
    using S = BwdShape<LPR>;
    const dim3 grid(static_cast<unsigned>((p.dim + S::ROWS - 1) / S::ROWS), static_cast<unsigned>(p.batch));
    const int smem = S::SMEM_FLOATS * static_cast<int>(sizeof(float));
    const void *k = in_dtype == 0 ? reinterpret_cast<const void *>(bwd_kernel<float, LPR>)
                                  : reinterpret_cast<const void *>(bwd_kernel<__nv_bfloat16, LPR>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    void *args[] = {const_cast<ScanParams *>(&p), const_cast<BwdParams *>(&q)};
    e = cudaLaunchKernel(k, grid, dim3(kBwdThreads), args, static_cast<size_t>(smem), stream);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(const ScanParams &p) {
    const int64_t nchunks = (p.seqlen + kT - 1) / kT;
    return static_cast<size_t>(p.batch * p.dim) * static_cast<size_t>(nchunks) * kN * sizeof(float);
}

cudaError_t launch_bwd(const ScanParams &p, const BwdParams &q, int in_dtype, cudaStream_t stream) {
    return launch_lpr<MS_BWD_LANES>(p, q, in_dtype, stream);
}

}  // namespace ms
