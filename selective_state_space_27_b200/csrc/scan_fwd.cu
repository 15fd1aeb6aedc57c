// Selective scan (S6) forward for sm_100a.
//
// What is computed ("Notas sobre Mamba", sections "O mecanismo de seleção (S6)"
// and "A varredura paralela ciente do hardware"; "Mamba-2 e State Space
// Duality (SSD)", section "Como o Mamba-1 alcançou complexidade linear"):
// for every row (b, d) and state index n,
//     h_t[n] = exp(delta_t A[d,n]) h_{t-1}[n] + delta_t B_t[n] u_t
//     y_t    = sum_n C_t[n] h_t[n] + D[d] u_t      (then * silu(z_t))
// with delta_t = softplus(delta_raw_t + delta_bias[d]).
//
// B200 design. The binding unit is the MUFU: one ex2 per (b, d, t, n) element
// at 16 results/clk/SM, against ~0.5 byte of HBM traffic per element, so the
// kernel is built to keep the MUFU busy and to spend as few other issue slots
// as possible per element (the SM issues 128 thread-instructions per clock,
// i.e. 8 per MUFU result):
//  * Every lane owns TWO channel rows (d, d+1) over the same 8 time steps, so
//    all float32 arithmetic runs as packed f32x2 operations (FMUL2/FFMA2)
//    with no register shuffling: one instruction serves both rows.
//  * A group of LG lanes covers one chunk of CH = 8 LG steps of a row pair.
//    Each lane composes its 8 pairs (Abar, Bbar u) sequentially, the group
//    combines the lane aggregates with an LG-lane Kogge-Stone scan over
//    shuffles, the carry of the previous chunk comes from shared memory, and
//    the fix-up h_i = P_i h_in + H_i feeds y_i += C_i h_i directly. The
//    expanded (b, d, t, n) state never leaves registers.
//  * One CTA per SM (or two), sized on the host so that the CTAs of a launch
//    fill the 148 SMs in one balanced wave. The CTA owns R rows of one batch
//    entry and walks the sequence chunk by chunk. B and C -- shared by every
//    row of the batch entry -- are staged once per chunk for all R rows:
//    cp.async brings the raw tiles in one chunk ahead, then the CTA widens
//    them to float32 and stores each value twice ((B_t, B_t) pairs), the
//    operand form of the packed multiply. u, delta and z arrive by cp.async,
//    also one chunk ahead.
//  * softplus uses one ex2 and a degree-6 polynomial for log1p on [0, 1]
//    (coefficients fitted by fit_log1p.py in this directory).
//  * Long sequences with too few rows are split into segments (grid z): a
//    summary pass writes each segment's zero-start end state and decay
//    product, and the main pass starts segment s from the carry composed from
//    the summaries of segments 0..s-1.
#include <mutex>
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kK = 8;            // time steps per lane per chunk
constexpr int kMaxN = 16;        // largest dstate
constexpr int kSegF2 = kK + 2;   // float2 slots per lane segment of the B/C tile (padded: no bank conflicts)

struct Layout {
    int bc, raw, x, a2, carry, carryP, fold, total;
};

// Per row pair: lane aggregates of two state indices ((P, H) of both rows)
// and the states entering each lane, padded so that the row pairs of a warp
// fall on different banks.
template <int LG> struct Fold {
    static constexpr int AGG_F = LG * 8 + 8;   // floats: [lane][u][P.x, H.x, P.y, H.y] + pad
    static constexpr int HIN_F = LG * 4 + 8;   // floats: [lane][u][h.x, h.y] + pad
    static constexpr int BYTES = (AGG_F + HIN_F) * 4;
};

// Shared-memory layout (bytes) of a CTA with W warps.
template <typename T, int LG>
__host__ __device__ __forceinline__ Layout layout(int W) {
    constexpr int CH = LG * kK, EB = sizeof(T);
    const int RP = W * (32 / LG), R = 2 * RP;
    Layout s;
    s.bc = 0;                                                   // [B,C][n][lane seg][kSegF2] float2
    s.raw = s.bc + 2 * kMaxN * LG * kSegF2 * 8;                 // [buf][B,C][n][CH] T
    s.x = s.raw + 2 * 2 * kMaxN * CH * EB;                      // [stage][u,delta,z][row][CH] T
    s.a2 = s.x + 2 * 3 * R * CH * EB;                           // [row pair][n] float2
    s.carry = s.a2 + RP * kMaxN * 8;                            // [2][row pair][n] float2
    s.carryP = s.carry + 2 * RP * kMaxN * 8;                    // [row pair][n] float2
    s.fold = s.carryP + RP * kMaxN * 8;                         // [row pair] Fold<LG>
    s.total = s.fold + RP * Fold<LG>::BYTES;
    return s;
}

__device__ __forceinline__ float2 shfl_up2(float2 v, int off, int width) {
    return f2(__shfl_up_sync(0xffffffffu, v.x, off, width), __shfl_up_sync(0xffffffffu, v.y, off, width));
}

// 64-bit register views of a float pair, for the predicated packed ops below.
__device__ __forceinline__ unsigned long long b64(float2 v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 unb64(unsigned long long v) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
    return f2(a, b);
}

// If `take`: (P, H) <- (Pu, Hu) o (P, H) = (P Pu, P Hu + H), the earlier
// segment (Pu, Hu) composed in front. Predicated packed ops instead of
// selects: no ALU work for the lanes that keep their value.
__device__ __forceinline__ void compose_if(int take, float2 &P, float2 &H, float2 Pu, float2 Hu) {
    unsigned long long p = b64(P), h = b64(H);
    asm("{\n\t.reg .pred q;\n\tsetp.ne.s32 q, %4, 0;\n\t"
        "@q fma.rn.f32x2 %1, %0, %3, %1;\n\t@q mul.rn.f32x2 %0, %0, %2;\n\t}"
        : "+l"(p), "+l"(h)
        : "l"(b64(Pu)), "l"(b64(Hu)), "r"(take));
    P = unb64(p);
    H = unb64(h);
}

// take ? Pe c + He : c  (the state entering a lane's steps; lane 0 of a group
// takes the chunk carry unchanged).
__device__ __forceinline__ float2 enter_state(int take, float2 Pe, float2 He, float2 c) {
    unsigned long long r = b64(c);
    asm("{\n\t.reg .pred q;\n\tsetp.ne.s32 q, %3, 0;\n\t@q fma.rn.f32x2 %0, %1, %0, %2;\n\t}"
        : "+l"(r)
        : "l"(b64(Pe)), "l"(b64(He)), "r"(take));
    return unb64(r);
}

// The lane's 8 steps of two consecutive rows of an input tile, as (row, row+1) pairs.
template <typename T>
__device__ __forceinline__ void lds_pair(const unsigned char *row0, int row_bytes, float2 (&v)[kK]) {
    if constexpr (std::is_same<T, float>::value) {
        const float4 *a = reinterpret_cast<const float4 *>(row0);
        const float4 *b = reinterpret_cast<const float4 *>(row0 + row_bytes);
#pragma unroll
        for (int q = 0; q < kK / 4; ++q) {
            const float4 x = a[q], y = b[q];
            v[4 * q + 0] = f2(x.x, y.x); v[4 * q + 1] = f2(x.y, y.y);
            v[4 * q + 2] = f2(x.z, y.z); v[4 * q + 3] = f2(x.w, y.w);
        }
    } else {
        const uint4 x = *reinterpret_cast<const uint4 *>(row0);
        const uint4 y = *reinterpret_cast<const uint4 *>(row0 + row_bytes);
        v[0] = f2(bf16_lo(x.x), bf16_lo(y.x)); v[1] = f2(bf16_hi(x.x), bf16_hi(y.x));
        v[2] = f2(bf16_lo(x.y), bf16_lo(y.y)); v[3] = f2(bf16_hi(x.y), bf16_hi(y.y));
        v[4] = f2(bf16_lo(x.z), bf16_lo(y.z)); v[5] = f2(bf16_hi(x.z), bf16_hi(y.z));
        v[6] = f2(bf16_lo(x.w), bf16_lo(y.w)); v[7] = f2(bf16_hi(x.w), bf16_hi(y.w));
    }
}

template <typename T>
__device__ __forceinline__ void store_row(T *dst, const float2 (&y)[kK], bool second, int64_t count,
                                          bool vec) {
    if (vec && count >= kK) {
        if constexpr (std::is_same<T, float>::value) {
            float4 *o = reinterpret_cast<float4 *>(dst);
            if (!second) {
                o[0] = make_float4(y[0].x, y[1].x, y[2].x, y[3].x);
                o[1] = make_float4(y[4].x, y[5].x, y[6].x, y[7].x);
            } else {
                o[0] = make_float4(y[0].y, y[1].y, y[2].y, y[3].y);
                o[1] = make_float4(y[4].y, y[5].y, y[6].y, y[7].y);
            }
        } else {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 h = second ? __floats2bfloat162_rn(y[2 * e].y, y[2 * e + 1].y)
                                                : __floats2bfloat162_rn(y[2 * e].x, y[2 * e + 1].x);
                w[e] = *reinterpret_cast<const uint32_t *>(&h);
            }
            *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < kK; ++i)
            if (i < count) dst[i] = from_f32<T>(second ? y[i].y : y[i].x);
    }
}

// One kernel configuration: lanes per row pair (LG), state indices processed
// together per loop body (NI, 2 doubles the independent dependency chains of a
// warp at the price of registers), and the launch bounds that set the register
// budget (MAXT threads per CTA, MINB CTAs per SM).
template <typename T, int LG, int NI, int MAXT, int MINB, bool VEC, bool SUMMARY>
__global__ void __launch_bounds__(MAXT, MINB)
scan_kernel(const ScanParams p) {
    constexpr int PG = 32 / LG, CH = LG * kK, EB = sizeof(T), VE = 16 / EB;
    constexpr int ROWB = CH * EB;
    constexpr int PPR = ROWB / 16;            // 16-byte pieces per input-tile row (divides 32)
    constexpr int PPN = CH / VE;              // 16-byte pieces per B/C tile row (divides 32)
    const int NT = blockDim.x, W = NT >> 5;
    const int RP = W * PG, R = 2 * RP;
    const Layout Ls = layout<T, LG>(W);

    extern __shared__ __align__(16) unsigned char smem[];
    float2 *bc = reinterpret_cast<float2 *>(smem + Ls.bc);
    unsigned char *raw = smem + Ls.raw;
    unsigned char *xs = smem + Ls.x;
    float2 *a2s = reinterpret_cast<float2 *>(smem + Ls.a2);
    float2 *carry = reinterpret_cast<float2 *>(smem + Ls.carry);
    float2 *carryP = reinterpret_cast<float2 *>(smem + Ls.carryP);
    float *fold_agg = reinterpret_cast<float *>(smem + Ls.fold);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane / LG, j = lane % LG;
    const int rp = warp * PG + g;                       // row pair within the CTA
    const int64_t b = blockIdx.y;
    const int64_t d0 = static_cast<int64_t>(blockIdx.x) * R;
    const int64_t dA = d0 + 2 * rp, dB = dA + 1;        // the lane's two rows
    const bool okA = dA < p.dim, okB = dB < p.dim;
    const int dstate = static_cast<int>(p.dstate);
    const int seg = blockIdx.z;
    const int64_t t_begin = static_cast<int64_t>(seg) * p.seg_len;
    const int64_t t_end = min64(p.seqlen, t_begin + p.seg_len);
    const int nchunks = static_cast<int>((t_end - t_begin + CH - 1) / CH);
    const bool has_z = !SUMMARY && p.z != nullptr;
    const int ntens = has_z ? 3 : 2;

    // Per row-pair constants (A log2 e) and the carry entering this segment.
    for (int i = tid; i < RP * kMaxN; i += NT) {
        const int r = i / kMaxN, n = i % kMaxN;
        float av[2] = {0.f, 0.f}, cv[2] = {0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t dd = d0 + 2 * r + h;
            if (dd < p.dim && n < dstate) {
                av[h] = p.A[dd * dstate + n] * kLog2e;
                if (!SUMMARY) {
                    const int64_t row = b * p.dim + dd;
                    float c = p.h0 ? p.h0[row * dstate + n] : 0.f;
                    for (int s = 0; s < seg; ++s) {
                        const int64_t w = (row * p.nseg + s) * kMaxN + n;
                        c = fmaf(p.ws_P[w], c, p.ws_H[w]);
                    }
                    cv[h] = c;
                }
            }
        }
        a2s[i] = f2(av[0], av[1]);
        carry[i] = f2(cv[0], cv[1]);
        carryP[i] = f2(1.f, 1.f);
    }

    // ---- staging ---------------------------------------------------------------
    // Thread tid always moves piece (tid % PPR) of rows tid / PPR, tid / PPR +
    // NT / PPR, ... -- no division inside the chunk loop.
    const int x_pc = tid % PPR, x_r0 = tid / PPR, x_rstep = NT / PPR;
    const int b_pc = tid % PPN, b_r0 = tid / PPN, b_rstep = NT / PPN;
    // u, delta (and z) of the CTA's R rows. Rows and steps outside the tensor read as 0.
    auto load_x = [&](int c, int stage) {
        const int64_t t = t_begin + static_cast<int64_t>(c) * CH + x_pc * VE;
        const int64_t valid_t = min64(VE, max64(0, p.seqlen - t));
        for (int r = x_r0; r < R; r += x_rstep) {
            const int64_t dd = d0 + r;
            const int64_t valid = dd < p.dim ? valid_t : 0;
            const int64_t ddc = min64(dd, p.dim - 1);
            for (int k = 0; k < ntens; ++k) {
                const void *base = k == 0 ? p.u : (k == 1 ? p.delta : p.z);
                const int64_t off = b * (k == 0 ? p.u_sb : (k == 1 ? p.dl_sb : p.z_sb)) +
                                    ddc * (k == 0 ? p.u_sd : (k == 1 ? p.dl_sd : p.z_sd));
                const T *src = static_cast<const T *>(base) + off;
                unsigned char *dst = xs + ((stage * 3 + k) * R + r) * ROWB + x_pc * 16;
                if constexpr (VEC) {
                    cp_async16(dst, valid > 0 ? static_cast<const void *>(src + t) : static_cast<const void *>(src),
                               static_cast<int>(valid) * EB);
                } else {
                    T *o = reinterpret_cast<T *>(dst);
#pragma unroll
                    for (int e = 0; e < VE; ++e) o[e] = e < valid ? src[t + e] : from_f32<T>(0.f);
                }
            }
        }
    };
    // Raw B and C tiles (dstate x CH) of the chunk: tile row rr = k * dstate + n.
    auto load_bc = [&](int c, int buf) {
        const int64_t t = t_begin + static_cast<int64_t>(c) * CH + b_pc * VE;
        const int64_t valid = min64(VE, max64(0, p.seqlen - t));
        for (int rr = b_r0; rr < 2 * dstate; rr += b_rstep) {
            const int k = rr >= dstate ? 1 : 0;
            const int n = rr - k * dstate;
            const T *src = static_cast<const T *>(k == 0 ? p.B : p.C) + b * (k == 0 ? p.B_sb : p.C_sb) +
                           n * (k == 0 ? p.B_sn : p.C_sn);
            unsigned char *dst = raw + (((buf * 2 + k) * kMaxN + n) * CH + b_pc * VE) * EB;
            if constexpr (VEC) {
                cp_async16(dst, valid > 0 ? static_cast<const void *>(src + t) : static_cast<const void *>(src),
                           static_cast<int>(valid) * EB);
            } else {
                T *o = reinterpret_cast<T *>(dst);
#pragma unroll
                for (int e = 0; e < VE; ++e) o[e] = e < valid ? src[t + e] : from_f32<T>(0.f);
            }
        }
    };
    // Widen the raw tiles into the (value, value) float32 pair tile.
    auto widen_bc = [&](int buf) {
        const int tt = b_pc * VE;
        for (int rr = b_r0; rr < 2 * dstate; rr += b_rstep) {
            const int k = rr >= dstate ? 1 : 0;
            const int n = rr - k * dstate;
            const unsigned char *srcp = raw + (((buf * 2 + k) * kMaxN + n) * CH + tt) * EB;
            float4 *dst = reinterpret_cast<float4 *>(bc + ((k * kMaxN + n) * LG + tt / kK) * kSegF2 + tt % kK);
            if constexpr (std::is_same<T, float>::value) {
                const float4 v = *reinterpret_cast<const float4 *>(srcp);
                dst[0] = make_float4(v.x, v.x, v.y, v.y);
                dst[1] = make_float4(v.z, v.z, v.w, v.w);
            } else {
                const uint4 w = *reinterpret_cast<const uint4 *>(srcp);
                const float v0 = bf16_lo(w.x), v1 = bf16_hi(w.x), v2 = bf16_lo(w.y), v3 = bf16_hi(w.y);
                const float v4 = bf16_lo(w.z), v5 = bf16_hi(w.z), v6 = bf16_lo(w.w), v7 = bf16_hi(w.w);
                dst[0] = make_float4(v0, v0, v1, v1);
                dst[1] = make_float4(v2, v2, v3, v3);
                dst[2] = make_float4(v4, v4, v5, v5);
                dst[3] = make_float4(v6, v6, v7, v7);
            }
        }
    };

    const float2 bias2 = f2((okA && p.delta_bias) ? p.delta_bias[dA] : 0.f,
                            (okB && p.delta_bias) ? p.delta_bias[dB] : 0.f);
    const float2 D2 = f2((!SUMMARY && okA && p.D) ? p.D[dA] : 0.f, (!SUMMARY && okB && p.D) ? p.D[dB] : 0.f);
    const float2 *a2row = a2s + rp * kMaxN;
    const float2 *Bt = bc + j * kSegF2;
    const float2 *Ct = bc + (kMaxN * LG + j) * kSegF2;

    if (nchunks > 0) {
        load_x(0, 0);
        load_bc(0, 0);
    }
    cp_async_commit();

    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        cp_async_wait_all();
        __syncthreads();            // chunk c staged; chunk c-1 fully consumed
        widen_bc(s);
        __syncthreads();            // pair tile of chunk c ready
        if (c + 1 < nchunks) {
            load_x(c + 1, s ^ 1);
            load_bc(c + 1, s ^ 1);
        }
        cp_async_commit();

        const int64_t tl = t_begin + static_cast<int64_t>(c) * CH + j * kK;   // lane's first step
        const int64_t count = t_end - tl;                                      // steps of the lane inside the segment
        const unsigned char *xrow = xs + ((s * 3) * R + 2 * rp) * ROWB + j * kK * EB;
        float2 dt2[kK], dtx2[kK], y2[kK];
        lds_pair<T>(xrow, ROWB, y2);                       // u (kept in y2 until y starts)
        lds_pair<T>(xrow + R * ROWB, ROWB, dt2);           // delta_raw
#pragma unroll
        for (int i = 0; i < kK; ++i) {
            float2 v = add2(dt2[i], bias2);
            if (p.softplus) v = softplus2(v);
            dt2[i] = v;
        }
        if (count < kK) {                                  // ragged last chunk: identity pairs (1, 0)
#pragma unroll
            for (int i = 0; i < kK; ++i)
                if (i >= count) dt2[i] = f2(0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kK; ++i) {
            dtx2[i] = mul2(dt2[i], y2[i]);
            y2[i] = mul2(D2, y2[i]);
        }

        const float2 *cin_buf = carry + s * RP * kMaxN + rp * kMaxN;
        float2 *cout_buf = carry + (s ^ 1) * RP * kMaxN + rp * kMaxN;
        // Local composition of the lane's 8 pairs for state n: P_i, H_i after each
        // step and the aggregate (P, H).
        auto chain_n = [&](int n, float2 (&Pi)[kK], float2 (&Hi)[kK], float2 &P, float2 &H) {
            const float2 a2 = a2row[n];
            const float2 *Bn = Bt + n * LG * kSegF2;
            P = f2(1.f, 1.f);
            H = f2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < kK; q += 2) {
                const float4 bb = *reinterpret_cast<const float4 *>(Bn + q);
                const float2 a0 = ex2x2(mul2(dt2[q], a2));
                const float2 a1 = ex2x2(mul2(dt2[q + 1], a2));
                H = fma2(a0, H, mul2(dtx2[q], f2(bb.x, bb.y)));
                P = mul2(P, a0);
                Pi[q] = P; Hi[q] = H;
                H = fma2(a1, H, mul2(dtx2[q + 1], f2(bb.z, bb.w)));
                P = mul2(P, a1);
                Pi[q + 1] = P; Hi[q + 1] = H;
            }
        };
        // Fix-up h_i = P_i h_in + H_i folded into y_i += C_i h_i.
        auto fixup_n = [&](int n, const float2 (&Pi)[kK], const float2 (&Hi)[kK], float2 hin) {
            const float2 *Cn = Ct + n * LG * kSegF2;
#pragma unroll
            for (int q = 0; q < kK; q += 2) {
                const float4 cc = *reinterpret_cast<const float4 *>(Cn + q);
                y2[q] = fma2(f2(cc.x, cc.y), fma2(Pi[q], hin, Hi[q]), y2[q]);
                y2[q + 1] = fma2(f2(cc.z, cc.w), fma2(Pi[q + 1], hin, Hi[q + 1]), y2[q + 1]);
            }
        };
        // Group scan of the lane aggregates, carry in/out, and the fix-up
        // h_i = P_i h_in + H_i folded into y_i += C_i h_i. `live` is false for a
        // padding state index (its results are dropped).
        auto finish_n = [&](int n, const float2 (&Pi)[kK], const float2 (&Hi)[kK], float2 P, float2 H,
                            bool live) {
            float2 Ps = P, Hs = H;
#pragma unroll
            for (int off = 1; off < LG; off <<= 1) {
                const float2 Pu = shfl_up2(Ps, off, LG), Hu = shfl_up2(Hs, off, LG);
                compose_if(j >= off, Ps, Hs, Pu, Hu);
            }
            const float2 Pe = shfl_up2(Ps, 1, LG), He = shfl_up2(Hs, 1, LG);
            const float2 cin = cin_buf[n];
            if (j == LG - 1 && live) {
                cout_buf[n] = fma2(Ps, cin, Hs);
                if constexpr (SUMMARY) carryP[rp * kMaxN + n] = mul2(carryP[rp * kMaxN + n], Ps);
            }
            if constexpr (!SUMMARY) {
                if (live) {
                    const float2 hin = enter_state(j > 0, Pe, He, cin);
                    const float2 *Cn = Ct + n * LG * kSegF2;
#pragma unroll
                    for (int q = 0; q < kK; q += 2) {
                        const float4 cc = *reinterpret_cast<const float4 *>(Cn + q);
                        y2[q] = fma2(f2(cc.x, cc.y), fma2(Pi[q], hin, Hi[q]), y2[q]);
                        y2[q + 1] = fma2(f2(cc.z, cc.w), fma2(Pi[q + 1], hin, Hi[q + 1]), y2[q + 1]);
                    }
                }
            }
        };

        if constexpr (NI == 0) {
            // dstate == 16: fully unrolled with two register sets in flight, so
            // the MUFU-heavy chain of state n+1 issues next to the shuffle scan
            // and fix-up of state n.
            float2 PiA[kK], HiA[kK], PiB[kK], HiB[kK], PA, HA, PB, HB;
            chain_n(0, PiA, HiA, PA, HA);
#pragma unroll
            for (int n = 0; n < kMaxN; n += 2) {
                chain_n(n + 1, PiB, HiB, PB, HB);
                finish_n(n, PiA, HiA, PA, HA, true);
                if (n + 2 < kMaxN) chain_n(n + 2, PiA, HiA, PA, HA);
                finish_n(n + 1, PiB, HiB, PB, HB, true);
            }
        } else if constexpr (NI == 1) {
            for (int n = 0; n < dstate; ++n) {
                float2 Pi[kK], Hi[kK], P, H;
                chain_n(n, Pi, Hi, P, H);
                finish_n(n, Pi, Hi, P, H, true);
            }
        } else {
            // Two state indices per pass; the lane aggregates go through shared
            // memory and four lanes of each group fold them serially from the
            // chunk carry: h_in(lane k+1) = P_k h_in(lane k) + H_k, one FFMA per
            // lane, no pair composition and no shuffles.
            float *agg = fold_agg + rp * (Fold<LG>::AGG_F + Fold<LG>::HIN_F);
            float *hin_buf = agg + Fold<LG>::AGG_F;
            for (int n0 = 0; n0 < dstate; n0 += 2) {
                const bool live1 = n0 + 1 < dstate;
                const int n1 = live1 ? n0 + 1 : n0;
                float2 PiA[kK], HiA[kK], PiB[kK], HiB[kK], PA, HA, PB, HB;
                chain_n(n0, PiA, HiA, PA, HA);
                chain_n(n1, PiB, HiB, PB, HB);
                reinterpret_cast<float4 *>(agg)[2 * j] = make_float4(PA.x, HA.x, PA.y, HA.y);
                reinterpret_cast<float4 *>(agg)[2 * j + 1] = make_float4(PB.x, HB.x, PB.y, HB.y);
                __syncwarp();
                if (j < 4) {
                    const int u = j >> 1, h = j & 1;
                    const int n = u ? n1 : n0;
                    float acc = reinterpret_cast<const float *>(cin_buf)[2 * n + h];
                    float accP = 1.f;
#pragma unroll
                    for (int k = 0; k < LG; ++k) {
                        const float2 ph = reinterpret_cast<const float2 *>(agg)[(2 * k + u) * 2 + h];
                        hin_buf[(2 * k + u) * 2 + h] = acc;
                        acc = fmaf(ph.x, acc, ph.y);
                        if constexpr (SUMMARY) accP *= ph.x;
                    }
                    if (u == 0 || live1) {
                        reinterpret_cast<float *>(cout_buf)[2 * n + h] = acc;
                        if constexpr (SUMMARY) reinterpret_cast<float *>(carryP + rp * kMaxN)[2 * n + h] *= accP;
                    }
                }
                __syncwarp();
                if constexpr (!SUMMARY) {
                    const float2 hinA = reinterpret_cast<const float2 *>(hin_buf)[2 * j];
                    const float2 hinB = reinterpret_cast<const float2 *>(hin_buf)[2 * j + 1];
                    fixup_n(n0, PiA, HiA, hinA);
                    if (live1) fixup_n(n1, PiB, HiB, hinB);
                }
            }
        }

        if constexpr (!SUMMARY) {
            if (has_z) {
                float2 z2[kK];
                lds_pair<T>(xrow + 2 * R * ROWB, ROWB, z2);
#pragma unroll
                for (int i = 0; i < kK; ++i) y2[i] = mul2(y2[i], silu2_out<T>(z2[i]));
            }
            if (count > 0) {
                if (okA) store_row<T>(static_cast<T *>(p.y) + b * p.y_sb + dA * p.y_sd + tl, y2, false, count, VEC);
                if (okB) store_row<T>(static_cast<T *>(p.y) + b * p.y_sb + dB * p.y_sd + tl, y2, true, count, VEC);
            }
        }
    }
    __syncthreads();

    // Outputs of the segment: the final state, or the summary of a non-last segment.
    const float2 *cfin = carry + (nchunks & 1) * RP * kMaxN + rp * kMaxN;
    for (int n = j; n < dstate; n += LG) {
        const float2 cv = cfin[n];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t dd = h ? dB : dA;
            if (dd >= p.dim) continue;
            const int64_t row = b * p.dim + dd;
            const float v = h ? cv.y : cv.x;
            if constexpr (SUMMARY) {
                const int64_t w = (row * p.nseg + seg) * kMaxN + n;
                p.ws_H[w] = v;
                p.ws_P[w] = h ? carryP[rp * kMaxN + n].y : carryP[rp * kMaxN + n].x;
            } else {
                if (p.hT && seg == p.nseg - 1) p.hT[row * dstate + n] = v;
            }
        }
    }
}

constexpr int kSmemLimit = 227 * 1024;

// The compiled configurations the planner chooses from. ni: 1 = one state
// index per loop body; 2 = two interleaved; 0 = dstate 16 only, fully
// unrolled and software pipelined. Kernels with ni != 1 keep up to 170
// registers (CTAs of <= 12 warps, one per SM); the ni = 1 kernels keep 128
// (CTAs of <= 16 warps). Summary passes and the unaligned path use ni = 1.
struct Config {
    int lg, ni, maxt, minb;
};
constexpr Config kConfigs[] = {
    {4, 1, 512, 1}, {8, 1, 512, 1}, {16, 1, 512, 1},
    {4, 2, 384, 1}, {8, 2, 384, 1}, {16, 2, 384, 1},
    {4, 0, 384, 1}, {8, 0, 384, 1}, {16, 0, 384, 1},
};
constexpr int kNumConfigs = sizeof(kConfigs) / sizeof(kConfigs[0]);

template <typename T, int LG, int NI, int MAXT, int MINB, bool VEC, bool SUMMARY>
const void *kernel_ptr() {
    return reinterpret_cast<const void *>(scan_kernel<T, LG, NI, MAXT, MINB, VEC, SUMMARY>);
}

template <typename T, int LG>
const void *basic_kernel(bool vec, bool summary) {
    if (summary) return vec ? kernel_ptr<T, LG, 1, 512, 1, true, true>() : kernel_ptr<T, LG, 1, 512, 1, false, true>();
    return vec ? kernel_ptr<T, LG, 1, 512, 1, true, false>() : kernel_ptr<T, LG, 1, 512, 1, false, false>();
}

// Kernel of configuration `ci` for the main pass (summary = false) or the
// summary pass; summaries and unaligned inputs always run the ni = 1 kernel of
// the same LG.
template <typename T>
const void *select_kernel(int ci, bool vec, bool summary) {
    const Config c = kConfigs[ci];
    if (summary || !vec || c.ni == 1) {
        switch (c.lg) {
            case 4: return basic_kernel<T, 4>(vec, summary);
            case 8: return basic_kernel<T, 8>(vec, summary);
            default: return basic_kernel<T, 16>(vec, summary);
        }
    }
    switch (ci) {
        case 3: return kernel_ptr<T, 4, 2, 384, 1, true, false>();
        case 4: return kernel_ptr<T, 8, 2, 384, 1, true, false>();
        case 5: return kernel_ptr<T, 16, 2, 384, 1, true, false>();
        case 6: return kernel_ptr<T, 4, 0, 384, 1, true, false>();
        case 7: return kernel_ptr<T, 8, 0, 384, 1, true, false>();
        default: return kernel_ptr<T, 16, 0, 384, 1, true, false>();
    }
}

const void *select_kernel_dt(int in_dtype, int ci, bool vec, bool summary) {
    return in_dtype == 0 ? select_kernel<float>(ci, vec, summary) : select_kernel<__nv_bfloat16>(ci, vec, summary);
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

int smem_bytes(int in_dtype, int lg, int W) {
    if (in_dtype == 0) {
        return lg == 4 ? layout<float, 4>(W).total : lg == 8 ? layout<float, 8>(W).total : layout<float, 16>(W).total;
    }
    return lg == 4 ? layout<__nv_bfloat16, 4>(W).total
                   : lg == 8 ? layout<__nv_bfloat16, 8>(W).total : layout<__nv_bfloat16, 16>(W).total;
}

// Relative issue cost per element of a configuration (scan depth log2 LG; the
// interleaved and pipelined kernels hide latency better with few warps).
double config_cost(const Config &c) {
    return (c.lg == 4 ? 7.3 : c.lg == 8 ? 7.7 : 8.1) * (c.ni == 0 ? 0.94 : c.ni == 2 ? 0.97 : 1.0);
}

// The sequential kernels (scan_rec.cu) follow the chunked configurations in
// the configuration index: lanes per row and their measured cost over the
// MUFU bound on a busy SM (shared-memory wavefronts of the step-tile and B/C
// loads grow with the lanes per row; fitted to B200 timings of Mamba-130M,
// Mamba-1.4B and 131k-token layers).
// Configurations kNumConfigs + 0 .. 3 have 2 I/O warps, + 4 .. 6 have 4.
constexpr int kRecLanes[] = {2, 4, 8, 16, 2, 4, 8};
constexpr int kRecIow[] = {2, 2, 2, 2, 4, 4, 4};
constexpr int kNumRec = sizeof(kRecLanes) / sizeof(kRecLanes[0]);
// SM clocks per (row, step) of a sequential configuration when m of its CTAs
// share an SM (m = 1 .. 4; larger m takes the last entry), measured on B200
// with bf16 Mamba-130M-, Mamba-1.4B- and 131k-token layers (the MUFU floor is
// 18/16 = 1.125: 16 exponentials of the states plus the softplus and the gate).
// One CTA alone on an SM leaves each sub-partition a single recurrence warp
// and runs markedly slower per row.
constexpr double kRecCycles[][4] = {
    {2.4, 1.85, 1.85, 1.85},   // 2 lanes per row, 2 I/O warps
    {2.51, 1.89, 1.69, 1.69},  // 4 lanes, 2 I/O warps
    {4.5, 2.57, 2.54, 2.54},   // 8 lanes, 2 I/O warps
    {9.0, 8.0, 6.5, 6.5},      // 16 lanes, 2 I/O warps
    {2.06, 1.68, 1.68, 1.68},  // 2 lanes, 4 I/O warps
    {2.59, 2.22, 2.2, 2.2},    // 4 lanes, 4 I/O warps
    {3.98, 3.25, 3.25, 3.25},  // 8 lanes, 4 I/O warps
};
double rec_cycles(int ri, int64_t m) { return kRecCycles[ri][m < 1 ? 0 : m > 4 ? 3 : m - 1]; }
// Relative cost of the persistent schedule's bookkeeping (piece table, carry
// hand-over) per unit of work.
constexpr double kRecPersistentCost = 1.01;
// SM clocks per unit of the chunked kernels' cost model (measured: a
// Mamba-130M layer on cfg 7, 11 warps, took 485k clocks for 1.30M units).
constexpr double kChunkedClocksPerUnit = 0.372;

// Registers per thread of a kernel, cached (cudaFuncGetAttributes is slow).
int kernel_regs(const void *k) {
    constexpr int kSlots = 64;
    static const void *keys[kSlots];
    static int vals[kSlots];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
        if (keys[i] == k) return vals[i];
    cudaFuncAttributes fa{};
    const int regs = cudaFuncGetAttributes(&fa, k) == cudaSuccess ? fa.numRegs : 128;
    if (used < kSlots) {
        keys[used] = k;
        vals[used] = regs;
        ++used;
    }
    return regs;
}

}  // namespace

// Launch planning. Every CTA does the same work (R rows x one segment), so the
// plan picks the kernel configuration, warps per CTA (W) and the number of
// segments that minimise the time of the busiest SM: its CTAs run in waves of
// as many as fit (registers, shared memory, warps), an SM with fewer than 8
// resident warps runs proportionally slower, and a segmented run costs 1.75x
// the arithmetic (summary pass + main pass).
ScanPlan plan_scan(const ScanParams &p, int in_dtype, int force_segments, int num_sms, bool persistent_ok) {
    const int eb = in_dtype == 0 ? 4 : 2;
    ScanPlan plan{};
    auto strides_ok = [&](int64_t s1, int64_t s2) { return (s1 * eb) % 16 == 0 && (s2 * eb) % 16 == 0; };
    plan.vec = aligned16(p.u) && aligned16(p.delta) && aligned16(p.B) && aligned16(p.C) &&
               aligned16(p.y) && (p.z == nullptr || aligned16(p.z)) && strides_ok(p.u_sb, p.u_sd) &&
               strides_ok(p.dl_sb, p.dl_sd) && strides_ok(p.B_sb, p.B_sn) && strides_ok(p.C_sb, p.C_sn) &&
               strides_ok(p.y_sb, p.y_sd) && (p.z == nullptr || strides_ok(p.z_sb, p.z_sd)) &&
               (p.lambda_raw == nullptr || (aligned16(p.lambda_raw) && strides_ok(p.lm_sb, p.lm_sd)));

    const int sms = num_sms > 0 ? num_sms : 148;
    // only sequential kernels fuse the convolution prologue or run the trapezoidal rule
    const int variant = rec_variant(p);
    double best = 1e300;
    // (checkpoints for the backward are written by the sequential kernels only)
    for (int ci = 0; ci < ((variant || p.ckpt) ? 0 : kNumConfigs); ++ci) {
        const Config cf = kConfigs[ci];
        if (cf.ni != 1 && !plan.vec) continue;
        if (cf.ni == 0 && p.dstate != kMaxN) continue;
        const int regs = kernel_regs(select_kernel_dt(in_dtype, ci, plan.vec, false));
        const int64_t chunk = cf.lg * kK;
        const int64_t nchunks = (p.seqlen + chunk - 1) / chunk;
        for (int W = 2; W * 32 <= cf.maxt; ++W) {
            const int smem = smem_bytes(in_dtype, cf.lg, W);
            if (smem > kSmemLimit) continue;
            const int64_t R = W * 64 / cf.lg;
            const int64_t per_sm = min64(min64(kSmemLimit / (smem + 1024), 64 / W),
                                         min64(65536 / (static_cast<int64_t>(regs) * 32 * W), 32));
            if (per_sm < 1) continue;
            const int64_t tiles = p.batch * ((p.dim + R - 1) / R);
            for (int64_t S = 1; S <= min64(nchunks, 4096); S *= 2) {
                if (force_segments > 0 && S != 1) break;
                const int64_t nseg = force_segments > 0 ? min64(force_segments, min64(nchunks, 65535)) : S;
                const int64_t ctas = tiles * nseg;
                const int64_t heavy = (ctas + sms - 1) / sms;   // CTAs on the busiest SM
                // The busiest SM runs its CTAs in waves of per_sm; a wave of m
                // CTAs takes m units of work at efficiency min(1, m W / 8).
                auto wave = [&](int64_t m) { return m * W >= 8 ? double(m) : 8.0 / W; };
                const double waves = (heavy / per_sm) * wave(per_sm) + (heavy % per_sm ? wave(heavy % per_sm) : 0.0);
                const double steps = static_cast<double>((nchunks + nseg - 1) / nseg) * chunk;
                const double t = waves * R * steps * config_cost(cf) * (nseg > 1 ? 1.75 : 1.0);
                if (t < best * 0.999) {
                    best = t;
                    plan.lg = cf.lg;
                    plan.config = ci;
                    plan.warps = W;
                    plan.nseg = static_cast<int>(nseg);
                }
            }
        }
    }
    // Sequential kernels: no segments; an SM runs its CTAs in waves of as many
    // as are resident, at the measured clocks per (row, step) for that many
    // CTAs per SM; with the persistent schedule every SM gets the same share.
    int rec = -1, rec_ctas = 0;
    if (force_segments <= 1 && p.dstate <= kMaxN) {
        best *= kChunkedClocksPerUnit;
        for (int ri = 0; ri < kNumRec; ++ri) {
            const int lpr = kRecLanes[ri], iow = kRecIow[ri];
            if (!rec_supports_variant(lpr, variant, iow)) continue;
            const int per_sm = rec_ctas_per_sm(in_dtype, lpr, plan.vec, variant, iow);
            if (per_sm < 1) continue;
            const int64_t R = rec_rows(lpr);
            const int64_t ctas = p.batch * ((p.dim + R - 1) / R);
            const int64_t heavy = (ctas + sms - 1) / sms;
            auto wave = [&](int64_t m) {   // m CTAs side by side on one SM, each R rows x L steps
                return static_cast<double>(m) * R * static_cast<double>(p.seqlen) * rec_cycles(ri, m);
            };
            const double t = (heavy / per_sm) * wave(per_sm) + (heavy % per_sm ? wave(heavy % per_sm) : 0.0);
            if (t < best * 0.999) {
                best = t;
                rec = ri;
                rec_ctas = 0;
            }
            // persistent schedule: m CTAs on every SM share the units' work exactly
            if (persistent_ok && p.batch * p.dim <= (int64_t(1) << 30) &&
                (p.seqlen + 15) / 16 < (int64_t(1) << 30)) {
                for (int m = 1; m <= per_sm && static_cast<int64_t>(m) * sms <= ctas; ++m) {
                    const double tp = static_cast<double>(ctas) * R * static_cast<double>(p.seqlen) / sms *
                                      rec_cycles(ri, m) * kRecPersistentCost;
                    if (tp < best * 0.999) {
                        best = tp;
                        rec = ri;
                        rec_ctas = m * sms;
                    }
                }
            }
        }
    }
    ScanPlan out = plan;
    if (rec >= 0) {
        make_plan(p, in_dtype, kNumConfigs + rec, rec_threads(kRecIow[rec]) / 32, 1, rec_ctas, sms, &out);
    } else {
        make_plan(p, in_dtype, plan.config, plan.warps, plan.nseg, 0, sms, &out);
    }
    return out;
}

bool make_plan(const ScanParams &p, int in_dtype, int config, int warps, int segments, int ctas, int num_sms,
               ScanPlan *out) {
    if (ctas < 0) return false;
    if (config >= kNumConfigs && config < kNumConfigs + kNumRec) {
        // sequential kernel: fixed CTA of rec_threads(), the whole sequence in one pass
        const int iow = kRecIow[config - kNumConfigs];
        if (warps != rec_threads(iow) / 32 || segments != 1 || p.dstate > kMaxN) return false;
        if (!rec_supports_variant(kRecLanes[config - kNumConfigs], rec_variant(p), iow)) return false;
        const int eb = in_dtype == 0 ? 4 : 2;
        auto strides_ok = [&](int64_t s1, int64_t s2) { return (s1 * eb) % 16 == 0 && (s2 * eb) % 16 == 0; };
        ScanPlan plan{};
        plan.kind = 1;
        plan.config = config;
        plan.iow = iow;
        plan.lg = kRecLanes[config - kNumConfigs];
        plan.warps = warps;
        plan.rows_per_cta = rec_rows(plan.lg);
        plan.chunk = rec_chunk();
        plan.vec = aligned16(p.u) && aligned16(p.delta) && aligned16(p.B) && aligned16(p.C) &&
                   aligned16(p.y) && (p.z == nullptr || aligned16(p.z)) && strides_ok(p.u_sb, p.u_sd) &&
                   strides_ok(p.dl_sb, p.dl_sd) && strides_ok(p.B_sb, p.B_sn) && strides_ok(p.C_sb, p.C_sn) &&
                   strides_ok(p.y_sb, p.y_sd) && (p.z == nullptr || strides_ok(p.z_sb, p.z_sd)) &&
                   (p.lambda_raw == nullptr || (aligned16(p.lambda_raw) && strides_ok(p.lm_sb, p.lm_sd)));
        plan.nseg = 1;
        plan.seg_len = p.seqlen;
        plan.ws_bytes = 0;
        plan.ctas = 0;
        if (ctas > 0) {
            // persistent schedule: every CTA resident, at most one per unit
            const int64_t units = p.batch * ((p.dim + plan.rows_per_cta - 1) / plan.rows_per_cta);
            if (units > (int64_t(1) << 30) || p.batch * p.dim > (int64_t(1) << 30) ||
                (p.seqlen + rec_chunk() - 1) / rec_chunk() >= (int64_t(1) << 30))
                return false;
            if (ctas > rec_max_ctas(p, in_dtype, plan.lg, plan.vec != 0, num_sms > 0 ? num_sms : 148, iow)) return false;
            plan.ctas = ctas;
            plan.ws_bytes = rec_persistent_ws_bytes(units, plan.rows_per_cta);
        }
        *out = plan;
        return true;
    }
    if (ctas != 0) return false;
    if (config < 0 || config >= kNumConfigs || segments < 1 || rec_variant(p) != 0) return false;
    const Config cf = kConfigs[config];
    ScanPlan plan{};
    const int eb = in_dtype == 0 ? 4 : 2;
    auto strides_ok = [&](int64_t s1, int64_t s2) { return (s1 * eb) % 16 == 0 && (s2 * eb) % 16 == 0; };
    plan.vec = aligned16(p.u) && aligned16(p.delta) && aligned16(p.B) && aligned16(p.C) &&
               aligned16(p.y) && (p.z == nullptr || aligned16(p.z)) && strides_ok(p.u_sb, p.u_sd) &&
               strides_ok(p.dl_sb, p.dl_sd) && strides_ok(p.B_sb, p.B_sn) && strides_ok(p.C_sb, p.C_sn) &&
               strides_ok(p.y_sb, p.y_sd) && (p.z == nullptr || strides_ok(p.z_sb, p.z_sd));
    if (cf.ni != 1 && !plan.vec) return false;
    if (cf.ni == 0 && p.dstate != kMaxN) return false;
    if (warps < 2 || warps * 32 > cf.maxt) return false;
    if (smem_bytes(in_dtype, cf.lg, warps) > kSmemLimit) return false;
    plan.config = config;
    plan.lg = cf.lg;
    plan.warps = warps;
    plan.rows_per_cta = warps * 64 / cf.lg;
    plan.chunk = cf.lg * kK;
    const int64_t nchunks = (p.seqlen + plan.chunk - 1) / plan.chunk;
    const int64_t nseg = min64(segments, min64(nchunks, 65535));
    const int64_t chunks_per_seg = (nchunks + nseg - 1) / nseg;
    plan.seg_len = chunks_per_seg * plan.chunk;
    plan.nseg = static_cast<int>((p.seqlen + plan.seg_len - 1) / plan.seg_len);
    plan.ws_bytes = plan.nseg > 1
                        ? 2 * static_cast<size_t>(p.batch * p.dim) * plan.nseg * kMaxN * sizeof(float)
                        : 0;
    *out = plan;
    return true;
}

int scan_num_configs() { return kNumConfigs + kNumRec; }

int scan_config_kind(int config) {
    if (config < 0 || config >= kNumConfigs + kNumRec) return -1;
    return config < kNumConfigs ? 0 : 1;
}

bool scan_config_info(int config, int *lanes, int *states_per_pass, int *max_warps) {
    if (config >= kNumConfigs && config < kNumConfigs + kNumRec) {
        const int lpr = kRecLanes[config - kNumConfigs];
        if (lanes) *lanes = lpr;
        if (states_per_pass) *states_per_pass = kMaxN / lpr;
        if (max_warps) *max_warps = rec_threads(kRecIow[config - kNumConfigs]) / 32;
        return true;
    }
    if (config < 0 || config >= kNumConfigs) return false;
    if (lanes) *lanes = kConfigs[config].lg;
    if (states_per_pass) *states_per_pass = kConfigs[config].ni;
    if (max_warps) *max_warps = kConfigs[config].maxt / 32;
    return true;
}

void bind_workspace(ScanParams &p, const ScanPlan &plan, void *workspace) {
    p.nseg = plan.nseg;
    p.seg_len = plan.seg_len;
    if (plan.ws_bytes == 0) return;
    if (plan.kind == 1) {
        const int64_t units = p.batch * ((p.dim + plan.rows_per_cta - 1) / plan.rows_per_cta);
        rec_bind_workspace(p, workspace, units, plan.ctas);
    } else {
        float *ws = static_cast<float *>(workspace);
        p.ws_P = ws;
        p.ws_H = ws + plan.ws_bytes / 2 / sizeof(float);
    }
}

cudaError_t launch_scan(const ScanParams &p, const ScanPlan &plan, int in_dtype, cudaStream_t stream) {
    if (plan.kind == 1) return launch_rec(p, plan.lg, plan.vec != 0, in_dtype, plan.iow, stream);
    const int W = plan.warps;
    const int smem = smem_bytes(in_dtype, plan.lg, W);
    const unsigned gx = static_cast<unsigned>((p.dim + plan.rows_per_cta - 1) / plan.rows_per_cta);
    void *args[] = {const_cast<ScanParams *>(&p)};
    auto go = [&](const void *kernel, unsigned gz) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e != cudaSuccess) return e;
        e = cudaLaunchKernel(kernel, dim3(gx, static_cast<unsigned>(p.batch), gz), dim3(W * 32), args,
                             static_cast<size_t>(smem), stream);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    };
    if (plan.nseg > 1) {
        const cudaError_t e = go(select_kernel_dt(in_dtype, plan.config, plan.vec, true), plan.nseg - 1);
        if (e != cudaSuccess) return e;
    }
    return go(select_kernel_dt(in_dtype, plan.config, plan.vec, false), plan.nseg);
}

}  // namespace ms
