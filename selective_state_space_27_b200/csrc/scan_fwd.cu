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
// Kernel design (B200: 148 SMs, MUFU ex2 at 16 results/clk/SM is the binding
// unit -- one ex2 per (b, d, t, n) element -- HBM traffic is ~4x below it):
//  * A CTA owns R rows (b, d0..d0+R) of one batch entry and walks the sequence
//    in chunks of CH = LG * 16 time steps. Inside a warp, a group of LG lanes
//    owns one row; each lane owns 16 consecutive time steps of the chunk.
//  * Per chunk the CTA stages the (dstate, CH) tiles of B and C -- shared by
//    all R rows -- in shared memory as float32 (bf16 inputs are widened once
//    here, not once per row), and u, delta, z tiles of its rows through
//    cp.async. Both are double buffered one chunk ahead.
//  * Each lane computes delta (softplus in registers) for its 16 steps, then,
//    for each n: Abar = ex2(delta * A log2e) and Bbar u in registers, the local
//    sequential composition (P, H) of its 16 pairs, an LG-lane Kogge-Stone
//    scan of the pairs (a1,b1)o(a2,b2) = (a1 a2, a2 b1 + b2) with shuffles, the
//    carry of the previous chunk from shared memory, and the fix-up
//    h_i = P_i h_in + H_i folded straight into y_i += C_i h_i. The expanded
//    (b, d, t, n) state exists only in registers.
//  * Long sequences with too few rows to fill the GPU are split into segments
//    (grid z). A summary pass computes each segment's zero-start end state and
//    decay product; the main pass starts each segment from the carry composed
//    from the summaries of the segments before it.
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kK = 16;      // time steps per lane per chunk
constexpr int kMaxN = 16;   // largest dstate
constexpr int kFSeg = kK + 4;  // floats per lane segment in the B/C tile (padded: no bank conflicts)

template <typename T, int LG, int W>
struct Cfg {
    static constexpr int G = 32 / LG;          // rows per warp
    static constexpr int R = W * G;            // rows per CTA
    static constexpr int CH = LG * kK;         // time steps per chunk
    static constexpr int NT = W * 32;          // threads per CTA
    static constexpr int EB = sizeof(T);
    static constexpr int VE = 16 / EB;         // elements per 16-byte piece
    static constexpr int ROWB = CH * EB;       // bytes of one row of an input tile
    static constexpr int NROWF = LG * kFSeg;   // floats of one state row of the B/C tile
    static constexpr int BC_BYTES = 2 /*buffers*/ * 2 /*B,C*/ * kMaxN * NROWF * 4;
    static constexpr int X_BYTES = 2 /*stages*/ * 3 /*u,delta,z*/ * R * ROWB;
    static constexpr int SMALL_BYTES = 3 * R * kMaxN * 4;  // A log2e, carry, decay product
    static constexpr int SMEM = BC_BYTES + X_BYTES + SMALL_BYTES;
    // 16-byte pieces of the B and C tiles per chunk, and per thread
    static constexpr int BC_PIECES = 2 * kMaxN * CH / VE;
    static constexpr int BC_PER_THREAD = (BC_PIECES + NT - 1) / NT;
};

// Load 16 consecutive values of a lane's segment from shared memory as float.
template <typename T>
__device__ __forceinline__ void lds_seg(const unsigned char *src, float (&v)[kK]) {
    if constexpr (std::is_same<T, float>::value) {
        const float4 *s = reinterpret_cast<const float4 *>(src);
#pragma unroll
        for (int q = 0; q < kK / 4; ++q) {
            const float4 f = s[q];
            v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
        }
    } else {
        const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
        for (int q = 0; q < kK / 8; ++q) {
            const uint4 w = s[q];
            v[8 * q + 0] = bf16_lo(w.x); v[8 * q + 1] = bf16_hi(w.x);
            v[8 * q + 2] = bf16_lo(w.y); v[8 * q + 3] = bf16_hi(w.y);
            v[8 * q + 4] = bf16_lo(w.z); v[8 * q + 5] = bf16_hi(w.z);
            v[8 * q + 6] = bf16_lo(w.w); v[8 * q + 7] = bf16_hi(w.w);
        }
    }
}

template <typename T, int LG, int W, bool VEC, bool SUMMARY>
__global__ void __launch_bounds__(W * 32)
scan_kernel(const ScanParams p) {
    using C_ = Cfg<T, LG, W>;
    constexpr int G = C_::G, R = C_::R, CH = C_::CH, NT = C_::NT, EB = C_::EB, VE = C_::VE;
    constexpr int ROWB = C_::ROWB, NROWF = C_::NROWF;

    extern __shared__ __align__(16) unsigned char smem[];
    float *bc = reinterpret_cast<float *>(smem);
    unsigned char *xs = smem + C_::BC_BYTES;
    float *a2s = reinterpret_cast<float *>(smem + C_::BC_BYTES + C_::X_BYTES);
    float *carry = a2s + R * kMaxN;
    float *carryP = carry + R * kMaxN;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane / LG, j = lane % LG;
    const int rloc = warp * G + g;
    const int64_t b = blockIdx.y;
    const int64_t d0 = static_cast<int64_t>(blockIdx.x) * R;
    const int64_t d = d0 + rloc;
    const bool row_ok = d < p.dim;
    const int dstate = static_cast<int>(p.dstate);
    const int seg = blockIdx.z;
    const int64_t t_begin = static_cast<int64_t>(seg) * p.seg_len;
    const int64_t t_end = min64(p.seqlen, t_begin + p.seg_len);
    const int nchunks = static_cast<int>((t_end - t_begin + CH - 1) / CH);
    const bool has_z = !SUMMARY && p.z != nullptr;
    const int ntens = has_z ? 3 : 2;

    // Per-row constants and the carry entering this segment.
    for (int i = tid; i < R * kMaxN; i += NT) {
        const int r = i / kMaxN, n = i % kMaxN;
        const int64_t dd = d0 + r;
        const bool ok = dd < p.dim && n < dstate;
        a2s[i] = ok ? p.A[dd * dstate + n] * kLog2e : 0.f;
        float c = 0.f;
        if (!SUMMARY && ok) {
            const int64_t row = b * p.dim + dd;
            if (p.h0) c = p.h0[row * dstate + n];
            for (int s = 0; s < seg; ++s) {
                const int64_t w = (row * p.nseg + s) * kMaxN + n;
                c = fmaf(p.ws_P[w], c, p.ws_H[w]);
            }
        }
        carry[i] = c;
        carryP[i] = 1.f;
    }

    // ---- staging of one chunk ------------------------------------------------
    // u, delta (and z): R rows x CH steps each, 16-byte pieces.
    auto load_x = [&](int c, int stage) {
        const int64_t t0 = t_begin + static_cast<int64_t>(c) * CH;
        constexpr int PPR = ROWB / 16;
        for (int q = tid; q < ntens * R * PPR; q += NT) {
            const int k = q / (R * PPR);
            const int r = (q / PPR) % R;
            const int pc = q % PPR;
            const int64_t dd = d0 + r;
            const int64_t t = t0 + static_cast<int64_t>(pc) * VE;
            const void *base = k == 0 ? p.u : (k == 1 ? p.delta : p.z);
            const int64_t sb = k == 0 ? p.u_sb : (k == 1 ? p.dl_sb : p.z_sb);
            const int64_t sd = k == 0 ? p.u_sd : (k == 1 ? p.dl_sd : p.z_sd);
            const T *src = static_cast<const T *>(base) + b * sb + min64(dd, p.dim - 1) * sd;
            const int64_t valid = dd < p.dim ? min64(VE, max64(0, p.seqlen - t)) : 0;
            unsigned char *dst = xs + ((stage * 3 + k) * R + r) * ROWB + pc * 16;
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

    // B and C: (dstate, CH) tiles stored as float32 in lane-segment layout.
    auto bc_dst = [&](int buf, int k, int n, int tt) -> float * {
        return bc + ((buf * 2 + k) * kMaxN + n) * NROWF + (tt / kK) * kFSeg + (tt % kK);
    };
    uint4 bcreg[C_::BC_PER_THREAD];
    auto bc_issue = [&](int c, int buf) {
        const int64_t t0 = t_begin + static_cast<int64_t>(c) * CH;
        constexpr int PPN = CH / VE;  // pieces per state row
#pragma unroll
        for (int i = 0; i < C_::BC_PER_THREAD; ++i) {
            const int q = tid + i * NT;
            const int k = q / (kMaxN * PPN);
            const int n = (q / PPN) % kMaxN;
            const int pc = q % PPN;
            const int64_t t = t0 + static_cast<int64_t>(pc) * VE;
            const bool live = q < C_::BC_PIECES && n < dstate;
            const T *src = live ? static_cast<const T *>(k == 0 ? p.B : p.C) +
                                      b * (k == 0 ? p.B_sb : p.C_sb) + n * (k == 0 ? p.B_sn : p.C_sn)
                                : nullptr;
            const int64_t valid = live ? min64(VE, max64(0, p.seqlen - t)) : 0;
            if constexpr (std::is_same<T, float>::value) {
                if (live) {
                    float *dst = bc_dst(buf, k, n, pc * VE);
                    if constexpr (VEC) {
                        cp_async16(dst, valid > 0 ? static_cast<const void *>(src + t) : static_cast<const void *>(src),
                                   static_cast<int>(valid) * EB);
                    } else {
#pragma unroll
                        for (int e = 0; e < VE; ++e) dst[e] = e < valid ? src[t + e] : 0.f;
                    }
                }
            } else {
                uint4 w = make_uint4(0u, 0u, 0u, 0u);
                if (VEC && valid == VE) {
                    w = *reinterpret_cast<const uint4 *>(src + t);
                } else if (valid > 0) {
                    const uint16_t *s16 = reinterpret_cast<const uint16_t *>(src + t);
                    uint32_t h[VE];
#pragma unroll
                    for (int e = 0; e < VE; ++e) h[e] = e < valid ? s16[e] : 0u;
                    w = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                   h[6] | (h[7] << 16));
                }
                bcreg[i] = w;
            }
        }
    };
    auto bc_store = [&](int buf) {  // bf16 only: widen the registers into the tile
        if constexpr (!std::is_same<T, float>::value) {
            constexpr int PPN = CH / VE;
#pragma unroll
            for (int i = 0; i < C_::BC_PER_THREAD; ++i) {
                const int q = tid + i * NT;
                const int k = q / (kMaxN * PPN);
                const int n = (q / PPN) % kMaxN;
                const int pc = q % PPN;
                if (q < C_::BC_PIECES && n < dstate) {
                    float *dst = bc_dst(buf, k, n, pc * VE);
                    const uint4 w = bcreg[i];
                    reinterpret_cast<float4 *>(dst)[0] =
                        make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
                    reinterpret_cast<float4 *>(dst)[1] =
                        make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
                }
            }
        }
    };

    const float bias = (row_ok && p.delta_bias) ? p.delta_bias[d] : 0.f;
    const float Dd = (!SUMMARY && row_ok && p.D) ? p.D[d] : 0.f;

    // prologue: chunk 0
    if (nchunks > 0) {
        load_x(0, 0);
        bc_issue(0, 0);
        cp_async_commit();
        bc_store(0);
        cp_async_wait_all();
    }
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        if (c + 1 < nchunks) {
            load_x(c + 1, s ^ 1);
            bc_issue(c + 1, s ^ 1);
        }
        cp_async_commit();

        const int64_t tl = t_begin + static_cast<int64_t>(c) * CH + j * kK;  // lane's first step
        float dt[kK], dtx[kK], y[kK];
        lds_seg<T>(xs + ((s * 3 + 0) * R + rloc) * ROWB + j * kK * EB, y);   // u, kept in y for now
        lds_seg<T>(xs + ((s * 3 + 1) * R + rloc) * ROWB + j * kK * EB, dt);
#pragma unroll
        for (int i = 0; i < kK; ++i) {
            float v = dt[i] + bias;
            if (p.softplus) v = softplus(v);
            if (!row_ok || tl + i >= t_end) v = 0.f;   // identity pair (1, 0) past the end
            dt[i] = v;
            dtx[i] = v * y[i];
            y[i] = Dd * y[i];
        }

        const float *Btile = bc + (s * 2 + 0) * kMaxN * NROWF + j * kFSeg;
        const float *Ctile = bc + (s * 2 + 1) * kMaxN * NROWF + j * kFSeg;
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) {
            if (n >= dstate) break;
            const float a2 = a2s[rloc * kMaxN + n];
            float Bv[kK];
#pragma unroll
            for (int q = 0; q < kK / 4; ++q) {
                const float4 f = reinterpret_cast<const float4 *>(Btile + n * NROWF)[q];
                Bv[4 * q] = f.x; Bv[4 * q + 1] = f.y; Bv[4 * q + 2] = f.z; Bv[4 * q + 3] = f.w;
            }
            // local composition of the lane's 16 pairs
            float P = 1.f, H = 0.f;
            float Pi[kK], Hi[kK];
#pragma unroll
            for (int i = 0; i < kK; ++i) {
                const float a = ex2_approx(dt[i] * a2);
                H = fmaf(a, H, dtx[i] * Bv[i]);
                P *= a;
                if constexpr (!SUMMARY) { Pi[i] = P; Hi[i] = H; }
            }
            // inclusive scan of (P, H) over the LG lanes of the row
            float Ps = P, Hs = H;
#pragma unroll
            for (int off = 1; off < LG; off <<= 1) {
                const float Pu = __shfl_up_sync(0xffffffffu, Ps, off, LG);
                const float Hu = __shfl_up_sync(0xffffffffu, Hs, off, LG);
                if (j >= off) { Hs = fmaf(Ps, Hu, Hs); Ps *= Pu; }
            }
            const float cin = carry[rloc * kMaxN + n];
            if constexpr (!SUMMARY) {
                float Pe = __shfl_up_sync(0xffffffffu, Ps, 1, LG);
                float He = __shfl_up_sync(0xffffffffu, Hs, 1, LG);
                if (j == 0) { Pe = 1.f; He = 0.f; }
                const float hin = fmaf(Pe, cin, He);
                float Cv[kK];
#pragma unroll
                for (int q = 0; q < kK / 4; ++q) {
                    const float4 f = reinterpret_cast<const float4 *>(Ctile + n * NROWF)[q];
                    Cv[4 * q] = f.x; Cv[4 * q + 1] = f.y; Cv[4 * q + 2] = f.z; Cv[4 * q + 3] = f.w;
                }
#pragma unroll
                for (int i = 0; i < kK; ++i) y[i] = fmaf(Cv[i], fmaf(Pi[i], hin, Hi[i]), y[i]);
            }
            __syncwarp();
            if (j == LG - 1) {
                carry[rloc * kMaxN + n] = fmaf(Ps, cin, Hs);
                if constexpr (SUMMARY) carryP[rloc * kMaxN + n] *= Ps;
            }
        }

        if constexpr (!SUMMARY) {
            if (has_z) {
                float zv[kK];
                lds_seg<T>(xs + ((s * 3 + 2) * R + rloc) * ROWB + j * kK * EB, zv);
#pragma unroll
                for (int i = 0; i < kK; ++i) y[i] *= silu(zv[i]);
            }
            if (row_ok) {
                T *yrow = static_cast<T *>(p.y) + b * p.y_sb + d * p.y_sd;
                if (VEC && tl + kK <= t_end) {
                    if constexpr (std::is_same<T, float>::value) {
#pragma unroll
                        for (int q = 0; q < kK / 4; ++q)
                            reinterpret_cast<float4 *>(yrow + tl)[q] =
                                make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < kK / 8; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 h2 = __floats2bfloat162_rn(y[8 * q + 2 * e], y[8 * q + 2 * e + 1]);
                                w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                            reinterpret_cast<uint4 *>(yrow + tl)[q] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kK; ++i)
                        if (tl + i < t_end) yrow[tl + i] = from_f32<T>(y[i]);
                }
            }
        }

        if (c + 1 < nchunks) bc_store(s ^ 1);
        cp_async_wait_all();
        __syncthreads();
    }

    // Outputs of the segment: final state, or the summary of a non-last segment.
    if (row_ok) {
        const int64_t row = b * p.dim + d;
        for (int n = j; n < dstate; n += LG) {
            if constexpr (SUMMARY) {
                const int64_t w = (row * p.nseg + seg) * kMaxN + n;
                p.ws_H[w] = carry[rloc * kMaxN + n];
                p.ws_P[w] = carryP[rloc * kMaxN + n];
            } else {
                if (p.hT && seg == p.nseg - 1) p.hT[row * dstate + n] = carry[rloc * kMaxN + n];
            }
        }
    }
}

template <typename T, int LG, int W>
cudaError_t launch_cfg(const ScanParams &p, const ScanPlan &plan, cudaStream_t stream) {
    using C_ = Cfg<T, LG, W>;
    const dim3 block(C_::NT);
    const unsigned gx = static_cast<unsigned>((p.dim + C_::R - 1) / C_::R);
    auto go = [&](auto kernel, unsigned gz) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C_::SMEM);
        if (e != cudaSuccess) return e;
        kernel<<<dim3(gx, static_cast<unsigned>(p.batch), gz), block, C_::SMEM, stream>>>(p);
        return cudaGetLastError();
    };
    cudaError_t e = cudaSuccess;
    if (plan.nseg > 1) {
        e = plan.vec ? go(scan_kernel<T, LG, W, true, true>, plan.nseg - 1)
                     : go(scan_kernel<T, LG, W, false, true>, plan.nseg - 1);
        if (e != cudaSuccess) return e;
    }
    return plan.vec ? go(scan_kernel<T, LG, W, true, false>, plan.nseg)
                    : go(scan_kernel<T, LG, W, false, false>, plan.nseg);
}

template <typename T>
cudaError_t launch_t(const ScanParams &p, const ScanPlan &plan, cudaStream_t stream) {
    switch (plan.lg) {
        case 4: return launch_cfg<T, 4, 4>(p, plan, stream);
        case 8: return launch_cfg<T, 8, 4>(p, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

ScanPlan plan_scan(const ScanParams &p, int in_dtype, int force_segments, int num_sms) {
    const int eb = in_dtype == 0 ? 4 : 2;
    ScanPlan plan{};
    auto strides_ok = [&](int64_t s1, int64_t s2) { return (s1 * eb) % 16 == 0 && (s2 * eb) % 16 == 0; };
    plan.vec = aligned16(p.u) && aligned16(p.delta) && aligned16(p.B) && aligned16(p.C) &&
               aligned16(p.y) && (p.z == nullptr || aligned16(p.z)) && strides_ok(p.u_sb, p.u_sd) &&
               strides_ok(p.dl_sb, p.dl_sd) && strides_ok(p.B_sb, p.B_sn) && strides_ok(p.C_sb, p.C_sn) &&
               strides_ok(p.y_sb, p.y_sd) && (p.z == nullptr || strides_ok(p.z_sb, p.z_sd));

    // Lanes per row: 4 when there are enough rows to give every SM sub-partition
    // a few warps, 8 otherwise.
    const int64_t warps_lg4 = p.batch * ((p.dim + 31) / 32) * 4;
    plan.lg = warps_lg4 >= static_cast<int64_t>(num_sms) * 8 ? 4 : 8;
    plan.warps = 4;
    plan.rows_per_cta = plan.warps * (32 / plan.lg);
    plan.chunk = plan.lg * kK;

    const int64_t nchunks = (p.seqlen + plan.chunk - 1) / plan.chunk;
    const int64_t warps = p.batch * ((p.dim + plan.rows_per_cta - 1) / plan.rows_per_cta) * plan.warps;
    int64_t nseg = 1;
    if (force_segments > 0) {
        nseg = force_segments;
    } else {
        // Split the sequence when the rows alone leave most of the GPU idle.
        const int64_t target = static_cast<int64_t>(num_sms) * 8;
        if (warps < target / 2) nseg = (target + warps - 1) / warps;
    }
    nseg = max64(1, min64(nseg, min64(nchunks, 65535)));
    const int64_t chunks_per_seg = (nchunks + nseg - 1) / nseg;
    plan.seg_len = chunks_per_seg * plan.chunk;
    plan.nseg = static_cast<int>((p.seqlen + plan.seg_len - 1) / plan.seg_len);
    plan.ws_bytes = plan.nseg > 1
                        ? 2 * static_cast<size_t>(p.batch * p.dim) * plan.nseg * kMaxN * sizeof(float)
                        : 0;
    return plan;
}

cudaError_t launch_scan(const ScanParams &p, const ScanPlan &plan, int in_dtype, cudaStream_t stream) {
    return in_dtype == 0 ? launch_t<float>(p, plan, stream) : launch_t<__nv_bfloat16>(p, plan, stream);
}

}  // namespace ms
