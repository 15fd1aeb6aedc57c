// Selective scan (S6) forward, sequential form, for sm_100a.
//
// Same operation as scan_fwd.cu ("Notas sobre Mamba", sections "O mecanismo de
// seleção (S6)" and "A varredura paralela ciente do hardware"; "Mamba-2 e
// State Space Duality (SSD)", section "Como o Mamba-1 alcançou complexidade
// linear"): for every row (b, d) and state index n
//     h_t[n] = exp(delta_t A[d,n]) h_{t-1}[n] + delta_t B_t[n] u_t
//     y_t    = sum_n C_t[n] h_t[n] + D[d] u_t      (then * silu(z_t))
// with delta_t = softplus(delta_raw_t + delta_bias[d]).
//
// Design. The recurrence runs exactly as written, one time step after the
// other, and the parallelism comes from the (row, state) pairs instead of the
// time axis: LPR lanes share a row and each owns NPL = 16 / LPR of its states
// in registers for the whole sequence. There is no scan, no carry and no
// second pass, so the per-element work is the minimum the recurrence needs --
// one ex2 on the MUFU plus, per pair of states, one packed multiply for
// delta A, one for delta u B, one packed FMA for h and one for the readout.
// The MUFU (16 results/clk/SM) is the bound. A (batch 8, d_inner 1536, N 16)
// layer already has 196,608 independent (row, state) chains.
//
// The CTA is warp-specialised so that the MUFU never waits for the per-row
// work around the recurrence:
//  * 4 recurrence warps (one per SM sub-partition) own R = 128 / LPR rows of
//    one batch entry and step their states through chunks of 16 steps,
//    leaving each lane's partial readout sum_{own n} C_t[n] h_t[n] in shared
//    memory;
//  * 2 I/O warps run up to two chunks ahead of the recurrence, preparing
//    chunk c -- delta = softplus(delta_raw + bias) and delta u, stored per
//    step pair, and the chunk's B and C tiles (shared by all rows) widened to
//    float32 -- and finishing chunk c - 2: sum the LPR partials, add D u,
//    apply the SiLU gate and store y. Their raw inputs arrive through a
//    cp.async ring three chunks ahead.
// The two groups hand the tiles over through three stage buffers and named
// hardware barriers (bar.arrive by the producer, bar.sync by the consumer; no
// spin loops). Steps past the end of the sequence get delta = 0 (Abar = 1,
// Bbar u = 0): the state reaches the final-state output unchanged.
#include <mutex>
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kScanThreads = 128;   // 4 recurrence warps
// I/O warps per CTA: 2, or 4 (one per SM sub-partition, so that every
// sub-partition carries the same share of the per-row work).
constexpr int kSteps = 16;          // time steps per chunk
constexpr int kStates = 16;         // states per row (smaller dstate is zero-padded)
constexpr int kTileStages = 3;      // step/readout tile buffers between the two warp groups

// Shared-memory layout of one of the kTileStages stages, in bytes. The step tile holds
// one float4 per (row, step pair): (delta_t, delta_t u_t, delta_t+1,
// delta_t+1 u_t+1), XR float4 per row (odd, so that the 8 rows a quarter-warp
// reads or writes fall on distinct banks). The readout tile holds, per row
// and state group, the group's partial readout of every step ([row][group]
// [step], YQ floats per group and YR per row). The B and C tiles are
// [step][state] float32.
//
// Lane mapping of the recurrence warps. A 128-bit shared load costs two
// wavefronts when every quarter-warp touches at most two distinct 16-byte
// addresses and four otherwise (measured on B200), so for LPR = 2 and 4 the
// lanes are group-major -- lane l of warp w takes row w (32 / LPR) + l %
// (32 / LPR) and state group l / (32 / LPR): a quarter-warp then reads one
// B/C address per step. For LPR = 8 and 16 (row-major, lane l takes row
// (32 w + l) / LPR and group l % LPR) a quarter-warp covers at most two rows.
// With the trapezoidal rule (TRAP) the step tile holds one float4 per step:
// (delta, lambda delta u, (1 - lambda) delta u_prev, 0).
template <int LPR, bool TRAP = false, int IOW = 2> struct Shape {
    static constexpr int IOT = 32 * IOW;                // I/O threads
    static constexpr int THREADS = kScanThreads + IOT;  // threads per CTA
    static constexpr int NPL = kStates / LPR;           // states per lane
    static constexpr int R = kScanThreads / LPR;        // rows per CTA
    static constexpr int IPR = IOT / R;                 // I/O threads per row
    static constexpr int IP = kSteps / IPR;             // steps per I/O thread
    static constexpr bool GROUP_MAJOR = LPR <= 4;
    // LPR 4 and 8: the groups of a row sit in one warp (lanes r + 8 q, or 8 r +
    // q) and sum their partial readouts with shuffles, LPR steps at a time; the
    // readout tile then holds one float per (row, step), YR floats per row (36
    // and 40: the stores of a warp fall on distinct banks).
    static constexpr bool WARP_SUM = LPR == 4 || LPR == 8;
    static constexpr int EW = WARP_SUM ? LPR : 4;      // steps per readout store
    static constexpr int QSTRIDE = GROUP_MAJOR ? 32 / LPR : 1;   // lane distance between a row's groups
    static constexpr int XR = TRAP ? kSteps + 1 : kSteps / 2 + 1;   // float4 per row of the step tile
    static constexpr int YQ = LPR <= 4 ? kSteps : kSteps + 4;
    static constexpr int YR = LPR == 2 ? 2 * kSteps + 4 : LPR == 4 ? kSteps + 20 : LPR == 8 ? kSteps + 24 : LPR * YQ + 8;
    static constexpr int X_OFF = 0;
    static constexpr int Y_OFF = X_OFF + R * XR * 16;
    static constexpr int B_OFF = Y_OFF + R * YR * 4;
    static constexpr int C_OFF = B_OFF + kSteps * kStates * 4;
    static constexpr int STAGE = C_OFF + kSteps * kStates * 4;
    static constexpr int BYTES = kTileStages * STAGE;
    // CTAs per SM the launch bounds provide registers for
    static constexpr int MINB = IOW == 4 ? (LPR == 8 ? 3 : 2) : LPR == 2 ? 2 : LPR == 4 ? 3 : LPR == 8 ? 4 : 5;
    static_assert(R * IPR == IOT && IP >= 2, "the I/O threads cover the rows, two steps or more each");
    static_assert(XR % 2 == 1, "odd row stride");
    static_assert(YQ >= kSteps && YQ % 4 == 0 && (WARP_SUM ? YR >= kSteps : YR >= LPR * YQ) && YR % 4 == 0,
                  "readout tile");
};

// The I/O warps' ring of raw inputs in shared memory, after the tile stages.
// It holds every chunk from the oldest one still to be finished (its u and z
// feed the readout) to the newest one in flight, RA chunks ahead of the
// one being widened. Each I/O thread fills and reads only its own 16-byte
// slots (its u, delta and z pieces of PB bytes each, then its B/C pieces),
// stored slot-major so that a warp's slot accesses are contiguous.
constexpr int kRawStages = 5;
// Kernel variants: 0 plain; 1 convolution prologue; 2 trapezoidal rule.
// With the convolution prologue every thread also copies the 16 bytes before
// its u piece (the convolution's look-back, VE >= 4 elements) into one more
// slot, and a skip tile per tile stage ([row][step] floats after the ring)
// carries D u from the widening to the readout. The trapezoidal rule uses the
// same look-back slot (for u_{t-1}) and stages lambda_raw pieces as well.
template <typename T, int LPR, int VAR = 0, int IOW = 2> struct Raw {
    static constexpr bool CONV = VAR == 1, TRAP = VAR == 2;
    using SH = Shape<LPR, TRAP, IOW>;
    static constexpr int IOT = SH::IOT;
    static constexpr int EB = static_cast<int>(sizeof(T));
    static constexpr int PB = SH::IP * EB;                           // bytes of one u/delta/z piece
    static constexpr int PS = (PB + 15) / 16;                        // slots per piece
    static constexpr int VE = 16 / EB;                               // elements in 16 bytes
    // B/C pieces: the chunk's 2 x kStates x kSteps B and C values split evenly
    // over the I/O threads, at most 16 bytes (VE elements) a piece
    static constexpr int VB = (2 * kStates * kSteps / IOT) < VE ? (2 * kStates * kSteps / IOT) : VE;
    static constexpr int BCB = VB * EB;                                      // bytes per B/C piece
    static constexpr int BC_TOTAL = 2 * kStates * (kSteps / VB);             // B/C pieces per chunk
    static constexpr int BC_PER = BC_TOTAL / IOT;                            // B/C pieces per thread
    static constexpr int HALO = 3 * PS + BC_PER;                     // slot of the look-back (variants 1, 2)
    static constexpr int LAM = HALO + 1;                             // first slot of lambda_raw (variant 2)
    static constexpr int SLOTS = 3 * PS + BC_PER + (VAR ? 1 : 0) + (TRAP ? PS : 0);
    static constexpr int STAGE = SLOTS * IOT * 16;
    // ring depth: one stage shorter for the convolution prologue, whose larger
    // slots and skip tiles must still leave room for 3 (LPR 4) CTAs per SM. The
    // trapezoidal rule keeps the full ring: its plans run 2 CTAs per SM, and
    // prefetching three chunks ahead beat a third CTA.
    static constexpr int RS = CONV ? kRawStages - 1 : kRawStages;
    static constexpr int RA = RS - kTileStages + 1;                   // chunks staged ahead
    static constexpr int OFF = SH::BYTES;
    static constexpr int SKR = kSteps + 4;                            // floats per row of the skip tile
    static constexpr int SK_OFF = OFF + RS * STAGE;
    static constexpr int SK_STAGE = SH::R * SKR * 4;
    static constexpr int BYTES = SK_OFF + (CONV ? kTileStages * SK_STAGE : 0);   // total dynamic shared memory
    static_assert(BC_PER * IOT == BC_TOTAL && BC_TOTAL * VB == 2 * kStates * kSteps && (BCB == 8 || BCB == 16),
                  "B/C pieces of 8 or 16 bytes, as many for every I/O thread");
    static_assert(PB == 4 || PB == 8 || PB % 16 == 0, "piece sizes cp.async can copy");
    static_assert(VAR == 0 || (PB % 16 == 0 && VE >= 4), "look-back: 16-byte aligned pieces, >= 3 earlier inputs");
    static_assert(RA >= 1, "at least one chunk staged ahead");
};

// Named barriers (0 is __syncthreads): the producer arrives, the consumer
// waits; all NT threads of the CTA complete each phase.
//   XF(s): the chunk in stage s is widened: its step and B/C tiles are ready
//          (I/O -> recurrence)
//   YF(s): the recurrence is done with the chunk in stage s: its readout
//          partials are ready (recurrence -> I/O)
// A stage needs no "free again" barriers: the I/O warps widen chunk c only
// after finishing chunk c - kTileStages (their own program order, one sync on
// YF before it), so by the time the recurrence sees XF for chunk c the readout
// tile it is about to overwrite has been read; and the I/O warps' sync on YF
// for chunk c - kTileStages, which precedes the widening of chunk c, already
// says that the recurrence has stopped reading that stage's step tile. (The
// protocol is model-checked on the CPU against random schedules.)
__device__ __forceinline__ int bar_xf(int s) { return 1 + s; }
__device__ __forceinline__ int bar_yf(int s) { return 1 + kTileStages + s; }
static_assert(2 * kTileStages + 1 <= 13, "named barriers per CTA (13 and 14 serve the recurrence warps)");
__device__ __forceinline__ int next_stage(int s, int n) { return s + 1 == n ? 0 : s + 1; }
template <int NT> __device__ __forceinline__ void bar_wait(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(NT) : "memory");
}
template <int NT> __device__ __forceinline__ void bar_signal(int id) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "n"(NT) : "memory");
}

// ---- Work schedule ----------------------------------------------------------
// A unit is one batch entry x one block of R rows; its sequence is cut into
// nc chunks of kSteps steps. Without the persistent schedule a CTA owns one
// unit (blockIdx.x = row block, blockIdx.y = batch entry). With it
// (p.sk_ctas > 0), the chunks of all units, unit after unit, form one list
// that is cut into sk_ctas equal ranges, one per CTA, so that every SM gets
// the same amount of recurrence whatever the number of units. A range is
// [us:cs, ue:ce) in (unit, chunk) coordinates; since there are at most as
// many CTAs as units it holds the end of unit us (from chunk cs), whole units
// us+1 .. ue-1 and the start of unit ue (up to chunk ce). The CTA first runs
// the start of ue, which begins at t = 0 and whose end state it hands over
// (sk_carry, sk_flag) to the CTA that owns the rest of ue; then the whole
// units; and last the end of us, from the state the previous CTA left. By
// then that CTA has long finished the start of us: it ran those chunks first,
// and there are fewer of them than the chunks this CTA ran before needing
// them.
struct Sched {
    int us, cs, ue, ce;   // the range (ce in 1 .. nc)
    int nc, blocks;       // chunks per unit, row blocks per batch entry
    int64_t K;            // chunks of this CTA
};

__device__ __forceinline__ Sched make_sched(const ScanParams &p, int R) {
    Sched s;
    s.nc = static_cast<int>((p.seqlen + kSteps - 1) / kSteps);
    s.blocks = static_cast<int>((p.dim + R - 1) / R);
    if (p.sk_ctas == 0) {
        s.us = s.ue = static_cast<int>(blockIdx.y) * s.blocks + static_cast<int>(blockIdx.x);
        s.cs = 0;
        s.ce = s.nc;
        s.K = s.nc;
    } else {
        const int64_t T = static_cast<int64_t>(p.sk_units) * s.nc;
        const int64_t G = p.sk_ctas, g = blockIdx.x, q = T / G, r = T % G;
        const int64_t a = g * q + (g * r) / G;                 // floor(g T / G) without overflow
        const int64_t e = (g + 1) * q + ((g + 1) * r) / G;
        s.us = static_cast<int>(a / s.nc);
        s.cs = static_cast<int>(a - static_cast<int64_t>(s.us) * s.nc);
        s.ue = static_cast<int>((e - 1) / s.nc);
        s.ce = static_cast<int>(e - static_cast<int64_t>(s.ue) * s.nc);
        s.K = e - a;
    }
    return s;
}

// The CTA's work as pieces, in processing order: piece 0 is the start of unit
// ue, pieces 1 .. n-2 the whole units us+1 .. ue-1, piece n-1 the end of unit
// us (a single piece when the range lies inside one unit).
struct PieceRange {
    int u, c0, c1;   // chunks [c0, c1) of unit u
};
__device__ __forceinline__ int num_pieces(const Sched &s) { return s.us == s.ue ? 1 : s.ue - s.us + 1; }
__device__ __forceinline__ PieceRange piece_at(const Sched &s, int i) {
    if (s.us == s.ue) return {s.us, s.cs, s.ce};
    if (i == 0) return {s.ue, 0, s.ce};
    if (i == s.ue - s.us) return {s.us, s.cs, s.nc};
    return {s.us + i, 0, s.nc};
}

// A position in the CTA's list of chunks (piece i, chunk c of unit u); next()
// reports when it enters a new piece, so that per-row data is looked up once
// per piece rather than once per chunk.
struct PCur {
    int i, c, c1, u;
    __device__ __forceinline__ void begin(const Sched &s) {
        const PieceRange pr = piece_at(s, 0);
        i = 0; c = pr.c0; c1 = pr.c1; u = pr.u;
    }
    __device__ __forceinline__ bool next(const Sched &s) {
        if (++c < c1) return false;
        if (++i < num_pieces(s)) {
            const PieceRange pr = piece_at(s, i);
            c = pr.c0; c1 = pr.c1; u = pr.u;
        }
        return true;
    }
};

// Batch entry and (clamped) channel row of the thread's row r in unit u.
struct UnitRow {
    int64_t b, dc;
    bool ok;
};
__device__ __forceinline__ UnitRow unit_row(const ScanParams &p, const Sched &s, int u, int R, int r) {
    UnitRow x;
    x.b = u / s.blocks;
    const int64_t d = static_cast<int64_t>(u - static_cast<int>(x.b) * s.blocks) * R + r;
    x.ok = d < p.dim;
    x.dc = x.ok ? d : p.dim - 1;
    return x;
}

// Carry hand-over between CTAs. The writer's threads store the states, fence,
// meet at a barrier of the recurrence warps, and one thread sets the flag with
// release semantics; the reader's first thread polls the flag with acquire
// semantics (sleeping between polls, giving up after kCarryWaitNs with
// MS_ERR_TIMEOUT in the status word), then the recurrence warps meet and read
// the states from L2.
constexpr int kBarRecA = 13, kBarRecB = 14;   // named barriers of the 128 recurrence threads
constexpr unsigned long long kCarryWaitNs = 4000000000ull;
constexpr int kStatusTimeout = 5;               // MS_ERR_TIMEOUT

__device__ __forceinline__ void rec_bar(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kScanThreads) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int *f) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int *f, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void wait_carry(const ScanParams &p, int unit, int tid) {
    if (tid == 0 && !ld_acquire(p.sk_flag + unit)) {
        const unsigned long long t0 = global_ns();
        while (!ld_acquire(p.sk_flag + unit)) {
            __nanosleep(200);
            if (global_ns() - t0 > kCarryWaitNs) {
                atomicExch(p.sk_status, kStatusTimeout);
                break;
            }
        }
    }
    rec_bar(kBarRecA);
}

// One step's B_t and C_t entries of a lane, as the pairs the packed
// instructions take.
template <int NPL> struct StepIn {
    float2 b[NPL > 1 ? NPL / 2 : 1], c[NPL > 1 ? NPL / 2 : 1];
};

template <int NPL>
__device__ __forceinline__ StepIn<NPL> load_bc_step(const float *Bl, const float *Cl) {
    StepIn<NPL> s;
    if constexpr (NPL == 1) {
        s.b[0] = f2(*Bl, 0.f);
        s.c[0] = f2(*Cl, 0.f);
    } else if constexpr (NPL == 2) {
        s.b[0] = *reinterpret_cast<const float2 *>(Bl);
        s.c[0] = *reinterpret_cast<const float2 *>(Cl);
    } else {
#pragma unroll
        for (int v = 0; v < NPL / 4; ++v) {
            const float4 b4 = reinterpret_cast<const float4 *>(Bl)[v];
            const float4 c4 = reinterpret_cast<const float4 *>(Cl)[v];
            s.b[2 * v] = f2(b4.x, b4.y); s.b[2 * v + 1] = f2(b4.z, b4.w);
            s.c[2 * v] = f2(c4.x, c4.y); s.c[2 * v + 1] = f2(c4.z, c4.w);
        }
    }
    return s;
}

// P consecutive elements of one row in 32-bit words (bf16 pairs or floats).
template <typename T, int P> struct Piece {
    static constexpr int W = P * static_cast<int>(sizeof(T)) / 4;
    uint32_t w[W];
};

template <typename T, int P>
__device__ __forceinline__ float elem(const Piece<T, P> &pc, int e) {
    if constexpr (std::is_same<T, float>::value) return __uint_as_float(pc.w[e]);
    else return (e & 1) ? bf16_hi(pc.w[e >> 1]) : bf16_lo(pc.w[e >> 1]);
}

// Load `valid` (<= P) elements from src; the rest read as zero and are not
// touched in memory. VEC: src is aligned to the piece size.
template <typename T, int P, bool VEC>
__device__ __forceinline__ void load_piece(Piece<T, P> &pc, const T *src, int64_t valid) {
    constexpr int W = Piece<T, P>::W;
    if (VEC && valid >= P) {
        if constexpr (W == 1) {
            pc.w[0] = __ldg(reinterpret_cast<const unsigned *>(src));
        } else if constexpr (W == 2) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
            pc.w[0] = v.x; pc.w[1] = v.y;
        } else {
#pragma unroll
            for (int i = 0; i < W / 4; ++i) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + i);
                pc.w[4 * i] = v.x; pc.w[4 * i + 1] = v.y; pc.w[4 * i + 2] = v.z; pc.w[4 * i + 3] = v.w;
            }
        }
    } else if constexpr (std::is_same<T, float>::value) {
#pragma unroll
        for (int e = 0; e < P; ++e) pc.w[e] = e < valid ? __float_as_uint(__ldg(src + e)) : 0u;
    } else {
        const unsigned short *s = reinterpret_cast<const unsigned short *>(src);
#pragma unroll
        for (int i = 0; i < W; ++i) {
            const uint32_t lo = 2 * i < valid ? __ldg(s + 2 * i) : 0u;
            const uint32_t hi = 2 * i + 1 < valid ? __ldg(s + 2 * i + 1) : 0u;
            pc.w[i] = lo | (hi << 16);
        }
    }
}

// Store the first `count` (<= P) of P float values as T.
template <typename T, int P, bool VEC>
__device__ __forceinline__ void store_piece(T *dst, const float (&v)[P], int64_t count) {
    if constexpr (std::is_same<T, float>::value) {
        if (VEC && count >= P) {
            if constexpr (P == 2) {
                *reinterpret_cast<float2 *>(dst) = make_float2(v[0], v[1]);
            } else {
#pragma unroll
                for (int i = 0; i < P / 4; ++i)
                    reinterpret_cast<float4 *>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < P; ++e)
                if (e < count) dst[e] = v[e];
        }
    } else {
        uint32_t w[P / 2];
#pragma unroll
        for (int i = 0; i < P / 2; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        if (VEC && count >= P) {
            if constexpr (P == 2) {
                *reinterpret_cast<uint32_t *>(dst) = w[0];
            } else if constexpr (P == 4) {
                *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
            } else {
#pragma unroll
                for (int i = 0; i < P / 8; ++i)
                    reinterpret_cast<uint4 *>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        } else {
            unsigned short *o = reinterpret_cast<unsigned short *>(dst);
#pragma unroll
            for (int e = 0; e < P; ++e)
                if (e < count) o[e] = static_cast<unsigned short>((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xffffu));
        }
    }
}

// Store the lane's NPL states (kept as pairs; NPL = 1 keeps one value in .x).
template <int NPL, int NP>
__device__ __forceinline__ void store_states(float *dst, const float2 (&hp)[NP]) {
    if constexpr (NPL == 1) {
        dst[0] = hp[0].x;
    } else if constexpr (NPL == 2) {
        *reinterpret_cast<float2 *>(dst) = hp[0];
    } else {
#pragma unroll
        for (int j = 0; j < NP; j += 2)
            reinterpret_cast<float4 *>(dst)[j / 2] = make_float4(hp[j].x, hp[j].y, hp[j + 1].x, hp[j + 1].y);
    }
}

// The recurrence warps: lane (r, q) owns states q NPL .. q NPL + NPL - 1 of
// row r of the unit being processed.
template <typename T, int LPR, bool TRAP, int IOW>
__device__ __forceinline__ void recurrence_role(const ScanParams &p, unsigned char *smem, int tid) {
    using S = Shape<LPR, TRAP, IOW>;
    constexpr int NT = S::THREADS;
    constexpr int NPL = S::NPL, R = S::R;
    constexpr int NP = NPL > 1 ? NPL / 2 : 1;
    constexpr int RW = 32 / LPR;   // rows per warp
    const int lane = tid & 31, warp = tid >> 5;
    const int r = S::GROUP_MAJOR ? warp * RW + lane % RW : tid / LPR;
    const int q = S::GROUP_MAJOR ? lane / RW : tid % LPR;
    const int dstate = static_cast<int>(p.dstate);
    const Sched sc = make_sched(p, R);
    const int n8 = static_cast<int>((p.seqlen + 7) / 8);   // 8-step checkpoints per row

    // A log2(e) and the state of the lane's states, kept as the register pairs
    // the packed instructions take (no moves in the loop); set at the start of
    // every piece of work.
    float2 ap[NP], hp[NP];
    float2 bprev[NP];   // trapezoidal rule: the lane's B_{t-1} entries (B_{-1} u_{-1} = 0 via its coefficient;
                        // a piece that starts inside a row reads B at its step before from memory)
    int s = 0;          // tile stage of chunk it
    int64_t it = 0;     // position in the CTA's list of chunks
    const int npieces = num_pieces(sc);
    for (int pi = 0; pi < npieces; ++pi) {
        const PieceRange pr = piece_at(sc, pi);
        // the rows of unit pr.u, entering state from the initial state (chunk
        // 0) or from the CTA that ran the unit's start
        const UnitRow ur = unit_row(p, sc, pr.u, R, r);
        const int64_t row = ur.b * p.dim + ur.dc;
        const bool carried = pr.c0 > 0;
        if (carried) wait_carry(p, pr.u, tid);
        // checkpoints of this row (the lane's states), if asked for
        float *ckpt_row = (p.ckpt && ur.ok) ? p.ckpt + row * n8 * kStates + q * NPL : nullptr;
        {
            const int64_t dc = ur.dc;
            const float *hsrc = carried ? p.sk_carry + (static_cast<int64_t>(pr.u) * R + r) * kStates
                                        : (p.h0 ? p.h0 + row * dstate : nullptr);
            const T *bsrc = nullptr;
            if constexpr (TRAP) {
                if (carried)
                    bsrc = static_cast<const T *>(p.B) + ur.b * p.B_sb + static_cast<int64_t>(pr.c0) * kSteps - 1;
            }
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                float a2[2] = {0.f, 0.f}, h2[2] = {0.f, 0.f}, b2[2] = {0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 2 && 2 * j + e < NPL; ++e) {
                    const int n = q * NPL + 2 * j + e;
                    if (n < dstate) {
                        a2[e] = __ldg(p.A + dc * dstate + n) * kLog2e;
                        if (hsrc) h2[e] = carried ? __ldcg(hsrc + n) : __ldg(hsrc + n);
                        if constexpr (TRAP) {
                            if (bsrc) b2[e] = to_f32<T>(bsrc[n * p.B_sn]);
                        }
                    }
                }
                ap[j] = f2(a2[0], a2[1]);
                hp[j] = f2(h2[0], h2[1]);
                bprev[j] = f2(b2[0], b2[1]);
            }
        }
        for (int c = pr.c0; c < pr.c1; ++c, ++it, s = next_stage(s, kTileStages)) {
        unsigned char *st = smem + s * S::STAGE;
        const float4 *xrow = reinterpret_cast<const float4 *>(st + S::X_OFF) + r * S::XR;
        float *yl = reinterpret_cast<float *>(st + S::Y_OFF) + r * S::YR + (S::WARP_SUM ? 0 : q * S::YQ);
        // The partial readouts of steps t0 .. t0 + EW - 1: stored per lane, or
        // (LPR 4 and 8) summed over the row's LPR groups in a transposed
        // reduction: each round a lane keeps half of its values, adds the
        // partner group's copy of that half, and passes on the other half, so
        // that after log2(LPR) rounds lane q holds the total of step t0 + q.
        auto emit = [&](int t0, const float (&o)[S::EW]) {
            if constexpr (S::WARP_SUM) {
                float v[LPR];
#pragma unroll
                for (int e = 0; e < LPR; ++e) v[e] = o[e];
#pragma unroll
                for (int half = LPR / 2; half >= 1; half /= 2) {
                    const bool hi = q & half;
#pragma unroll
                    for (int e = 0; e < half; ++e) {
                        const float keep = hi ? v[e + half] : v[e];
                        const float send = hi ? v[e] : v[e + half];
                        v[e] = keep + __shfl_xor_sync(0xffffffffu, send, S::QSTRIDE * half);
                    }
                }
                yl[t0 + q] = v[0];
            } else {
                *reinterpret_cast<float4 *>(yl + t0) = make_float4(o[0], o[1], o[2], o[3]);
            }
        };
        const float *Bl = reinterpret_cast<const float *>(st + S::B_OFF) + q * NPL;
        const float *Cl = reinterpret_cast<const float *>(st + S::C_OFF) + q * NPL;
        bar_wait<NT>(bar_xf(s));

        // Software pipelined over the chunk: step pairs are read one pair
        // ahead, B and C one step ahead, and the ex2 of step t + 1 is issued
        // before the FMAs of step t, so neither shared-memory nor MUFU latency
        // sits on the state's dependency chain. Partial readouts leave in
        // float4 stores every 4 steps.
        auto decay = [&](float dt, float2 (&a)[NP]) {
            if constexpr (NPL == 1) {
                a[0] = f2(ex2_approx(dt * ap[0].x), 0.f);
            } else {
#pragma unroll
                for (int j = 0; j < NP; ++j) a[j] = ex2x2(mul2(f2(dt, dt), ap[j]));
            }
        };
        if constexpr (TRAP) {
            // h_t = a_t (h_{t-1} + p_t B_{t-1}) + q_t B_t with p_t = (1 - lambda_t)
            // delta_t u_{t-1} and q_t = lambda_t delta_t u_t (one float4 per step)
            float4 xc = xrow[0], xn = xrow[1];
            float2 acur[NP];
            decay(xc.x, acur);
            StepIn<NPL> cur = load_bc_step<NPL>(Bl, Cl);
            float outs[4];
#pragma unroll
            for (int t = 0; t < kSteps; ++t) {
                StepIn<NPL> nxt = cur;
                float2 anxt[NP];
                float4 xnn = xn;
                if (t + 1 < kSteps) {
                    nxt = load_bc_step<NPL>(Bl + (t + 1) * kStates, Cl + (t + 1) * kStates);
                    decay(xn.x, anxt);
                    if (t + 2 < kSteps) xnn = xrow[t + 2];
                }
                const float qv = xc.y, pv = xc.z;
                if constexpr (NPL == 1) {
                    hp[0].x = fmaf(acur[0].x, fmaf(pv, bprev[0].x, hp[0].x), qv * cur.b[0].x);
                    outs[t & 3] = cur.c[0].x * hp[0].x;
                } else {
                    float2 acc;
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        hp[j] = fma2(acur[j], fma2(f2(pv, pv), bprev[j], hp[j]), mul2(f2(qv, qv), cur.b[j]));
                        acc = j == 0 ? mul2(cur.c[j], hp[j]) : fma2(cur.c[j], hp[j], acc);
                    }
                    outs[t & 3] = acc.x + acc.y;
                }
                if ((t & 3) == 3) emit(t - 3, outs);
#pragma unroll
                for (int j = 0; j < NP; ++j) bprev[j] = cur.b[j];
                if (t + 1 < kSteps) {
                    cur = nxt;
#pragma unroll
                    for (int j = 0; j < NP; ++j) acur[j] = anxt[j];
                    xc = xn;
                    xn = xnn;
                }
            }
        } else {
        // B and C of step t + D and its exponentials are issued while step t
        // runs (D = 2 when the lane holds 4 states or fewer, else 1), so that
        // with one recurrence warp on a sub-partition neither the shared-memory
        // nor the MUFU latency reaches the state's dependency chain. xw holds
        // the step pairs t/2, t/2 + 1 and t/2 + 2 of the step tile.
        constexpr int D = NPL <= 4 ? 2 : 1;
        float4 xw[3] = {xrow[0], xrow[1], xrow[2]};
        auto dlt = [&](int step, int t) -> float {
            const float4 &w = xw[(step >> 1) - (t >> 1)];
            return (step & 1) ? w.z : w.x;
        };
        StepIn<NPL> bq[D + 1];
        float2 aq[D + 1][NP];
#pragma unroll
        for (int k = 0; k < D; ++k) {
            bq[k] = load_bc_step<NPL>(Bl + k * kStates, Cl + k * kStates);
            decay(dlt(k, 0), aq[k]);
        }
        float outs[S::EW];
#pragma unroll
        for (int t = 0; t < kSteps; ++t) {
            if (t + D < kSteps) {
                bq[(t + D) % (D + 1)] = load_bc_step<NPL>(Bl + (t + D) * kStates, Cl + (t + D) * kStates);
                decay(dlt(t + D, t), aq[(t + D) % (D + 1)]);
            }
            const StepIn<NPL> &cur = bq[t % (D + 1)];
            const float2 (&acur)[NP] = aq[t % (D + 1)];
            const float du = (t & 1) ? xw[0].w : xw[0].y;
            constexpr int E = S::EW;
            if constexpr (NPL == 1) {
                hp[0].x = fmaf(acur[0].x, hp[0].x, du * cur.b[0].x);
                outs[t % E] = cur.c[0].x * hp[0].x;
            } else {
                float2 acc;
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    hp[j] = fma2(acur[j], hp[j], mul2(f2(du, du), cur.b[j]));
                    acc = j == 0 ? mul2(cur.c[j], hp[j]) : fma2(cur.c[j], hp[j], acc);
                }
                outs[t % E] = acc.x + acc.y;
            }
            if (t % E == E - 1) emit(t - E + 1, outs);
            if ((t & 7) == 7 && ckpt_row) {   // the state after step 8 k + 7 of the sequence
                const int k8 = 2 * c + t / 8;
                if (k8 < n8) store_states<NPL>(ckpt_row + static_cast<int64_t>(k8) * kStates, hp);
            }
            if (t & 1) {   // the pair (t + 1, t + 2) becomes current
                xw[0] = xw[1];
                xw[1] = xw[2];
                if ((t >> 1) + 3 < kSteps / 2) xw[2] = xrow[(t >> 1) + 3];
            }
        }
        }
        bar_signal<NT>(bar_yf(s));
        }

        if (pr.c1 == sc.nc) {   // the end of the sequence: the final state
            if (ur.ok && p.hT) {
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int n = q * NPL + i;
                    if (n < dstate) p.hT[row * dstate + n] = (i & 1) ? hp[i / 2].y : hp[i / 2].x;
                }
            }
        } else {   // hand the state over to the CTA that continues this unit
            float *dst = p.sk_carry + (static_cast<int64_t>(pr.u) * R + r) * kStates;
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                const int n = q * NPL + i;
                if (n < dstate) dst[n] = (i & 1) ? hp[i / 2].y : hp[i / 2].x;
            }
            __threadfence();
            rec_bar(kBarRecB);
            if (tid == 0) st_release(p.sk_flag + pr.u, 1);
        }
    }
}

// The I/O warps: thread (r, k) handles steps k IP .. k IP + IP - 1 of row r in
// every chunk, plus BC_PER 16-byte pieces of the chunk's B/C tiles. Its raw
// inputs travel through the ring RA chunks ahead of use (cp.async on
// the aligned path, plain loads otherwise); a thread waits only for its own
// copies, so the ring needs no barrier.
template <typename T, int LPR, bool VEC, int VAR, int IOW>
__device__ __forceinline__ void io_role(const ScanParams &p, unsigned char *smem, int i) {
    constexpr bool CONV = VAR == 1, TRAP = VAR == 2;
    using S = Shape<LPR, TRAP, IOW>;
    using RW = Raw<T, LPR, VAR, IOW>;
    constexpr int NT = S::THREADS, IOT = S::IOT;
    constexpr int R = S::R, IP = S::IP, IPR = S::IPR, EB = RW::EB, PB = RW::PB, PS = RW::PS;
    constexpr int VE = RW::VE, VB = RW::VB, BCB = RW::BCB, BC_PER = RW::BC_PER;
    static_assert(IP % 2 == 0, "pieces hold step pairs");
    const int r = i / IPR, k = i % IPR;
    const int dstate = static_cast<int>(p.dstate);
    const int64_t L = p.seqlen;
    const bool has_z = p.z != nullptr;
    const int tk = k * IP;   // the thread's first step within a chunk
    const Sched sc = make_sched(p, R);
    const int nfull = static_cast<int>(L / kSteps);   // chunks with all kSteps steps inside the sequence

    // The thread's B/C pieces: tensor (0 = B, 1 = C), state n, steps bt .. bt + VB - 1.
    int bc_off[BC_PER], bc_t[BC_PER], bc_n[BC_PER], bc_tensor[BC_PER], bc_bytes[BC_PER];
#pragma unroll
    for (int j = 0; j < BC_PER; ++j) {
        const int pc = i + j * IOT;
        bc_tensor[j] = pc / (kStates * (kSteps / VB));
        const int rem = pc % (kStates * (kSteps / VB));
        bc_n[j] = rem % kStates;
        bc_t[j] = (rem / kStates) * VB;
        bc_off[j] = (bc_tensor[j] == 0 ? S::B_OFF : S::C_OFF) + (bc_t[j] * kStates + bc_n[j]) * 4;
        bc_bytes[j] = bc_n[j] < dstate ? BCB : 0;   // states past dstate read as zero
    }

    // Per-piece data of the three steps, looked up when a step enters a new
    // piece and then advanced chunk by chunk: the input pointers of the
    // thread's steps of the chunk to stage; the bias (and convolution taps)
    // for widening; the output pointer and D for finishing.
    const T *srow[3], *lrow = nullptr, *bsrc[BC_PER];
    auto stage_ctx = [&](int u, int c) {
        const UnitRow x = unit_row(p, sc, u, R, r);
        const int64_t t = static_cast<int64_t>(c) * kSteps + tk;
        srow[0] = static_cast<const T *>(p.u) + x.b * p.u_sb + x.dc * p.u_sd + t;
        srow[1] = static_cast<const T *>(p.delta) + x.b * p.dl_sb + x.dc * p.dl_sd + t;
        srow[2] = has_z ? static_cast<const T *>(p.z) + x.b * p.z_sb + x.dc * p.z_sd + t : srow[0];
        if constexpr (TRAP) lrow = static_cast<const T *>(p.lambda_raw) + x.b * p.lm_sb + x.dc * p.lm_sd + t;
#pragma unroll
        for (int j = 0; j < BC_PER; ++j) {
            const T *base = bc_tensor[j] == 0 ? static_cast<const T *>(p.B) + x.b * p.B_sb
                                              : static_cast<const T *>(p.C) + x.b * p.C_sb;
            bsrc[j] = (bc_bytes[j] ? base + bc_n[j] * (bc_tensor[j] == 0 ? p.B_sn : p.C_sn) : base) + bc_t[j] +
                      static_cast<int64_t>(c) * kSteps;
        }
    };
    auto stage_advance = [&]() {
#pragma unroll
        for (int t = 0; t < 3; ++t) srow[t] += kSteps;
        if constexpr (TRAP) lrow += kSteps;
#pragma unroll
        for (int j = 0; j < BC_PER; ++j) bsrc[j] += kSteps;
    };
    // Convolution taps right-aligned in a window of 4 (leading taps beyond
    // the width stay 0): cw[3] weighs the current input.
    float bias = 0.f, cw[4] = {0.f, 0.f, 0.f, 0.f}, cb = 0.f, Dw = 0.f;
    auto widen_ctx = [&](int u) {
        const UnitRow x = unit_row(p, sc, u, R, r);
        bias = p.delta_bias ? __ldg(p.delta_bias + x.dc) : 0.f;
        if constexpr (CONV) {
            const int K = p.conv_width;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (j >= 4 - K) cw[j] = __ldg(p.conv_w + x.dc * K + (j - (4 - K)));
            cb = p.conv_b ? __ldg(p.conv_b + x.dc) : 0.f;
            Dw = p.D ? __ldg(p.D + x.dc) : 0.f;
        }
    };
    T *yrow = nullptr;
    float Df = 0.f;
    bool fok = false;
    auto finish_ctx = [&](int u, int c) {
        const UnitRow x = unit_row(p, sc, u, R, r);
        fok = x.ok;
        Df = p.D ? __ldg(p.D + x.dc) : 0.f;
        yrow = static_cast<T *>(p.y) + x.b * p.y_sb + x.dc * p.y_sd + static_cast<int64_t>(c) * kSteps + tk;
    };

    unsigned char *ring = smem + RW::OFF;
    auto slot = [&](int rs, int sl) { return ring + rs * RW::STAGE + (sl * IOT + i) * 16; };

    // Issue the copies of the raw inputs of chunk c (the staging step's
    // pointers point at it) into ring stage rs. Chunks inside the sequence
    // take fixed-size copies; the ragged last chunk copies what exists and
    // zero-fills the rest.
    // shared-window address of the thread's slot 0 in ring stage 0
    const unsigned ring_s = static_cast<unsigned>(__cvta_generic_to_shared(ring)) + i * 16;
    auto stage_chunk = [&](int c, int rs, bool known_full = false) {
        const bool full = known_full || c < nfull;
        if constexpr (VEC) {
            // (the variants' look-back lies before t = 0 in the sequence's first chunk: general path)
            if (full && (!(CONV || TRAP) || c > 0 || tk >= VE)) {
                // chunks inside the sequence: fixed-size copies from the running pointers
                const unsigned sb = ring_s + rs * RW::STAGE;
                constexpr int SB = PB < 16 ? PB : 16;
#pragma unroll
                for (int tsr = 0; tsr < 3; ++tsr) {
                    if (tsr == 2 && !has_z) break;
#pragma unroll
                    for (int sl = 0; sl < PS; ++sl)
                        cp_async_full<SB>(sb + (tsr * PS + sl) * IOT * 16,
                                          reinterpret_cast<const unsigned char *>(srow[tsr]) + sl * 16);
                }
#pragma unroll
                for (int j = 0; j < BC_PER; ++j) {
                    const unsigned dst = sb + (3 * PS + j) * IOT * 16;
                    if (bc_bytes[j]) {
                        cp_async_full<BCB>(dst, bsrc[j]);
                    } else {   // a state past dstate: zeros
                        if constexpr (BCB == 16) cp_async16(slot(rs, 3 * PS + j), p.B, 0);
                        else cp_async_small<BCB>(slot(rs, 3 * PS + j), p.B, 0);
                    }
                }
                if constexpr (TRAP) {
#pragma unroll
                    for (int sl = 0; sl < PS; ++sl)
                        cp_async_full<16>(sb + (RW::LAM + sl) * IOT * 16,
                                          reinterpret_cast<const unsigned char *>(lrow) + sl * 16);
                }
                if constexpr (CONV || TRAP) cp_async_full<16>(sb + RW::HALO * IOT * 16, srow[0] - VE);
                return;
            }
        }
        const int64_t t0 = static_cast<int64_t>(c) * kSteps;
        const int valid = full ? IP : static_cast<int>(min64(IP, max64(0, L - (t0 + tk))));
        constexpr int SB = PB < 16 ? PB : 16;   // bytes per slot
        // an in-bounds, aligned address for copies of zero bytes (nothing is read)
        const void *const tbase[3] = {p.u, p.delta, has_z ? p.z : p.u};
#pragma unroll
        for (int tsr = 0; tsr < 3; ++tsr) {
            if (tsr == 2 && !has_z) break;
            const T *src = srow[tsr];
            if constexpr (VEC) {
#pragma unroll
                for (int sl = 0; sl < PS; ++sl) {
                    int bytes = SB;
                    if (!full) {
                        const int have = valid * EB - sl * 16;
                        bytes = have < 0 ? 0 : (have > SB ? SB : have);
                    }
                    const void *g = bytes > 0 ? static_cast<const void *>(reinterpret_cast<const unsigned char *>(src) + sl * 16)
                                              : tbase[tsr];
                    if constexpr (PB >= 16) cp_async16(slot(rs, tsr * PS + sl), g, bytes);
                    else cp_async_small<PB>(slot(rs, tsr * PS + sl), g, bytes);
                }
            } else {
                Piece<T, IP> pc;
                load_piece<T, IP, false>(pc, src, valid);
#pragma unroll
                for (int w = 0; w < Piece<T, IP>::W; ++w)
                    reinterpret_cast<uint32_t *>(slot(rs, tsr * PS + w / 4))[w % 4] = pc.w[w];
            }
        }
        if constexpr (TRAP) {
            const T *src = lrow;
            if constexpr (VEC) {
#pragma unroll
                for (int sl = 0; sl < PS; ++sl) {
                    const int have = valid * EB - sl * 16;
                    const int bytes = have < 0 ? 0 : (have > 16 ? 16 : have);
                    cp_async16(slot(rs, RW::LAM + sl),
                               bytes > 0 ? static_cast<const void *>(reinterpret_cast<const unsigned char *>(src) + sl * 16)
                                         : p.lambda_raw,
                               bytes);
                }
            } else {
                Piece<T, IP> pc;
                load_piece<T, IP, false>(pc, src, valid);
#pragma unroll
                for (int w = 0; w < Piece<T, IP>::W; ++w)
                    reinterpret_cast<uint32_t *>(slot(rs, RW::LAM + w / 4))[w % 4] = pc.w[w];
            }
        }
        if constexpr (CONV || TRAP) {
            // the VE inputs before the piece (the convolution's look-back; the
            // trapezoidal rule's u_{t-1}); for the first piece of the sequence
            // they lie before t = 0 and read as 0
            const int64_t th = t0 + tk - VE;
            const int hv = th < 0 ? 0 : static_cast<int>(min64(VE, max64(0, L - th)));
            const T *hsrc = hv > 0 ? srow[0] - VE : static_cast<const T *>(p.u);
            if constexpr (VEC) {
                cp_async16(slot(rs, RW::HALO), hsrc, hv * EB);
            } else {
                Piece<T, VE> pc;
                load_piece<T, VE, false>(pc, hsrc, hv);
                *reinterpret_cast<uint4 *>(slot(rs, RW::HALO)) = make_uint4(pc.w[0], pc.w[1], pc.w[2], pc.w[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < BC_PER; ++j) {
            int bytes = bc_bytes[j];
            if (!full && bytes) bytes = static_cast<int>(min64(VB, max64(0, L - (t0 + bc_t[j])))) * EB;
            if constexpr (VEC) {
                const void *g = bytes > 0 ? static_cast<const void *>(bsrc[j]) : p.B;
                if constexpr (BCB == 16) cp_async16(slot(rs, 3 * PS + j), g, bytes);
                else cp_async_small<BCB>(slot(rs, 3 * PS + j), g, bytes);
            } else {
                Piece<T, VB> pc;
                load_piece<T, VB, false>(pc, bsrc[j], bytes / EB);
#pragma unroll
                for (int w = 0; w < Piece<T, VB>::W; ++w)
                    reinterpret_cast<uint32_t *>(slot(rs, 3 * PS + j))[w] = pc.w[w];
            }
        }
    };
    // The thread's piece starting at slot `first` of ring stage rs.
    auto ring_slots = [&](int rs, int first) {
        Piece<T, IP> pc;
        if constexpr (PB == 4) {
            pc.w[0] = *reinterpret_cast<const uint32_t *>(slot(rs, first));
        } else if constexpr (PB == 8) {
            const uint2 v = *reinterpret_cast<const uint2 *>(slot(rs, first));
            pc.w[0] = v.x; pc.w[1] = v.y;
        } else {
#pragma unroll
            for (int sl = 0; sl < PS; ++sl) {
                const uint4 v = *reinterpret_cast<const uint4 *>(slot(rs, first + sl));
                pc.w[4 * sl] = v.x; pc.w[4 * sl + 1] = v.y; pc.w[4 * sl + 2] = v.z; pc.w[4 * sl + 3] = v.w;
            }
        }
        return pc;
    };
    // The thread's piece of tensor tsr (0 u, 1 delta, 2 z) from ring stage rs.
    auto ring_piece = [&](int rs, int tsr) { return ring_slots(rs, tsr * PS); };
    // Readout of chunk c in two parts. finish_pre (before the wait for the
    // recurrence) takes what does not depend on it from ring stage rs: D u
    // and the gate; finish then adds the partial sums from tile stage s and
    // stores.
    float2 fskip[IP / 2], fgate[IP / 2];   // D u and silu(z) of the chunk to finish
    auto finish_pre = [&](int s, int rs) {
        if constexpr (CONV) {
            const float *sk = reinterpret_cast<const float *>(smem + RW::SK_OFF + s * RW::SK_STAGE) + r * RW::SKR + tk;
#pragma unroll
            for (int e = 0; e < IP; e += 2) fskip[e / 2] = *reinterpret_cast<const float2 *>(sk + e);
        } else {
            const float Dd = Df;
            const Piece<T, IP> u = ring_piece(rs, 0);
#pragma unroll
            for (int e = 0; e < IP; e += 2) fskip[e / 2] = mul2(f2(Dd, Dd), f2(elem(u, e), elem(u, e + 1)));
        }
        if (has_z) {
            const Piece<T, IP> z = ring_piece(rs, 2);
#pragma unroll
            for (int e = 0; e < IP; e += 2) fgate[e / 2] = silu2_out<T>(f2(elem(z, e), elem(z, e + 1)));
        }
    };
    auto finish = [&](int c_, int s, bool known_full = false) {
        const int64_t c = c_;
        const int64_t cnt = (known_full || c_ < nfull) ? IP : L - (c * kSteps + tk);
        if (!fok || cnt <= 0) return;
        const float *yp = reinterpret_cast<const float *>(smem + s * S::STAGE + S::Y_OFF) + r * S::YR + tk;
        float2 sum[IP / 2];
#pragma unroll
        for (int e = 0; e < IP / 2; ++e) sum[e] = f2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < (S::WARP_SUM ? 1 : LPR); ++j) {
            if constexpr (IP == 2) {
                sum[0] = add2(sum[0], *reinterpret_cast<const float2 *>(yp + j * S::YQ));
            } else {
#pragma unroll
                for (int v = 0; v < IP / 4; ++v) {
                    const float4 a = reinterpret_cast<const float4 *>(yp + j * S::YQ)[v];
                    sum[2 * v] = add2(sum[2 * v], f2(a.x, a.y));
                    sum[2 * v + 1] = add2(sum[2 * v + 1], f2(a.z, a.w));
                }
            }
        }
        float outv[IP];
#pragma unroll
        for (int e = 0; e < IP; e += 2) {
            float2 yv = add2(fskip[e / 2], sum[e / 2]);
            if (has_z) yv = mul2(yv, fgate[e / 2]);
            outv[e] = yv.x;
            outv[e + 1] = yv.y;
        }
        store_piece<T, IP, VEC>(yrow, outv, cnt);
    };
    // Chunk c's step tile (step pairs of delta, delta u) and B/C tiles from
    // ring stage rs into tile stage s.
    auto widen = [&](int c_, int s, int rs, bool known_full = false) {
        const int64_t c = c_;
        const float Dd = Dw;
        unsigned char *st = smem + s * S::STAGE;
        float4 *xrow = reinterpret_cast<float4 *>(st + S::X_OFF) + r * S::XR + (TRAP ? tk : tk / 2);
        const Piece<T, IP> xin = ring_piece(rs, 0), dl = ring_piece(rs, 1);
        // the SSM input u: the raw u, or the convolution prologue applied to x
        float2 u2[IP / 2];
        if constexpr (CONV) {
            const uint4 hw = *reinterpret_cast<const uint4 *>(slot(rs, RW::HALO));
            Piece<T, VE> hl;
            hl.w[0] = hw.x; hl.w[1] = hw.y; hl.w[2] = hw.z; hl.w[3] = hw.w;
            // input j of the window [look-back | piece]
            auto win = [&](int j) { return j < VE ? elem(hl, j) : elem(xin, j - VE); };
            float* sk = reinterpret_cast<float *>(smem + RW::SK_OFF + s * RW::SK_STAGE) + r * RW::SKR + tk;
#pragma unroll
            for (int e = 0; e < IP; e += 2) {
                float a0 = cb, a1 = cb;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    a0 = fmaf(cw[m], win(e + VE - 3 + m), a0);
                    a1 = fmaf(cw[m], win(e + 1 + VE - 3 + m), a1);
                }
                float2 uv = f2(a0, a1);
                if (p.conv_silu) uv = silu2_out<T>(uv);
                u2[e / 2] = uv;
                *reinterpret_cast<float2 *>(sk + e) = mul2(f2(Dd, Dd), uv);
            }
        } else {
#pragma unroll
            for (int e = 0; e < IP; e += 2) u2[e / 2] = f2(elem(xin, e), elem(xin, e + 1));
        }
        const bool full = known_full || c_ < nfull;
        const int64_t cnt = L - (c * kSteps + tk);
        float uprev = 0.f;   // trapezoidal rule: u_{t-1} of the piece's first step
        Piece<T, IP> lam;
        if constexpr (TRAP) {
            const uint4 hw = *reinterpret_cast<const uint4 *>(slot(rs, RW::HALO));
            Piece<T, VE> hl;
            hl.w[0] = hw.x; hl.w[1] = hw.y; hl.w[2] = hw.z; hl.w[3] = hw.w;
            uprev = elem(hl, VE - 1);
            lam = ring_slots(rs, RW::LAM);
        }
#pragma unroll
        for (int e = 0; e < IP; e += 2) {
            float2 v = add2(f2(elem(dl, e), elem(dl, e + 1)), f2(bias, bias));
            if (p.softplus) v = softplus2(v);
            if (!full) {   // steps past the end: delta = 0
                if (e >= cnt) v.x = 0.f;
                if (e + 1 >= cnt) v.y = 0.f;
            }
            if constexpr (TRAP) {
                // lambda = sigmoid(lambda_raw); q = lambda delta u_t, p = (1 - lambda) delta u_{t-1}
                const float2 lr = f2(elem(lam, e), elem(lam, e + 1));
                const float2 ex = ex2x2(mul2(lr, f2(-kLog2e, -kLog2e)));
                const float2 lm = f2(__fdividef(1.f, 1.f + ex.x), __fdividef(1.f, 1.f + ex.y));
                const float2 ld = mul2(lm, v);                          // lambda delta
                const float2 q = mul2(ld, u2[e / 2]);
                const float2 prev = f2(e == 0 ? uprev : u2[e / 2 - 1].y, u2[e / 2].x);
                const float2 pq = mul2(add2(v, f2(-ld.x, -ld.y)), prev);   // (1 - lambda) delta u_{t-1}
                xrow[e] = make_float4(v.x, q.x, pq.x, 0.f);
                xrow[e + 1] = make_float4(v.y, q.y, pq.y, 0.f);
            } else {
                const float2 du = mul2(v, u2[e / 2]);
                xrow[e / 2] = make_float4(v.x, du.x, v.y, du.y);
            }
        }
#pragma unroll
        for (int j = 0; j < BC_PER; ++j) {
            Piece<T, VB> pc;
            if constexpr (BCB == 16) {
                const uint4 w = *reinterpret_cast<const uint4 *>(slot(rs, 3 * PS + j));
                pc.w[0] = w.x; pc.w[1] = w.y; pc.w[2] = w.z; pc.w[3] = w.w;
            } else {
                const uint2 w = *reinterpret_cast<const uint2 *>(slot(rs, 3 * PS + j));
                pc.w[0] = w.x; pc.w[1] = w.y;
            }
            float *dst = reinterpret_cast<float *>(st + bc_off[j]);
#pragma unroll
            for (int e = 0; e < VB; ++e) dst[e * kStates] = elem(pc, e);
        }
    };

    // Chunk it (of the CTA's list) is widened in iteration it, finished in
    // iteration it + kTileStages - 1 (or after the loop), and its raw inputs
    // are staged RA = RS - kTileStages + 1 iterations before its widening into
    // the ring stage that the chunk finished in the same iteration releases.
    // Prologue: chunks 0 .. RA - 1 in flight, one commit group per chunk
    // (empty past the end: the count stays uniform). Each of the three steps
    // follows the CTA's work with its own cursor.
    const int64_t K = sc.K;
    PCur ka, kw, kf;
    ka.begin(sc);
    kw = ka;
    kf = ka;
    stage_ctx(ka.u, ka.c);
    widen_ctx(kw.u);
    finish_ctx(kf.u, kf.c);
    auto stage_next = [&]() {
        if (ka.next(sc)) stage_ctx(ka.u, ka.c);
        else stage_advance();
    };
    auto finish_next = [&]() {
        if (kf.next(sc)) finish_ctx(kf.u, kf.c);
        else yrow += kSteps;
    };
#pragma unroll
    for (int c0 = 0; c0 < RW::RA; ++c0) {
        if (c0 < K) {
            stage_chunk(ka.c, c0);
            stage_next();
        }
        cp_async_commit();
    }
    int s = 0, rs = 0;                    // tile and ring stage of chunk it
    int sf = 0, rf = 0;                   // tile and ring stage of the next chunk to finish
    int ra = RW::RA % RW::RS;             // ring stage of chunk it + RA
    for (int64_t it = 0; it < K; ++it) {
        // Steady state: while the three cursors stay inside their pieces, the
        // chunks they touch are whole and both the finish and the staging of
        // this iteration are due, a lean body runs with no cursor or bounds
        // logic; it stops one chunk before any of them would cross, and the
        // general body below takes that chunk.
        if (it >= kTileStages - 1) {
            auto room = [&](const PCur &k) {
                const int left = k.c1 - k.c;   // chunks left in the piece, this one included
                const int whole = nfull - k.c;
                return left < whole ? left : whole;
            };
            int64_t n = K - RW::RA - it;      // iterations that still stage a chunk
            n = min64(n, room(kw));
            n = min64(n, room(kf));
            n = min64(n, room(ka));
            for (int64_t m = 1; m < n; ++m, ++it) {
                cp_async_wait<RW::RA - 1>();
                widen(kw.c, s, rs, true);
                bar_signal<NT>(bar_xf(s));
                finish_pre(sf, rf);
                bar_wait<NT>(bar_yf(sf));
                finish(kf.c, sf, true);
                stage_chunk(ka.c, ra, true);
                cp_async_commit();
                ++kw.c;
                ++kf.c;
                ++ka.c;
                stage_advance();
                yrow += kSteps;
                s = next_stage(s, kTileStages);
                rs = next_stage(rs, RW::RS);
                ra = next_stage(ra, RW::RS);
                sf = next_stage(sf, kTileStages);
                rf = next_stage(rf, RW::RS);
            }
        }
        cp_async_wait<RW::RA - 1>();      // chunk it's copies have landed
        widen(kw.c, s, rs);
        bar_signal<NT>(bar_xf(s));
        const int64_t j = it - (kTileStages - 1);
        if (j >= 0) {
            finish_pre(sf, rf);
            bar_wait<NT>(bar_yf(sf));
            finish(kf.c, sf);
            sf = next_stage(sf, kTileStages);
            rf = next_stage(rf, RW::RS);
            finish_next();
        }
        if (it + RW::RA < K) {
            stage_chunk(ka.c, ra);
            stage_next();
        }
        cp_async_commit();
        s = next_stage(s, kTileStages);
        rs = next_stage(rs, RW::RS);
        ra = next_stage(ra, RW::RS);
        if (kw.next(sc)) widen_ctx(kw.u);
    }
    for (int64_t j = max64(K - (kTileStages - 1), 0); j < K; ++j) {
        finish_pre(sf, rf);
        bar_wait<NT>(bar_yf(sf));
        finish(kf.c, sf);
        sf = next_stage(sf, kTileStages);
        rf = next_stage(rf, RW::RS);
        finish_next();
    }
    cp_async_wait<0>();
}

// ONE: the instantiation for launches with at most one CTA per SM, whose
// threads may take every register the SM has.
template <typename T, int LPR, bool VEC, int VAR, int IOW, bool ONE = false>
__global__ void __launch_bounds__(Shape<LPR, VAR == 2, IOW>::THREADS, ONE ? 1 : Shape<LPR, VAR == 2, IOW>::MINB)
    rec_kernel(const ScanParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    if (threadIdx.x < kScanThreads) {
        recurrence_role<T, LPR, VAR == 2, IOW>(p, smem, threadIdx.x);
    } else {
        io_role<T, LPR, VEC, VAR, IOW>(p, smem, threadIdx.x - kScanThreads);
    }
}

// Compiled variants: every lanes-per-row count with 2 I/O warps for the plain
// scan, the convolution prologue (2 and 4 lanes) and the trapezoidal rule (2
// and 4 lanes); 4 I/O warps for the plain scan with 2, 4 or 8 lanes.
bool variant_compiled(int lpr, int variant, int iow) {
    if (iow == 2) return variant == 0 || lpr == 2 || lpr == 4;
    return iow == 4 && variant == 0 && (lpr == 2 || lpr == 4 || lpr == 8);
}

template <typename T, int LPR, int VAR, int IOW>
const void *rec_ptr_v(bool vec, bool one = false) {
    if constexpr (VAR == 0 && LPR <= 8) {   // one CTA per SM: the aligned plain scan
        if (vec && one) return reinterpret_cast<const void *>(rec_kernel<T, LPR, true, VAR, IOW, true>);
    }
    return vec ? reinterpret_cast<const void *>(rec_kernel<T, LPR, true, VAR, IOW>)
               : reinterpret_cast<const void *>(rec_kernel<T, LPR, false, VAR, IOW>);
}

template <typename T, int LPR>
const void *rec_ptr(bool vec, int variant, int iow, bool one) {
    if constexpr (LPR != 16) {
        if (iow == 4) return rec_ptr_v<T, LPR, 0, 4>(vec, one);
    }
    if constexpr (LPR == 2 || LPR == 4) {   // the variants need 16-byte pieces
        if (variant == 1) return rec_ptr_v<T, LPR, 1, 2>(vec);
        if (variant == 2) return rec_ptr_v<T, LPR, 2, 2>(vec);
    }
    return rec_ptr_v<T, LPR, 0, 2>(vec, one);
}

template <typename T>
const void *rec_select(int lpr, bool vec, int variant, int iow, bool one) {
    switch (lpr) {
        case 2: return rec_ptr<T, 2>(vec, variant, iow, one);
        case 4: return rec_ptr<T, 4>(vec, variant, iow, one);
        case 8: return rec_ptr<T, 8>(vec, variant, iow, one);
        default: return rec_ptr<T, 16>(vec, variant, iow, one);
    }
}

const void *rec_kernel_for(int in_dtype, int lpr, bool vec, int variant, int iow, bool one) {
    return in_dtype == 0 ? rec_select<float>(lpr, vec, variant, iow, one)
                         : rec_select<__nv_bfloat16>(lpr, vec, variant, iow, one);
}

// Streaming multiprocessors of the current device (cached per device).
int device_sms() {
    static int cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) cached[dev] = n;
    }
    return cached[dev];
}

template <typename T, int LPR>
int smem_bytes_lpr(int variant, int iow) {
    if constexpr (LPR != 16) {
        if (iow == 4) return Raw<T, LPR, 0, 4>::BYTES;
    }
    if constexpr (LPR == 2 || LPR == 4) {
        if (variant == 1) return Raw<T, LPR, 1, 2>::BYTES;
        if (variant == 2) return Raw<T, LPR, 2, 2>::BYTES;
    }
    return Raw<T, LPR, 0, 2>::BYTES;
}

template <typename T>
int smem_bytes_t(int lpr, int variant, int iow) {
    switch (lpr) {
        case 2: return smem_bytes_lpr<T, 2>(variant, iow);
        case 4: return smem_bytes_lpr<T, 4>(variant, iow);
        case 8: return smem_bytes_lpr<T, 8>(variant, iow);
        default: return smem_bytes_lpr<T, 16>(variant, iow);
    }
}

}  // namespace

int rec_variant(const ScanParams &p) { return p.lambda_raw ? 2 : p.conv_w ? 1 : 0; }

int rec_smem_bytes(int in_dtype, int lpr, int variant, int iow) {
    return in_dtype == 0 ? smem_bytes_t<float>(lpr, variant, iow) : smem_bytes_t<__nv_bfloat16>(lpr, variant, iow);
}

bool rec_supports_variant(int lpr, int variant, int iow) { return variant_compiled(lpr, variant, iow); }
int rec_chunk() { return kSteps; }
int rec_threads(int iow) { return kScanThreads + 32 * iow; }
int rec_rows(int lpr) { return kScanThreads / lpr; }

// Resident CTAs per SM of a sequential kernel (cached per kernel; the
// shared-memory bound when no device answers).
int rec_ctas_per_sm(int in_dtype, int lpr, bool vec, int variant, int iow) {
    constexpr int kSlots = 64;
    static const void *keys[kSlots];
    static int vals[kSlots];
    static int used = 0;
    static std::mutex mu;
    const void *k = rec_kernel_for(in_dtype, lpr, vec, variant, iow, false);
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
        if (keys[i] == k) return vals[i];
    const int smem = rec_smem_bytes(in_dtype, lpr, variant, iow);
    int n = 0;
    bool asked = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess &&
                 cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, rec_threads(iow), smem) == cudaSuccess;
    if (!asked) {
        cudaGetLastError();
        n = (228 * 1024) / (smem + 1024);
    } else if (used < kSlots) {
        keys[used] = k;
        vals[used] = n;
        ++used;
    }
    return n;
}

namespace {
constexpr size_t kStatusBytes = 256;
size_t round256(size_t n) { return (n + 255) / 256 * 256; }
}  // namespace

size_t rec_persistent_clear_bytes(int64_t units) {
    return kStatusBytes + round256(static_cast<size_t>(units) * sizeof(int));
}

size_t rec_persistent_ws_bytes(int64_t units, int rows_per_unit) {
    return rec_persistent_clear_bytes(units) +
           static_cast<size_t>(units) * static_cast<size_t>(rows_per_unit) * kStates * sizeof(float);
}

void rec_bind_workspace(ScanParams &p, void *ws, int64_t units, int ctas) {
    unsigned char *w = static_cast<unsigned char *>(ws);
    p.sk_ctas = ctas;
    p.sk_units = static_cast<int>(units);
    p.sk_status = reinterpret_cast<int *>(w);
    p.sk_flag = reinterpret_cast<int *>(w + kStatusBytes);
    p.sk_carry = reinterpret_cast<float *>(w + rec_persistent_clear_bytes(units));
}

int rec_max_ctas(const ScanParams &p, int in_dtype, int lpr, bool vec, int num_sms, int iow) {
    const int per_sm = rec_ctas_per_sm(in_dtype, lpr, vec, rec_variant(p), iow);
    const int64_t R = kScanThreads / lpr;
    const int64_t units = p.batch * ((p.dim + R - 1) / R);
    return static_cast<int>(min64(units, static_cast<int64_t>(per_sm) * num_sms));
}

// Persistent launches (p.sk_ctas > 0) are cooperative: the runtime starts them
// only if every CTA can be resident at once, so a CTA that waits for another
// one's carry never waits for a CTA that has not started. The flags and the
// status word are cleared on the stream first.
cudaError_t launch_rec(const ScanParams &p, int lpr, bool vec, int in_dtype, int iow, cudaStream_t stream) {
    const int variant = rec_variant(p);
    if (!rec_supports_variant(lpr, variant, iow) || (p.conv_w && p.lambda_raw)) return cudaErrorInvalidValue;
    if (p.sk_ctas > 0 && (!p.sk_carry || !p.sk_flag || !p.sk_status)) return cudaErrorInvalidValue;
    // a persistent launch with at most one CTA per SM takes the instantiation
    // without the occupancy bound on registers
    const bool one = p.sk_ctas > 0 && p.sk_ctas <= device_sms();
    const void *k = rec_kernel_for(in_dtype, lpr, vec, variant, iow, one);
    const int smem = rec_smem_bytes(in_dtype, lpr, variant, iow);
    const int threads = rec_threads(iow);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int R = kScanThreads / lpr;
    void *args[] = {const_cast<ScanParams *>(&p)};
    if (p.sk_ctas == 0) {
        const dim3 grid(static_cast<unsigned>((p.dim + R - 1) / R), static_cast<unsigned>(p.batch));
        e = cudaLaunchKernel(k, grid, dim3(threads), args, static_cast<size_t>(smem), stream);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    e = cudaMemsetAsync(p.sk_status, 0, rec_persistent_clear_bytes(p.sk_units), stream);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(p.sk_ctas));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeCooperative;
    attr.val.cooperative = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelExC(&cfg, k, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ms
