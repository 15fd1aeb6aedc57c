// ssd_fwd.cu -- Mamba-2 scalar-decay SSM forward (the structured state space
// duality, SSD) in chunks of 128 tokens on the sm_100a tensor cores.
//
// What it computes, per batch b and head h (the recurrent definition):
//   delta_t = softplus(dt[b,t,h] + dt_bias[h]),  a_t = exp(delta_t A[h])
//   H_t = a_t H_{t-1} + (delta_t x_t) B_t^T   (H: headdim x dstate = 64 x 128)
//   y_t = H_t C_t + D[h] x_t,  y_t *= silu(z_t)
// ("Notas sobre Mamba", sections "A forma dual: atenção mascarada" and "O
// algoritmo SSD"; "Mamba-2 e State Space Duality (SSD)", section "O algoritmo
// de decomposição em blocos do SSD").
//
// How: the pages' chunked algorithm. Within a chunk of Q = 128 tokens, with
// s_t the running sum of delta A inside the chunk (s_end its last value):
//   G     = C B^T                                   (Q x Q, contraction over N)
//   M'_ji = [i <= j] exp(s_j - s_i) delta_i G_ji     (decay mask and step)
//   Yd    = M' X                                    (diagonal block)
//   Yo    = C H_prev^T,  y_j = Yd_j + exp(s_j) Yo_j + D x_j   (off-diagonal)
//   Xt_i  = exp(s_end - s_i) delta_i X_i,  S = B^T Xt  (chunk state)
//   H     = exp(s_end) H_prev + S^T                 (state passing)
// The four products are tcgen05 MMAs (bf16 operands from shared memory,
// fp32 accumulators in tensor memory); the decay, the state passing, the
// skip and the gate run in the epilogue warps. A CTA walks the chunks of a
// (b, h) in order, so the state stays on the SM: one CTA per (b, h), or, when
// the pairs would leave the last wave partly empty, one resident CTA per SM
// taking an even share of all pairs' chunks, where a pair cut between two CTAs
// hands its state over through global memory (see the schedule below).
//
// Roles (576 threads): warps 0-15 epilogue (warp w reads TMEM lanes
// 32 (w % 4) .. +31, i.e. rows of the chunk, and handles column quarter
// w / 4); warp 16 issues the TMA loads and computes each chunk's step sizes
// and decay sums ahead of time; warp 17 owns the tensor memory and issues the
// MMAs. Every wait on an mbarrier gives up after about a second, records
// MS_ERR_TIMEOUT in the status word and lets the CTA drain and exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_math.cuh"
#include "launch.h"
#include "mambascan.h"

namespace {

constexpr int kQ = 128;          // tokens per chunk
constexpr int kP = 64;           // headdim
constexpr int kN = 128;          // dstate
constexpr int kStages = 2;       // input stages (X, B, C of one chunk each)
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = kEpiThreads + 64;
constexpr int kTmaWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;

// Shared memory, from a 1024-byte aligned base. Every operand tile is made of
// 128-byte-swizzled atoms (rows of 128 bytes, 8-row groups of 1024 bytes).
constexpr uint32_t kXTile = kQ * 128;                    // 128 tokens x 64 bf16
constexpr uint32_t kBCTile = 2 * kQ * 128;               // 128 tokens x 128 bf16, two 64-wide atoms
constexpr uint32_t kStageBytes = kXTile + 2 * kBCTile;   // X, B, C
constexpr uint32_t kOffM = kStages * kStageBytes;        // M' (128 x 128 bf16, two atoms along i)
constexpr uint32_t kOffXt = kOffM + 2 * kQ * 128;        // Xt (128 tokens x 64 bf16)
constexpr uint32_t kOffH = kOffXt + kXTile;              // H (128 rows n x 64 bf16 along p)
// step data of two chunks: float delta[2][Q], float s2[2][Q], bf16 cf[2][Q]; then int abort
constexpr uint32_t kOffStep = kOffH + kN * 128;
constexpr uint32_t kOffAbort = kOffStep + 2 * kQ * 10;
constexpr uint32_t kOffBar = kOffAbort + 16;
// mbarriers and their phases (chunk c completes phase c of a single barrier, or
// phase c / 2 of barrier c % 2 of a pair; waits use that parity):
//   full[c%2]   TMA bytes of stage c landed          <- producer expect_tx + TMA
//   empty[c%2]  stage c no longer read                <- 16 epilogue warps after y(c)
//   gfull[c%2]  G(c) in TMEM buffer c%2               <- tcgen05.commit
//   pready      M'(c), Xt(c) written (phase c)        <- 16 epilogue warps
//   sfull/yfull S(c) / Yd(c) done (phase c)           <- tcgen05.commit
//   hready      H_{c-1} in its tile (phase c; phase 0 is the initial state)
//   yfree       Yd/Yo of chunk c read (phase c)       <- 16 epilogue warps
//   step[c%2]   step data of chunk c written           <- 32 producer lanes
// No waiter can fall two phases behind: every barrier's next phase needs an
// event that itself follows the wait (e.g. gfull[c%2] for chunk c + 2 needs
// pready(c + 1), which follows the epilogue's wait on gfull for chunk c + 1;
// full[c%2] for chunk c + 2 needs empty(c), which follows the waits on
// full[c%2] for chunk c; hready phase c + 1 needs S(c), issued after the
// issuer's wait on hready phase c).
enum Bar { kFull0, kFull1, kEmpty0, kEmpty1, kGFull0, kGFull1, kPReady, kSFull, kYFull, kHReady, kYFree, kDrain,
           kStep0, kStep1, kNumBars };
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffSched = kOffTmemSlot + 8;          // the CTA's SsdSched (seven ints)
constexpr uint32_t kSmemBytes = kOffSched + 32;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kOffM % 1024 == 0 && kOffXt % 1024 == 0 && kOffH % 1024 == 0 && kStageBytes % 1024 == 0,
              "swizzle atoms need 1024-byte alignment");

// Tensor memory: 512 columns x 128 lanes of fp32.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0;      // two buffers of 128 columns
constexpr uint32_t kColYd = 256;   // 64 columns
constexpr uint32_t kColYo = 320;   // 64 columns
constexpr uint32_t kColS = 384;    // 64 columns

constexpr uint32_t kStageTx = kStageBytes;   // bytes the TMA delivers per stage
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

// ---- small PTX wrappers ----------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// One test of the phase; while it is incomplete the warp is suspended (it
// issues nothing) until the phase completes or about 20 us pass, so waiting
// warps leave the issue slots to the warps that work.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(20000u)
        : "memory");
    return done != 0;
}

// Wait for the phase of the given parity to complete; false after about a
// second (the caller then records a timeout and stops).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_test(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_test(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs)
            return false;
    return true;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1,
                                            int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }


// Shared-memory matrix descriptor of a 128-byte-swizzled operand: start
// address, leading and stride byte offsets (16-byte units), version 1,
// layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of a kind::f16 MMA with bf16 A and B, fp32 D.
// a_mn / b_mn select the MN-major (instead of K-major) operand layout.
__host__ __device__ constexpr uint32_t bf16_idesc(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 16 consecutive fp32 columns of this warp's 32 lanes; thread i gets lane i.
// The wait is part of the same statement so no use can move above it.
__device__ __forceinline__ void tmem_load16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// 8 consecutive fp32 columns of this warp's lanes, without waiting; pair with
// tmem_wait_regs on the same registers before using them.
__device__ __forceinline__ void tmem_load8_async(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

#define MS_R8(a, j) "+r"(a[j][0]), "+r"(a[j][1]), "+r"(a[j][2]), "+r"(a[j][3]), "+r"(a[j][4]), "+r"(a[j][5]), \
                    "+r"(a[j][6]), "+r"(a[j][7])
// Wait for this thread's outstanding tensor-memory loads; the registers are
// operands so that no use of them is scheduled above the wait.
template <int G> __device__ __forceinline__ void tmem_wait_regs(uint32_t (&a)[G][8]);
template <> __device__ __forceinline__ void tmem_wait_regs<1>(uint32_t (&a)[1][8])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MS_R8(a, 0) : : "memory");
}
template <> __device__ __forceinline__ void tmem_wait_regs<2>(uint32_t (&a)[2][8])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MS_R8(a, 0), MS_R8(a, 1) : : "memory");
}
template <> __device__ __forceinline__ void tmem_wait_regs<3>(uint32_t (&a)[3][8])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MS_R8(a, 0), MS_R8(a, 1), MS_R8(a, 2) : : "memory");
}
template <> __device__ __forceinline__ void tmem_wait_regs<4>(uint32_t (&a)[4][8])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MS_R8(a, 0), MS_R8(a, 1), MS_R8(a, 2), MS_R8(a, 3) : : "memory");
}
#undef MS_R8

__device__ __forceinline__ float ex2(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// silu(z) = z sigmoid(z) = z (1 + tanh(z / 2)) / 2, one MUFU operation.
__device__ __forceinline__ float silu_fast(float z)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    const float hz = 0.5f * z;
    return fmaf(hz, t, hz);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of 16-byte chunk q of row r inside a 128-byte-swizzled atom.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t q) { return r * 128u + ((q ^ (r & 7u)) << 4); }

// A bounded wait that also gives up at once when another role of the CTA has
// already given up (abort flag in shared memory).
__device__ __forceinline__ bool role_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, uint64_t limit_ns)
{
    if (mbar_test(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_test(bar, parity)) {
        if (*abort_flag || global_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

__device__ __forceinline__ void give_up(int *status, volatile int *abort_flag)
{
    *abort_flag = 1;
    atomicExch(status, (int)MS_ERR_TIMEOUT);
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float load_bf16(const void *p, int64_t i)
{
    return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(p)[i] << 16);
}

// The running state H[p][n] of this thread (n = its row r, p = 16 hq + j) as
// bf16 into the MN-major operand tile of the Yo product (rows K = n, p
// contiguous): the thread's 16 values are two 16-byte chunks of row r.
__device__ __forceinline__ void store_state_tile(uint32_t tile, int r, int hq, const float (&H)[16])
{
#pragma unroll
    for (int q = 0; q < 2; ++q)
        st_shared_v4(tile + sw128((uint32_t)r, (uint32_t)(2 * hq + q)), pack_bf16(H[8 * q], H[8 * q + 1]),
                     pack_bf16(H[8 * q + 2], H[8 * q + 3]), pack_bf16(H[8 * q + 4], H[8 * q + 5]),
                     pack_bf16(H[8 * q + 6], H[8 * q + 7]));
}

// M' for row r (row block K, this warp's quarter hq): column groups of 8 at
// 32 j + 8 hq for j = 0..K. Groups below the diagonal block use the factored
// decay exp(s_r - s_e(j)) exp(s_e(j) - s_i) delta_i (cf); the group in the
// diagonal block takes exp(s_r - s_i) directly and masks i > r.
// Groups j = J0 .. J0 + G - 1 of build_mask_rows, loaded together.
template <int K, int J0, int G>
__device__ __forceinline__ void build_mask_groups(uint32_t tg, uint32_t m_tile, int r, int hq, float sr,
                                                  const float *dl, const float *s2, const uint16_t *cf)
{
    uint32_t g[G][8];
#pragma unroll
    for (int u = 0; u < G; ++u)
        tmem_load8_async(tg + 32u * (uint32_t)(J0 + u) + 8u * (uint32_t)hq, g[u]);
    tmem_wait_regs<G>(g);
#pragma unroll
    for (int u = 0; u < G; ++u) {
        const int j = J0 + u;
        const int i0 = 32 * j + 8 * hq;
        float m[8];
        if (j < K) {
            const float rf = ex2(sr - s2[32 * j + 31]);
            const uint4 cw = *reinterpret_cast<const uint4 *>(cf + i0);
            const float ci[8] = {bf16_lo(cw.x), bf16_hi(cw.x), bf16_lo(cw.y), bf16_hi(cw.y),
                                 bf16_lo(cw.z), bf16_hi(cw.z), bf16_lo(cw.w), bf16_hi(cw.w)};
#pragma unroll
            for (int e = 0; e < 8; ++e)
                m[e] = __uint_as_float(g[u][e]) * ci[e] * rf;
        } else {
            const float4 sa = *reinterpret_cast<const float4 *>(s2 + i0);
            const float4 sb4 = *reinterpret_cast<const float4 *>(s2 + i0 + 4);
            const float4 da = *reinterpret_cast<const float4 *>(dl + i0);
            const float4 db4 = *reinterpret_cast<const float4 *>(dl + i0 + 4);
            const float si[8] = {sa.x, sa.y, sa.z, sa.w, sb4.x, sb4.y, sb4.z, sb4.w};
            const float di[8] = {da.x, da.y, da.z, da.w, db4.x, db4.y, db4.z, db4.w};
#pragma unroll
            for (int e = 0; e < 8; ++e)
                m[e] = i0 + e <= r ? __uint_as_float(g[u][e]) * ex2(sr - si[e]) * di[e] : 0.f;
        }
        st_shared_v4(m_tile + (uint32_t)(i0 >> 6) * (kQ * 128) + sw128((uint32_t)r, (uint32_t)((i0 & 63) >> 3)),
                     pack_bf16(m[0], m[1]), pack_bf16(m[2], m[3]), pack_bf16(m[4], m[5]), pack_bf16(m[6], m[7]));
    }
}

// M' for row r (row block K, this warp's quarter hq): column groups of 8 at
// 32 j + 8 hq for j = 0..K. Groups below the diagonal block use the factored
// decay exp(s_r - s_e(j)) exp(s_e(j) - s_i) delta_i (cf); the group in the
// diagonal block takes exp(s_r - s_i) directly and masks i > r. Every warp of
// an SMSP thus gets one diagonal group and K lower groups.
template <int K>
__device__ __forceinline__ void build_mask_rows(uint32_t tg, uint32_t m_tile, int r, int hq, float sr,
                                                const float *dl, const float *s2, const uint16_t *cf)
{
    if constexpr (K < 2) {
        build_mask_groups<K, 0, K + 1>(tg, m_tile, r, hq, sr, dl, s2, cf);
    } else {
        build_mask_groups<K, 0, 2>(tg, m_tile, r, hq, sr, dl, s2, cf);
        build_mask_groups<K, 2, K - 1>(tg, m_tile, r, hq, sr, dl, s2, cf);
    }
}

// ---- schedule ----------------------------------------------------------------
// One CTA per (batch, head) walks that sequence's chunks; or, persistent, CTA g
// of G takes chunks [g T / G, (g + 1) T / G) of the list of all T chunks
// (sequence u = b * nheads + h, chunk c at u * nc + c). Such a range is the
// tail of sequence us from chunk cs, whole sequences, and the head of sequence
// ue up to chunk ce. The CTA runs the head first (its end state goes to the
// next CTA), then the whole sequences, then the tail (which starts from the
// state the previous CTA handed over): by then that state is ready whenever the
// range holds at least one sequence's worth of chunks.
struct SsdSched {
    int us, cs, ue, ce, nc, np;   // np pieces
    int K;                        // chunks of this CTA
};
struct SsdPiece {
    int u, c0, c1;   // chunks [c0, c1) of sequence u
};

__device__ __forceinline__ SsdSched ssd_sched(const ms::SsdParams &p, int nc)
{
    SsdSched s;
    s.nc = nc;
    if (p.sk_ctas == 0) {
        s.us = s.ue = (int)blockIdx.x;
        s.cs = 0;
        s.ce = nc;
        s.K = nc;
        s.np = nc > 0 ? 1 : 0;
        return s;
    }
    const int64_t T = p.batch * p.nheads * (int64_t)nc, G = p.sk_ctas, g = blockIdx.x;
    const int64_t q = T / G, rm = T % G;
    const int64_t a = g * q + (g * rm) / G, e = (g + 1) * q + ((g + 1) * rm) / G;
    s.K = (int)(e - a);
    if (s.K <= 0) {
        s.us = s.ue = s.cs = s.ce = 0;
        s.np = 0;
        s.K = 0;
        return s;
    }
    s.us = (int)(a / nc);
    s.cs = (int)(a % nc);
    s.ue = (int)((e - 1) / nc);
    s.ce = (int)((e - 1) % nc) + 1;
    s.np = s.ue - s.us + 1;
    return s;
}

__device__ __forceinline__ SsdPiece ssd_piece(const SsdSched &s, int i)
{
    if (s.us == s.ue)
        return {s.us, s.cs, s.ce};
    if (i == 0)
        return {s.ue, 0, s.ce};
    if (i < s.np - 1)
        return {s.us + i, 0, s.nc};
    return {s.us, s.cs, s.nc};
}

__device__ __forceinline__ int ld_acquire_gpu(const int *f)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(int *f, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}

// Barrier of the 512 epilogue threads (named barrier 1).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
ssd_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap b_map,
           const __grid_constant__ CUtensorMap c_map, const ms::SsdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = (int)p.seqlen;
    const int hpg = (int)(p.nheads / p.ngroups);
    SsdSched *sched = reinterpret_cast<SsdSched *>(smem + kOffSched);
    const uint32_t base = smem_addr(smem);
    if (base & 1023u) {   // the swizzled tiles need a 1024-byte aligned window
        if (threadIdx.x == 0)
            atomicExch(p.status, (int)MS_ERR_ALIGNMENT);
        return;
    }
    auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffAbort);
    const uint64_t wlim = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        mbar_init(bar(kFull0), 1);
        mbar_init(bar(kFull1), 1);
        mbar_init(bar(kEmpty0), kEpiWarps);
        mbar_init(bar(kEmpty1), kEpiWarps);
        mbar_init(bar(kGFull0), 1);
        mbar_init(bar(kGFull1), 1);
        mbar_init(bar(kPReady), kEpiWarps);
        mbar_init(bar(kSFull), 1);
        mbar_init(bar(kYFull), 1);
        mbar_init(bar(kHReady), kEpiWarps);
        mbar_init(bar(kYFree), kEpiWarps);
        mbar_init(bar(kDrain), 1);
        mbar_init(bar(kStep0), 32);
        mbar_init(bar(kStep1), 32);
        *abort_flag = 0;
        *sched = ssd_sched(p, (L + kQ - 1) / kQ);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp)
        tmem_alloc(base + kOffTmemSlot, kTmemCols);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffTmemSlot);
    const int K = sched->K;

    if (warp == kTmaWarp) {
        // ---- producer: X, B and C of chunk i into stage i % 2 (lane 0), and the chunk's step
        // data (all lanes, four tokens each) into step buffer i % 2 ----
        float *dl_all = reinterpret_cast<float *>(smem + kOffStep);
        float *s2_all = dl_all + 2 * kQ;
        uint16_t *cf_all = reinterpret_cast<uint16_t *>(s2_all + 2 * kQ);
        int issued = 0;            // chunks whose loads went out (or were withheld)
        unsigned withheld = 0u;    // bit i % 2: chunk i's loads withheld
        bool stop = false;
        int i = 0;
        const int np = sched->np;
        for (int pi = 0; pi < np && !stop; ++pi) {
            const SsdPiece pc = ssd_piece(*sched, pi);
            const int b = pc.u / (int)p.nheads, h = pc.u - b * (int)p.nheads, g = h / hpg;
            const float Ah2 = p.A[h] * kLog2e;
            const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
            const uint16_t *dtp = reinterpret_cast<const uint16_t *>(p.dt) + b * p.dt_sb + h;
            auto load_dt = [&](int c, float (&v)[4]) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int t = c * kQ + 4 * lane + k;
                    v[k] = t < L ? load_bf16(dtp, (int64_t)t * p.dt_st) : 0.f;
                }
            };
            float dtv[4];
            load_dt(pc.c0, dtv);
            for (int c = pc.c0; c < pc.c1; ++c, ++i) {
                const int st = i & 1;
                if (i >= 2 &&
                    !__all_sync(0xffffffffu, role_wait(bar(kEmpty0 + st), ((i >> 1) + 1) & 1, abort_flag, wlim))) {
                    if (lane == 0)
                        give_up(p.status, abort_flag);
                    stop = true;
                    break;
                }
                // (a test can withhold one block's loads: its full barrier then never completes)
                const bool hold = c + 1 == p.withhold_block;
                withheld = hold ? (withheld | (1u << st)) : (withheld & ~(1u << st));
                if (lane == 0 && !hold) {
                    const uint32_t sx = base + (uint32_t)st * kStageBytes, sb = sx + kXTile, sc2 = sb + kBCTile;
                    const uint32_t full = bar(kFull0 + st);
                    mbar_arrive_tx(full, kStageTx);
                    tma_load_3d(sx, &x_map, full, (int)(h * kP), c * kQ, (int)b);
                    tma_load_3d(sb, &b_map, full, (int)(g * kN), c * kQ, (int)b);
                    tma_load_3d(sb + kQ * 128, &b_map, full, (int)(g * kN + 64), c * kQ, (int)b);
                    tma_load_3d(sc2, &c_map, full, (int)(g * kN), c * kQ, (int)b);
                    tma_load_3d(sc2 + kQ * 128, &c_map, full, (int)(g * kN + 64), c * kQ, (int)b);
                }
                issued = i + 1;
                // step sizes of tokens 4 lane .. 4 lane + 3 and the running sum of delta A (log2 units)
                float d[4], v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int t = c * kQ + 4 * lane + k;
                    d[k] = 0.f;
                    if (t < L) {
                        d[k] = dtv[k] + bias;
                        if (p.softplus)
                            d[k] = ms::softplus(d[k]);
                    }
                }
                if (c + 1 < pc.c1)
                    load_dt(c + 1, dtv);
                v[0] = d[0] * Ah2;
#pragma unroll
                for (int k = 1; k < 4; ++k)
                    v[k] = fmaf(d[k], Ah2, v[k - 1]);
                float incl = v[3];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o)
                        incl += u;
                }
                const float excl = incl - v[3];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[k] += excl;
                // s at the last token of this 32-token block (lanes 8 j .. 8 j + 7 hold block j)
                const float vend = __shfl_sync(0xffffffffu, v[3], (lane & ~7) | 7);
                float cfv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    cfv[k] = ex2(vend - v[k]) * d[k];
                *reinterpret_cast<float4 *>(dl_all + st * kQ + 4 * lane) = make_float4(d[0], d[1], d[2], d[3]);
                *reinterpret_cast<float4 *>(s2_all + st * kQ + 4 * lane) = make_float4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<uint2 *>(cf_all + st * kQ + 4 * lane) =
                    make_uint2(pack_bf16(cfv[0], cfv[1]), pack_bf16(cfv[2], cfv[3]));
                mbar_arrive(bar(kStep0 + st));
            }
        }
        // the loads in flight must land before the CTA leaves
        if (lane == 0)
            for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c)
                if (!(withheld & (1u << (c & 1))))
                    mbar_wait(bar(kFull0 + (c & 1)), (c >> 1) & 1);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---- MMA issue (one thread) ----
        if (lane == 0) {
            constexpr uint32_t id_g = bf16_idesc(128, 128, false, false);   // G = C B^T
            constexpr uint32_t id_yo = bf16_idesc(128, 64, false, true);    // Yo = C H^T
            constexpr uint32_t id_s = bf16_idesc(128, 64, true, true);      // S = B^T Xt
            constexpr uint32_t id_yd = bf16_idesc(128, 64, false, true);    // Yd = M' X
            for (int c = 0; c < K; ++c) {   // c: position in the CTA's list of chunks
                const int st = c & 1;
                const uint32_t sx = base + (uint32_t)st * kStageBytes, sb = sx + kXTile, sc = sb + kBCTile;
                if (!role_wait(bar(kFull0 + st), (c >> 1) & 1, abort_flag, wlim)) {
                    give_up(p.status, abort_flag);
                    break;
                }
                tc_after_sync();
                const uint32_t tg = tmem + kColG + 128u * (uint32_t)(c & 1);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (uint32_t)(k >> 2) * (kQ * 128) + (uint32_t)(k & 3) * 32u;
                    mma_bf16(tg, sw128_desc(sc + off, 16, 1024), sw128_desc(sb + off, 16, 1024), id_g, k > 0);
                }
                mma_commit(bar(kGFull0 + (c & 1)));
                // Yo needs the state of the previous chunk and the Y columns free
                if (!role_wait(bar(kHReady), c & 1, abort_flag, wlim) ||
                    (c > 0 && !role_wait(bar(kYFree), (c - 1) & 1, abort_flag, wlim))) {
                    give_up(p.status, abort_flag);
                    break;
                }
                tc_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t offc = (uint32_t)(k >> 2) * (kQ * 128) + (uint32_t)(k & 3) * 32u;
                    mma_bf16(tmem + kColYo, sw128_desc(sc + offc, 16, 1024),
                             sw128_desc(base + kOffH + (uint32_t)k * 2048u, kXTile, 1024), id_yo, k > 0);
                }
                // S and Yd need M' and Xt of this chunk
                if (!role_wait(bar(kPReady), c & 1, abort_flag, wlim)) {
                    give_up(p.status, abort_flag);
                    break;
                }
                tc_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16(tmem + kColS, sw128_desc(sb + (uint32_t)k * 2048u, kQ * 128, 1024),
                             sw128_desc(base + kOffXt + (uint32_t)k * 2048u, kXTile, 1024), id_s, k > 0);
                mma_commit(bar(kSFull));
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t offm = (uint32_t)(k >> 2) * (kQ * 128) + (uint32_t)(k & 3) * 32u;
                    mma_bf16(tmem + kColYd, sw128_desc(base + kOffM + offm, 16, 1024),
                             sw128_desc(sx + (uint32_t)k * 2048u, kXTile, 1024), id_yd, k > 0);
                }
                mma_commit(bar(kYFull));
            }
            // every MMA issued must finish before the tensor memory is freed
            mma_commit(bar(kDrain));
            mbar_wait(bar(kDrain), 0);
        }
        __syncwarp();
    } else {
        // ---- epilogue: warps 0-15; thread = row r of the chunk, column quarter hq ----
        // Software-pipelined over chunks: while the tensor core computes S and Yd of
        // chunk c + 1, the warps gate and store y of chunk c.
        const int sub = warp & 3, hq = warp >> 2;
        const int r = sub * 32 + lane;
        const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
        const float *dl_all = reinterpret_cast<const float *>(smem + kOffStep);
        const float *s2_all = dl_all + 2 * kQ;
        const uint16_t *cf_all = reinterpret_cast<const uint16_t *>(s2_all + 2 * kQ);
        bool ok = true;
        auto epi_wait = [&](uint32_t barrier, uint32_t parity) {
            if (ok)
                ok = __all_sync(0xffffffffu, role_wait(barrier, parity, abort_flag, wlim));
            if (!ok && lane == 0)
                give_up(p.status, abort_flag);
            return ok;
        };

        // this thread keeps H[p][n] for n = r and p = 16 hq + j
        float H[16];
        // The state a piece starts from: the initial state (or zero) at the start of a
        // sequence, else the one the previous CTA handed over (bounded wait for its flag).
        auto load_state = [&](const SsdPiece &pc) {
            if (pc.c0 > 0) {
                const int src = (int)blockIdx.x - 1;
                bool got = true;
                if (lane == 0 && ok) {
                    got = ld_acquire_gpu(p.sk_flag + src) != 0;
                    if (!got) {
                        const uint64_t t0 = global_ns();
                        while (!(got = ld_acquire_gpu(p.sk_flag + src) != 0)) {
                            if (*abort_flag || global_ns() - t0 > wlim)
                                break;
                            __nanosleep(256);
                        }
                    }
                }
                if (!__all_sync(0xffffffffu, got) && ok) {
                    ok = false;
                    if (lane == 0)
                        give_up(p.status, abort_flag);
                }
                const float *src_h = p.sk_carry + ((int64_t)src * kP + 16 * hq) * kN + r;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    H[j] = ok ? __ldcg(src_h + (int64_t)j * kN) : 0.f;
            } else {
                const int64_t hoff = ((int64_t)pc.u * kP + 16 * hq) * kN + r;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    H[j] = p.h0 ? p.h0[hoff + (int64_t)j * kN] : 0.f;
            }
        };
        // The state a piece ends with: the final state at the end of a sequence, else
        // the hand-over to the next CTA (stored, fenced, then the flag raised once all
        // 512 threads have stored; raised even after a timeout so no CTA waits on it).
        auto save_state = [&](const SsdPiece &pc, int nc) {
            if (pc.c1 == nc) {
                if (ok && p.hT) {
                    const int64_t hoff = ((int64_t)pc.u * kP + 16 * hq) * kN + r;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        p.hT[hoff + (int64_t)j * kN] = H[j];
                }
            } else {
                float *dst = p.sk_carry + ((int64_t)blockIdx.x * kP + 16 * hq) * kN + r;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    __stcg(dst + (int64_t)j * kN, H[j]);
                __threadfence();
                epi_bar();
                if (threadIdx.x == 0)
                    st_release_gpu(p.sk_flag + blockIdx.x, 1);
            }
        };

        // position: piece pi, chunk c of its sequence, `left` chunks to the piece's end
        int pi = 0, c = 0, left = 0;
        if (sched->np > 0) {
            const SsdPiece f = ssd_piece(*sched, 0);
            c = f.c0;
            left = f.c1 - f.c0;
            load_state(f);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                H[j] = 0.f;
        }
        // rows of block sub: M' columns in blocks above the diagonal are zero (causal mask)
        // and are written once, this warp taking the groups 32 j + 8 hq
        for (int j = sub + 1; j < 4; ++j) {
            const int i0 = 32 * j + 8 * hq;
            st_shared_v4(base + kOffM + (uint32_t)(i0 >> 6) * (kQ * 128) +
                             sw128((uint32_t)r, (uint32_t)((i0 & 63) >> 3)),
                         0u, 0u, 0u, 0u);
        }
        store_state_tile(base + kOffH, r, hq, H);
        async_proxy_fence();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar(kHReady));

        // Build the operands M' and Xt of chunk k from its step data; returns s_r and s_end.
        auto prepare = [&](int k, float &sr, float &se) {
            const int stk = k & 1;
            const float *dl = dl_all + stk * kQ, *s2 = s2_all + stk * kQ;
            const uint16_t *cf = cf_all + stk * kQ;
            epi_wait(bar(kStep0 + stk), (k >> 1) & 1);
            epi_wait(bar(kFull0 + stk), (k >> 1) & 1);
            epi_wait(bar(kGFull0 + (k & 1)), (k >> 1) & 1);
            sr = s2[r];
            se = s2[kQ - 1];
            if (ok) {
                tc_after_sync();
                const uint32_t tg = tmem + lane_base + kColG + 128u * (uint32_t)(k & 1);
                switch (sub) {
                case 0: build_mask_rows<0>(tg, base + kOffM, r, hq, sr, dl, s2, cf); break;
                case 1: build_mask_rows<1>(tg, base + kOffM, r, hq, sr, dl, s2, cf); break;
                case 2: build_mask_rows<2>(tg, base + kOffM, r, hq, sr, dl, s2, cf); break;
                default: build_mask_rows<3>(tg, base + kOffM, r, hq, sr, dl, s2, cf); break;
                }
                // Xt: the 1024 16-byte pieces (token i, 8 p each) go mostly to the
                // sub-partitions with the fewest mask groups: 4, 3, 1 and 0
                // pieces per thread on sub-partitions 0..3.
                const uint32_t sx = base + (uint32_t)stk * kStageBytes;
                const int tsub = hq * 32 + lane;
                const int npc = sub == 0 ? 4 : sub == 1 ? 3 : sub == 2 ? 1 : 0;
                const int pc0 = sub == 0 ? 0 : sub == 1 ? 512 : 896;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (k < npc) {
                        const int pc = pc0 + 128 * k + tsub;
                        const int i = pc >> 3;
                        const float wr = ex2(se - s2[i]) * dl[i];
                        const uint32_t off = sw128((uint32_t)i, (uint32_t)(pc & 7));
                        const uint4 v = ld_shared_v4(sx + off);
                        st_shared_v4(base + kOffXt + off, pack_bf16(bf16_lo(v.x) * wr, bf16_hi(v.x) * wr),
                                     pack_bf16(bf16_lo(v.y) * wr, bf16_hi(v.y) * wr),
                                     pack_bf16(bf16_lo(v.z) * wr, bf16_hi(v.z) * wr),
                                     pack_bf16(bf16_lo(v.w) * wr, bf16_hi(v.w) * wr));
                    }
                }
            }
            async_proxy_fence();
            tc_before_sync();
            __syncwarp();
            if (lane == 0 && ok)
                mbar_arrive(bar(kPReady));
        };

        // per piece: this thread's columns of y and z at token 0 of the sequence, and D
        const uint16_t *zcol = nullptr;
        uint16_t *ycol = nullptr;
        float Dh = 0.f;
        auto enter = [&](int u) {
            const int b = u / (int)p.nheads, h = u - b * (int)p.nheads;
            Dh = p.D ? p.D[h] : 0.f;
            ycol = reinterpret_cast<uint16_t *>(p.y) + (int64_t)b * p.y_sb + (int64_t)h * kP + 16 * hq;
            if (p.z)
                zcol = reinterpret_cast<const uint16_t *>(p.z) + (int64_t)b * p.z_sb + (int64_t)h * kP + 16 * hq;
        };
        float sr_c = 0.f, se_c = 0.f;   // s_r and s_end of the chunk being finished
        if (K > 0) {
            enter(ssd_piece(*sched, 0).u);
            prepare(0, sr_c, se_c);
        }
        for (int i = 0; i < K; ++i) {
            const int st = i & 1, t0 = c * kQ;
            const bool live = t0 + r < L;
            const uint32_t sx = base + (uint32_t)st * kStageBytes;
            // the gate of this thread's 16 outputs
            uint4 zq[2] = {};
            if (p.z && live) {
                const uint4 *zp = reinterpret_cast<const uint4 *>(zcol + (int64_t)(t0 + r) * p.z_st);
                zq[0] = __ldg(zp);
                zq[1] = __ldg(zp + 1);
            }
            const float Dc = Dh;
            const uint16_t *ycol_c = ycol;   // the piece's, before a change of piece below

            // (2) state passing: H = exp(s_end) H + S^T; at the end of a piece the state
            // leaves (final state or hand-over) and the next piece's initial state enters
            epi_wait(bar(kSFull), i & 1);
            if (ok) {
                tc_after_sync();
                float sv[16];
                tmem_load16(tmem + lane_base + kColS + 16u * hq, sv);
                const float ac = ex2(se_c);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    H[j] = fmaf(ac, H[j], sv[j]);
                // (stored at once inside a piece: the Yo product of the next chunk waits for it)
                if (left > 1)
                    store_state_tile(base + kOffH, r, hq, H);
            }
            ++c;
            if (--left == 0) {
                const SsdSched s2 = *sched;
                save_state(ssd_piece(s2, pi), s2.nc);
                if (pi + 1 < s2.np) {
                    const SsdPiece nx = ssd_piece(s2, ++pi);
                    load_state(nx);
                    enter(nx.u);
                    c = nx.c0;
                    left = nx.c1 - nx.c0;
                }
                if (ok)
                    store_state_tile(base + kOffH, r, hq, H);
            }
            async_proxy_fence();
            tc_before_sync();
            __syncwarp();
            if (lane == 0 && ok)
                mbar_arrive(bar(kHReady));

            // (3a) y = Yd + exp(s_r) Yo + D x into registers; the Y columns and the stage are then free
            float yv[16];
            epi_wait(bar(kYFull), i & 1);
            if (ok) {
                tc_after_sync();
                float yd[16];
                tmem_load16(tmem + lane_base + kColYd + 16u * hq, yd);
                tmem_load16(tmem + lane_base + kColYo + 16u * hq, yv);
                tc_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(kYFree));
                const float er = ex2(sr_c);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint4 xv = ld_shared_v4(sx + sw128((uint32_t)r, (uint32_t)(2 * hq + q)));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * q + 2 * e;
                        yv[j] = fmaf(er, yv[j], fmaf(Dc, bf16_lo(xw[e]), yd[j]));
                        yv[j + 1] = fmaf(er, yv[j + 1], fmaf(Dc, bf16_hi(xw[e]), yd[j + 1]));
                    }
                }
            }
            __syncwarp();
            if (lane == 0 && ok)
                mbar_arrive(bar(kEmpty0 + st));

            // (1) operands of the next chunk, so that its products overlap the rest of this one
            float sr_n = 0.f, se_n = 0.f;
            if (i + 1 < K)
                prepare(i + 1, sr_n, se_n);

            // (3b) gate and store y of this chunk
            if (ok && live) {
                uint4 out[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t zw[4] = {zq[q].x, zq[q].y, zq[q].z, zq[q].w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * q + 2 * e;
                        float o0 = yv[j], o1 = yv[j + 1];
                        if (p.z) {
                            o0 *= silu_fast(bf16_lo(zw[e]));
                            o1 *= silu_fast(bf16_hi(zw[e]));
                        }
                        ow[e] = pack_bf16(o0, o1);
                    }
                    out[q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
                uint4 *yp = reinterpret_cast<uint4 *>(const_cast<uint16_t *>(ycol_c) + (int64_t)(t0 + r) * p.y_st);
                yp[0] = out[0];
                yp[1] = out[1];
            }
            sr_c = sr_n;
            se_c = se_n;
        }
    }
    tc_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_after_sync();
        tmem_free(tmem, kTmemCols);
    }
}

}  // namespace

namespace ms {
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime.
EncodeTiled encoder()
{
    static const EncodeTiled fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiled>(nullptr);
        return reinterpret_cast<EncodeTiled>(ptr);
    }();
    return fn;
}

// A bf16 map over (inner, tokens, batch) delivering 64 x 128 x 1 boxes into
// 128-byte-swizzled shared memory; rows past the last token read as zero.
// L2 fills: 256 bytes for B and C (a chunk reads both 128-byte halves of each
// row), 128 bytes for x (one head's 128 bytes of a token; the other half of a
// 256-byte fill is another head's, which the persistent schedule reaches at
// another time).
bool encode_map(CUtensorMap *m, const void *ptr, int64_t inner, int64_t tokens, int64_t batch, int64_t token_stride,
                int64_t batch_stride, CUtensorMapL2promotion promo)
{
    const EncodeTiled fn = encoder();
    if (!fn)
        return false;
    if (batch == 1)
        batch_stride = token_stride * tokens;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)tokens, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)token_stride * 2u, (cuuint64_t)batch_stride * 2u};
    const cuuint32_t box[3] = {64u, (cuuint32_t)kQ, 1u};
    const cuuint32_t elem[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// The persistent schedule pays when the (batch, head) pairs leave the last wave
// of one-CTA-per-pair partly empty: it then takes ceil(T / SMs) chunk times plus
// about one for the hand-over, against waves x chunks. Each CTA must hold at
// least one sequence's worth of chunks so that no hand-over waits.
int ssd_persistent_ctas(int64_t batch, int64_t nheads, int64_t seqlen, int num_sms)
{
    const int64_t units = batch * nheads, nc = (seqlen + kQ - 1) / kQ;
    if (num_sms <= 0 || nc < 2 || units <= num_sms || units % num_sms == 0)
        return 0;
    if (units * nc / num_sms >= (int64_t(1) << 30))   // a CTA's count of chunks is kept in an int
        return 0;
    const int64_t waves = (units + num_sms - 1) / num_sms;
    const int64_t per_cta = (units * nc + num_sms - 1) / num_sms;
    return per_cta + 2 < waves * nc ? num_sms : 0;
}

size_t ssd_flag_offset() { return 256; }

size_t ssd_carry_offset(int ctas) { return 256 + (((size_t)ctas * sizeof(int) + 255) / 256) * 256; }

size_t ssd_persistent_ws_bytes(int ctas) { return ssd_carry_offset(ctas) + (size_t)ctas * kP * kN * sizeof(float); }

cudaError_t launch_ssd(const SsdParams &p, cudaStream_t stream)
{
    CUtensorMap xm, bm, cm;
    if (!encode_map(&xm, p.x, p.nheads * kP, p.seqlen, p.batch, p.x_st, p.x_sb, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
        !encode_map(&bm, p.B, p.ngroups * kN, p.seqlen, p.batch, p.B_st, p.B_sb, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !encode_map(&cm, p.C, p.ngroups * kN, p.seqlen, p.batch, p.C_st, p.C_sb, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
        return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(ssd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess)
        return e;
    if (p.sk_ctas == 0) {
        e = cudaMemsetAsync(p.status, 0, sizeof(int), stream);
        if (e != cudaSuccess)
            return e;
        ssd_kernel<<<(unsigned)(p.batch * p.nheads), kThreads, kSmemBytes, stream>>>(xm, bm, cm, p);
        return cudaGetLastError();
    }
    // status word and flags, then a cooperative launch: every CTA is resident, so a
    // CTA waiting for its predecessor's hand-over never waits for one that has not started
    if (!p.sk_flag || !p.sk_carry)
        return cudaErrorInvalidValue;
    e = cudaMemsetAsync(p.status, 0, ssd_carry_offset(p.sk_ctas), stream);
    if (e != cudaSuccess)
        return e;
    void *args[] = {&xm, &bm, &cm, const_cast<SsdParams *>(&p)};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)p.sk_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeCooperative;
    attr.val.cooperative = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void *>(ssd_kernel), args);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace ms
