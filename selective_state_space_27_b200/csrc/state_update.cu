// Single-token selective state update (decode) for sm_100a, optionally with
// the causal depthwise convolution prologue in front ("Notas sobre Mamba",
// section "O bloco Mamba": short convolution + SiLU before the SSM).
//
// The recurrence for one step ("Mamba-2 e State Space Duality (SSD)", section
// "Como o Mamba-1 alcançou complexidade linear", the decode step; "Notas sobre
// Mamba", section "O mecanismo de seleção (S6)"):
//     delta = softplus(delta_raw + delta_bias[d])
//     h[n]  = exp(delta A[d,n]) h[n] + delta B[n] x        (in place)
//     y     = (sum_n C[n] h[n] + D[d] x) * silu(z)
//
// Decode reads and writes the whole float32 state once per token: the step is
// bound by HBM bandwidth (~168 MB of state traffic per step for 256 x 5120 x
// 16), so the kernel is built to keep many bytes in flight with few
// instructions per byte. The grid is (dim blocks, batch): no index division.
// With 16 states, two consecutive threads share a row (b, d): thread q owns
// the float4 pieces q and q + 2 of the row's state, so each of its two
// state loads (and stores) covers whole 32-byte sectors across the warp, and
// the per-row work (softplus of the step, skip, gate) is done twice per row
// instead of four times. A thread takes the same row of two batch entries,
// loading A once. Measured on B200 for 256 x 5120 x 16, each step on a state
// that is not in L2 (four layers' states cycled): 31.5 us per step, against
// 34.9 us with one batch entry per thread and 30.8 us for a plain in-place
// float4 copy-update of the same state. The two partial readouts are summed
// with one shuffle. Other state sizes take a scalar path with four threads per
// row.
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kBlock = 256;
constexpr int kRowGroups = kBlock / 4;         // rows per block on the scalar path (4 threads each)
constexpr int kVecRows = kBlock / 2;           // rows per block on the vector path (2 threads each)
constexpr int kVecBatch = 2;                   // batch entries per thread on the vector path

template <typename T>
__device__ __forceinline__ float ldg1(const void *base, int64_t i) {
    return to_f32<T>(__ldg(static_cast<const T *>(base) + i));
}

// Four consecutive elements starting at `p` (aligned to 4 elements).
template <typename T>
__device__ __forceinline__ float4 ldg4(const T *p) {
    if constexpr (std::is_same<T, float>::value) {
        return __ldg(reinterpret_cast<const float4 *>(p));
    } else {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
    }
}

// Convolution prologue of one decode step for row (b, d): the state
// (conv_width inputs, oldest first) drops its oldest entry and takes x; the
// return value is act(bias + sum_k w[k] window[k]). Called by one lane per row.
template <typename T>
__device__ __forceinline__ float conv_step(const UpdateParams &p, int64_t b, int64_t d, float x, bool store) {
    T *cs = static_cast<T *>(p.conv_state) + b * p.cs_sb + d * p.cs_sd;
    const int K = p.conv_width;
    const float *w = p.conv_w + d * K;
    float acc = p.conv_b ? __ldg(p.conv_b + d) : 0.f;
    float prev[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) prev[j] = (j + 1 < K) ? to_f32<T>(cs[j + 1]) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < K) {
            const float v = (j + 1 < K) ? prev[j] : x;
            acc = fmaf(__ldg(w + j), v, acc);
            if (store) cs[j] = from_f32<T>(v);
        }
    }
    return p.conv_silu ? silu(acc) : acc;
}

// dstate == 16, state rows, A rows and B/C rows aligned for vector access:
// two threads per row, thread q owning the float4 pieces q and q + 2 of the
// rows (b, d) of kVecBatch consecutive batch entries. The thread loads its
// pieces of A once for all of them and issues every entry's state loads
// before any arithmetic, so 64 bytes of state per thread are in flight. The
// state is read and written with evict-first hints: a decode step touches
// each row once, and the next touch (the next token) comes after the other
// layers' states have passed through L2.
template <typename T, bool CONV>
__global__ void __launch_bounds__(kBlock) state_update_vec_kernel(const UpdateParams p) {
    const int tid = threadIdx.x;
    const int q = tid & 1;
    const int64_t b0 = static_cast<int64_t>(blockIdx.y) * kVecBatch;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * kVecRows + (tid >> 1);
    const bool dok = d < p.dim;
    const int64_t dc = dok ? d : p.dim - 1;
    const float4 *ar = reinterpret_cast<const float4 *>(p.A + dc * 16);
    float4 h[kVecBatch][2];
    bool ok[kVecBatch];
    int64_t bc[kVecBatch];
#pragma unroll
    for (int i = 0; i < kVecBatch; ++i) {
        ok[i] = dok && b0 + i < p.batch;
        bc[i] = b0 + i < p.batch ? b0 + i : p.batch - 1;
        const float4 *st = reinterpret_cast<const float4 *>(p.state + bc[i] * p.s_sb + dc * p.s_sd);
        h[i][0] = __ldcs(st + q);
        h[i][1] = __ldcs(st + q + 2);
    }
    const float4 a0 = __ldg(ar + q), a1 = __ldg(ar + q + 2);
    const float bias = p.delta_bias ? __ldg(p.delta_bias + dc) : 0.f;
    const float Dd = p.D ? __ldg(p.D + dc) : 0.f;
    float xs[kVecBatch], dts[kVecBatch];
#pragma unroll
    for (int i = 0; i < kVecBatch; ++i) {
        xs[i] = ldg1<T>(p.x, bc[i] * p.x_sb + dc);
        dts[i] = ldg1<T>(p.delta, bc[i] * p.dl_sb + dc);
    }
#pragma unroll
    for (int i = 0; i < kVecBatch; ++i) {
        const int64_t b = bc[i];
        float x = xs[i];
        const float4 B0 = ldg4<T>(static_cast<const T *>(p.B) + b * p.B_sb + 4 * q);
        const float4 B1 = ldg4<T>(static_cast<const T *>(p.B) + b * p.B_sb + 4 * q + 8);
        const float4 C0 = ldg4<T>(static_cast<const T *>(p.C) + b * p.C_sb + 4 * q);
        const float4 C1 = ldg4<T>(static_cast<const T *>(p.C) + b * p.C_sb + 4 * q + 8);
        if constexpr (CONV) {
            // the row's first lane steps the convolution state; u reaches the
            // other lane of the row by shuffle
            float u = 0.f;
            if (q == 0) u = conv_step<T>(p, b, dc, x, ok[i]);
            x = __shfl_sync(0xffffffffu, u, (tid & 31) & ~1);
        }
        float v = dts[i] + bias;
        if (p.softplus) v = softplus(v);
        const float v2 = v * kLog2e, dtx = v * x;
        const float4 h0 = h[i][0], h1 = h[i][1];
        float4 o0, o1;
        o0.x = fmaf(ex2_approx(v2 * a0.x), h0.x, dtx * B0.x);
        o0.y = fmaf(ex2_approx(v2 * a0.y), h0.y, dtx * B0.y);
        o0.z = fmaf(ex2_approx(v2 * a0.z), h0.z, dtx * B0.z);
        o0.w = fmaf(ex2_approx(v2 * a0.w), h0.w, dtx * B0.w);
        o1.x = fmaf(ex2_approx(v2 * a1.x), h1.x, dtx * B1.x);
        o1.y = fmaf(ex2_approx(v2 * a1.y), h1.y, dtx * B1.y);
        o1.z = fmaf(ex2_approx(v2 * a1.z), h1.z, dtx * B1.z);
        o1.w = fmaf(ex2_approx(v2 * a1.w), h1.w, dtx * B1.w);
        if (ok[i]) {
            float4 *st = reinterpret_cast<float4 *>(p.state + b * p.s_sb + dc * p.s_sd);
            __stcs(st + q, o0);
            __stcs(st + q + 2, o1);
        }
        float acc = fmaf(C0.x, o0.x, fmaf(C0.y, o0.y, fmaf(C0.z, o0.z, C0.w * o0.w)));
        acc = fmaf(C1.x, o1.x, fmaf(C1.y, o1.y, fmaf(C1.z, o1.z, fmaf(C1.w, o1.w, acc))));
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        if (ok[i] && q == 0) {
            float yv = acc + Dd * x;
            if (p.z) yv *= silu(ldg1<T>(p.z, b * p.z_sb + dc));
            static_cast<T *>(p.y)[b * p.y_sb + dc] = from_f32<T>(yv);
        }
    }
}

// Any dstate <= 16 or unaligned rows: four threads per row, thread q taking
// the states n = q, q + 4, ... with scalar accesses.
template <typename T, bool CONV>
__global__ void __launch_bounds__(kBlock) state_update_kernel(const UpdateParams p) {
    const int tid = threadIdx.x;
    const int q = tid & 3;
    const int64_t b = blockIdx.y;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * kRowGroups + (tid >> 2);
    const int dstate = static_cast<int>(p.dstate);
    const bool ok = d < p.dim;
    const int64_t dc = ok ? d : p.dim - 1;
    float x = ldg1<T>(p.x, b * p.x_sb + dc);
    const float dt = ldg1<T>(p.delta, b * p.dl_sb + dc);
    if constexpr (CONV) {
        float u = 0.f;
        if (q == 0) u = conv_step<T>(p, b, dc, x, ok);
        x = __shfl_sync(0xffffffffu, u, (tid & 31) & ~3);
    }
    float v = dt;
    if (p.delta_bias) v += __ldg(p.delta_bias + dc);
    if (p.softplus) v = softplus(v);
    const float dtx = v * x;
    float *st = p.state + b * p.s_sb + dc * p.s_sd;
    float acc = 0.f;
    for (int n = q; n < dstate; n += 4) {
        const float an = ex2_approx(v * (__ldg(p.A + dc * dstate + n) * kLog2e));
        float hn = st[n];
        hn = fmaf(an, hn, dtx * ldg1<T>(p.B, b * p.B_sb + n));
        acc = fmaf(ldg1<T>(p.C, b * p.C_sb + n), hn, acc);
        if (ok) st[n] = hn;
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (ok && q == 0) {
        float yv = acc + (p.D ? __ldg(p.D + dc) * x : 0.f);
        if (p.z) yv *= silu(ldg1<T>(p.z, b * p.z_sb + dc));
        static_cast<T *>(p.y)[b * p.y_sb + dc] = from_f32<T>(yv);
    }
}

template <typename T>
cudaError_t launch_t(const UpdateParams &p, cudaStream_t stream) {
    const int eb = sizeof(T);
    auto al = [](const void *ptr, int bytes) { return (reinterpret_cast<uintptr_t>(ptr) % bytes) == 0; };
    const bool vec = p.dstate == 16 && al(p.state, 16) && (p.s_sb % 4) == 0 && (p.s_sd % 4) == 0 &&
                     al(p.A, 16) && al(p.B, 4 * eb) && al(p.C, 4 * eb) && (p.B_sb % 4) == 0 &&
                     (p.C_sb % 4) == 0;
    const bool conv = p.conv_w != nullptr;
    if (vec) {
        const dim3 grid(static_cast<unsigned>((p.dim + kVecRows - 1) / kVecRows),
                        static_cast<unsigned>((p.batch + kVecBatch - 1) / kVecBatch));
        conv ? state_update_vec_kernel<T, true><<<grid, kBlock, 0, stream>>>(p)
             : state_update_vec_kernel<T, false><<<grid, kBlock, 0, stream>>>(p);
    } else {
        const dim3 grid(static_cast<unsigned>((p.dim + kRowGroups - 1) / kRowGroups), static_cast<unsigned>(p.batch));
        conv ? state_update_kernel<T, true><<<grid, kBlock, 0, stream>>>(p)
             : state_update_kernel<T, false><<<grid, kBlock, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const UpdateParams &p, int in_dtype, cudaStream_t stream) {
    return in_dtype == 0 ? launch_t<float>(p, stream) : launch_t<__nv_bfloat16>(p, stream);
}

}  // namespace ms
