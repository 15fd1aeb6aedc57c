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
// Four consecutive threads share a row (b, d); thread q owns state entries
// [4q, 4q+4), so every state access is a fully coalesced 16-byte load and
// store and its A, B and C entries arrive as one vector load each. (A thread
// may own several rows, kRowGroups apart, loading all of them before
// computing; one row per thread at full occupancy measured faster.) The
// partial readouts are summed with two butterfly shuffles.
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kRowGroups = 64;                // row groups per block (4 threads each)
constexpr int kBlock = kRowGroups * 4;

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

// VEC: dstate == 16 with state rows, A rows and B/C rows aligned for vector
// access. A thread owns state entries [4q, 4q+4) of kRowsPerThread rows and
// issues all of their loads before any arithmetic, so that enough bytes are in
// flight to cover HBM latency.
template <typename T, bool VEC, int kRowsPerThread, bool CONV>
__global__ void __launch_bounds__(kBlock) state_update_kernel(const UpdateParams p) {
    constexpr int kRowsPerBlock = kRowGroups * kRowsPerThread;
    const int tid = threadIdx.x;
    const int q = tid & 3;
    const int64_t b = blockIdx.y;
    const int64_t d0 = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + (tid >> 2);
    const int dstate = static_cast<int>(p.dstate);

    int64_t dd[kRowsPerThread];
    bool ok[kRowsPerThread];
    float x[kRowsPerThread], dt[kRowsPerThread];
#pragma unroll
    for (int k = 0; k < kRowsPerThread; ++k) {
        const int64_t d = d0 + k * kRowGroups;
        ok[k] = d < p.dim;
        dd[k] = ok[k] ? d : p.dim - 1;
        x[k] = ldg1<T>(p.x, b * p.x_sb + dd[k]);
        dt[k] = ldg1<T>(p.delta, b * p.dl_sb + dd[k]);
        if constexpr (CONV) {
            // the row's first lane steps the convolution state; u reaches the
            // other three lanes of the row by shuffle
            float u = 0.f;
            if (q == 0) u = conv_step<T>(p, b, dd[k], x[k], ok[k]);
            x[k] = __shfl_sync(0xffffffffu, u, (tid & 31) & ~3);
        }
    }
    if constexpr (VEC) {
        float4 h[kRowsPerThread], a[kRowsPerThread];
#pragma unroll
        for (int k = 0; k < kRowsPerThread; ++k) {
            h[k] = reinterpret_cast<const float4 *>(p.state + b * p.s_sb + dd[k] * p.s_sd)[q];
            a[k] = __ldg(reinterpret_cast<const float4 *>(p.A + dd[k] * 16) + q);
        }
        const float4 Bv = ldg4<T>(static_cast<const T *>(p.B) + b * p.B_sb + 4 * q);
        const float4 Cv = ldg4<T>(static_cast<const T *>(p.C) + b * p.C_sb + 4 * q);
#pragma unroll
        for (int k = 0; k < kRowsPerThread; ++k) {
            float v = dt[k];
            if (p.delta_bias) v += __ldg(p.delta_bias + dd[k]);
            if (p.softplus) v = softplus(v);
            const float dtx = v * x[k];
            float4 o;
            o.x = fmaf(ex2_approx(v * (a[k].x * kLog2e)), h[k].x, dtx * Bv.x);
            o.y = fmaf(ex2_approx(v * (a[k].y * kLog2e)), h[k].y, dtx * Bv.y);
            o.z = fmaf(ex2_approx(v * (a[k].z * kLog2e)), h[k].z, dtx * Bv.z);
            o.w = fmaf(ex2_approx(v * (a[k].w * kLog2e)), h[k].w, dtx * Bv.w);
            float acc = fmaf(Cv.x, o.x, fmaf(Cv.y, o.y, fmaf(Cv.z, o.z, Cv.w * o.w)));
            if (ok[k]) reinterpret_cast<float4 *>(p.state + b * p.s_sb + dd[k] * p.s_sd)[q] = o;
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (ok[k] && q == 0) {
                float yv = acc + (p.D ? __ldg(p.D + dd[k]) * x[k] : 0.f);
                if (p.z) yv *= silu(ldg1<T>(p.z, b * p.z_sb + dd[k]));
                static_cast<T *>(p.y)[b * p.y_sb + dd[k]] = from_f32<T>(yv);
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < kRowsPerThread; ++k) {
            float v = dt[k];
            if (p.delta_bias) v += __ldg(p.delta_bias + dd[k]);
            if (p.softplus) v = softplus(v);
            const float dtx = v * x[k];
            float *st = p.state + b * p.s_sb + dd[k] * p.s_sd;
            float acc = 0.f;
            for (int n = q; n < dstate; n += 4) {
                const float an = ex2_approx(v * (__ldg(p.A + dd[k] * dstate + n) * kLog2e));
                float hn = st[n];
                hn = fmaf(an, hn, dtx * ldg1<T>(p.B, b * p.B_sb + n));
                acc = fmaf(ldg1<T>(p.C, b * p.C_sb + n), hn, acc);
                if (ok[k]) st[n] = hn;
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (ok[k] && q == 0) {
                float yv = acc + (p.D ? __ldg(p.D + dd[k]) * x[k] : 0.f);
                if (p.z) yv *= silu(ldg1<T>(p.z, b * p.z_sb + dd[k]));
                static_cast<T *>(p.y)[b * p.y_sb + dd[k]] = from_f32<T>(yv);
            }
        }
    }
}

template <typename T>
cudaError_t launch_t(const UpdateParams &p, cudaStream_t stream) {
    const int eb = sizeof(T);
    auto al = [](const void *ptr, int bytes) { return (reinterpret_cast<uintptr_t>(ptr) % bytes) == 0; };
    const bool vec = p.dstate == 16 && al(p.state, 16) && (p.s_sb % 4) == 0 && (p.s_sd % 4) == 0 &&
                     al(p.A, 16) && al(p.B, 4 * eb) && al(p.C, 4 * eb) && (p.B_sb % 4) == 0 &&
                     (p.C_sb % 4) == 0;
    constexpr int kRows = 1;   // rows per thread (occupancy beats per-thread batching here)
    const dim3 grid(static_cast<unsigned>((p.dim + kRowGroups * kRows - 1) / (kRowGroups * kRows)),
                    static_cast<unsigned>(p.batch));
    const bool conv = p.conv_w != nullptr;
    if (vec)
        conv ? state_update_kernel<T, true, kRows, true><<<grid, kBlock, 0, stream>>>(p)
             : state_update_kernel<T, true, kRows, false><<<grid, kBlock, 0, stream>>>(p);
    else
        conv ? state_update_kernel<T, false, kRows, true><<<grid, kBlock, 0, stream>>>(p)
             : state_update_kernel<T, false, kRows, false><<<grid, kBlock, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const UpdateParams &p, int in_dtype, cudaStream_t stream) {
    return in_dtype == 0 ? launch_t<float>(p, stream) : launch_t<__nv_bfloat16>(p, stream);
}

}  // namespace ms
