// Single-token selective state update (decode) for sm_100a.
//
// The recurrence for one step ("Mamba-2 e State Space Duality (SSD)", section
// "Como o Mamba-1 alcançou complexidade linear", the decode step; "Notas sobre
// Mamba", section "O mecanismo de seleção (S6)"):
//     delta = softplus(delta_raw + delta_bias[d])
//     h[n]  = exp(delta A[d,n]) h[n] + delta B[n] x        (in place)
//     y     = (sum_n C[n] h[n] + D[d] x) * silu(z)
//
// Decode reads and writes the whole float32 state once per token, so the step
// is bound by memory bandwidth. Four consecutive threads own one row (b, d);
// thread q owns state entries [4q, 4q+4), which makes every state access a
// fully coalesced 16-byte load and store. The partial readouts are summed with
// two butterfly shuffles.
#include <type_traits>

#include "device_math.cuh"
#include "launch.h"

namespace ms {
namespace {

constexpr int kThreadsPerRow = 4;
constexpr int kBlock = 256;

template <typename T>
__device__ __forceinline__ float ld(const void *base, int64_t i) {
    return to_f32<T>(static_cast<const T *>(base)[i]);
}

template <typename T, bool VEC16>
__global__ void __launch_bounds__(kBlock) state_update_kernel(const UpdateParams p) {
    const int64_t gt = static_cast<int64_t>(blockIdx.x) * kBlock + threadIdx.x;
    const int64_t row = gt / kThreadsPerRow;
    const int q = static_cast<int>(gt % kThreadsPerRow);
    const int64_t rows = p.batch * p.dim;
    const bool ok = row < rows;
    const int64_t r = ok ? row : rows - 1;
    const int64_t b = r / p.dim, d = r % p.dim;
    const int dstate = static_cast<int>(p.dstate);

    const float x = ld<T>(p.x, b * p.x_sb + d);
    float dt = ld<T>(p.delta, b * p.dl_sb + d);
    if (p.delta_bias) dt += p.delta_bias[d];
    if (p.softplus) dt = softplus(dt);
    const float dtx = dt * x;

    float *st = p.state + b * p.s_sb + d * p.s_sd;
    const float *Arow = p.A + d * dstate;
    float acc = 0.f;
    if constexpr (VEC16) {
        // dstate == 16, state rows 16-byte aligned
        const int n0 = 4 * q;
        float4 h = ok ? reinterpret_cast<const float4 *>(st)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 a4 = reinterpret_cast<const float4 *>(Arow)[q];
        float hv[4] = {h.x, h.y, h.z, h.w};
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = ex2_approx(dt * (av[e] * kLog2e));
            const float Bn = ld<T>(p.B, b * p.B_sb + n0 + e);
            hv[e] = fmaf(a, hv[e], dtx * Bn);
            acc = fmaf(ld<T>(p.C, b * p.C_sb + n0 + e), hv[e], acc);
        }
        if (ok) reinterpret_cast<float4 *>(st)[q] = make_float4(hv[0], hv[1], hv[2], hv[3]);
    } else {
        for (int n = q; n < dstate; n += kThreadsPerRow) {
            const float a = ex2_approx(dt * (Arow[n] * kLog2e));
            float h = ok ? st[n] : 0.f;
            h = fmaf(a, h, dtx * ld<T>(p.B, b * p.B_sb + n));
            acc = fmaf(ld<T>(p.C, b * p.C_sb + n), h, acc);
            if (ok) st[n] = h;
        }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (ok && q == 0) {
        float yv = acc + (p.D ? p.D[d] * x : 0.f);
        if (p.z) yv *= silu(ld<T>(p.z, b * p.z_sb + d));
        static_cast<T *>(p.y)[b * p.y_sb + d] = from_f32<T>(yv);
    }
}

template <typename T>
cudaError_t launch_t(const UpdateParams &p, cudaStream_t stream) {
    const int64_t threads = p.batch * p.dim * kThreadsPerRow;
    const int64_t blocks = (threads + kBlock - 1) / kBlock;
    const bool vec16 = p.dstate == 16 && (reinterpret_cast<uintptr_t>(p.state) & 15u) == 0 &&
                       (p.s_sb % 4) == 0 && (p.s_sd % 4) == 0 &&
                       (reinterpret_cast<uintptr_t>(p.A) & 15u) == 0;
    if (vec16)
        state_update_kernel<T, true><<<static_cast<unsigned>(blocks), kBlock, 0, stream>>>(p);
    else
        state_update_kernel<T, false><<<static_cast<unsigned>(blocks), kBlock, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const UpdateParams &p, int in_dtype, cudaStream_t stream) {
    return in_dtype == 0 ? launch_t<float>(p, stream) : launch_t<__nv_bfloat16>(p, stream);
}

}  // namespace ms
