// Device-side helpers shared by the scan and state-update kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ms {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// log2(e): exp(v) = 2^(v * log2 e). A is pre-scaled once per (d, n) so that the
// discretised transition Abar = exp(delta * A) costs one multiply and one ex2.
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log1p(e) = e p(e) on [0, 1], p of degree 6 (max relative error of log1p
// 1.7e-6 in float32 evaluation); coefficients fitted by fit_log1p.py.
__device__ __forceinline__ float log1p_unit(float e) {
    float p = 0.014539077877998352f;
    p = fmaf(p, e, -0.06759698688983917f);
    p = fmaf(p, e, 0.15056990087032318f);
    p = fmaf(p, e, -0.23573748767375946f);
    p = fmaf(p, e, 0.3312585949897766f);
    p = fmaf(p, e, -0.499883770942688f);
    p = fmaf(p, e, 0.999998927116394f);
    return p * e;
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(exp(-|v|)). Above v = 20 the
// second term is below 2.1e-9, under half an ulp of v, so the float32 result
// is v itself (the "identity above 20" rule, without a branch).
__device__ __forceinline__ float softplus(float v) {
    return fmaxf(v, 0.f) + log1p_unit(ex2_approx(-fabsf(v) * kLog2e));
}

// SiLU(z) = z * sigmoid(z) = z / (1 + e^-z).
__device__ __forceinline__ float silu(float z) {
    return __fdividef(z, 1.f + __expf(-z));
}

// Packed float32 pairs: one f32x2 instruction serves two independent lanes of
// work (two rows, two states or two time steps).
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 ex2x2(float2 v) { return f2(ex2_approx(v.x), ex2_approx(v.y)); }

__device__ __forceinline__ float2 log1p_unit2(float2 e) {
    float2 p = f2(0.014539077877998352f, 0.014539077877998352f);
    p = fma2(p, e, f2(-0.06759698688983917f, -0.06759698688983917f));
    p = fma2(p, e, f2(0.15056990087032318f, 0.15056990087032318f));
    p = fma2(p, e, f2(-0.23573748767375946f, -0.23573748767375946f));
    p = fma2(p, e, f2(0.3312585949897766f, 0.3312585949897766f));
    p = fma2(p, e, f2(-0.499883770942688f, -0.499883770942688f));
    p = fma2(p, e, f2(0.999998927116394f, 0.999998927116394f));
    return mul2(p, e);
}

// softplus and SiLU of a pair (same formulas as the scalar versions above).
__device__ __forceinline__ float2 softplus2(float2 v) {
    const float2 m = mul2(f2(fabsf(v.x), fabsf(v.y)), f2(-kLog2e, -kLog2e));
    const float2 l = log1p_unit2(ex2x2(m));
    return add2(f2(fmaxf(v.x, 0.f), fmaxf(v.y, 0.f)), l);
}
__device__ __forceinline__ float2 silu2(float2 z) {
    const float2 e = ex2x2(mul2(z, f2(-kLog2e, -kLog2e)));
    const float2 s = add2(e, f2(1.f, 1.f));
    return f2(__fdividef(z.x, s.x), __fdividef(z.y, s.y));
}

// SiLU of a pair as (z/2)(1 + tanh(z/2)) with tanh.approx: one MUFU operation
// per value instead of two, relative error near 2^-11. Used only where the
// result feeds a bfloat16 output (whose rounding is 2^-9); float32 paths keep
// silu2.
__device__ __forceinline__ float2 silu2_tanh(float2 z) {
    const float2 hz = mul2(z, f2(0.5f, 0.5f));
    float t0, t1;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(hz.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(hz.y));
    return fma2(hz, f2(t0, t1), hz);
}
template <typename T> __device__ __forceinline__ float2 silu2_out(float2 z) {
    if constexpr (sizeof(T) == 4) return silu2(z);
    else return silu2_tanh(z);
}

// bfloat16 <-> float32. Widening is exact (the bf16 bits are the top half of
// the float); narrowing rounds to nearest even.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Asynchronous 16-byte global->shared copy; bytes beyond `src_bytes` (0..16)
// are zero-filled and not read.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
                 "r"(src_bytes)
                 : "memory");
}
// 4- or 8-byte asynchronous copy (same zero-fill rule).
template <int BYTES>
__device__ __forceinline__ void cp_async_small(void *smem, const void *gmem, int src_bytes) {
    static_assert(BYTES == 4 || BYTES == 8, "cp.async.ca copies 4, 8 or 16 bytes");
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;\n" ::"r"(s), "l"(gmem), "n"(BYTES),
                 "r"(src_bytes)
                 : "memory");
}
// Asynchronous copy of BYTES (4, 8 or 16) bytes, all read, to a shared-memory
// address given as a 32-bit shared-window offset.
template <int BYTES>
__device__ __forceinline__ void cp_async_full(unsigned smem_addr, const void *gmem) {
    static_assert(BYTES == 4 || BYTES == 8 || BYTES == 16, "cp.async copies 4, 8 or 16 bytes");
    if constexpr (BYTES == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr), "l"(gmem) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(smem_addr), "l"(gmem), "n"(BYTES) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

}  // namespace ms
