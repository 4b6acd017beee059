// common.cuh -- device helpers shared by the mixer-core kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// Load / store VEC consecutive elements (VEC * sizeof(T) is 16 bytes for the
// vector paths, or one element for the scalar paths).
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T *p, float (&out)[VEC])
{
    if constexpr (VEC * sizeof(T) == 16) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p));
        const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
        for (int i = 0; i < VEC; ++i) out[i] = to_f32(e[i]);
    } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) out[i] = to_f32(p[i]);
    }
}

template <typename T, int VEC>
__device__ __forceinline__ void store_vec(T *p, const float (&v)[VEC])
{
    if constexpr (VEC * sizeof(T) == 16) {
        uint4 raw;
        T *e = reinterpret_cast<T *>(&raw);
#pragma unroll
        for (int i = 0; i < VEC; ++i) e[i] = from_f32<T>(v[i]);
        *reinterpret_cast<uint4 *>(p) = raw;
    } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) p[i] = from_f32<T>(v[i]);
    }
}

// Raw 16-byte global load kept in registers (software prefetch).
__device__ __forceinline__ uint4 ldg16(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

template <typename T, int VEC>
__device__ __forceinline__ void unpack16(const uint4 &raw, float (&out)[VEC])
{
    static_assert(VEC * sizeof(T) == 16, "16-byte vectors only");
    const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
    for (int i = 0; i < VEC; ++i) out[i] = to_f32(e[i]);
}

// ---------------------------------------------------------------------------
// math
// ---------------------------------------------------------------------------

// 2^x on the special-function unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2_approx(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// ---------------------------------------------------------------------------
// packed fp32x2 arithmetic (sm_100a): one instruction, two IEEE fp32 lanes
// ---------------------------------------------------------------------------
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pk2(float lo, float hi)
{
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void upk2(f32x2 v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b)
{
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// silu(v) = v * sigmoid(v); exp(-v) overflowing to +inf gives -0 for v << 0.
__device__ __forceinline__ float silu_f(float v)
{
    return __fdividef(v, 1.0f + __expf(-v));
}

// softplus(v) = log(1 + e^v), taken as v itself above 20 where the two agree
// to fp32 precision.
__device__ __forceinline__ float softplus_f(float v)
{
    return v > 20.0f ? v : log1pf(__expf(v));
}

// Clamp a sequence offset into [0, tok] so that a malformed cu_seqlens array
// can never push an access out of bounds.
__device__ __forceinline__ int64_t clamp_off(int64_t v, int64_t tok)
{
    return v < 0 ? 0 : (v > tok ? tok : v);
}

}  // namespace ssm
