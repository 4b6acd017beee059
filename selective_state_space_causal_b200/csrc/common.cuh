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

__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b)
{
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for two values on the FMA pipe instead of the special-function unit.
// x is clamped to [-126, 126] and split as n + f with n = round(x) (adding and
// subtracting 1.5 * 2^23 rounds to an integer held in the low mantissa bits)
// and f in [-0.5, 0.5]; 2^f comes from a degree-5 polynomial, the minimax
// fit for relative error on [-0.5, 0.5] with its coefficients rounded to fp32
// (1.5e-7 in exact arithmetic, 2.3e-7 when evaluated in fp32;
// tests/test_fastmath_fit.py re-derives the fit), and 2^n is added into the exponent bits:
// the float bits of x + 1.5 * 2^23 are 0x4B400000 + n, and shifting them left
// by 23 leaves exactly n << 23 (mod 2^32).
__device__ __forceinline__ void exp2_fma2(float x0, float x1, float &r0, float &r1)
{
    x0 = fminf(fmaxf(x0, -126.0f), 126.0f);
    x1 = fminf(fmaxf(x1, -126.0f), 126.0f);
    const f32x2 X = pk2(x0, x1);
    const f32x2 T = add2(X, pk2(12582912.0f, 12582912.0f));
    const f32x2 N = add2(T, pk2(-12582912.0f, -12582912.0f));  // exact
    const f32x2 F = fma2(N, pk2(-1.0f, -1.0f), X);                // x - n, exact
    f32x2 P = fma2(pk2(0.00132764782756567f, 0.00132764782756567f), F,
                   pk2(0.009675521403551102f, 0.009675521403551102f));
    P = fma2(P, F, pk2(0.05550713092088699f, 0.05550713092088699f));
    P = fma2(P, F, pk2(0.24022120237350464f, 0.24022120237350464f));
    P = fma2(P, F, pk2(0.6931469440460205f, 0.6931469440460205f));
    P = fma2(P, F, pk2(1.0000001192092896f, 1.0000001192092896f));
    float p0, p1, t0, t1;
    upk2(P, p0, p1);
    upk2(T, t0, t1);
    r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// softplus of two values as softplus_fast, with exp on the FMA pipe.
__device__ __forceinline__ void softplus2(float v0, float v1, float &d0, float &d1)
{
    float e0, e1;
    exp2_fma2(-fabsf(v0) * kLog2e, -fabsf(v1) * kLog2e, e0, e1);
    const f32x2 S = pk2(__fdividef(e0, 2.0f + e0), __fdividef(e1, 2.0f + e1));
    const f32x2 X = mul2(S, S);
    f32x2 P = fma2(pk2(0.28178291674498446f, 0.28178291674498446f), X,
                   pk2(0.27960550702657632f, 0.27960550702657632f));
    P = fma2(P, X, pk2(0.40024919874690540f, 0.40024919874690540f));
    P = fma2(P, X, pk2(0.66666314227845440f, 0.66666314227845440f));
    P = fma2(P, X, pk2(2.0000000079702546f, 2.0000000079702546f));
    float l0, l1;
    upk2(mul2(S, P), l0, l1);
    d0 = fmaxf(v0, 0.0f) + l0;
    d1 = fmaxf(v1, 0.0f) + l1;
}

// silu of two values, exp on the FMA pipe: z / (1 + 2^(-z log2 e)).
__device__ __forceinline__ void silu2(float z0, float z1, float &g0, float &g1)
{
    float e0, e1;
    exp2_fma2(-z0 * kLog2e, -z1 * kLog2e, e0, e1);
    g0 = __fdividef(z0, 1.0f + e0);
    g1 = __fdividef(z1, 1.0f + e1);
}

// silu(v) = v * sigmoid(v); exp(-v) overflowing to +inf gives -0 for v << 0.
__device__ __forceinline__ float silu_f(float v)
{
    return __fdividef(v, 1.0f + __expf(-v));
}

// softplus(v) = max(v, 0) + log1p(e) with e = exp(-|v|) in (0, 1], and
// log1p(e) = 2 atanh(s), s = e / (2 + e) in (0, 1/3]. 2 atanh(s) / s is a
// polynomial in s^2; the degree-4 coefficients below are the minimax fit for
// relative error on [0, 1/9] (max 4e-9, below fp32 resolution;
// tests/test_fastmath_fit.py re-derives it). Two
// special-function ops (2^x and 1/x) and ten FMA-pipe ops; relative error of
// the result ~5e-7.
__device__ __forceinline__ float softplus_fast(float v)
{
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-fabsf(v) * kLog2e));
    const float s = __fdividef(e, 2.0f + e);
    const float x = s * s;
    float p = 0.28178291674498446f;
    p = fmaf(p, x, 0.27960550702657632f);
    p = fmaf(p, x, 0.40024919874690540f);
    p = fmaf(p, x, 0.66666314227845440f);
    p = fmaf(p, x, 2.0000000079702546f);
    return fmaxf(v, 0.0f) + s * p;
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
