// scan_pipe.cuh -- the chunk-pipelined selective scan (schedules 9 to 12,
// sm_100a). Included by scan_pipe.cu (the kernels as the forward uses them)
// and scan_pipe_ckpt.cu (the same kernels, also writing the state before every
// 8th token of each sequence for the backward pass); the two compile apart.
#pragma once
//
// Math (tp_builder.py, TensorRT-Model-Connect Mamba family, _add_mamba_tp_layer;
// reset at every cu_seqlens boundary as in "PackMamba", abstract):
//   delta = softplus(dt + dt_bias)      dA[n] = exp(delta * A[c, n])
//   h[n]  = dA[n] * h[n] + delta * u * B_t[n]
//   y     = (sum_n C_t[n] h[n] + Dskip[c] * u) * silu(z)
//
// The scan is bound by the special-function unit: 16 ex2 per (token, channel)
// against ~8 bytes of DRAM traffic. A channel's 16 states are split over
// TPC = 16 / NPT lanes; every warp-wide ex2 occupies a sub-partition's
// special-function unit for 8 cycles, so the rest of a token's work must fit
// in the issue slots around the exponentials and must not stall the warp.
//
// A CTA owns one sequence and CH channels and walks the sequence in chunks of
// TCH tokens, in groups of TPC tokens. Lane `sub` of a channel owns the
// channel's tokens sub, sub + TPC, ... of every chunk:
//   pre-pass   for its own tokens: delta = softplus(dt + dt_bias) and delta*u
//              (shared memory, one (delta, delta*u) pair per token and channel
//              for all TPC lanes of the channel), Dskip*u and silu(z) (kept in
//              registers for its own skip and gate); B and C rows to fp32
//              (cooperative)
//   recurrence NPT states per lane in packed fp32x2 registers, one ex2 per
//              state and token; after each group a transposed shuffle butterfly
//              over the channel's TPC lanes leaves token `sub` of the group in
//              full in lane `sub`, which applies skip and gate and stores y
// Within a warp a channel's TPC lanes sit WCH = 32 / TPC lanes apart. Shared
// memory, not the special-function unit, is the limit to design for: every
// shared load shares the MIO path with ex2, and a 16-byte load costs two
// wavefronts when groups of lanes read one address but four when neighbouring
// lanes differ; with this lane order a token's B and C rows cost two each and
// its (delta, delta*u) pair (8 bytes) two.
// The state-free part of a token (shared loads, exponent arguments, ex2,
// delta*u*B) is issued TPC tokens ahead of its state chain, so a warp keeps a
// group's exponentials in flight while it runs the previous group's chain.
// With CK the lanes also store their states after every 8th token of the
// sequence (the backward pass's checkpoints).
// Iteration k runs the recurrence of chunk k together with the pre-pass of
// chunk k+1 in one loop body (the pre-pass's loads at the top, its stores at
// the bottom), so the compiler fills the recurrence's latency gaps with the
// pre-pass's independent arithmetic; a chunk costs one CTA barrier.
//
// Data movement: the raw u, dt, z (TCH x CH) and B, C (TCH x 16) tiles of a
// chunk arrive by TMA (cp.async.bulk.tensor, mbarrier completion; plain
// per-CTA copies of this GPU's memory, no multicast) into one of RS = 4 stages:
// chunk j's copy is issued at the start of iteration j-RS, three iterations
// before its pre-pass (iteration j-1), which covers the DRAM latency. The loop
// is unrolled by two so every shared-buffer index is a constant.
// Tokens past the sequence end within its last chunk get delta = 0 and
// delta*u = 0, which leaves the state unchanged; their outputs are not stored.
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "scan_parts.cuh"
#include "tma.cuh"

namespace ssm {

namespace {

// Set by a pipelined kernel whose bounded wait on a TMA completion gave up
// (reported through ssm_device_status with the scan's other kernels). One per
// translation unit that includes this header, each read by its own
// read_tu_pipe_status.
__device__ int g_pipe_status = 0;

struct Maps {
    CUtensorMap u, dt, z, b, c;
};

// 1/x on the special-function unit (flushes subnormals).
__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Shared loads as packed fp32x2 pairs: one 16-byte load as two pairs, one
// 8-byte load as a pair. Plain loads (not inline assembly), so the compiler
// addresses them off a register with constant offsets and keeps the pairs in
// the load's aligned registers.
__device__ __forceinline__ void lds_2x2(const void *p, f32x2 &a, f32x2 &b)
{
    const float4 v = *reinterpret_cast<const float4 *>(p);
    a = pk2(v.x, v.y);
    b = pk2(v.z, v.w);
}
__device__ __forceinline__ f32x2 lds_x2(const void *p)
{
    const float2 v = *reinterpret_cast<const float2 *>(p);
    return pk2(v.x, v.y);
}

// y[...] = v when pred, as one predicated store.
__device__ __forceinline__ void stg_if(__nv_bfloat16 *dst, __nv_bfloat16 v, bool pred)
{
    asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %2, 0;\n @q st.global.b16 [%0], %1;\n}\n"
                 :: "l"(dst), "h"(*reinterpret_cast<unsigned short *>(&v)), "r"((unsigned)pred)
                 : "memory");
}
__device__ __forceinline__ void stg_if(float *dst, float v, bool pred)
{
    asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %2, 0;\n @q st.global.f32 [%0], %1;\n}\n"
                 :: "l"(dst), "f"(v), "r"((unsigned)pred) : "memory");
}

// Tokens per checkpoint of the state written for the backward pass.
constexpr int kCkTok = 8;

// Packed sequences run longest first. In the one-lane-per-channel kernels,
// without a precomputed order (no workspace) and with at most kRankMax
// sequences, each CTA ranks the lengths itself (their longest chains are twice
// as long as the split-lane kernels', so the order matters more there): cu_seqlens into shared memory, one rank per thread (ties by index),
// and the CTA takes the blockIdx.y-th longest. Otherwise sequence blockIdx.y.
// The branch is the same for the whole CTA, and every thread must call this
// (it holds two CTA barriers).
constexpr int kRankMax = 128;

__device__ __forceinline__ int64_t ranked_seq(const Params &p)
{
    __shared__ int cu_s[kRankMax + 1];
    __shared__ int seq_s;
    if (p.order) return (int64_t)p.order[blockIdx.y];
    if (!p.cu || p.S <= 1 || p.S > kRankMax) return (int64_t)blockIdx.y;
    const int S = (int)p.S;
    for (int i = threadIdx.x; i <= S; i += blockDim.x) cu_s[i] = (int)clamp_off(p.cu[i], p.tok);
    if (threadIdx.x == 0) seq_s = (int)blockIdx.y;
    __syncthreads();
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
        const int li = max(cu_s[i + 1] - cu_s[i], 0);
        int rank = 0;
        for (int j = 0; j < S; ++j) {
            const int lj = max(cu_s[j + 1] - cu_s[j], 0);
            rank += (lj > li) || (lj == li && j < i);
        }
        if (rank == (int)blockIdx.y) seq_s = i;
    }
    __syncthreads();
    return (int64_t)seq_s;
}

template <typename T, int NPT_, int CH_, int TCH_, int MINB_ = 3>
struct PipeCfg {
    static constexpr int NPT = NPT_, CH = CH_, TCH = TCH_;
    // resident CTAs per SM the register budget must allow: 3 (up to 168
    // registers a thread) or, for grids of at most two CTAs per SM, 2 (up to
    // 255), which gives the compiler room to keep more of the look-ahead live
    static constexpr int MINB = MINB_;
    static constexpr int NP = NPT / 2;                       // packed state pairs per lane
    static constexpr int TPC = kN / NPT;                     // lanes per channel = tokens per group
    static constexpr int THREADS = CH * TPC;
    static constexpr int G = TCH / TPC;                      // token groups per chunk
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CH;
    static constexpr size_t RAW_BC = sizeof(T) * TCH * kN;
    static constexpr size_t STAGE = 3 * align128(RAW_ACT) + 2 * align128(RAW_BC);
    static constexpr int WCH = 32 / TPC;                     // channels per warp
    // (delta, delta*u) of (token t, channel c) at t * ROWD + c: 64 bytes of
    // padding per row put the pre-pass's four-token stores on two bank halves
    static constexpr int ROWD = CH + 8;
    static constexpr size_t DD_BUF = 8 * (size_t)TCH * ROWD;
    static constexpr size_t BC_BUF = 4 * (size_t)TCH * kN;
    static constexpr int RS = 4;                             // raw tile stages
    static constexpr size_t OFF_RAW = 0;
    static constexpr size_t OFF_DD = OFF_RAW + RS * STAGE;
    static constexpr size_t OFF_B = align128(OFF_DD + 2 * DD_BUF);
    static constexpr size_t OFF_C = align128(OFF_B + 2 * BC_BUF);
    static constexpr size_t OFF_BAR = align128(OFF_C + 2 * BC_BUF);
    static constexpr size_t SMEM = OFF_BAR + 8 * RS;
    // B and C rows are widened to fp32 in pieces of PE elements, one or more
    // pieces per thread (at most 16 bytes of raw data a piece)
    static constexpr int PE = (TCH * kN / THREADS) < (16 / (int)sizeof(T)) ? (TCH * kN / THREADS)
                                                                           : (16 / (int)sizeof(T));
    static constexpr int BCP = TCH * kN / PE;                // pieces of B (or C) per chunk
    static constexpr int BPT = BCP / THREADS;                // pieces per thread
    static constexpr int PW = PE * sizeof(T) / 4;            // 32-bit words of a raw piece
    static_assert(NPT == 2 || NPT == 4 || NPT == 8, "states per lane");
    static_assert(G % 2 == 0, "token pairs per lane");
    static_assert(BCP % THREADS == 0, "whole B and C pieces per thread");
    static_assert(PE >= 2 && (PE & (PE - 1)) == 0, "B and C pieces of 2, 4 or 8 elements");
    static_assert(TCH % TPC == 0, "whole token groups per chunk");
    static_assert(TCH % kCkTok == 0, "checkpoints fall on chunk boundaries");
    static_assert(RAW_ACT % 128 == 0 && RAW_BC % 128 == 0, "TMA tiles stay 128-byte aligned");
    static_assert((CH * sizeof(T)) % 16 == 0, "TMA box rows are whole 16-byte units");
    static_assert(THREADS <= 1024 && THREADS % 32 == 0, "block size");
};

// softplus(v) = max(v, 0) + log1p(e), e = 2^(-|v| log2 e), as
// log1p(e) = 2 atanh(s) = s q(s^2) with s = e / (2 + e) (q: the degree-4
// polynomial of softplus_fast), and silu(z) = z / (1 + e'), e' = 2^(-z log2 e)
// clamped below 2^64 (silu is then below 2^-64 |z|, i.e. zero for any output).
// Both reciprocals come from one: with a = 2 + e and b = 1 + e',
// r = 1 / (a b), 1/a = r b, 1/b = r a. Two channels at a time in packed
// fp32x2; three special-function operations per channel (two ex2, one
// reciprocal); relative error about 5e-7.
__device__ __forceinline__ void softplus_silu2(f32x2 v, f32x2 z, f32x2 &d, f32x2 &g)
{
    float v0, v1, z0, z1;
    upk2(v, v0, v1);
    upk2(z, z0, z1);
    const f32x2 e = pk2(ex2_approx(-fabsf(v0) * kLog2e), ex2_approx(-fabsf(v1) * kLog2e));
    float n0, n1;
    upk2(mul2(z, pk2(-kLog2e, -kLog2e)), n0, n1);
    const f32x2 e2 = pk2(ex2_approx(fminf(n0, 64.0f)), ex2_approx(fminf(n1, 64.0f)));
    const f32x2 a = add2(e, pk2(2.0f, 2.0f)), b = add2(e2, pk2(1.0f, 1.0f));
    float ab0, ab1;
    upk2(mul2(a, b), ab0, ab1);
    const f32x2 r = pk2(rcp_approx(ab0), rcp_approx(ab1));
    const f32x2 s = mul2(e, mul2(r, b));
    const f32x2 x = mul2(s, s);
    f32x2 q = fma2(pk2(0.28178291674498446f, 0.28178291674498446f), x,
                   pk2(0.27960550702657632f, 0.27960550702657632f));
    q = fma2(q, x, pk2(0.40024919874690540f, 0.40024919874690540f));
    q = fma2(q, x, pk2(0.66666314227845440f, 0.66666314227845440f));
    q = fma2(q, x, pk2(2.0000000079702546f, 2.0000000079702546f));
    d = fma2(s, q, pk2(fmaxf(v0, 0.0f), fmaxf(v1, 0.0f)));
    g = mul2(z, mul2(r, a));
}

__device__ __forceinline__ f32x2 softplus2p(f32x2 v)
{
    float v0, v1;
    upk2(v, v0, v1);
    const f32x2 e = pk2(ex2_approx(-fabsf(v0) * kLog2e), ex2_approx(-fabsf(v1) * kLog2e));
    float a0, a1;
    upk2(add2(e, pk2(2.0f, 2.0f)), a0, a1);
    const f32x2 s = mul2(e, pk2(rcp_approx(a0), rcp_approx(a1)));
    const f32x2 x = mul2(s, s);
    f32x2 q = fma2(pk2(0.28178291674498446f, 0.28178291674498446f), x,
                   pk2(0.27960550702657632f, 0.27960550702657632f));
    q = fma2(q, x, pk2(0.40024919874690540f, 0.40024919874690540f));
    q = fma2(q, x, pk2(0.66666314227845440f, 0.66666314227845440f));
    q = fma2(q, x, pk2(2.0000000079702546f, 2.0000000079702546f));
    return fma2(s, q, pk2(fmaxf(v0, 0.0f), fmaxf(v1, 0.0f)));
}

__device__ __forceinline__ f32x2 silu2p(f32x2 z)
{
    float n0, n1;
    upk2(mul2(z, pk2(-kLog2e, -kLog2e)), n0, n1);
    float b0, b1;
    upk2(add2(pk2(ex2_approx(fminf(n0, 64.0f)), ex2_approx(fminf(n1, 64.0f))), pk2(1.0f, 1.0f)),
         b0, b1);
    return mul2(z, pk2(rcp_approx(b0), rcp_approx(b1)));
}

__device__ __forceinline__ float raw_f32(const __nv_bfloat16 *p)
{
    return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short *>(p)) << 16);
}
__device__ __forceinline__ float raw_f32(const float *p) { return *p; }

template <class K, typename T, bool SP, bool GZ, bool CK>
struct Pipe {
    static constexpr int NPT = K::NPT, NP = K::NP, TPC = K::TPC, CH = K::CH;
    static constexpr int TCH = K::TCH, G = K::G, THREADS = K::THREADS;

    unsigned char *smem;
    const Params &p;
    int tid, lane, cl, sub;
    int64_t cbase, c0;
    bool cvalid;
    float dtb, dsk;
    f32x2 A2p[NP], hp[NP];  // A * log2(e) and the state, two states per register
    float gdu[2][G], gg[2][G];  // Dskip*u and silu(z) of my tokens, per chunk buffer
    float *ckb;  // this lane's state checkpoints for the backward pass, or null

    // The lane's NPT states as checkpoint j of its sequence (the state before
    // the sequence's token 8j).
    __device__ __forceinline__ void store_ckpt(int64_t j) const
    {
        float *dst = ckb + j * p.D * kN;
        if constexpr (NPT == 2) {
            float a, b;
            upk2(hp[0], a, b);
            *reinterpret_cast<float2 *>(dst) = make_float2(a, b);
        } else {
#pragma unroll
            for (int q = 0; q < NP; q += 2) {
                float4 v;
                upk2(hp[q], v.x, v.y);
                upk2(hp[q + 1], v.z, v.w);
                *reinterpret_cast<float4 *>(dst + 2 * q) = v;
            }
        }
    }

    __device__ __forceinline__ Pipe(unsigned char *s, const Params &p_) : smem(s), p(p_) {}

    __device__ __forceinline__ T *raw(int stage, int which) const
    {
        size_t off = K::OFF_RAW + (size_t)stage * K::STAGE;
        off += which < 3 ? (size_t)which * align128(K::RAW_ACT)
                         : 3 * align128(K::RAW_ACT) + (size_t)(which - 3) * align128(K::RAW_BC);
        return reinterpret_cast<T *>(smem + off);
    }
    __device__ __forceinline__ float2 *sDD(int buf) const
    {
        return reinterpret_cast<float2 *>(smem + K::OFF_DD + buf * K::DD_BUF);
    }
    __device__ __forceinline__ float *sB(int buf) const
    {
        return reinterpret_cast<float *>(smem + K::OFF_B + buf * K::BC_BUF);
    }
    __device__ __forceinline__ float *sC(int buf) const
    {
        return reinterpret_cast<float *>(smem + K::OFF_C + buf * K::BC_BUF);
    }

    // ---- pre-pass of one chunk: loads at the top, stores at the bottom -------
    struct Pre {
        float dt[G], u[G], z[G];
        uint32_t rb[K::BPT][K::PW], rc[K::BPT][K::PW];  // pieces of B and C, raw
    };

    __device__ __forceinline__ void pre_load(Pre &q, int stage) const
    {
        const T *rU = raw(stage, 0), *rDT = raw(stage, 1), *rZ = raw(stage, 2);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int o = (sub + TPC * g) * CH + cl;
            q.dt[g] = raw_f32(rDT + o);
            q.u[g] = raw_f32(rU + o);
            if (GZ) q.z[g] = raw_f32(rZ + o);
        }
#pragma unroll
        for (int i = 0; i < K::BPT; ++i) {
            const uint32_t *rb = reinterpret_cast<const uint32_t *>(raw(stage, 3)) + (tid + i * THREADS) * K::PW;
            const uint32_t *rc = reinterpret_cast<const uint32_t *>(raw(stage, 4)) + (tid + i * THREADS) * K::PW;
            if constexpr (K::PW == 4) {
                const uint4 b4 = *reinterpret_cast<const uint4 *>(rb), c4 = *reinterpret_cast<const uint4 *>(rc);
                q.rb[i][0] = b4.x; q.rb[i][1] = b4.y; q.rb[i][2] = b4.z; q.rb[i][3] = b4.w;
                q.rc[i][0] = c4.x; q.rc[i][1] = c4.y; q.rc[i][2] = c4.z; q.rc[i][3] = c4.w;
            } else if constexpr (K::PW == 2) {
                const uint2 b2 = *reinterpret_cast<const uint2 *>(rb), c2 = *reinterpret_cast<const uint2 *>(rc);
                q.rb[i][0] = b2.x; q.rb[i][1] = b2.y;
                q.rc[i][0] = c2.x; q.rc[i][1] = c2.y;
            } else {
                q.rb[i][0] = *rb;
                q.rc[i][0] = *rc;
            }
        }
    }

    // Pre-pass arithmetic and stores of my tokens g and g + 1 for chunk
    // buffer BUF (nt valid tokens).
    template <int BUF, bool MASK>
    __device__ __forceinline__ void pre_pair(const Pre &q, int g, int nt)
    {
        float2 *dd = sDD(BUF);
        const f32x2 v = add2(pk2(q.dt[g], q.dt[g + 1]), pk2(dtb, dtb));
        const f32x2 u = pk2(q.u[g], q.u[g + 1]);
        f32x2 d, gt = pk2(1.0f, 1.0f);
        if (SP && GZ) {
            softplus_silu2(v, pk2(q.z[g], q.z[g + 1]), d, gt);
        } else if (SP) {
            d = softplus2p(v);
        } else {
            d = v;
            if (GZ) gt = silu2p(pk2(q.z[g], q.z[g + 1]));
        }
        float d0, d1, x0, x1;
        upk2(d, d0, d1);
        upk2(mul2(d, u), x0, x1);
        upk2(mul2(pk2(dsk, dsk), u), gdu[BUF][g], gdu[BUF][g + 1]);
        upk2(gt, gg[BUF][g], gg[BUF][g + 1]);
        if (MASK) {
            const bool l0 = sub + TPC * g < nt, l1 = sub + TPC * (g + 1) < nt;
            d0 = l0 ? d0 : 0.f;
            x0 = l0 ? x0 : 0.f;
            d1 = l1 ? d1 : 0.f;
            x1 = l1 ? x1 : 0.f;
        }
        dd[(sub + TPC * g) * K::ROWD + cl] = make_float2(d0, x0);
        dd[(sub + TPC * (g + 1)) * K::ROWD + cl] = make_float2(d1, x1);
    }

    // B and C rows to fp32 for chunk buffer BUF (tokens past the sequence end
    // only meet delta*u = 0 and unstored outputs).
    template <int BUF>
    __device__ __forceinline__ void pre_bc(const Pre &q) const
    {
#pragma unroll
        for (int i = 0; i < K::BPT; ++i) {
            float fb[K::PE], fc[K::PE];
#pragma unroll
            for (int w = 0; w < K::PW; ++w) {
                if constexpr (sizeof(T) == 2) {
                    fb[2 * w] = __uint_as_float(q.rb[i][w] << 16);
                    fb[2 * w + 1] = __uint_as_float(q.rb[i][w] & 0xffff0000u);
                    fc[2 * w] = __uint_as_float(q.rc[i][w] << 16);
                    fc[2 * w + 1] = __uint_as_float(q.rc[i][w] & 0xffff0000u);
                } else {
                    fb[w] = __uint_as_float(q.rb[i][w]);
                    fc[w] = __uint_as_float(q.rc[i][w]);
                }
            }
            float *b = sB(BUF) + (tid + i * THREADS) * K::PE;
            float *c = sC(BUF) + (tid + i * THREADS) * K::PE;
#pragma unroll
            for (int e = 0; e < K::PE; e += 2) {
                *reinterpret_cast<float2 *>(b + e) = make_float2(fb[e], fb[e + 1]);
                *reinterpret_cast<float2 *>(c + e) = make_float2(fc[e], fc[e + 1]);
            }
        }
    }

    template <int BUF, bool MASK>
    __device__ __forceinline__ void pre_store(const Pre &q, int nt)
    {
#pragma unroll
        for (int g = 0; g < G; g += 2) pre_pair<BUF, MASK>(q, g, nt);
        pre_bc<BUF>(q);
    }

    // ---- recurrence of one chunk ----------------------------------------------
    // A token's state-free part (shared loads, exponent arguments, ex2, the
    // input terms delta*u*B) runs LA = TPC tokens ahead of its state chain,
    // token by token, so every warp issues its exponentials at an even rate
    // (four per token between the chain steps) instead of in bursts.
    static constexpr int LA = TPC;
    struct Tok {
        f32x2 dA[NP], bx[NP];
    };
    struct Cv {
        f32x2 c[NP];
    };

    __device__ __forceinline__ void front_tok(Tok &E, int buf, int t) const
    {
        const float2 *dd = sDD(buf);
        const float *b = sB(buf);
        f32x2 bb[NP];
        const float2 v = dd[t * K::ROWD + cl];
        const f32x2 dv = pk2(v.x, v.x), xv = pk2(v.y, v.y);
#pragma unroll
        for (int j = 0; j < NP; j += 2) {
            if (j + 1 < NP) lds_2x2(b + t * kN + sub * NPT + 2 * j, bb[j], bb[j + 1]);
            else bb[j] = lds_x2(b + t * kN + sub * NPT + 2 * j);
        }
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            float a0, a1;
            upk2(mul2(dv, A2p[j]), a0, a1);
            E.dA[j] = pk2(ex2_approx(a0), ex2_approx(a1));
            E.bx[j] = mul2(xv, bb[j]);
        }
    }

    __device__ __forceinline__ void load_c(Cv &C, int buf, int t) const
    {
        const float *c = sC(buf);
#pragma unroll
        for (int j = 0; j < NP; j += 2) {
            if (j + 1 < NP) lds_2x2(c + t * kN + sub * NPT + 2 * j, C.c[j], C.c[j + 1]);
            else C.c[j] = lds_x2(c + t * kN + sub * NPT + 2 * j);
        }
    }

    // State chain of one token; returns the lane's partial readout.
    __device__ __forceinline__ float chain_tok(const Tok &E, const Cv &C)
    {
        f32x2 acc = 0ull;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            hp[j] = fma2(E.dA[j], hp[j], E.bx[j]);
            acc = j == 0 ? mul2(C.c[0], hp[0]) : fma2(C.c[j], hp[j], acc);
        }
        float s0, s1;
        upk2(acc, s0, s1);
        return s0 + s1;
    }

    // The butterfly over the channel's lanes for a group's partials, then
    // skip, gate and store of token g * TPC + sub.
    template <int BUF, bool FULL>
    __device__ __forceinline__ void group_out(float (&P)[TPC], int g, int64_t t0, int nt) const
    {
        // transposed butterfly: after log2(TPC) steps P[0] of lane `sub` is
        // the channel's full readout of token g * TPC + sub
#pragma unroll
        for (int w = TPC / 2; w >= 1; w >>= 1) {
            const bool upper = (sub & w) != 0;
#pragma unroll
            for (int i = 0; i < w; ++i) {
                const float send = upper ? P[i] : P[i + w];
                const float keep = upper ? P[i + w] : P[i];
                P[i] = keep + __shfl_xor_sync(0xffffffffu, send, w * K::WCH);
            }
        }
        const int t = g * TPC + sub;
        const T yv = from_f32<T>((P[0] + gdu[BUF][g]) * gg[BUF][g]);
        T *dst = static_cast<T *>(p.y) + (t0 + t) * p.D + c0;
        if (FULL) {
            if (cvalid) *dst = yv;
        } else {
            if (cvalid && t < nt) *dst = yv;
        }
    }

    // Iteration: the recurrence of the chunk in buffer BUF (nt valid tokens
    // from t0) and, if PRE, the pre-pass of the next chunk (raw stage `stage`,
    // buffer BUF ^ 1, ntn valid tokens).
    // kc: the checkpoint index of the chunk's first token (its offset in the
    // sequence / 8); without PRE this is the sequence's last chunk.
    template <int BUF, bool PRE, bool MASK, bool FULL>
    __device__ __forceinline__ void iteration(int64_t t0, int nt, int ntn, int stage, int64_t kc)
    {
        Pre q;
        if (PRE) pre_load(q, stage);
        Tok E[2 * LA];
        Cv C[2];
#pragma unroll
        for (int t = 0; t < LA; ++t) front_tok(E[t], BUF, t);
        load_c(C[0], BUF, 0);
        float P[TPC];
#pragma unroll
        for (int t = 0; t < TCH; ++t) {
            if (t + LA < TCH) front_tok(E[(t + LA) % (2 * LA)], BUF, t + LA);
            if (t + 1 < TCH) load_c(C[(t + 1) & 1], BUF, t + 1);
            P[t % TPC] = chain_tok(E[t % (2 * LA)], C[t & 1]);
            // after every 8th token of the sequence, unless it was the last
            if constexpr (CK) {
                if (t % kCkTok == kCkTok - 1 && ckb && (PRE || t + 1 < nt))
                    store_ckpt(kc + (t + 1) / kCkTok);
            }
            if (t % TPC == TPC - 1) group_out<BUF, FULL>(P, t / TPC, t0, nt);
            // the next chunk's pre-pass arithmetic, spread over the chunk
            if (PRE && t % (TCH / (G / 2)) == TCH / (G / 2) - 1)
                pre_pair<BUF ^ 1, MASK>(q, 2 * (t / (TCH / (G / 2))), ntn);
        }
        if (PRE) pre_bc<BUF ^ 1>(q);
    }
};

template <int V> struct BufTag { static constexpr int value = V; };

// One warp per CTA needs only a warp barrier between the phases.
template <int THREADS>
__device__ __forceinline__ void cta_sync()
{
    if constexpr (THREADS == 32) __syncwarp();
    else __syncthreads();
}

// At least MINB 4-warp CTAs per SM: with three (up to 168 registers a thread)
// every (sequence, channel) warp of the Mamba-130M layer is resident at once.
template <class K, typename T, bool SP, bool GZ, bool CK>
__global__ void __launch_bounds__(K::THREADS, K::MINB)
scan_pipe_kernel(const Params p, const __grid_constant__ Maps m)
{
    constexpr int TCH = K::TCH, CH = K::CH, NPT = K::NPT, TPC = K::TPC;
    extern __shared__ __align__(128) unsigned char smem[];
    Pipe<K, T, SP, GZ, CK> P(smem, p);
    uint64_t *const bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);

    P.tid = threadIdx.x;
    // lane = sub * WCH + channel-in-warp: a channel's TPC lanes sit WCH apart,
    // so shared loads of B and C rows (one address per `sub`) serve groups of
    // WCH neighbouring lanes in two wavefronts
    P.lane = P.tid & 31;
    P.cl = (P.tid >> 5) * K::WCH + P.lane % K::WCH;
    P.sub = P.lane / K::WCH;
    P.cbase = (int64_t)blockIdx.x * CH;
    P.c0 = P.cbase + P.cl;
    P.cvalid = P.c0 < p.D;
    int64_t seq = p.order ? (int64_t)p.order[blockIdx.y] : (int64_t)blockIdx.y;
    seq = seq < 0 ? 0 : (seq >= p.S ? p.S - 1 : seq);
    int64_t start, end;
    if (p.cu) {
        start = clamp_off(p.cu[seq], p.tok);
        end = max(clamp_off(p.cu[seq + 1], p.tok), start);
    } else {
        start = seq * p.L;
        end = start + p.L;
    }
    const int nch = (int)((end - start + TCH - 1) / TCH);
    constexpr uint32_t tx_bytes = (uint32_t)((GZ ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);

    if (P.tid == 0) {
#pragma unroll
        for (int st = 0; st < K::RS; ++st) mbar_init(&bar[st]);
    }
    cta_sync<K::THREADS>();
    auto issue = [&](int j) {  // TMA of chunk j into stage j % RS
        const int stage = j % K::RS;
        mbar_expect_tx(&bar[stage], tx_bytes);
        const int x = (int)P.cbase, y = (int)(start + (int64_t)j * TCH);
        tma_2d(P.raw(stage, 0), &m.u, &bar[stage], x, y);
        tma_2d(P.raw(stage, 1), &m.dt, &bar[stage], x, y);
        if (GZ) tma_2d(P.raw(stage, 2), &m.z, &bar[stage], x, y);
        tma_2d(P.raw(stage, 3), &m.b, &bar[stage], 0, y);
        tma_2d(P.raw(stage, 4), &m.c, &bar[stage], 0, y);
    };
    if (P.tid == 0) {
        for (int j = 0; j < K::RS && j < nch; ++j) issue(j);
    }

#pragma unroll
    for (int j = 0; j < NPT; j += 2) {
        const int64_t ai = P.c0 * kN + P.sub * NPT + j;
        const int64_t hi = (seq * p.D + P.c0) * kN + P.sub * NPT + j;
        P.A2p[j / 2] = P.cvalid ? pk2(__ldg(p.A + ai) * kLog2e, __ldg(p.A + ai + 1) * kLog2e) : 0ull;
        P.hp[j / 2] = (P.cvalid && p.h0) ? pk2(p.h0[hi], p.h0[hi + 1]) : 0ull;
    }
    P.dtb = (P.cvalid && p.dt_bias) ? __ldg(p.dt_bias + P.c0) : 0.f;
    // checkpoint j of sequence `seq` (the state before its token 8j) lives in
    // row floor(start / 8) + seq + j of D x 16 floats: sequences never collide
    P.ckb = (CK && P.cvalid)
                ? p.ckpt + ((start / kCkTok + seq) * p.D + P.c0) * kN + P.sub * NPT
                : nullptr;
    if (CK && P.ckb && end > start) P.store_ckpt(0);
    P.dsk = (P.cvalid && p.Dskip) ? __ldg(p.Dskip + P.c0) : 0.f;

    bool failed = false;
    auto ntok = [&](int j) { return (int)min((int64_t)TCH, end - start - (int64_t)j * TCH); };
    auto wait_raw = [&](int j) {
        mbar_wait(&bar[j % K::RS], (uint32_t)((j / K::RS) & 1), failed, &g_pipe_status, 1);
    };
    if (nch > 0) {
        wait_raw(0);
        typename Pipe<K, T, SP, GZ, CK>::Pre q;
        P.pre_load(q, 0);
        if (nch == 1) P.template pre_store<0, true>(q, ntok(0));
        else P.template pre_store<0, false>(q, TCH);
    }
    cta_sync<K::THREADS>();

    // iteration k: chunk buffer k & 1, next chunk's raw stage (k + 1) % RS;
    // only the last chunk may be partial
    auto step = [&](auto tag, int k) {
        constexpr int BUF = decltype(tag)::value;
        const int64_t t0 = start + (int64_t)k * TCH;
        const int64_t kc = (int64_t)k * (TCH / kCkTok);
        if (P.tid == 0 && k + K::RS < nch) {
            // stage k % RS was last read by the pre-pass of chunk k, before
            // the last barrier
            fence_proxy_async();
            issue(k + K::RS);
        }
        if (k + 1 < nch) {
            wait_raw(k + 1);
            if (k + 2 < nch) P.template iteration<BUF, true, false, true>(t0, TCH, TCH, (k + 1) % K::RS, kc);
            else P.template iteration<BUF, true, true, true>(t0, TCH, ntok(k + 1), (k + 1) % K::RS, kc);
        } else {
            P.template iteration<BUF, false, false, false>(t0, ntok(k), 0, 0, kc);
        }
        cta_sync<K::THREADS>();
    };
    int k = 0;
    for (; k + 1 < nch; k += 2) {
        step(BufTag<0>{}, k);
        step(BufTag<1>{}, k + 1);
    }
    if (k < nch) step(BufTag<0>{}, k);

    if (p.h_final && P.cvalid) {
#pragma unroll
        for (int j = 0; j < NPT; j += 2) {
            float lo, hi;
            upk2(P.hp[j / 2], lo, hi);
            const int64_t o = (seq * p.D + P.c0) * kN + P.sub * NPT + j;
            p.h_final[o] = lo;
            p.h_final[o + 1] = hi;
        }
    }
}

template <class K, typename T, bool SP, bool GZ, bool CK>
cudaError_t run_pipe_t(const Params &p, const Maps &m, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
    cudaError_t e = cudaFuncSetAttribute(scan_pipe_kernel<K, T, SP, GZ, CK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_pipe_kernel<K, T, SP, GZ, CK><<<grid, K::THREADS, K::SMEM, stream>>>(p, m);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T, bool CK>
cudaError_t run_pipe(const Params &p, cudaStream_t stream, int *launches)
{
    Maps m;
    const bool bf = sizeof(T) == 2;
    bool ok = p.tok > 0 && encode_2d(&m.u, p.u, bf, p.D, p.tok, K::CH, K::TCH) &&
              encode_2d(&m.dt, p.delta, bf, p.D, p.tok, K::CH, K::TCH) &&
              encode_2d(&m.b, p.B, bf, kN, p.tok, kN, K::TCH) &&
              encode_2d(&m.c, p.C, bf, kN, p.tok, kN, K::TCH);
    if (ok) {
        if (p.z) ok = encode_2d(&m.z, p.z, bf, p.D, p.tok, K::CH, K::TCH);
        else m.z = m.u;  // never loaded
    }
    if (!ok) return cudaErrorNotSupported;
    if (p.delta_softplus)
        return p.z ? run_pipe_t<K, T, true, true, CK>(p, m, stream, launches)
                   : run_pipe_t<K, T, true, false, CK>(p, m, stream, launches);
    return p.z ? run_pipe_t<K, T, false, true, CK>(p, m, stream, launches)
               : run_pipe_t<K, T, false, false, CK>(p, m, stream, launches);
}

template <bool CK>
cudaError_t launch_wide_cfg(const Params &p, bool bf16, cudaStream_t stream, int *launches);

template <bool CK>
cudaError_t launch_pipe_cfg(const Params &p, bool bf16, int npt, int sched, cudaStream_t stream,
                            int *launches)
{
    if (sched == 12) return launch_wide_cfg<CK>(p, bf16, stream, launches);
    const bool lng = sched == 10;
    if (bf16) {
        using T = __nv_bfloat16;
        if (sched == 11) return run_pipe<PipeCfg<T, 4, 32, 32, 2>, T, CK>(p, stream, launches);
        if (npt == 8) return lng ? run_pipe<PipeCfg<T, 8, 64, 32>, T, CK>(p, stream, launches)
                                 : run_pipe<PipeCfg<T, 8, 64, 16>, T, CK>(p, stream, launches);
        if (npt == 2) return run_pipe<PipeCfg<T, 2, 16, 32>, T, CK>(p, stream, launches);
        return lng ? run_pipe<PipeCfg<T, 4, 32, 32>, T, CK>(p, stream, launches)
                   : run_pipe<PipeCfg<T, 4, 32, 16>, T, CK>(p, stream, launches);
    }
    if (npt == 8) return run_pipe<PipeCfg<float, 8, 64, 16>, float, CK>(p, stream, launches);
    if (npt == 2) return run_pipe<PipeCfg<float, 2, 16, 32>, float, CK>(p, stream, launches);
    return run_pipe<PipeCfg<float, 4, 32, 16>, float, CK>(p, stream, launches);
}

// ---------------------------------------------------------------------------
// Schedule 12: one lane per channel, all 16 states of the channel in the lane.
//
// For shapes with many (sequence, channel) pairs per SM. With a channel's
// states in one lane the readout needs no shuffles, every lane of a warp reads
// a token's B and C rows at one address (one shared-memory wavefront per
// 16-byte load, where the split-lane kernels pay two), and the per-token
// pre-pass (softplus, silu, delta*u) stays in the lane's registers instead of
// going through shared memory. Per token and warp that is 8 broadcast loads
// and 3 two-byte column loads against 16 warp-wide ex2, about half the
// shared-memory wavefronts per exponential of the 8-state kernel. The price is
// a longer chain: a lane walks all 16 exponentials of each token, so one
// sequence takes twice as long as with 8 states per lane, and the kernel needs
// enough (sequence, channel) pairs to fill the SMs (the packed workload has
// 43 x 5120).
//
// A CTA of 128 lanes owns one sequence and 128 channels. Raw u, dt, z tiles
// (TCH x 128) and B, C rows (TCH x 16) arrive by TMA (plain per-CTA copies of
// this GPU's memory, no multicast) into one of RS stages; chunk j is issued
// after the barrier that ends iteration j - RS, so RS - 1 chunks are in
// flight. Iteration k runs chunk k's tokens straight from its raw stage and
// its fp32 B and C rows, then widens chunk k+1's B and C rows to fp32 (bf16
// inputs; fp32 rows are read from the raw stage), then one CTA barrier.
// Tokens past the sequence end get delta = 0 and delta*u = 0 (the state is
// unchanged) and are not stored.
template <typename T, int TCH_, int RS_, int MINB_>
struct WideCfg {
    static constexpr int CH = 128, THREADS = 128, TCH = TCH_, RS = RS_, MINB = MINB_;
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CH;
    static constexpr size_t RAW_BC = sizeof(T) * TCH * kN;
    static constexpr size_t STAGE = 3 * align128(RAW_ACT) + 2 * align128(RAW_BC);
    static constexpr size_t BCF = 4 * (size_t)TCH * kN;   // one chunk's B (or C) rows in fp32
    static constexpr size_t OFF_B = RS * STAGE;
    static constexpr size_t OFF_C = OFF_B + 2 * BCF;
    static constexpr size_t OFF_BAR = align128(OFF_C + 2 * BCF);
    static constexpr size_t SMEM = OFF_BAR + 8 * RS;
    // B or C elements one thread widens per chunk (threads 0-63: B, 64-127: C)
    static constexpr int EPT = TCH * kN / (THREADS / 2);
    static_assert(TCH % 2 == 0, "token pairs");
    static_assert(sizeof(T) == 4 || EPT == 4 || EPT == 8, "8- or 16-byte raw B and C pieces");
    static_assert(RAW_ACT % 128 == 0 && RAW_BC % 128 == 0, "TMA tiles stay 128-byte aligned");
    static_assert(RS >= 2, "at least one chunk in flight");
};

template <class K, typename T, bool SP, bool GZ, bool CK>
struct Wide {
    static constexpr int TCH = K::TCH, CH = K::CH;
    static_assert(TCH % kCkTok == 0, "checkpoints fall on chunk boundaries");
    unsigned char *smem;
    const Params &p;
    int tid;
    int64_t c0, end;
    bool cvalid;
    float dtb, dsk;
    f32x2 A2p[8], hp[8];  // A * log2(e) and the state, two states per register
    float *ckb;  // this lane's state checkpoints for the backward pass, or null

    // The lane's 16 states as checkpoint j of its sequence (the state before
    // the sequence's token 8j).
    __device__ __forceinline__ void store_ckpt(int64_t j) const
    {
        float4 *dst = reinterpret_cast<float4 *>(ckb + j * p.D * kN);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 v;
            upk2(hp[2 * q], v.x, v.y);
            upk2(hp[2 * q + 1], v.z, v.w);
            dst[q] = v;
        }
    }

    __device__ __forceinline__ Wide(unsigned char *s, const Params &p_) : smem(s), p(p_) {}

    __device__ __forceinline__ T *raw(int stage, int which) const
    {
        size_t off = (size_t)stage * K::STAGE;
        off += which < 3 ? (size_t)which * align128(K::RAW_ACT)
                         : 3 * align128(K::RAW_ACT) + (size_t)(which - 3) * align128(K::RAW_BC);
        return reinterpret_cast<T *>(smem + off);
    }
    // fp32 B (which 0) or C (which 1) rows of the chunk in `stage` / buffer `buf`
    __device__ __forceinline__ const float *bc(int which, int buf, int stage) const
    {
        if constexpr (sizeof(T) == 4) {
            (void)buf;
            return reinterpret_cast<const float *>(raw(stage, 3 + which));
        } else {
            (void)stage;
            return reinterpret_cast<const float *>(smem + (which ? K::OFF_C : K::OFF_B) + buf * K::BCF);
        }
    }

    // B and C rows of the chunk in `stage` to fp32 buffer BUF (bf16 only).
    template <int BUF>
    __device__ __forceinline__ void widen(int stage) const
    {
        if constexpr (sizeof(T) == 2) {
            const int which = tid >= K::THREADS / 2, i = tid & (K::THREADS / 2 - 1);
            const uint32_t *src = reinterpret_cast<const uint32_t *>(raw(stage, 3 + which)) + i * (K::EPT / 2);
            float *dst = reinterpret_cast<float *>(smem + (which ? K::OFF_C : K::OFF_B) + BUF * K::BCF) +
                         i * K::EPT;
            if constexpr (K::EPT == 4) {
                const uint2 v = *reinterpret_cast<const uint2 *>(src);
                *reinterpret_cast<float4 *>(dst) = make_float4(
                    __uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                    __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
            } else {
                const uint4 v = *reinterpret_cast<const uint4 *>(src);
                *reinterpret_cast<float4 *>(dst) = make_float4(
                    __uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                    __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(
                    __uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                    __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
            }
        } else {
            (void)stage;
        }
    }

    // One token: 16 exponentials, the state update, the readout, skip, gate.
    __device__ __forceinline__ float token(float d, float du, const float *b, const float *c)
    {
        const f32x2 dv = pk2(d, d), xv = pk2(du, du);
        f32x2 bb[8], cc[8];
#pragma unroll
        for (int j = 0; j < 8; j += 2) lds_2x2(b + 2 * j, bb[j], bb[j + 1]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a0, a1;
            upk2(mul2(dv, A2p[j]), a0, a1);
            hp[j] = fma2(pk2(ex2_approx(a0), ex2_approx(a1)), hp[j], mul2(xv, bb[j]));
        }
#pragma unroll
        for (int j = 0; j < 8; j += 2) lds_2x2(c + 2 * j, cc[j], cc[j + 1]);
        f32x2 acc0 = mul2(cc[0], hp[0]), acc1 = mul2(cc[1], hp[1]);
#pragma unroll
        for (int j = 2; j < 8; j += 2) {
            acc0 = fma2(cc[j], hp[j], acc0);
            acc1 = fma2(cc[j + 1], hp[j + 1], acc1);
        }
        float s0, s1;
        upk2(add2(acc0, acc1), s0, s1);
        return s0 + s1;
    }

    // The tokens of chunk k (nt valid, starting at t0) from raw stage `stage`
    // and B/C buffer BUF; kc: the checkpoint index of the chunk's first token.
    template <int BUF, bool MASK>
    __device__ __forceinline__ void chunk(int stage, int64_t t0, int nt, int64_t kc)
    {
        const T *rU = raw(stage, 0), *rDT = raw(stage, 1), *rZ = raw(stage, 2);
        const float *b = bc(0, BUF, stage), *c = bc(1, BUF, stage);
        T *dst = static_cast<T *>(p.y) + t0 * p.D + c0;
        // one token pair per trip: unrolled further, the compiler hoists the
        // B and C rows of later tokens (174 registers at two pairs per trip,
        // 255 and spills at a full chunk), which leaves two CTAs per SM
        // instead of three, and ran slower (packed workload 0.62 against
        // 0.68 of the ex2 peak)
#pragma unroll 1
        for (int t = 0; t < TCH; t += 2) {
            const f32x2 v = add2(pk2(raw_f32(rDT + t * CH + tid), raw_f32(rDT + (t + 1) * CH + tid)),
                                 pk2(dtb, dtb));
            const f32x2 u = pk2(raw_f32(rU + t * CH + tid), raw_f32(rU + (t + 1) * CH + tid));
            f32x2 d, gt = pk2(1.0f, 1.0f);
            if (SP && GZ) {
                softplus_silu2(v, pk2(raw_f32(rZ + t * CH + tid), raw_f32(rZ + (t + 1) * CH + tid)), d, gt);
            } else if (SP) {
                d = softplus2p(v);
            } else {
                d = v;
                if (GZ) gt = silu2p(pk2(raw_f32(rZ + t * CH + tid), raw_f32(rZ + (t + 1) * CH + tid)));
            }
            float d0, d1, x0, x1, s0, s1, g0, g1;
            upk2(d, d0, d1);
            upk2(mul2(d, u), x0, x1);
            upk2(mul2(pk2(dsk, dsk), u), s0, s1);
            upk2(gt, g0, g1);
            if (MASK) {
                d0 = t < nt ? d0 : 0.f;
                x0 = t < nt ? x0 : 0.f;
                d1 = t + 1 < nt ? d1 : 0.f;
                x1 = t + 1 < nt ? x1 : 0.f;
            }
            const float r0 = token(d0, x0, b + t * kN, c + t * kN);
            const float r1 = token(d1, x1, b + (t + 1) * kN, c + (t + 1) * kN);
            const T y0 = from_f32<T>((r0 + s0) * g0), y1 = from_f32<T>((r1 + s1) * g1);
            if (MASK) {
                if (cvalid && t < nt) dst[(int64_t)t * p.D] = y0;
                if (cvalid && t + 1 < nt) dst[(int64_t)(t + 1) * p.D] = y1;
            } else if (cvalid) {
                dst[(int64_t)t * p.D] = y0;
                dst[(int64_t)(t + 1) * p.D] = y1;
            }
            // after every 8th token of the sequence, unless it was the last
            if constexpr (CK) {
                if ((t + 2) % kCkTok == 0 && ckb && t0 + t + 2 < end) store_ckpt(kc + (t + 2) / kCkTok);
            }
        }
    }
};

// RK: the CTAs rank the sequences themselves (no order given, at most
// kRankMax packed sequences); a separate instantiation, so that the kernel
// with an order (or without packing) keeps its own register allocation.
template <class K, typename T, bool SP, bool GZ, bool CK, bool RK>
__global__ void __launch_bounds__(K::THREADS, K::MINB)
scan_wide_kernel(const Params p, const __grid_constant__ Maps m)
{
    constexpr int TCH = K::TCH;
    extern __shared__ __align__(128) unsigned char smem[];
    Wide<K, T, SP, GZ, CK> W(smem, p);
    uint64_t *const bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);
    W.tid = threadIdx.x;
    const int64_t cbase = (int64_t)blockIdx.x * K::CH;
    W.c0 = cbase + W.tid;
    W.cvalid = W.c0 < p.D;
    int64_t seq;
    if constexpr (RK) seq = ranked_seq(p);
    else seq = p.order ? (int64_t)p.order[blockIdx.y] : (int64_t)blockIdx.y;
    seq = seq < 0 ? 0 : (seq >= p.S ? p.S - 1 : seq);
    int64_t start, end;
    if (p.cu) {
        start = clamp_off(p.cu[seq], p.tok);
        end = max(clamp_off(p.cu[seq + 1], p.tok), start);
    } else {
        start = seq * p.L;
        end = start + p.L;
    }
    W.end = end;
    const int nch = (int)((end - start + TCH - 1) / TCH);
    constexpr uint32_t tx_bytes = (uint32_t)((GZ ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);

    if (W.tid == 0) {
#pragma unroll
        for (int st = 0; st < K::RS; ++st) mbar_init(&bar[st]);
    }
    __syncthreads();
    auto issue = [&](int j) {  // TMA of chunk j into stage j % RS
        const int stage = j % K::RS;
        mbar_expect_tx(&bar[stage], tx_bytes);
        const int x = (int)cbase, y = (int)(start + (int64_t)j * TCH);
        tma_2d(W.raw(stage, 0), &m.u, &bar[stage], x, y);
        tma_2d(W.raw(stage, 1), &m.dt, &bar[stage], x, y);
        if (GZ) tma_2d(W.raw(stage, 2), &m.z, &bar[stage], x, y);
        tma_2d(W.raw(stage, 3), &m.b, &bar[stage], 0, y);
        tma_2d(W.raw(stage, 4), &m.c, &bar[stage], 0, y);
    };
    if (W.tid == 0) {
        for (int j = 0; j < K::RS && j < nch; ++j) issue(j);
    }

    if (W.cvalid) {
        const float4 *a4 = reinterpret_cast<const float4 *>(p.A + W.c0 * kN);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 a = __ldg(a4 + q);
            W.A2p[2 * q] = pk2(a.x * kLog2e, a.y * kLog2e);
            W.A2p[2 * q + 1] = pk2(a.z * kLog2e, a.w * kLog2e);
        }
        if (p.h0) {
            const float4 *h4 = reinterpret_cast<const float4 *>(p.h0 + (seq * p.D + W.c0) * kN);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 h = h4[q];
                W.hp[2 * q] = pk2(h.x, h.y);
                W.hp[2 * q + 1] = pk2(h.z, h.w);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) W.hp[j] = 0ull;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            W.A2p[j] = 0ull;
            W.hp[j] = 0ull;
        }
    }
    W.dtb = (W.cvalid && p.dt_bias) ? __ldg(p.dt_bias + W.c0) : 0.f;
    W.dsk = (W.cvalid && p.Dskip) ? __ldg(p.Dskip + W.c0) : 0.f;
    // checkpoint j of sequence `seq` (the state before its token 8j) lives in
    // row floor(start / 8) + seq + j of D x 16 floats: sequences never collide
    W.ckb = (CK && W.cvalid) ? p.ckpt + ((start / kCkTok + seq) * p.D + W.c0) * kN : nullptr;
    if (CK && W.ckb && end > start) W.store_ckpt(0);

    bool failed = false;
    auto wait_raw = [&](int j) {
        mbar_wait(&bar[j % K::RS], (uint32_t)((j / K::RS) & 1), failed, &g_pipe_status, 1);
    };
    if (nch > 0) {
        wait_raw(0);
        W.template widen<0>(0);
    }
    __syncthreads();

    // iteration k: chunk k from stage k % RS and B/C buffer k & 1; then chunk
    // k+1's B and C rows widened into buffer (k+1) & 1
    auto step = [&](auto tag, int k) {
        constexpr int BUF = decltype(tag)::value;
        // stage (k-1) % RS was last read in iteration k-1, before the last barrier
        if (W.tid == 0 && k >= 1 && k - 1 + K::RS < nch) {
            fence_proxy_async();
            issue(k - 1 + K::RS);
        }
        const int64_t t0 = start + (int64_t)k * TCH;
        const int64_t kc = (int64_t)k * (TCH / kCkTok);
        const int nt = (int)min((int64_t)TCH, end - t0);
        if (nt == TCH) W.template chunk<BUF, false>(k % K::RS, t0, TCH, kc);
        else W.template chunk<BUF, true>(k % K::RS, t0, nt, kc);
        if (k + 1 < nch) {
            wait_raw(k + 1);
            W.template widen<BUF ^ 1>((k + 1) % K::RS);
        }
        __syncthreads();
    };
    int k = 0;
    for (; k + 1 < nch; k += 2) {
        step(BufTag<0>{}, k);
        step(BufTag<1>{}, k + 1);
    }
    if (k < nch) step(BufTag<0>{}, k);

    if (p.h_final && W.cvalid) {
        float4 *o4 = reinterpret_cast<float4 *>(p.h_final + (seq * p.D + W.c0) * kN);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 v;
            upk2(W.hp[2 * q], v.x, v.y);
            upk2(W.hp[2 * q + 1], v.z, v.w);
            o4[q] = v;
        }
    }
}

template <class K, typename T, bool SP, bool GZ, bool CK, bool RK>
cudaError_t run_wide_k(const Params &p, const Maps &m, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
    cudaError_t e = cudaFuncSetAttribute(scan_wide_kernel<K, T, SP, GZ, CK, RK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_wide_kernel<K, T, SP, GZ, CK, RK><<<grid, K::THREADS, K::SMEM, stream>>>(p, m);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T, bool SP, bool GZ, bool CK>
cudaError_t run_wide_t(const Params &p, const Maps &m, cudaStream_t stream, int *launches)
{
    if (!p.order && p.cu && p.S > 1 && p.S <= kRankMax)
        return run_wide_k<K, T, SP, GZ, CK, true>(p, m, stream, launches);
    return run_wide_k<K, T, SP, GZ, CK, false>(p, m, stream, launches);
}

template <class K, typename T, bool CK>
cudaError_t run_wide(const Params &p, cudaStream_t stream, int *launches)
{
    Maps m;
    const bool bf = sizeof(T) == 2;
    bool ok = p.tok > 0 && encode_2d(&m.u, p.u, bf, p.D, p.tok, K::CH, K::TCH) &&
              encode_2d(&m.dt, p.delta, bf, p.D, p.tok, K::CH, K::TCH) &&
              encode_2d(&m.b, p.B, bf, kN, p.tok, kN, K::TCH) &&
              encode_2d(&m.c, p.C, bf, kN, p.tok, kN, K::TCH);
    if (ok) {
        if (p.z) ok = encode_2d(&m.z, p.z, bf, p.D, p.tok, K::CH, K::TCH);
        else m.z = m.u;  // never loaded
    }
    if (!ok) return cudaErrorNotSupported;
    if (p.delta_softplus)
        return p.z ? run_wide_t<K, T, true, true, CK>(p, m, stream, launches)
                   : run_wide_t<K, T, true, false, CK>(p, m, stream, launches);
    return p.z ? run_wide_t<K, T, false, true, CK>(p, m, stream, launches)
               : run_wide_t<K, T, false, false, CK>(p, m, stream, launches);
}

// Schedule 12 (one lane per channel); cudaErrorNotSupported when the tensor
// maps cannot be encoded. bf16: 32-token chunks in two stages (60 KB of
// shared memory), 142 registers, three CTAs (12 warps) per SM. Measured on
// the packed and uniform workloads against 16-token chunks in three or four
// stages (0.661-0.669 / 0.628-0.634 of the ex2 peak) and four CTAs per SM
// capped at 128 registers (0.623 / 0.647): 0.684 / 0.657.
template <bool CK>
cudaError_t launch_wide_cfg(const Params &p, bool bf16, cudaStream_t stream, int *launches)
{
    if (bf16) return run_wide<WideCfg<__nv_bfloat16, 32, 2, 3>, __nv_bfloat16, CK>(p, stream, launches);
    return run_wide<WideCfg<float, 16, 3, 2>, float, CK>(p, stream, launches);
}

// This translation unit's status word (-1 when it cannot be read).
inline int read_tu_pipe_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_pipe_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_pipe_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace

}  // namespace ssm
