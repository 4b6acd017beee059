// scan_parts.cuh -- pieces of the register-prefetch selective scan (schedule 1)
// shared by the scan kernels (scan.cu) and the fused conv -> scan kernel
// (conv_scan.cu): launch parameters, the tile configuration, the cooperative
// pre-pass, the recurrence over a staged chunk with its transposed-butterfly
// readout, the output pass, and the per-lane state load and store.
//
// The math is that of tp_builder.py (TensorRT-Model-Connect, Mamba family),
// _add_mamba_tp_layer: delta = softplus(dt + dt_bias), dA = exp(delta A),
// h = dA h + delta u B, y = (C . h + Dskip u) silu(z).
#pragma once

#include "common.cuh"

namespace ssm {

// Launch parameters of every forward scan kernel (external linkage: the
// schedules live in more than one translation unit).
struct Params {
    const void *u, *delta, *B, *C, *z;
    const float *A, *Dskip, *dt_bias, *h0;
    const int32_t *cu;
    const int32_t *order;
    void *y;
    float *h_final;
    int64_t S, tok, D, L;
    int delta_softplus;
    // the state before every 8th token of each sequence, for the backward
    // pass (written by the pipelined kernel only), or null
    float *ckpt = nullptr;
};

namespace {

constexpr int kN = 16;

constexpr size_t align128(size_t v) { return (v + 127) / 128 * 128; }

template <typename T, int NPT_, int BATCH_, int CH_, int TCH_, int VEC_>
struct Cfg {
    static constexpr int NPT = NPT_, BATCH = BATCH_, CH = CH_, TCH = TCH_, VEC = VEC_;
    static constexpr int TPC = kN / NPT;                  // lanes per channel
    static constexpr int THREADS = CH * TPC;
    static constexpr int CV = CH / VEC;                   // channel vectors per row
    static constexpr int ITEMS = TCH * CV;                // (token, vector) items per chunk
    static constexpr int IPT = (ITEMS + THREADS - 1) / THREADS;  // items per thread (last partial)
    static constexpr int ROW2 = CH + 2 * (CH / 16);       // padded smem row, in float2
    static constexpr int BCVEC = 16 / sizeof(T);          // B/C elements per 16 bytes
    static constexpr int BCN = TCH * kN / BCVEC;          // 16-byte B (or C) pieces per chunk
    static constexpr int BPT = (BCN + THREADS - 1) / THREADS;
    // shared memory: derived arrays, then (TMA kernel only) the raw tiles
    static constexpr size_t OFF_DX = 0;
    static constexpr size_t OFF_UG = align128(OFF_DX + sizeof(float2) * TCH * ROW2);
    static constexpr size_t OFF_B = align128(OFF_UG + sizeof(float2) * TCH * ROW2);
    static constexpr size_t OFF_C = align128(OFF_B + sizeof(float) * TCH * kN);
    static constexpr size_t SMEM = align128(OFF_C + sizeof(float) * TCH * kN);
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CH;   // one u / dt / z tile
    static constexpr size_t RAW_BC = sizeof(T) * TCH * kN;    // one B / C tile
    static constexpr size_t OFF_RU = SMEM;
    static constexpr size_t OFF_RDT = OFF_RU + align128(RAW_ACT);
    static constexpr size_t OFF_RZ = OFF_RDT + align128(RAW_ACT);
    static constexpr size_t OFF_RB = OFF_RZ + align128(RAW_ACT);
    static constexpr size_t OFF_RC = OFF_RB + align128(RAW_BC);
    static constexpr size_t OFF_BAR = OFF_RC + align128(RAW_BC);
    static constexpr size_t SMEM_TMA = OFF_BAR + 128;
    static_assert(CH % 16 == 0, "channel tile is a multiple of 16");
    static_assert(NPT % 2 == 0, "states come in packed pairs");
    static_assert(THREADS % CV == 0, "each thread keeps one channel vector");
    static_assert(TCH % TPC == 0, "chunk must hold whole token groups");
    static_assert(THREADS <= 1024 && (THREADS % 32) == 0, "block size");
    static_assert(RAW_ACT % 128 == 0 && RAW_BC % 128 == 0, "TMA tiles stay 128-byte aligned");
};

// Column of channel c in a padded float2 row: 16 B of padding after every 16
// channels keeps both the 16-byte pre-pass stores and the per-token reads free
// of bank conflicts.
__device__ __forceinline__ int col2(int c) { return c + 2 * (c >> 4); }

// Store VEC consecutive float2 values (16-byte aligned when VEC is even).
template <int VEC>
__device__ __forceinline__ void st_pairs(float2 *dst, const float (&a)[VEC], const float (&b)[VEC])
{
    if constexpr (VEC % 2 == 0) {
#pragma unroll
        for (int e = 0; e < VEC; e += 2)
            *reinterpret_cast<float4 *>(dst + e) = make_float4(a[e], b[e], a[e + 1], b[e + 1]);
    } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = make_float2(a[e], b[e]);
    }
}

// Derived per-(token, channel) values of one pre-pass item.
template <int VEC>
__device__ __forceinline__ void prepass_item(float2 *dx_row, float2 *ug_row, bool live,
                                             const float (&fdt)[VEC], const float (&fu)[VEC],
                                             const float (&fz)[VEC], bool has_z,
                                             const float (&dtb)[VEC], int softplus)
{
    float vd[VEC], vdx[VEC], vu[VEC], vg[VEC];
    if constexpr (VEC % 2 == 0) {
        // in pairs, with the exponentials on the FMA pipe: the special-function
        // unit is left to the recurrence's decays
#pragma unroll
        for (int e = 0; e < VEC; e += 2) {
            float d0 = fdt[e] + dtb[e], d1 = fdt[e + 1] + dtb[e + 1];
            if (softplus) softplus2(d0, d1, d0, d1);
            float g0 = 1.f, g1 = 1.f;
            if (has_z) silu2(fz[e], fz[e + 1], g0, g1);
            vd[e] = live ? d0 : 0.f;
            vd[e + 1] = live ? d1 : 0.f;
            vdx[e] = live ? d0 * fu[e] : 0.f;
            vdx[e + 1] = live ? d1 * fu[e + 1] : 0.f;
            vu[e] = live ? fu[e] : 0.f;
            vu[e + 1] = live ? fu[e + 1] : 0.f;
            vg[e] = live ? g0 : 0.f;
            vg[e + 1] = live ? g1 : 0.f;
        }
    } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            float d = fdt[e] + dtb[e];
            if (softplus) d = softplus_fast(d);
            vd[e] = live ? d : 0.f;
            vdx[e] = live ? d * fu[e] : 0.f;
            vu[e] = live ? fu[e] : 0.f;
            vg[e] = live ? (has_z ? silu_f(fz[e]) : 1.f) : 0.f;
        }
    }
    st_pairs<VEC>(dx_row, vd, vdx);
    st_pairs<VEC>(ug_row, vu, vg);
}

// Recurrence over one staged chunk for one lane: NPT states of channel `mycol`
// (padded column), tokens [0, ntr) of the chunk in groups of TPC.
template <class K>
__device__ __forceinline__ void recur_chunk(const float2 *__restrict__ sDX, float2 *sUG,
                                            const float *__restrict__ sB,
                                            const float *__restrict__ sC, int ntr, int mycol,
                                            int sub, const f32x2 (&A2p)[K::NPT / 2],
                                            f32x2 (&hp)[K::NPT / 2], float dsk)
{
    constexpr int NPT = K::NPT, TPC = K::TPC, ROW2 = K::ROW2, NP = K::NPT / 2;
    auto group = [&](const int tt) {
        float yp[TPC];
        if constexpr (K::BATCH) {
            // all exponentials of the group first, then the dependent FMAs
            f32x2 dA[TPC][NP], bx[TPC][NP], cc[TPC][NP];
#pragma unroll
            for (int q = 0; q < TPC; ++q) {
                const int tq = tt + q;
                const float2 v = sDX[tq * ROW2 + mycol];
                const f32x2 dd = pk2(v.x, v.x), xx = pk2(v.y, v.y);
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const float2 b2 = *reinterpret_cast<const float2 *>(sB + tq * kN + sub * NPT + 2 * j);
                    const float2 c2 = *reinterpret_cast<const float2 *>(sC + tq * kN + sub * NPT + 2 * j);
                    float a0, a1;
                    upk2(mul2(dd, A2p[j]), a0, a1);
                    dA[q][j] = pk2(ex2_approx(a0), ex2_approx(a1));
                    bx[q][j] = mul2(xx, pk2(b2.x, b2.y));
                    cc[q][j] = pk2(c2.x, c2.y);
                }
            }
#pragma unroll
            for (int q = 0; q < TPC; ++q) {
                f32x2 acc = 0ull;
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    hp[j] = fma2(dA[q][j], hp[j], bx[q][j]);
                    acc = fma2(cc[q][j], hp[j], acc);
                }
                float s0, s1;
                upk2(acc, s0, s1);
                yp[q] = s0 + s1;
            }
        } else {
#pragma unroll
            for (int q = 0; q < TPC; ++q) {
                const int tq = tt + q;
                const float2 v = sDX[tq * ROW2 + mycol];
                const f32x2 dd = pk2(v.x, v.x), xx = pk2(v.y, v.y);
                f32x2 acc = 0ull;
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const float2 b2 = *reinterpret_cast<const float2 *>(sB + tq * kN + sub * NPT + 2 * j);
                    const float2 c2 = *reinterpret_cast<const float2 *>(sC + tq * kN + sub * NPT + 2 * j);
                    float a0, a1;
                    upk2(mul2(dd, A2p[j]), a0, a1);
                    const f32x2 dA = pk2(ex2_approx(a0), ex2_approx(a1));
                    hp[j] = fma2(dA, hp[j], mul2(xx, pk2(b2.x, b2.y)));
                    acc = fma2(pk2(c2.x, c2.y), hp[j], acc);
                }
                float s0, s1;
                upk2(acc, s0, s1);
                yp[q] = s0 + s1;
            }
        }
        // transposed butterfly: lane `sub` ends with the full sum of token tt+sub
#pragma unroll
        for (int w = TPC / 2; w >= 1; w >>= 1) {
            const bool upper = (sub & w) != 0;
#pragma unroll
            for (int i = 0; i < w; ++i) {
                const float send = upper ? yp[i] : yp[i + w];
                const float keep = upper ? yp[i + w] : yp[i];
                yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
            }
        }
        float2 *q2 = sUG + (tt + sub) * ROW2 + mycol;
        const float2 ug = *q2;
        q2->x = (yp[0] + dsk * ug.x) * ug.y;
    };
    // full chunks run fully unrolled, so one group's loads and exponentials
    // can overlap the previous group's readout butterfly
    if (ntr == K::TCH) {
#pragma unroll
        for (int tt = 0; tt < K::TCH; tt += TPC) group(tt);
    } else {
        for (int tt = 0; tt < ntr; tt += TPC) group(tt);
    }
}

// Writes y for this thread's pre-pass items of the chunk (y sits in sUG.x).
template <class K, typename T>
__device__ __forceinline__ void store_y(T *Y, const float2 *sUG, int tid, int nt, bool vvalid,
                                        int vcol, int64_t t0, int64_t D, int64_t cg)
{
    constexpr int VEC = K::VEC;
#pragma unroll
    for (int i = 0; i < K::IPT; ++i) {
        if (tid + i * K::THREADS >= K::ITEMS) break;
        const int tl = (tid + i * K::THREADS) / K::CV;
        if (tl < nt && vvalid) {
            float out[VEC];
            const float2 *src = sUG + tl * K::ROW2 + vcol;
            if constexpr (VEC % 2 == 0) {
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + e);
                    out[e] = v.x;
                    out[e + 1] = v.z;
                }
            } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) out[e] = src[e].x;
            }
            store_vec<T, VEC>(Y + (t0 + tl) * D + cg, out);
        }
    }
}

// Per-CTA setup shared by both kernels.
struct Lane {
    int64_t seq, start, end, cbase, c0, cg;
    int sub, mycol, cvl, vcol;
    bool cvalid, vvalid;
};

template <class K>
__device__ __forceinline__ Lane lane_setup(const Params &p)
{
    Lane l;
    const int tid = threadIdx.x;
    l.sub = tid % K::TPC;
    const int cl = tid / K::TPC;
    l.cbase = (int64_t)blockIdx.x * K::CH;
    l.c0 = l.cbase + cl;
    l.cvalid = l.c0 < p.D;
    int64_t seq = p.order ? (int64_t)p.order[blockIdx.y] : (int64_t)blockIdx.y;
    l.seq = seq < 0 ? 0 : (seq >= p.S ? p.S - 1 : seq);
    if (p.cu) {
        l.start = clamp_off(p.cu[l.seq], p.tok);
        l.end = max(clamp_off(p.cu[l.seq + 1], p.tok), l.start);
    } else {
        l.start = l.seq * p.L;
        l.end = l.start + p.L;
    }
    l.mycol = col2(cl);
    l.cvl = tid % K::CV;
    l.cg = l.cbase + (int64_t)l.cvl * K::VEC;
    l.vvalid = l.cg < p.D;  // D % VEC == 0 on the vector paths
    l.vcol = col2(l.cvl * K::VEC);
    return l;
}

template <class K>
__device__ __forceinline__ void load_state(const Params &p, const Lane &l, f32x2 (&A2p)[K::NPT / 2],
                                           f32x2 (&hp)[K::NPT / 2])
{
#pragma unroll
    for (int j = 0; j < K::NPT; j += 2) {
        const int64_t ai = l.c0 * kN + l.sub * K::NPT + j;
        const int64_t hi = (l.seq * p.D + l.c0) * kN + l.sub * K::NPT + j;
        A2p[j / 2] = l.cvalid ? pk2(__ldg(p.A + ai) * kLog2e, __ldg(p.A + ai + 1) * kLog2e) : 0ull;
        hp[j / 2] = (l.cvalid && p.h0) ? pk2(p.h0[hi], p.h0[hi + 1]) : 0ull;
    }
}

template <class K>
__device__ __forceinline__ void save_state(const Params &p, const Lane &l,
                                           const f32x2 (&hp)[K::NPT / 2])
{
    if (p.h_final && l.cvalid) {
#pragma unroll
        for (int j = 0; j < K::NPT; j += 2) {
            float lo, hi;
            upk2(hp[j / 2], lo, hi);
            const int64_t o = (l.seq * p.D + l.c0) * kN + l.sub * K::NPT + j;
            p.h_final[o] = lo;
            p.h_final[o + 1] = hi;
        }
    }
}

template <typename T, int VEC> struct Raw { using type = uint4; };
template <typename T> struct Raw<T, 1> { using type = T; };

template <typename T, int VEC>
__device__ __forceinline__ typename Raw<T, VEC>::type ld_raw(const T *p)
{
    if constexpr (VEC == 1) return *p;
    else return ldg16(p);
}

template <typename T, int VEC>
__device__ __forceinline__ void unpack(const typename Raw<T, VEC>::type &r, float (&o)[VEC])
{
    if constexpr (VEC == 1) o[0] = to_f32(r);
    else unpack16<T, VEC>(r, o);
}

}  // namespace
}  // namespace ssm
