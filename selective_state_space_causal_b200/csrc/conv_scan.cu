// conv_scan.cu -- fused causal depthwise conv1d + SiLU -> selective scan (sm_100a).
//
// One pass over the packed sequences that computes the conv output xc and
// feeds it straight into the scan, without writing xc to memory and reading it
// back: the mixer's dataflow of "Scaling State-Space Models on Multiple GPUs
// with Tensor Parallelism", Fig. 1 (conv, then the state update), with the
// per-token math of tp_builder.py (TensorRT-Model-Connect, Mamba family),
// _add_mamba_tp_layer, and no flow across a cu_seqlens boundary ("PackMamba",
// abstract). The conv window of each sequence starts from its carried conv
// state (or zeros), and the sequence's last K-1 inputs become its new conv
// state.
//
// The kernel is the register-prefetch scan (schedule 1) with the conv in its
// per-chunk pre-pass: the chunk's raw x rows (prefetched into registers one
// chunk ahead, as u is in the plain scan) sit as fp32 in a shared-memory tile
// below K-1 halo rows (the previous chunk's last inputs, or the carried state
// at a sequence start); each pre-pass item forms its conv output from the
// tile, applies SiLU and proceeds as the plain scan's pre-pass with that value
// as u. Two tiles alternate, so the next chunk's tile is filled during this
// chunk and no extra barrier is needed. The conv takes the same operations in
// the same order as the conv kernel (taps oldest first, bias first, SiLU as
// x * 1/(1 + 2^(-x log2 e))), and xc stays in fp32.
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "scan_parts.cuh"
#include "scan_pipe.cuh"

namespace ssm {

namespace {

struct ConvParams {
    const void *x;          // (tok, D) raw conv input
    const float *w, *bias;  // (D, KW) taps, (D) or null
    const void *state_in;   // (S, D, KW-1) or null (= zeros)
    void *state_out;        // (S, D, KW-1) or null; may be state_in
    void *xc;               // (tok, D) or null: copy of the conv output
};

__device__ __forceinline__ float rcp_fast(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// SiLU as the conv kernels compute it: z * 1/(1 + 2^(-z log2 e)).
__device__ __forceinline__ float conv_silu_f(float z)
{
    return z * rcp_fast(ex2_approx(z * -kLog2e) + 1.f);
}

template <class K, int KW>
struct ConvSmem {
    static constexpr int ROWS = K::TCH + KW - 1;
    static constexpr int RS = K::CH + 4;  // row stride: 16 bytes of padding per row
    static constexpr size_t OFF_X = K::SMEM;                          // fp32 [2][ROWS][RS]
    static constexpr size_t OFF_W = align128(OFF_X + sizeof(float) * 2 * ROWS * RS);
    static constexpr size_t OFF_BIAS = OFF_W + sizeof(float) * K::CH * KW;
    static constexpr size_t SMEM = align128(OFF_BIAS + sizeof(float) * K::CH);
};

template <class K, typename T, typename TS, int KW>
__global__ void __launch_bounds__(K::THREADS)
conv_scan_kernel(const Params p, const ConvParams cp)
{
    constexpr int VEC = K::VEC, IPT = K::IPT, THREADS = K::THREADS, CV = K::CV, TCH = K::TCH;
    constexpr int CH = K::CH;
    using G = ConvSmem<K, KW>;
    using RawT = typename Raw<T, VEC>::type;
    extern __shared__ __align__(128) unsigned char smem[];
    float2 *sDX = reinterpret_cast<float2 *>(smem + K::OFF_DX);
    float2 *sUG = reinterpret_cast<float2 *>(smem + K::OFF_UG);
    float *sB = reinterpret_cast<float *>(smem + K::OFF_B);
    float *sC = reinterpret_cast<float *>(smem + K::OFF_C);
    // tile row r holds position t0 - (KW-1) + r; rows are RS floats apart so
    // that the 16-byte reads of items of different tokens hit different banks
    float *sX = reinterpret_cast<float *>(smem + G::OFF_X);
    float *sW = reinterpret_cast<float *>(smem + G::OFF_W);   // [KW][CH], tap-major
    constexpr int RS = G::RS;
    float *sBias = reinterpret_cast<float *>(smem + G::OFF_BIAS);

    const int tid = threadIdx.x;
    const Lane l = lane_setup<K>(p);
    const T *X = static_cast<const T *>(cp.x);
    const T *DT = static_cast<const T *>(p.delta);
    const T *Z = static_cast<const T *>(p.z);
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    const TS *SIN = static_cast<const TS *>(cp.state_in);
    TS *SOUT = static_cast<TS *>(cp.state_out);
    T *XC = static_cast<T *>(cp.xc);

    // conv taps and bias of the CTA's channels; the carried state as halo rows
    for (int e = tid; e < CH * KW; e += THREADS) {
        const int k = e / CH;
        const int64_t c = l.cbase + e % CH;
        sW[e] = c < p.D ? __ldg(cp.w + c * KW + k) : 0.f;
    }
    for (int e = tid; e < CH; e += THREADS) {
        const int64_t c = l.cbase + e;
        sBias[e] = (c < p.D && cp.bias) ? __ldg(cp.bias + c) : 0.f;
    }
    for (int e = tid; e < (KW - 1) * CH; e += THREADS) {
        const int r = e / CH, cl = e % CH;
        const int64_t c = l.cbase + cl;
        sX[r * RS + cl] = (SIN && c < p.D) ? to_f32(SIN[(l.seq * p.D + c) * (KW - 1) + r]) : 0.f;
    }

    f32x2 A2p[K::NPT / 2], hp[K::NPT / 2];
    load_state<K>(p, l, A2p, hp);
    const float dsk = (l.cvalid && p.Dskip) ? __ldg(p.Dskip + l.c0) : 0.f;
    float dtb[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) dtb[i] = (l.vvalid && p.dt_bias) ? __ldg(p.dt_bias + l.cg + i) : 0.f;
    const int cvl = l.cvl * VEC;  // this thread's first channel within the CTA

    RawT rdt[IPT], rx[IPT], rz[IPT];
    uint4 rb[K::BPT], rc[K::BPT];
    auto prefetch = [&](int64_t t0) {
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int64_t row = t0 + (tid + i * THREADS) / CV;
            if (row < l.end && l.vvalid) {
                const int64_t off = row * p.D + l.cg;
                rdt[i] = ld_raw<T, VEC>(DT + off);
                rx[i] = ld_raw<T, VEC>(X + off);
                if (Z) rz[i] = ld_raw<T, VEC>(Z + off);
            }
        }
#pragma unroll
        for (int i = 0; i < K::BPT; ++i) {
            const int q = tid + i * THREADS;
            const int64_t row = t0 + (q * K::BCVEC) / kN;
            if (q < K::BCN && row < l.end) {
                const int64_t off = t0 * kN + (int64_t)q * K::BCVEC;
                rb[i] = ldg16(Bp + off);
                rc[i] = ldg16(Cp + off);
            }
        }
    };

    // Two tiles: chunk k convolves from tile k mod 2 and fills tile (k+1) mod 2
    // for the next chunk (its halo rows from chunk k's last inputs during the
    // pre-pass, its own rows from the prefetched registers after the
    // recurrence), so the chunk needs no barrier beyond the scan's own.
    float *const tile0 = sX, *const tile1 = sX + G::ROWS * RS;
    auto put = [&](float *row, const float (&fx)[VEC]) {
        if constexpr (VEC % 4 == 0) {
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4 *>(row + e) = make_float4(fx[e], fx[e + 1], fx[e + 2], fx[e + 3]);
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) row[e] = fx[e];
        }
    };
    // the raw x rows of the chunk starting at t1 (prefetched) into a tile
    auto put_chunk = [&](float *tile, int64_t t1) {
        const int n1 = (int)min((int64_t)TCH, l.end - t1);
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int tl = (tid + i * THREADS) / CV;
            float fx[VEC];
            if (tl < n1 && l.vvalid) unpack<T, VEC>(rx[i], fx);
            else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) fx[e] = 0.f;
            }
            put(tile + (KW - 1 + tl) * RS + cvl, fx);
        }
    };

    int nt_last = 0;
    float *tile_last = tile0;
    if (l.start < l.end) {
        prefetch(l.start);
        put_chunk(tile0, l.start);
    }
    __syncthreads();  // taps, bias, carried state and the first chunk's rows are staged
    float wr[KW][VEC], br[VEC];  // this thread's taps and bias (its channel vector is fixed)
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        br[e] = sBias[cvl + e];
#pragma unroll
        for (int k = 0; k < KW; ++k) wr[k][e] = sW[k * CH + cvl + e];
    }
    int cur = 0;
    for (int64_t t0 = l.start; t0 < l.end; t0 += TCH) {
        const int nt = (int)min((int64_t)TCH, l.end - t0);
        const bool more = t0 + TCH < l.end;  // then this chunk is full (nt = TCH >= KW - 1)
        float *tc = cur ? tile1 : tile0, *tn = cur ? tile0 : tile1;
        nt_last = nt;
        tile_last = tc;
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int tl = (tid + i * THREADS) / CV;
            float fdt[VEC], fu[VEC], fz[VEC];
            const bool live = tl < nt && l.vvalid;
            if (live) {
                unpack<T, VEC>(rdt[i], fdt);
                if (Z) unpack<T, VEC>(rz[i], fz);
                float win[KW][VEC];
#pragma unroll
                for (int k = 0; k < KW; ++k) {
                    const float *src = tc + (tl + k) * RS + cvl;
                    if constexpr (VEC % 4 == 0) {
#pragma unroll
                        for (int e = 0; e < VEC; e += 4) {
                            const float4 v4 = *reinterpret_cast<const float4 *>(src + e);
                            win[k][e] = v4.x; win[k][e + 1] = v4.y;
                            win[k][e + 2] = v4.z; win[k][e + 3] = v4.w;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < VEC; ++e) win[k][e] = src[e];
                    }
                }
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    float acc = br[e];
#pragma unroll
                    for (int k = 0; k < KW; ++k) acc = fmaf(wr[k][e], win[k][e], acc);
                    fu[e] = conv_silu_f(acc);
                }
                if (XC) store_vec<T, VEC>(XC + (t0 + tl) * p.D + l.cg, fu);
                // the next chunk's halo rows: this chunk's last KW-1 inputs
                if (more && tl >= nt - (KW - 1)) put(tn + (tl - (nt - (KW - 1))) * RS + cvl, win[KW - 1]);
            } else if (more && tl >= nt - (KW - 1)) {
                float zero[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) zero[e] = 0.f;
                put(tn + (tl - (nt - (KW - 1))) * RS + cvl, zero);
            }
            prepass_item<VEC>(sDX + tl * K::ROW2 + l.vcol, sUG + tl * K::ROW2 + l.vcol, live, fdt,
                              fu, fz, Z != nullptr, dtb, p.delta_softplus);
        }
#pragma unroll
        for (int i = 0; i < K::BPT; ++i) {
            const int q = tid + i * THREADS;
            if (q < K::BCN) {
                const int e0 = q * K::BCVEC;
                const bool live = e0 / kN < nt;
                float fb[K::BCVEC], fc[K::BCVEC];
                unpack16<T, K::BCVEC>(rb[i], fb);
                unpack16<T, K::BCVEC>(rc[i], fc);
#pragma unroll
                for (int e = 0; e < K::BCVEC; ++e) {
                    sB[e0 + e] = live ? fb[e] : 0.f;
                    sC[e0 + e] = live ? fc[e] : 0.f;
                }
            }
        }
        __syncthreads();
        if (more) prefetch(t0 + TCH);
        const int ntr = ((nt + K::TPC - 1) / K::TPC) * K::TPC;
        recur_chunk<K>(sDX, sUG, sB, sC, ntr, l.mycol, l.sub, A2p, hp, dsk);
        if (more) put_chunk(tn, t0 + TCH);  // the loads have had the recurrence to land
        __syncthreads();
        store_y<K, T>(static_cast<T *>(p.y), sUG, tid, nt, l.vvalid, l.vcol, t0, p.D, l.cg);
        cur ^= 1;
    }
    save_state<K>(p, l, hp);
    // new conv state: the last KW-1 positions of [carried state || x_seq], which
    // sit in rows nt_last .. nt_last + KW-2 of the last chunk's tile (rows 0.. of
    // the first tile when the sequence is empty); every write to it preceded a
    // barrier
    if (SOUT) {
        for (int e = tid; e < (KW - 1) * CH; e += THREADS) {
            const int j = e / CH, cl = e % CH;
            const int64_t c = l.cbase + cl;
            if (c < p.D)
                SOUT[(l.seq * p.D + c) * (KW - 1) + j] =
                    from_f32<TS>(tile_last[(nt_last + j) * RS + cl]);
        }
    }
}

template <class K, typename T, typename TS, int KW>
cudaError_t run_fused(const Params &p, const ConvParams &cp, cudaStream_t stream, int *launches)
{
    using G = ConvSmem<K, KW>;
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
    cudaError_t e = cudaFuncSetAttribute(conv_scan_kernel<K, T, TS, KW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G::SMEM);
    if (e != cudaSuccess) return e;
    conv_scan_kernel<K, T, TS, KW><<<grid, K::THREADS, G::SMEM, stream>>>(p, cp);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, typename TS, int KW>
cudaError_t by_npt(const Params &p, const ConvParams &cp, int npt, bool vec, cudaStream_t s,
                   int *n)
{
    constexpr int VEC = 16 / sizeof(T);
    if (!vec) return run_fused<Cfg<T, 4, 0, 32, 64, 1>, T, TS, KW>(p, cp, s, n);
    if (npt == 8) return run_fused<Cfg<T, 8, 0, 64, 64, VEC>, T, TS, KW>(p, cp, s, n);
    return run_fused<Cfg<T, 4, 0, 32, 64, VEC>, T, TS, KW>(p, cp, s, n);
}

template <typename T, typename TS>
cudaError_t by_kw(const Params &p, const ConvParams &cp, int K, int npt, bool vec, cudaStream_t s,
                  int *n)
{
    switch (K) {
    case 2: return by_npt<T, TS, 2>(p, cp, npt, vec, s, n);
    case 3: return by_npt<T, TS, 3>(p, cp, npt, vec, s, n);
    default: return by_npt<T, TS, 4>(p, cp, npt, vec, s, n);
    }
}


// ---------------------------------------------------------------------------
// One lane per channel (the scan's schedule 12) with the conv in the lane.
//
// A lane walks its channel's tokens in order, so the conv window is the
// lane's last KW-1 inputs, kept in registers across chunks (the sequence's
// carried conv state at its start): no halo rows and no shared-memory tile.
// Each token's conv output is formed with the conv kernel's operations in its
// order (bias first, taps oldest first, SiLU as x / (1 + 2^(-x log2 e))),
// stays in fp32 as the scan's u and is optionally stored as xc. The rest is
// scan_wide_kernel: raw x, dt, z tiles and B, C rows by TMA in two stages of 32
// tokens, B and C widened to fp32 once per CTA, one lane per channel with all
// 16 states, no shuffles. Packed sequences run longest first: with at most
// kRankMax sequences each CTA ranks the lengths itself (the entry point takes
// no workspace for an order); above that, in index order.

template <class K, typename T, typename TS, int KW>
struct FusedWide {
    static constexpr int TCH = K::TCH, CH = K::CH;
    unsigned char *smem;
    const Params &p;
    const ConvParams &cp;
    int tid;
    int64_t c0;
    bool cvalid, sp, gz;
    float dtb, dsk, cb;
    float cw[KW], win[KW - 1];  // conv taps; the channel's last KW-1 inputs, oldest first
    f32x2 A2p[8], hp[8];        // A * log2(e) and the state, two states per register

    __device__ __forceinline__ FusedWide(unsigned char *s, const Params &p_, const ConvParams &cp_)
        : smem(s), p(p_), cp(cp_) {}

    __device__ __forceinline__ T *raw(int stage, int which) const
    {
        size_t off = (size_t)stage * K::STAGE;
        off += which < 3 ? (size_t)which * align128(K::RAW_ACT)
                         : 3 * align128(K::RAW_ACT) + (size_t)(which - 3) * align128(K::RAW_BC);
        return reinterpret_cast<T *>(smem + off);
    }
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
    template <int BUF>
    __device__ __forceinline__ void widen(int stage) const
    {
        if constexpr (sizeof(T) == 2) {
            const int which = tid >= K::THREADS / 2, i = tid & (K::THREADS / 2 - 1);
            const uint32_t *src = reinterpret_cast<const uint32_t *>(raw(stage, 3 + which)) + i * (K::EPT / 2);
            float *dst = reinterpret_cast<float *>(smem + (which ? K::OFF_C : K::OFF_B) + BUF * K::BCF) +
                         i * K::EPT;
#pragma unroll
            for (int e = 0; e < K::EPT / 2; e += 2)
                *reinterpret_cast<float4 *>(dst + 2 * e) = make_float4(
                    __uint_as_float(src[e] << 16), __uint_as_float(src[e] & 0xffff0000u),
                    __uint_as_float(src[e + 1] << 16), __uint_as_float(src[e + 1] & 0xffff0000u));
        } else {
            (void)stage;
        }
    }

    // One token of the recurrence and its readout (as scan_wide_kernel).
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

    template <int BUF, bool MASK>
    __device__ __forceinline__ void chunk(int stage, int64_t t0, int nt)
    {
        const T *rX = raw(stage, 0), *rDT = raw(stage, 1), *rZ = raw(stage, 2);
        const float *b = bc(0, BUF, stage), *c = bc(1, BUF, stage);
        T *dst = static_cast<T *>(p.y) + t0 * p.D + c0;
        T *xcd = cp.xc ? static_cast<T *>(cp.xc) + t0 * p.D + c0 : nullptr;
#pragma unroll 1
        for (int t = 0; t < TCH; t += 2) {
            // the conv of tokens t and t + 1 over [window, x_t, x_t+1]
            float ext[KW + 1];
#pragma unroll
            for (int k = 0; k < KW - 1; ++k) ext[k] = win[k];
            ext[KW - 1] = raw_f32(rX + t * CH + tid);
            ext[KW] = raw_f32(rX + (t + 1) * CH + tid);
            float a0 = cb, a1 = cb;
#pragma unroll
            for (int k = 0; k < KW; ++k) {
                a0 = fmaf(cw[k], ext[k], a0);
                a1 = fmaf(cw[k], ext[k + 1], a1);
            }
            const float u0 = conv_silu_f(a0), u1 = conv_silu_f(a1);
            const bool l0 = !MASK || t < nt, l1 = !MASK || t + 1 < nt;
#pragma unroll
            for (int k = 0; k < KW - 1; ++k) win[k] = l1 ? ext[k + 2] : (l0 ? ext[k + 1] : ext[k]);

            const f32x2 v = add2(pk2(raw_f32(rDT + t * CH + tid), raw_f32(rDT + (t + 1) * CH + tid)),
                                 pk2(dtb, dtb));
            const f32x2 u = pk2(u0, u1);
            f32x2 d, gt = pk2(1.0f, 1.0f);
            if (sp && gz) {
                softplus_silu2(v, pk2(raw_f32(rZ + t * CH + tid), raw_f32(rZ + (t + 1) * CH + tid)), d, gt);
            } else if (sp) {
                d = softplus2p(v);
            } else {
                d = v;
                if (gz) gt = silu2p(pk2(raw_f32(rZ + t * CH + tid), raw_f32(rZ + (t + 1) * CH + tid)));
            }
            float d0, d1, x0, x1, s0, s1, g0, g1;
            upk2(d, d0, d1);
            upk2(mul2(d, u), x0, x1);
            upk2(mul2(pk2(dsk, dsk), u), s0, s1);
            upk2(gt, g0, g1);
            if (MASK) {
                d0 = l0 ? d0 : 0.f;
                x0 = l0 ? x0 : 0.f;
                d1 = l1 ? d1 : 0.f;
                x1 = l1 ? x1 : 0.f;
            }
            const float r0 = token(d0, x0, b + t * kN, c + t * kN);
            const float r1 = token(d1, x1, b + (t + 1) * kN, c + (t + 1) * kN);
            if (cvalid) {
                if (l0) dst[(int64_t)t * p.D] = from_f32<T>((r0 + s0) * g0);
                if (l1) dst[(int64_t)(t + 1) * p.D] = from_f32<T>((r1 + s1) * g1);
                if (xcd) {
                    if (l0) xcd[(int64_t)t * p.D] = from_f32<T>(u0);
                    if (l1) xcd[(int64_t)(t + 1) * p.D] = from_f32<T>(u1);
                }
            }
        }
    }
};

template <class K, typename T, typename TS, int KW>
__global__ void __launch_bounds__(K::THREADS, K::MINB)
conv_scan_wide_kernel(const Params p, const ConvParams cp, const __grid_constant__ Maps m)
{
    constexpr int TCH = K::TCH;
    extern __shared__ __align__(128) unsigned char smem[];
    FusedWide<K, T, TS, KW> W(smem, p, cp);
    uint64_t *const bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);
    W.tid = threadIdx.x;
    const int64_t cbase = (int64_t)blockIdx.x * K::CH;
    W.c0 = cbase + W.tid;
    W.cvalid = W.c0 < p.D;
    W.sp = p.delta_softplus != 0;
    W.gz = p.z != nullptr;

    // longest first (ranked by the CTA when there is no order and at most
    // kRankMax sequences)
    int64_t seq = ranked_seq(p);
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
    const uint32_t tx_bytes = (uint32_t)((W.gz ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);

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
        if (W.gz) tma_2d(W.raw(stage, 2), &m.z, &bar[stage], x, y);
        tma_2d(W.raw(stage, 3), &m.b, &bar[stage], 0, y);
        tma_2d(W.raw(stage, 4), &m.c, &bar[stage], 0, y);
    };
    if (W.tid == 0) {
        for (int j = 0; j < K::RS && j < nch; ++j) issue(j);
    }

    const TS *SIN = static_cast<const TS *>(cp.state_in);
    TS *SOUT = static_cast<TS *>(cp.state_out);
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
#pragma unroll
        for (int k = 0; k < KW; ++k) W.cw[k] = __ldg(cp.w + W.c0 * KW + k);
#pragma unroll
        for (int k = 0; k < KW - 1; ++k)
            W.win[k] = SIN ? to_f32(SIN[(seq * p.D + W.c0) * (KW - 1) + k]) : 0.f;
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            W.A2p[j] = 0ull;
            W.hp[j] = 0ull;
        }
#pragma unroll
        for (int k = 0; k < KW; ++k) W.cw[k] = 0.f;
#pragma unroll
        for (int k = 0; k < KW - 1; ++k) W.win[k] = 0.f;
    }
    W.cb = (W.cvalid && cp.bias) ? __ldg(cp.bias + W.c0) : 0.f;
    W.dtb = (W.cvalid && p.dt_bias) ? __ldg(p.dt_bias + W.c0) : 0.f;
    W.dsk = (W.cvalid && p.Dskip) ? __ldg(p.Dskip + W.c0) : 0.f;

    bool failed = false;
    auto wait_raw = [&](int j) {
        mbar_wait(&bar[j % K::RS], (uint32_t)((j / K::RS) & 1), failed, &g_pipe_status, 1);
    };
    if (nch > 0) {
        wait_raw(0);
        W.template widen<0>(0);
    }
    __syncthreads();

    auto step = [&](auto tag, int k) {
        constexpr int BUF = decltype(tag)::value;
        // stage (k-1) % RS was last read in iteration k-1, before the last barrier
        if (W.tid == 0 && k >= 1 && k - 1 + K::RS < nch) {
            fence_proxy_async();
            issue(k - 1 + K::RS);
        }
        const int64_t t0 = start + (int64_t)k * TCH;
        const int nt = (int)min((int64_t)TCH, end - t0);
        if (nt == TCH) W.template chunk<BUF, false>(k % K::RS, t0, TCH);
        else W.template chunk<BUF, true>(k % K::RS, t0, nt);
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

    if (W.cvalid) {
        if (p.h_final) {
            float4 *o4 = reinterpret_cast<float4 *>(p.h_final + (seq * p.D + W.c0) * kN);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float4 v;
                upk2(W.hp[2 * q], v.x, v.y);
                upk2(W.hp[2 * q + 1], v.z, v.w);
                o4[q] = v;
            }
        }
        // the sequence's last KW-1 inputs (the carried state where it is
        // shorter); the lane read its own entries of the input state above
        if (SOUT) {
#pragma unroll
            for (int k2 = 0; k2 < KW - 1; ++k2)
                SOUT[(seq * p.D + W.c0) * (KW - 1) + k2] = from_f32<TS>(W.win[k2]);
        }
    }
}

template <class K, typename T, typename TS, int KW>
cudaError_t run_fused_wide(const Params &p, const ConvParams &cp, cudaStream_t stream, int *launches)
{
    Maps m;
    const bool bf = sizeof(T) == 2;
    bool ok = p.tok > 0 && encode_2d(&m.u, cp.x, bf, p.D, p.tok, K::CH, K::TCH) &&
              encode_2d(&m.dt, p.delta, bf, p.D, p.tok, K::CH, K::TCH) &&
              encode_2d(&m.b, p.B, bf, kN, p.tok, kN, K::TCH) &&
              encode_2d(&m.c, p.C, bf, kN, p.tok, kN, K::TCH);
    if (ok) {
        if (p.z) ok = encode_2d(&m.z, p.z, bf, p.D, p.tok, K::CH, K::TCH);
        else m.z = m.u;  // never loaded
    }
    if (!ok) return cudaErrorNotSupported;
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
    cudaError_t e = cudaFuncSetAttribute(conv_scan_wide_kernel<K, T, TS, KW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM);
    if (e != cudaSuccess) return e;
    conv_scan_wide_kernel<K, T, TS, KW><<<grid, K::THREADS, K::SMEM, stream>>>(p, cp, m);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, typename TS>
cudaError_t wide_by_kw(const Params &p, const ConvParams &cp, int KW, cudaStream_t s, int *n)
{
    using K = std::conditional_t<sizeof(T) == 2, WideCfg<__nv_bfloat16, 32, 2, 3>, WideCfg<float, 16, 3, 2>>;
    switch (KW) {
    case 2: return run_fused_wide<K, T, TS, 2>(p, cp, s, n);
    case 3: return run_fused_wide<K, T, TS, 3>(p, cp, s, n);
    default: return run_fused_wide<K, T, TS, 4>(p, cp, s, n);
    }
}

}  // namespace

struct ConvScanArgs {
    const void *x;
    const float *w, *bias;
    const void *state_in;
    void *state_out;
    void *xc;
    int K;
    DType state_dtype;
    ScanArgs scan;
};

// This translation unit's status word of bounded TMA waits (-1 when it
// cannot be read).
int read_conv_scan_status(bool clear) { return read_tu_pipe_status(clear); }

// The fused kernel: one lane per channel where the scan would take schedule
// 12 and every row is 16-byte aligned; else 16-byte channel vectors (4 or 8
// states per lane, as the scan's variant choice says) where every row is
// 16-byte aligned, else scalar channels with 4 states per lane.
cudaError_t launch_conv_scan(const ConvScanArgs &a, int npt, int sched, cudaStream_t stream,
                             int *launches)
{
    const ScanArgs &s = a.scan;
    if (s.S == 0) return cudaSuccess;
    const size_t es = s.dtype == DType::BF16 ? 2 : 4;
    const uintptr_t mis = (uintptr_t)a.x | (uintptr_t)s.delta | (uintptr_t)s.z | (uintptr_t)s.y |
                          (uintptr_t)a.xc;
    const bool vec = mis % 16 == 0 && (s.D * (int64_t)es) % 16 == 0;
    Params p;
    p.u = a.x; p.delta = s.delta; p.B = s.B; p.C = s.C; p.z = s.z;
    p.A = s.A; p.Dskip = s.Dskip; p.dt_bias = s.dt_bias; p.h0 = s.h0;
    p.cu = s.cu; p.order = nullptr; p.y = s.y; p.h_final = s.h_final;  // sequences in index order
    p.S = s.S; p.tok = s.tok; p.D = s.D; p.L = s.cu ? 0 : s.tok / s.S;
    p.delta_softplus = s.delta_softplus;
    ConvParams cp{a.x, a.w, a.bias, a.state_in, a.state_out, a.xc};
    const bool xb = s.dtype == DType::BF16, sb = a.state_dtype == DType::BF16;
    if (sched == 12 && vec && s.tok > 0) {
        cudaError_t e;
        if (xb && sb) e = wide_by_kw<__nv_bfloat16, __nv_bfloat16>(p, cp, a.K, stream, launches);
        else if (xb) e = wide_by_kw<__nv_bfloat16, float>(p, cp, a.K, stream, launches);
        else if (sb) e = wide_by_kw<float, __nv_bfloat16>(p, cp, a.K, stream, launches);
        else e = wide_by_kw<float, float>(p, cp, a.K, stream, launches);
        if (e != cudaErrorNotSupported) return e;
    }
    if (xb && sb) return by_kw<__nv_bfloat16, __nv_bfloat16>(p, cp, a.K, npt, vec, stream, launches);
    if (xb) return by_kw<__nv_bfloat16, float>(p, cp, a.K, npt, vec, stream, launches);
    if (sb) return by_kw<float, __nv_bfloat16>(p, cp, a.K, npt, vec, stream, launches);
    return by_kw<float, float>(p, cp, a.K, npt, vec, stream, launches);
}

}  // namespace ssm
