// scan.cu -- selective scan over packed variable-length sequences (sm_100a).
//
// Math (tp_builder.py, TensorRT-Model-Connect Mamba family, _add_mamba_tp_layer:
// dt softplus, discretisation, state update, C readout, D skip, silu(z) gate;
// run over each sequence as Fig. 1 of "Scaling State-Space Models on Multiple
// GPUs with Tensor Parallelism" describes; reset at every cu_seqlens boundary as
// in "PackMamba", abstract):
//   delta = softplus(dt + dt_bias)      dA[n] = exp(delta * A[c, n])
//   h[n]  = dA[n] * h[n] + delta * u * B_t[n]
//   y     = (sum_n C_t[n] h[n] + Dskip[c] * u) * silu(z)
//
// Design. The scan is bound by the special-function unit: every (token,
// channel) needs N = 16 exponentials against ~8 bytes of DRAM traffic in bf16,
// so the kernel spends as few issue slots and as little latency as it can on
// anything but the 16 dA exponentials:
//
// * A CTA owns one sequence and CH channels. A channel's 16 states are split
//   over TPC = 16 / NPT adjacent lanes (NPT states each); h stays in fp32
//   registers, two states per packed fp32x2 register, for the whole sequence.
// * The sequence is walked in chunks of TCH tokens. The chunk's tiles of u, dt,
//   z (TCH x CH) and B, C (TCH x 16) are brought into shared memory by TMA
//   (cp.async.bulk.tensor, completion on an mbarrier) one chunk ahead, so no
//   registers are held by loads in flight. Where TMA cannot be used (rows not
//   16-byte aligned) a variant prefetches the next chunk into registers.
// * Each chunk's per-(token, channel) work (softplus, delta*u, silu(z), bf16
//   unpacking) is done once, in a cooperative pre-pass into shared memory.
// * The recurrence runs on packed fp32x2 FMUL/FFMA (sm_100a), one MUFU ex2 per
//   state and token, and the TPC partial readouts are combined with a
//   transposed butterfly over shuffles: after log2(TPC) steps lane `sub` holds
//   the full sum of token `sub` of the group, which it gates and writes back.
// * Tokens past a sequence's end are padded with delta = 0 (dA = 1, no input),
//   which leaves h unchanged, so the inner loop needs no tail branch.
// * Packed sequences are scheduled longest-first when scratch is supplied.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "scan_parts.cuh"
#include "tma.cuh"

namespace ssm {

// Set by a kernel whose bounded wait on a TMA completion gave up.
__device__ int g_scan_status = 0;

namespace {

// ---------------------------------------------------------------------------
// Variant 1: next chunk prefetched into registers (any alignment).
// ---------------------------------------------------------------------------
template <class K, typename T>
__global__ void __launch_bounds__(K::THREADS)
scan_kernel(const Params p)
{
    constexpr int VEC = K::VEC, IPT = K::IPT, THREADS = K::THREADS, CV = K::CV, TCH = K::TCH;
    using RawT = typename Raw<T, VEC>::type;
    extern __shared__ __align__(128) unsigned char smem[];
    float2 *sDX = reinterpret_cast<float2 *>(smem + K::OFF_DX);
    float2 *sUG = reinterpret_cast<float2 *>(smem + K::OFF_UG);
    float *sB = reinterpret_cast<float *>(smem + K::OFF_B);
    float *sC = reinterpret_cast<float *>(smem + K::OFF_C);

    const int tid = threadIdx.x;
    const Lane l = lane_setup<K>(p);
    const T *U = static_cast<const T *>(p.u);
    const T *DT = static_cast<const T *>(p.delta);
    const T *Z = static_cast<const T *>(p.z);
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);

    f32x2 A2p[K::NPT / 2], hp[K::NPT / 2];
    load_state<K>(p, l, A2p, hp);
    const float dsk = (l.cvalid && p.Dskip) ? __ldg(p.Dskip + l.c0) : 0.f;
    float dtb[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) dtb[i] = (l.vvalid && p.dt_bias) ? __ldg(p.dt_bias + l.cg + i) : 0.f;

    RawT rdt[IPT], ru[IPT], rz[IPT];
    uint4 rb[K::BPT], rc[K::BPT];
    auto prefetch = [&](int64_t t0) {
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int64_t row = t0 + (tid + i * THREADS) / CV;
            if (row < l.end && l.vvalid) {
                const int64_t off = row * p.D + l.cg;
                rdt[i] = ld_raw<T, VEC>(DT + off);
                ru[i] = ld_raw<T, VEC>(U + off);
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

    if (l.start < l.end) prefetch(l.start);
    for (int64_t t0 = l.start; t0 < l.end; t0 += TCH) {
        const int nt = (int)min((int64_t)TCH, l.end - t0);
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int tl = (tid + i * THREADS) / CV;
            float fdt[VEC], fu[VEC], fz[VEC];
            const bool live = tl < nt && l.vvalid;
            if (live) {
                unpack<T, VEC>(rdt[i], fdt);
                unpack<T, VEC>(ru[i], fu);
                if (Z) unpack<T, VEC>(rz[i], fz);
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
        if (t0 + TCH < l.end) prefetch(t0 + TCH);
        const int ntr = ((nt + K::TPC - 1) / K::TPC) * K::TPC;
        recur_chunk<K>(sDX, sUG, sB, sC, ntr, l.mycol, l.sub, A2p, hp, dsk);
        __syncthreads();
        store_y<K, T>(static_cast<T *>(p.y), sUG, tid, nt, l.vvalid, l.vcol, t0, p.D, l.cg);
        // The next pre-pass rewrites only slots this thread just read (sUG) or
        // slots no thread reads after the barrier above, so no barrier here.
    }
    save_state<K>(p, l, hp);
}

// ---------------------------------------------------------------------------
// Variant 2: tiles brought in by TMA one chunk ahead (16-byte aligned rows).
// ---------------------------------------------------------------------------
struct Maps {
    CUtensorMap u, dt, z, b, c;
};

// ---------------------------------------------------------------------------
// Schedule 8: the layout and readout of schedule 1 (per-token float2 arrays,
// shuffle-butterfly readout into the gate slot) with the raw tiles brought in
// by TMA instead of register prefetch: one stage, issued as soon as the
// pre-pass has read the previous one. Fewest registers of the staged kernels,
// which suits shapes with few (sequence, channel) pairs.
// ---------------------------------------------------------------------------
template <class K, typename T>
__global__ void __launch_bounds__(K::THREADS)
scan_staged_kernel(const Params p, const __grid_constant__ Maps m, const int has_z)
{
    constexpr int VEC = K::VEC, IPT = K::IPT, THREADS = K::THREADS, CV = K::CV, TCH = K::TCH;
    constexpr int CH = K::CH;
    extern __shared__ __align__(128) unsigned char smem[];
    float2 *sDX = reinterpret_cast<float2 *>(smem + K::OFF_DX);
    float2 *sUG = reinterpret_cast<float2 *>(smem + K::OFF_UG);
    float *sB = reinterpret_cast<float *>(smem + K::OFF_B);
    float *sC = reinterpret_cast<float *>(smem + K::OFF_C);
    T *rU = reinterpret_cast<T *>(smem + K::OFF_RU);
    T *rDT = reinterpret_cast<T *>(smem + K::OFF_RDT);
    T *rZ = reinterpret_cast<T *>(smem + K::OFF_RZ);
    T *rB = reinterpret_cast<T *>(smem + K::OFF_RB);
    T *rC = reinterpret_cast<T *>(smem + K::OFF_RC);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);

    const int tid = threadIdx.x;
    const Lane l = lane_setup<K>(p);
    const uint32_t tx_bytes = (uint32_t)((has_z ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);

    if (tid == 0) mbar_init(bar);
    __syncthreads();
    auto issue = [&](int64_t t0) {
        mbar_expect_tx(bar, tx_bytes);
        const int x = (int)l.cbase, y = (int)t0;
        tma_2d(rU, &m.u, bar, x, y);
        tma_2d(rDT, &m.dt, bar, x, y);
        if (has_z) tma_2d(rZ, &m.z, bar, x, y);
        tma_2d(rB, &m.b, bar, 0, y);
        tma_2d(rC, &m.c, bar, 0, y);
    };
    if (tid == 0 && l.start < l.end) issue(l.start);

    f32x2 A2p[K::NPT / 2], hp[K::NPT / 2];
    load_state<K>(p, l, A2p, hp);
    const float dsk = (l.cvalid && p.Dskip) ? __ldg(p.Dskip + l.c0) : 0.f;
    float dtb[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) dtb[i] = (l.vvalid && p.dt_bias) ? __ldg(p.dt_bias + l.cg + i) : 0.f;

    uint32_t parity = 0;
    bool failed = false;
    for (int64_t t0 = l.start; t0 < l.end; t0 += TCH) {
        const int nt = (int)min((int64_t)TCH, l.end - t0);
        mbar_wait(bar, parity, failed, &g_scan_status, 1);
        parity ^= 1u;
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int tl = (tid + i * THREADS) / CV;
            const int ro = tl * CH + l.cvl * VEC;
            float fdt[VEC], fu[VEC], fz[VEC];
            unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rDT + ro), fdt);
            unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rU + ro), fu);
            if (has_z) unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rZ + ro), fz);
            prepass_item<VEC>(sDX + tl * K::ROW2 + l.vcol, sUG + tl * K::ROW2 + l.vcol,
                              tl < nt && l.vvalid, fdt, fu, fz, has_z != 0, dtb,
                              p.delta_softplus);
        }
#pragma unroll
        for (int i = 0; i < K::BPT; ++i) {
            const int q = tid + i * THREADS;
            if (q < K::BCN) {
                const int e0 = q * K::BCVEC;
                const bool live = e0 / kN < nt;
                float fb[K::BCVEC], fc[K::BCVEC];
                unpack16<T, K::BCVEC>(*reinterpret_cast<const uint4 *>(rB + e0), fb);
                unpack16<T, K::BCVEC>(*reinterpret_cast<const uint4 *>(rC + e0), fc);
#pragma unroll
                for (int e = 0; e < K::BCVEC; ++e) {
                    sB[e0 + e] = live ? fb[e] : 0.f;
                    sC[e0 + e] = live ? fc[e] : 0.f;
                }
            }
        }
        __syncthreads();
        if (tid == 0 && t0 + TCH < l.end) {
            // the raw tiles were read through the generic proxy; order those
            // reads before the next asynchronous-proxy writes into them
            fence_proxy_async();
            issue(t0 + TCH);
        }
        const int ntr = ((nt + K::TPC - 1) / K::TPC) * K::TPC;
        recur_chunk<K>(sDX, sUG, sB, sC, ntr, l.mycol, l.sub, A2p, hp, dsk);
        __syncthreads();
        store_y<K, T>(static_cast<T *>(p.y), sUG, tid, nt, l.vvalid, l.vcol, t0, p.D, l.cg);
    }
    save_state<K>(p, l, hp);
}


// Shapes of the TMA-staged kernel. Per (token, channel) shared memory holds
// (delta, delta, delta*u, delta*u) as one float4, so a lane gets both packed
// operands of its recurrence from one 16-byte load, and TPC partial readouts.
// The raw u, dt, z, B, C tiles are double-buffered: chunk k+1 lands while
// chunk k is computed, and chunk k's u and z stay readable for its output.
template <typename T, int NPT_, int CH_, int TCH_>
struct TmaCfg {
    static constexpr int NPT = NPT_, CH = CH_, TCH = TCH_;
    static constexpr int TPC = kN / NPT, NP = NPT / 2;
    static constexpr int THREADS = CH * TPC;
    static constexpr int VEC = 16 / sizeof(T);
    static constexpr int CV = CH / VEC;
    static constexpr int ITEMS = TCH * CV;
    static constexpr int IPT = (ITEMS + THREADS - 1) / THREADS;
    static constexpr int ROWP = CH + CH / 8;               // float4 per row of sDD
    static constexpr int ROWY = CH * TPC + (CH / 8) * 4;   // floats per row of sYP
    static constexpr int BCN = TCH * kN / VEC;             // 16-byte B (or C) pieces
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CH;
    static constexpr size_t RAW_BC = sizeof(T) * TCH * kN;
    static constexpr size_t STAGE = 3 * align128(RAW_ACT) + 2 * align128(RAW_BC);
    static constexpr size_t OFF_DD = 0;
    static constexpr size_t OFF_YP = align128(OFF_DD + 16 * (size_t)TCH * ROWP);
    static constexpr size_t OFF_B = align128(OFF_YP + 4 * (size_t)TCH * ROWY);
    static constexpr size_t OFF_C = align128(OFF_B + 4 * (size_t)TCH * kN);
    static constexpr size_t OFF_RAW = align128(OFF_C + 4 * (size_t)TCH * kN);
    static constexpr size_t OFF_BAR = OFF_RAW + 2 * STAGE;
    static constexpr size_t SMEM = OFF_BAR + 128;
    static_assert(NPT % 2 == 0 && CH % 8 == 0, "shape");
    static_assert(VEC == 8 || VEC == 4, "16-byte vectors");
    static_assert(THREADS % CV == 0, "each thread keeps one channel vector");
    static_assert(THREADS <= 1024 && THREADS % 32 == 0, "block size");
};

// float4 column of channel c in a padded sDD row (16 B after every 8 channels).
__device__ __forceinline__ int col4(int c) { return c + (c >> 3); }
// float offset of (channel c, lane sub) in a padded sYP row.
template <int TPC>
__device__ __forceinline__ int coly(int c, int sub) { return c * TPC + sub + 4 * (c >> 3); }

template <class K, typename T>
__global__ void __launch_bounds__(K::THREADS)
scan_tma_kernel(const Params p, const __grid_constant__ Maps m, const int has_z)
{
    constexpr int NPT = K::NPT, NP = K::NP, TPC = K::TPC, CH = K::CH, TCH = K::TCH;
    constexpr int VEC = K::VEC, CV = K::CV, IPT = K::IPT, THREADS = K::THREADS;
    constexpr int ROWP = K::ROWP, ROWY = K::ROWY;
    extern __shared__ __align__(128) unsigned char smem[];
    float4 *sDD = reinterpret_cast<float4 *>(smem + K::OFF_DD);
    float *sYP = reinterpret_cast<float *>(smem + K::OFF_YP);
    float *sB = reinterpret_cast<float *>(smem + K::OFF_B);
    float *sC = reinterpret_cast<float *>(smem + K::OFF_C);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);
    auto raw = [&](int stage, int which) -> T * {
        size_t off = K::OFF_RAW + (size_t)stage * K::STAGE;
        off += which < 3 ? (size_t)which * align128(K::RAW_ACT)
                         : 3 * align128(K::RAW_ACT) + (size_t)(which - 3) * align128(K::RAW_BC);
        return reinterpret_cast<T *>(smem + off);
    };  // which: 0 u, 1 dt, 2 z, 3 B, 4 C

    const int tid = threadIdx.x;
    const int cl = tid / TPC, sub = tid % TPC;
    const int64_t cbase = (int64_t)blockIdx.x * CH;
    const int64_t c0 = cbase + cl;
    const bool cvalid = c0 < p.D;
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
    const uint32_t tx_bytes = (uint32_t)((has_z ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);

    if (tid == 0) {
        mbar_init(&bar[0]);
        mbar_init(&bar[1]);
    }
    __syncthreads();
    auto issue = [&](int64_t t0, int stage) {
        mbar_expect_tx(&bar[stage], tx_bytes);
        const int x = (int)cbase, y = (int)t0;
        tma_2d(raw(stage, 0), &m.u, &bar[stage], x, y);
        tma_2d(raw(stage, 1), &m.dt, &bar[stage], x, y);
        if (has_z) tma_2d(raw(stage, 2), &m.z, &bar[stage], x, y);
        tma_2d(raw(stage, 3), &m.b, &bar[stage], 0, y);
        tma_2d(raw(stage, 4), &m.c, &bar[stage], 0, y);
    };
    if (tid == 0 && start < end) issue(start, 0);

    // recurrence lane: A * log2(e) and the state, two states per register
    f32x2 A2p[NP], hp[NP];
#pragma unroll
    for (int j = 0; j < NPT; j += 2) {
        const int64_t ai = c0 * kN + sub * NPT + j;
        const int64_t hi = (seq * p.D + c0) * kN + sub * NPT + j;
        A2p[j / 2] = cvalid ? pk2(__ldg(p.A + ai) * kLog2e, __ldg(p.A + ai + 1) * kLog2e) : 0ull;
        hp[j / 2] = (cvalid && p.h0) ? pk2(p.h0[hi], p.h0[hi + 1]) : 0ull;
    }
    const int mycol = col4(cl);
    const int myy = coly<TPC>(cl, sub);

    // pre-pass / output lane: one 16-byte channel vector
    const int cvl = tid % CV;
    const int64_t cg = cbase + (int64_t)cvl * VEC;
    const bool vvalid = cg < p.D;
    float dtb[VEC], dsk[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        dtb[i] = (vvalid && p.dt_bias) ? __ldg(p.dt_bias + cg + i) : 0.f;
        dsk[i] = (vvalid && p.Dskip) ? __ldg(p.Dskip + cg + i) : 0.f;
    }
    const int vcol = col4(cvl * VEC);
    const int vy = coly<TPC>(cvl * VEC, 0);

    bool failed = false;
    int k = 0;
    for (int64_t t0 = start; t0 < end; t0 += TCH, ++k) {
        const int stage = k & 1;
        const int nt = (int)min((int64_t)TCH, end - t0);
        mbar_wait(&bar[stage], (uint32_t)((k >> 1) & 1), failed, &g_scan_status, 1);

        // ---- pre-pass: (delta, delta, delta*u, delta*u) per (token, channel) ----
        const T *rU = raw(stage, 0), *rDT = raw(stage, 1);
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int tl = (tid + i * THREADS) / CV;
            const bool live = tl < nt && vvalid;
            float fdt[VEC], fu[VEC];
            unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rDT + tl * CH + cvl * VEC), fdt);
            unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rU + tl * CH + cvl * VEC), fu);
            float4 *dst = sDD + tl * ROWP + vcol;
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                float d0 = fdt[e] + dtb[e], d1 = fdt[e + 1] + dtb[e + 1];
                if (p.delta_softplus) softplus2(d0, d1, d0, d1);
                d0 = live ? d0 : 0.f;
                d1 = live ? d1 : 0.f;
                float x0, x1;
                upk2(mul2(pk2(d0, d1), pk2(fu[e], fu[e + 1])), x0, x1);
                dst[e] = make_float4(d0, d0, x0, x0);
                dst[e + 1] = make_float4(d1, d1, x1, x1);
            }
        }
        {
            const T *rB = raw(stage, 3), *rC = raw(stage, 4);
            for (int q = tid; q < K::BCN; q += THREADS) {
                const int e0 = q * VEC;
                const bool live = e0 / kN < nt;
                float fb[VEC], fc[VEC];
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rB + e0), fb);
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rC + e0), fc);
#pragma unroll
                for (int e = 0; e < VEC; e += 4) {
                    *reinterpret_cast<float4 *>(sB + e0 + e) = live
                        ? make_float4(fb[e], fb[e + 1], fb[e + 2], fb[e + 3])
                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4 *>(sC + e0 + e) = live
                        ? make_float4(fc[e], fc[e + 1], fc[e + 2], fc[e + 3])
                        : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && t0 + TCH < end) {
            // the other stage was last read by the previous chunk's output pass,
            // which every thread finished before the barrier above
            fence_proxy_async();
            issue(t0 + TCH, stage ^ 1);
        }

        // ---- recurrence: packed fp32x2, one ex2 per state and token ----
        auto step = [&](const int tq) {
            const float4 v = sDD[tq * ROWP + mycol];
            const f32x2 dd = pk2(v.x, v.y), xx = pk2(v.z, v.w);
            f32x2 acc = 0ull;
#pragma unroll
            for (int j = 0; j + 1 < NP; j += 2) {
                const float4 b4 = *reinterpret_cast<const float4 *>(sB + tq * kN + sub * NPT + 2 * j);
                const float4 c4 = *reinterpret_cast<const float4 *>(sC + tq * kN + sub * NPT + 2 * j);
                float a0, a1, a2, a3;
                upk2(mul2(dd, A2p[j]), a0, a1);
                upk2(mul2(dd, A2p[j + 1]), a2, a3);
                const f32x2 dA0 = pk2(ex2_approx(a0), ex2_approx(a1));
                const f32x2 dA1 = pk2(ex2_approx(a2), ex2_approx(a3));
                hp[j] = fma2(dA0, hp[j], mul2(xx, pk2(b4.x, b4.y)));
                hp[j + 1] = fma2(dA1, hp[j + 1], mul2(xx, pk2(b4.z, b4.w)));
                acc = fma2(pk2(c4.x, c4.y), hp[j], acc);
                acc = fma2(pk2(c4.z, c4.w), hp[j + 1], acc);
            }
            if constexpr (NP % 2 == 1) {  // NPT == 2: one pair
                const float2 b2 = *reinterpret_cast<const float2 *>(sB + tq * kN + sub * NPT);
                const float2 c2 = *reinterpret_cast<const float2 *>(sC + tq * kN + sub * NPT);
                float a0, a1;
                upk2(mul2(dd, A2p[NP - 1]), a0, a1);
                const f32x2 dA = pk2(ex2_approx(a0), ex2_approx(a1));
                hp[NP - 1] = fma2(dA, hp[NP - 1], mul2(xx, pk2(b2.x, b2.y)));
                acc = fma2(pk2(c2.x, c2.y), hp[NP - 1], acc);
            }
            float s0, s1;
            upk2(acc, s0, s1);
            sYP[tq * ROWY + myy] = s0 + s1;
        };
        // full chunks run fully unrolled, so every shared-memory offset is an
        // immediate; only a sequence's ragged last chunk takes the plain loop
        if (nt == TCH) {
#pragma unroll
            for (int tq = 0; tq < TCH; ++tq) step(tq);
        } else {
#pragma unroll 1
            for (int tq = 0; tq < nt; ++tq) step(tq);
        }
        __syncthreads();

        // ---- output: sum the partial readouts, skip, gate, store y ----
        const T *rU2 = raw(stage, 0), *rZ = raw(stage, 2);
        T *Y = static_cast<T *>(p.y);
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            if (tid + i * THREADS >= K::ITEMS) break;
            const int tl = (tid + i * THREADS) / CV;
            if (tl < nt && vvalid) {
                float fu[VEC], fz[VEC], out[VEC];
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rU2 + tl * CH + cvl * VEC), fu);
                if (has_z) unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rZ + tl * CH + cvl * VEC), fz);
                const float *yp = sYP + tl * ROWY + vy;
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    float sum = 0.f;
                    if constexpr (TPC >= 4) {
#pragma unroll
                        for (int q = 0; q < TPC; q += 4) {
                            const float4 v4 = *reinterpret_cast<const float4 *>(yp + e * TPC + q);
                            sum += (v4.x + v4.y) + (v4.z + v4.w);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < TPC; ++q) sum += yp[e * TPC + q];
                    }
                    out[e] = fmaf(dsk[e], fu[e], sum);
                }
                if (has_z) {
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        float g0, g1;
                        silu2(fz[e], fz[e + 1], g0, g1);
                        out[e] *= g0;
                        out[e + 1] *= g1;
                    }
                }
                store_vec<T, VEC>(Y + (t0 + tl) * p.D + cg, out);
            }
        }
        // next chunk's pre-pass and recurrence rewrite sDD, sB, sC, sYP only
        // after its first barrier, which follows every thread's output pass
    }
    if (p.h_final && cvalid) {
#pragma unroll
        for (int j = 0; j < NPT; j += 2) {
            float lo, hi;
            upk2(hp[j / 2], lo, hi);
            const int64_t o = (seq * p.D + c0) * kN + sub * NPT + j;
            p.h_final[o] = lo;
            p.h_final[o + 1] = hi;
        }
    }
}

// ---------------------------------------------------------------------------
// Warp-specialized variant (TMA staging). REC threads run the recurrence; HELP
// helper threads run, for the same CTA, the per-token pre-pass one chunk ahead
// and the output pass one chunk behind, so the recurrence warps keep the
// special-function unit busy while the helpers unpack, softplus, gate and
// store. The two roles hand chunks over through double-buffered shared
// arrays and mbarriers; the raw TMA tiles are triple-buffered so each load is
// issued a full chunk before it is needed. Every wait is bounded.
//   raw_full[3] : TMA landed           (count 1 + transaction bytes)
//   dd_full[2]  : pre-pass written     (count HELP)
//   rec_done[2] : recurrence finished  (count REC; sDD free, sYP written)
//   out_done[2] : output finished      (count HELP; sYP and the raw stage free)
// ---------------------------------------------------------------------------
template <typename T, int NPT_, int CH_, int TCH_, int HELP_>
struct WsCfg {
    static constexpr int NPT = NPT_, CH = CH_, TCH = TCH_, HELP = HELP_;
    static constexpr int TPC = kN / NPT, NP = NPT / 2;
    static constexpr int REC = CH * TPC;
    static constexpr int THREADS = REC + HELP;
    static constexpr int VEC = 16 / sizeof(T);
    static constexpr int CV = CH / VEC;
    static constexpr int ITEMS = TCH * CV;
    static constexpr int IPT = (ITEMS + HELP - 1) / HELP;
    static constexpr int ROWP = CH + CH / 8;
    static constexpr int ROWY = CH * TPC + (CH / 8) * 4;
    static constexpr int BCN = TCH * kN / VEC;
    static constexpr size_t DD = 16 * (size_t)TCH * ROWP;
    static constexpr size_t YP = 4 * (size_t)TCH * ROWY;
    static constexpr size_t BC = 4 * (size_t)TCH * kN;
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CH;
    static constexpr size_t RAW_BC = sizeof(T) * TCH * kN;
    static constexpr size_t RAWSTAGE = 3 * align128(RAW_ACT) + 2 * align128(RAW_BC);
    static constexpr size_t OFF_DD = 0;
    static constexpr size_t OFF_YP = OFF_DD + 2 * align128(DD);
    static constexpr size_t OFF_B = OFF_YP + 2 * align128(YP);
    static constexpr size_t OFF_C = OFF_B + 2 * align128(BC);
    static constexpr size_t OFF_RAW = OFF_C + 2 * align128(BC);
    static constexpr size_t OFF_BAR = OFF_RAW + 3 * RAWSTAGE;
    static constexpr size_t SMEM = OFF_BAR + 128;
    static_assert(NPT % 2 == 0 && CH % 8 == 0, "shape");
    static_assert(HELP % 32 == 0 && REC % 32 == 0 && THREADS <= 1024, "roles are whole warps");
    static_assert(HELP % CV == 0, "each helper keeps one channel vector");
};

template <class K, typename T>
__global__ void __launch_bounds__(K::THREADS)
scan_ws_kernel(const Params p, const __grid_constant__ Maps m, const int has_z)
{
    constexpr int NPT = K::NPT, NP = K::NP, TPC = K::TPC, CH = K::CH, TCH = K::TCH;
    constexpr int VEC = K::VEC, CV = K::CV, IPT = K::IPT, REC = K::REC, HELP = K::HELP;
    constexpr int ROWP = K::ROWP, ROWY = K::ROWY;
    extern __shared__ __align__(128) unsigned char smem[];
    auto sDD = [&](int s) { return reinterpret_cast<float4 *>(smem + K::OFF_DD + s * align128(K::DD)); };
    auto sYP = [&](int s) { return reinterpret_cast<float *>(smem + K::OFF_YP + s * align128(K::YP)); };
    auto sB = [&](int s) { return reinterpret_cast<float *>(smem + K::OFF_B + s * align128(K::BC)); };
    auto sC = [&](int s) { return reinterpret_cast<float *>(smem + K::OFF_C + s * align128(K::BC)); };
    auto raw = [&](int stage, int which) -> T * {
        size_t off = K::OFF_RAW + (size_t)stage * K::RAWSTAGE;
        off += which < 3 ? (size_t)which * align128(K::RAW_ACT)
                         : 3 * align128(K::RAW_ACT) + (size_t)(which - 3) * align128(K::RAW_BC);
        return reinterpret_cast<T *>(smem + off);
    };  // which: 0 u, 1 dt, 2 z, 3 B, 4 C
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);
    uint64_t *raw_full = bars, *dd_full = bars + 3, *rec_done = bars + 5, *out_done = bars + 7;

    const int tid = threadIdx.x;
    const int64_t cbase = (int64_t)blockIdx.x * CH;
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
    const int nchunks = (int)((end - start + TCH - 1) / TCH);

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init_n(&raw_full[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init_n(&dd_full[i], HELP);
            mbar_init_n(&rec_done[i], REC);
            mbar_init_n(&out_done[i], HELP);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    bool failed = false;

    if (tid >= REC) {
        // ================= helpers: TMA, pre-pass, output =================
        const int hid = tid - REC;
        const uint32_t tx_bytes = (uint32_t)((has_z ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);
        auto issue = [&](int j) {
            const int st = j % 3;
            mbar_expect_tx(&raw_full[st], tx_bytes);
            const int x = (int)cbase, y = (int)(start + (int64_t)j * TCH);
            tma_2d(raw(st, 0), &m.u, &raw_full[st], x, y);
            tma_2d(raw(st, 1), &m.dt, &raw_full[st], x, y);
            if (has_z) tma_2d(raw(st, 2), &m.z, &raw_full[st], x, y);
            tma_2d(raw(st, 3), &m.b, &raw_full[st], 0, y);
            tma_2d(raw(st, 4), &m.c, &raw_full[st], 0, y);
        };
        if (hid == 0)
            for (int j = 0; j < 3 && j < nchunks; ++j) issue(j);

        const int cvl = hid % CV;
        const int64_t cg = cbase + (int64_t)cvl * VEC;
        const bool vvalid = cg < p.D;
        float dtb[VEC], dsk[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            dtb[i] = (vvalid && p.dt_bias) ? __ldg(p.dt_bias + cg + i) : 0.f;
            dsk[i] = (vvalid && p.Dskip) ? __ldg(p.Dskip + cg + i) : 0.f;
        }
        const int vcol = col4(cvl * VEC);
        const int vy = coly<TPC>(cvl * VEC, 0);
        T *Y = static_cast<T *>(p.y);

        auto output = [&](int j) {
            const int s = j & 1, st = j % 3;
            const int64_t t0 = start + (int64_t)j * TCH;
            const int nt = (int)min((int64_t)TCH, end - t0);
            mbar_wait(&rec_done[s], (uint32_t)((j >> 1) & 1), failed, &g_scan_status, 1);
            const T *rU = raw(st, 0), *rZ = raw(st, 2);
            const float *yp0 = sYP(s);
#pragma unroll
            for (int i = 0; i < IPT; ++i) {
                const int it = hid + i * HELP;
                if (it >= K::ITEMS) break;
                const int tl = it / CV;
                if (tl < nt && vvalid) {
                    float fu[VEC], fz[VEC], out[VEC];
                    unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rU + tl * CH + cvl * VEC), fu);
                    if (has_z) unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rZ + tl * CH + cvl * VEC), fz);
                    const float *yp = yp0 + tl * ROWY + vy;
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        float sum = 0.f;
                        if constexpr (TPC >= 4) {
#pragma unroll
                            for (int q = 0; q < TPC; q += 4) {
                                const float4 v4 = *reinterpret_cast<const float4 *>(yp + e * TPC + q);
                                sum += (v4.x + v4.y) + (v4.z + v4.w);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < TPC; ++q) sum += yp[e * TPC + q];
                        }
                        out[e] = fmaf(dsk[e], fu[e], sum);
                    }
                    if (has_z) {
#pragma unroll
                        for (int e = 0; e < VEC; e += 2) {
                            float g0, g1;
                            silu2(fz[e], fz[e + 1], g0, g1);
                            out[e] *= g0;
                            out[e + 1] *= g1;
                        }
                    }
                    store_vec<T, VEC>(Y + (t0 + tl) * p.D + cg, out);
                }
            }
            mbar_arrive(&out_done[s]);
            if (hid == 0 && j + 3 < nchunks) {
                // every helper has finished with raw stage j % 3
                mbar_wait(&out_done[s], (uint32_t)((j >> 1) & 1), failed, &g_scan_status, 1);
                fence_proxy_async();
                issue(j + 3);
            }
        };

        for (int k = 0; k < nchunks; ++k) {
            const int s = k & 1, st = k % 3;
            const int64_t t0 = start + (int64_t)k * TCH;
            const int nt = (int)min((int64_t)TCH, end - t0);
            mbar_wait(&raw_full[st], (uint32_t)((k / 3) & 1), failed, &g_scan_status, 1);
            // sDD/sB/sC stage s were released by the recurrence of chunk k-2,
            // which output(k-2) waited for before this iteration
            const T *rU = raw(st, 0), *rDT = raw(st, 1);
            float4 *dd = sDD(s);
#pragma unroll
            for (int i = 0; i < IPT; ++i) {
                const int it = hid + i * HELP;
                if (it >= K::ITEMS) break;
                const int tl = it / CV;
                const bool live = tl < nt && vvalid;
                float fdt[VEC], fu[VEC];
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rDT + tl * CH + cvl * VEC), fdt);
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rU + tl * CH + cvl * VEC), fu);
                float4 *dst = dd + tl * ROWP + vcol;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    float d0 = fdt[e] + dtb[e], d1 = fdt[e + 1] + dtb[e + 1];
                    if (p.delta_softplus) softplus2(d0, d1, d0, d1);
                    d0 = live ? d0 : 0.f;
                    d1 = live ? d1 : 0.f;
                    float x0, x1;
                    upk2(mul2(pk2(d0, d1), pk2(fu[e], fu[e + 1])), x0, x1);
                    dst[e] = make_float4(d0, d0, x0, x0);
                    dst[e + 1] = make_float4(d1, d1, x1, x1);
                }
            }
            {
                const T *rB = raw(st, 3), *rC = raw(st, 4);
                float *b = sB(s), *c = sC(s);
                for (int q = hid; q < K::BCN; q += HELP) {
                    const int e0 = q * VEC;
                    const bool live = e0 / kN < nt;
                    float fb[VEC], fc[VEC];
                    unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rB + e0), fb);
                    unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rC + e0), fc);
#pragma unroll
                    for (int e = 0; e < VEC; e += 4) {
                        *reinterpret_cast<float4 *>(b + e0 + e) = live
                            ? make_float4(fb[e], fb[e + 1], fb[e + 2], fb[e + 3])
                            : make_float4(0.f, 0.f, 0.f, 0.f);
                        *reinterpret_cast<float4 *>(c + e0 + e) = live
                            ? make_float4(fc[e], fc[e + 1], fc[e + 2], fc[e + 3])
                            : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            }
            mbar_arrive(&dd_full[s]);
            if (k >= 1) output(k - 1);
        }
        if (nchunks >= 1) output(nchunks - 1);
    } else {
        // ================= recurrence =================
        const int cl = tid / TPC, sub = tid % TPC;
        const int64_t c0 = cbase + cl;
        const bool cvalid = c0 < p.D;
        f32x2 A2p[NP], hp[NP];
#pragma unroll
        for (int j = 0; j < NPT; j += 2) {
            const int64_t ai = c0 * kN + sub * NPT + j;
            const int64_t hi = (seq * p.D + c0) * kN + sub * NPT + j;
            A2p[j / 2] = cvalid ? pk2(__ldg(p.A + ai) * kLog2e, __ldg(p.A + ai + 1) * kLog2e) : 0ull;
            hp[j / 2] = (cvalid && p.h0) ? pk2(p.h0[hi], p.h0[hi + 1]) : 0ull;
        }
        const int mycol = col4(cl);
        const int myy = coly<TPC>(cl, sub);
        for (int k = 0; k < nchunks; ++k) {
            const int s = k & 1;
            const int64_t t0 = start + (int64_t)k * TCH;
            const int nt = (int)min((int64_t)TCH, end - t0);
            mbar_wait(&dd_full[s], (uint32_t)((k >> 1) & 1), failed, &g_scan_status, 1);
            if (k >= 2) mbar_wait(&out_done[s], (uint32_t)(((k - 2) >> 1) & 1), failed, &g_scan_status, 1);
            const float4 *dd = sDD(s);
            const float *b = sB(s), *c = sC(s);
            float *yp = sYP(s);
#pragma unroll 4
            for (int tq = 0; tq < nt; ++tq) {
                const float4 v = dd[tq * ROWP + mycol];
                const f32x2 ddv = pk2(v.x, v.y), xx = pk2(v.z, v.w);
                f32x2 acc = 0ull;
#pragma unroll
                for (int j = 0; j + 1 < NP; j += 2) {
                    const float4 b4 = *reinterpret_cast<const float4 *>(b + tq * kN + sub * NPT + 2 * j);
                    const float4 c4 = *reinterpret_cast<const float4 *>(c + tq * kN + sub * NPT + 2 * j);
                    float a0, a1, a2, a3;
                    upk2(mul2(ddv, A2p[j]), a0, a1);
                    upk2(mul2(ddv, A2p[j + 1]), a2, a3);
                    const f32x2 dA0 = pk2(ex2_approx(a0), ex2_approx(a1));
                    const f32x2 dA1 = pk2(ex2_approx(a2), ex2_approx(a3));
                    hp[j] = fma2(dA0, hp[j], mul2(xx, pk2(b4.x, b4.y)));
                    hp[j + 1] = fma2(dA1, hp[j + 1], mul2(xx, pk2(b4.z, b4.w)));
                    acc = fma2(pk2(c4.x, c4.y), hp[j], acc);
                    acc = fma2(pk2(c4.z, c4.w), hp[j + 1], acc);
                }
                if constexpr (NP % 2 == 1) {
                    const float2 b2 = *reinterpret_cast<const float2 *>(b + tq * kN + sub * NPT);
                    const float2 c2 = *reinterpret_cast<const float2 *>(c + tq * kN + sub * NPT);
                    float a0, a1;
                    upk2(mul2(ddv, A2p[NP - 1]), a0, a1);
                    const f32x2 dA = pk2(ex2_approx(a0), ex2_approx(a1));
                    hp[NP - 1] = fma2(dA, hp[NP - 1], mul2(xx, pk2(b2.x, b2.y)));
                    acc = fma2(pk2(c2.x, c2.y), hp[NP - 1], acc);
                }
                float s0, s1;
                upk2(acc, s0, s1);
                yp[tq * ROWY + myy] = s0 + s1;
            }
            mbar_arrive(&rec_done[s]);
        }
        if (p.h_final && cvalid) {
#pragma unroll
            for (int j = 0; j < NPT; j += 2) {
                float lo, hi;
                upk2(hp[j / 2], lo, hi);
                const int64_t o = (seq * p.D + c0) * kN + sub * NPT + j;
                p.h_final[o] = lo;
                p.h_final[o + 1] = hi;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Warp-autonomous variant. A CTA is one warp that owns CPW = 32 / TPC channels
// of one sequence; nothing is shared between warps, so there is no CTA-wide
// barrier and the warps of an SM drift into different phases: while some run
// the exponential-heavy recurrence, others unpack, softplus, gate and store,
// and the special-function unit stays busy. Per chunk of TCH tokens:
//   1. TMA has landed the raw u, dt, z (TCH x CPW) and B, C (TCH x 16) tiles
//      (two stages, issued two chunks ahead by lane 0; bounded mbarrier wait).
//   2. B and C are widened to fp32; lane (channel, sub) computes delta and
//      delta*u for tokens sub, sub + TPC, ... of its channel into sDX, and
//      keeps D*u and silu(z) of those tokens in registers.
//   3. Recurrence over the chunk (fully unrolled); the lane's partial readout
//      of each token goes to the raw stage, which is dead by then.
//   4. The lane that owns a token sums its channel's TPC partials, applies
//      skip and gate and stores y.
// ---------------------------------------------------------------------------
template <typename T, int NPT_, int TCH_>
struct WarpCfg {
    static constexpr int NPT = NPT_, TCH = TCH_;
    static constexpr int TPC = kN / NPT;            // lanes per channel
    static constexpr int CPW = 32 / TPC;            // channels per warp
    static constexpr int TPL = TCH / TPC;           // tokens per lane in steps 2 and 4
    static constexpr int VEC = 16 / sizeof(T);
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CPW;
    static constexpr size_t RAW_BC = sizeof(T) * TCH * kN;
    static constexpr size_t RAW = 3 * align128(RAW_ACT) + 2 * align128(RAW_BC);
    static constexpr size_t YP = sizeof(float) * TCH * 32;
    static constexpr size_t STAGE = align128(RAW > YP ? RAW : YP);
    static constexpr size_t OFF_B = 2 * STAGE;
    static constexpr size_t OFF_C = OFF_B + align128(sizeof(float) * TCH * kN);
    static constexpr size_t OFF_DX = OFF_C + align128(sizeof(float) * TCH * kN);
    static constexpr size_t OFF_BAR = OFF_DX + align128(sizeof(float2) * TCH * CPW);
    static constexpr size_t SMEM = OFF_BAR + 16;
    static_assert(NPT % 4 == 0, "states are read four at a time");
    static_assert(TPL % 2 == 0, "per-token work goes in packed pairs");
    static_assert((CPW * sizeof(T)) % 16 == 0, "TMA rows are whole 16-byte pieces");
    static_assert((TCH * kN) % VEC == 0, "B and C tiles are whole 16-byte pieces");
};

template <class K, typename T>
__global__ void __launch_bounds__(32)
scan_warp_kernel(const Params p, const __grid_constant__ Maps m, const int has_z)
{
    constexpr int NPT = K::NPT, TPC = K::TPC, CPW = K::CPW, TCH = K::TCH, TPL = K::TPL;
    constexpr int VEC = K::VEC;
    extern __shared__ __align__(128) unsigned char smem[];
    float *sB = reinterpret_cast<float *>(smem + K::OFF_B);
    float *sC = reinterpret_cast<float *>(smem + K::OFF_C);
    float2 *sDX = reinterpret_cast<float2 *>(smem + K::OFF_DX);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);
    auto raw = [&](int st, int which) -> T * {
        size_t off = (size_t)st * K::STAGE;
        off += which < 3 ? (size_t)which * align128(K::RAW_ACT)
                         : 3 * align128(K::RAW_ACT) + (size_t)(which - 3) * align128(K::RAW_BC);
        return reinterpret_cast<T *>(smem + off);
    };  // which: 0 u, 1 dt, 2 z, 3 B, 4 C

    const int lane = threadIdx.x;
    const int cl = lane / TPC, sub = lane % TPC;
    const int64_t cbase = (int64_t)blockIdx.x * CPW;
    const int64_t c = cbase + cl;
    const bool cvalid = c < p.D;
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
    const int nchunks = (int)((end - start + TCH - 1) / TCH);

    if (lane == 0) {
        mbar_init_n(&bar[0], 1);
        mbar_init_n(&bar[1], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const uint32_t tx_bytes = (uint32_t)((has_z ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);
    auto issue = [&](int j) {
        const int st = j & 1;
        mbar_expect_tx(&bar[st], tx_bytes);
        const int x = (int)cbase, y = (int)(start + (int64_t)j * TCH);
        tma_2d(raw(st, 0), &m.u, &bar[st], x, y);
        tma_2d(raw(st, 1), &m.dt, &bar[st], x, y);
        if (has_z) tma_2d(raw(st, 2), &m.z, &bar[st], x, y);
        tma_2d(raw(st, 3), &m.b, &bar[st], 0, y);
        tma_2d(raw(st, 4), &m.c, &bar[st], 0, y);
    };
    if (lane == 0) {
        if (nchunks > 0) issue(0);
        if (nchunks > 1) issue(1);
    }

    f32x2 A2p[NPT / 2], hp[NPT / 2];
#pragma unroll
    for (int j = 0; j < NPT; j += 4) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), h = a;
        if (cvalid) {
            a = __ldg(reinterpret_cast<const float4 *>(p.A + c * kN + sub * NPT + j));
            if (p.h0) h = *reinterpret_cast<const float4 *>(p.h0 + (seq * p.D + c) * kN + sub * NPT + j);
        }
        A2p[j / 2] = pk2(a.x * kLog2e, a.y * kLog2e);
        A2p[j / 2 + 1] = pk2(a.z * kLog2e, a.w * kLog2e);
        hp[j / 2] = pk2(h.x, h.y);
        hp[j / 2 + 1] = pk2(h.z, h.w);
    }
    const float dtb = (cvalid && p.dt_bias) ? __ldg(p.dt_bias + c) : 0.f;
    const float dsk = (cvalid && p.Dskip) ? __ldg(p.Dskip + c) : 0.f;
    T *Y = static_cast<T *>(p.y);

    bool failed = false;
    for (int k = 0; k < nchunks; ++k) {
        const int st = k & 1;
        const int64_t t0 = start + (int64_t)k * TCH;
        const int nt = (int)min((int64_t)TCH, end - t0);
        mbar_wait(&bar[st], (uint32_t)((k >> 1) & 1), failed, &g_scan_status, 1);

        // ---- step 2: widen B, C; delta, delta*u, D*u, silu(z) of this lane's tokens ----
        {
            const T *rB = raw(st, 3), *rC = raw(st, 4);
#pragma unroll
            for (int q = lane; q < TCH * kN / VEC; q += 32) {
                float fb[VEC], fc[VEC];
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rB + q * VEC), fb);
                unpack16<T, VEC>(*reinterpret_cast<const uint4 *>(rC + q * VEC), fc);
#pragma unroll
                for (int e = 0; e < VEC; e += 4) {
                    *reinterpret_cast<float4 *>(sB + q * VEC + e) =
                        make_float4(fb[e], fb[e + 1], fb[e + 2], fb[e + 3]);
                    *reinterpret_cast<float4 *>(sC + q * VEC + e) =
                        make_float4(fc[e], fc[e + 1], fc[e + 2], fc[e + 3]);
                }
            }
        }
        float skip[TPL], gate[TPL];
        {
            const T *rU = raw(st, 0), *rDT = raw(st, 1), *rZ = raw(st, 2);
#pragma unroll
            for (int i = 0; i < TPL; i += 2) {
                const int ta = sub + TPC * i, tb = ta + TPC;
                float da = to_f32(rDT[ta * CPW + cl]) + dtb, db = to_f32(rDT[tb * CPW + cl]) + dtb;
                if (p.delta_softplus) softplus2(da, db, da, db);
                const float ua = to_f32(rU[ta * CPW + cl]), ub = to_f32(rU[tb * CPW + cl]);
                float xa, xb;
                upk2(mul2(pk2(da, db), pk2(ua, ub)), xa, xb);
                sDX[ta * CPW + cl] = make_float2(da, xa);
                sDX[tb * CPW + cl] = make_float2(db, xb);
                skip[i] = dsk * ua;
                skip[i + 1] = dsk * ub;
                if (has_z) {
                    silu2(to_f32(rZ[ta * CPW + cl]), to_f32(rZ[tb * CPW + cl]), gate[i], gate[i + 1]);
                } else {
                    gate[i] = gate[i + 1] = 1.f;
                }
            }
        }
        __syncwarp();

        // ---- step 3: recurrence; partial readouts into the (now dead) raw stage ----
        float *sYP = reinterpret_cast<float *>(smem + (size_t)st * K::STAGE);
#pragma unroll
        for (int t = 0; t < TCH; ++t) {
            if (t >= nt) break;
            const float2 v = sDX[t * CPW + cl];
            const f32x2 dd = pk2(v.x, v.x), xx = pk2(v.y, v.y);
            f32x2 acc = 0ull;
#pragma unroll
            for (int q = 0; q < NPT / 4; ++q) {
                const float4 b4 = *reinterpret_cast<const float4 *>(sB + t * kN + sub * NPT + 4 * q);
                const float4 c4 = *reinterpret_cast<const float4 *>(sC + t * kN + sub * NPT + 4 * q);
                float a0, a1, a2, a3;
                upk2(mul2(dd, A2p[2 * q]), a0, a1);
                upk2(mul2(dd, A2p[2 * q + 1]), a2, a3);
                const f32x2 dA0 = pk2(ex2_approx(a0), ex2_approx(a1));
                const f32x2 dA1 = pk2(ex2_approx(a2), ex2_approx(a3));
                hp[2 * q] = fma2(dA0, hp[2 * q], mul2(xx, pk2(b4.x, b4.y)));
                hp[2 * q + 1] = fma2(dA1, hp[2 * q + 1], mul2(xx, pk2(b4.z, b4.w)));
                acc = fma2(pk2(c4.x, c4.y), hp[2 * q], acc);
                acc = fma2(pk2(c4.z, c4.w), hp[2 * q + 1], acc);
            }
            float s0, s1;
            upk2(acc, s0, s1);
            sYP[t * 32 + lane] = s0 + s1;
        }
        __syncwarp();

        // ---- step 4: sum partials, skip, gate, store ----
#pragma unroll
        for (int i = 0; i < TPL; ++i) {
            const int t = sub + TPC * i;
            if (t < nt && cvalid) {
                const float *yp = sYP + t * 32 + cl * TPC;
                float sum = 0.f;
                if constexpr (TPC >= 4) {
#pragma unroll
                    for (int q = 0; q < TPC; q += 4) {
                        const float4 v4 = *reinterpret_cast<const float4 *>(yp + q);
                        sum += (v4.x + v4.y) + (v4.z + v4.w);
                    }
                } else if constexpr (TPC == 2) {
                    const float2 v2 = *reinterpret_cast<const float2 *>(yp);
                    sum = v2.x + v2.y;
                } else {
                    sum = yp[0];
                }
                Y[(t0 + t) * p.D + c] = from_f32<T>((sum + skip[i]) * gate[i]);
            }
        }
        __syncwarp();
        if (lane == 0 && k + 2 < nchunks) {
            // every lane's reads of this stage (raw tiles, then partials) are done
            fence_proxy_async();
            issue(k + 2);
        }
    }
    if (p.h_final && cvalid) {
        float *hf = p.h_final + (seq * p.D + c) * kN + sub * NPT;
#pragma unroll
        for (int j = 0; j < NPT; j += 4) {
            float x0, x1, x2, x3;
            upk2(hp[j / 2], x0, x1);
            upk2(hp[j / 2 + 1], x2, x3);
            *reinterpret_cast<float4 *>(hf + j) = make_float4(x0, x1, x2, x3);
        }
    }
}

// ---------------------------------------------------------------------------
// Variant 3: time-split chunks (TMA staging). A chunk of SEG x TS tokens is
// cut into SEG segments handled by different warps, which multiplies the
// warps available to sequences x channels pairs that are too few to fill the
// GPU. Each segment first runs its tokens from a zero state, keeping dA and
// delta*u*B in registers and forming its decay product P = prod dA and local
// state hl; the segments' (P, hl) pairs meet in shared memory, every warp
// folds those of the segments before its own onto the chunk's incoming state
// (h_in = P * h_in + hl), and then replays its tokens from the true state
// with the register-resident dA, so every exponential is computed once.
// ---------------------------------------------------------------------------
template <typename T, int NPT_, int SEG_, int TS_, int CH_>
struct TsCfg {
    static constexpr int NPT = NPT_, SEG = SEG_, TS = TS_, CH = CH_;
    static constexpr int TPC = kN / NPT, NP = NPT / 2;
    static constexpr int TCH = SEG * TS;                  // tokens per chunk
    static constexpr int LANES = CH * TPC;                // threads per segment
    static constexpr int THREADS = SEG * LANES;
    static constexpr int PV = 2;                          // channels per pre-pass item
    static constexpr int ITEMS = TCH * CH / PV;
    static constexpr int IPT = (ITEMS + THREADS - 1) / THREADS;
    static constexpr int ROW2 = CH + 2 * (CH / 16);
    static constexpr int BCE = TCH * kN;                  // B (or C) elements per chunk
    static constexpr size_t OFF_DX = 0;
    static constexpr size_t OFF_UG = align128(OFF_DX + sizeof(float2) * TCH * ROW2);
    static constexpr size_t OFF_B = align128(OFF_UG + sizeof(float2) * TCH * ROW2);
    static constexpr size_t OFF_C = align128(OFF_B + sizeof(float) * BCE);
    static constexpr size_t OFF_XF = align128(OFF_C + sizeof(float) * BCE);
    static constexpr size_t RAW_ACT = sizeof(T) * TCH * CH;
    static constexpr size_t RAW_BC = sizeof(T) * BCE;
    static constexpr size_t OFF_RU = align128(OFF_XF + sizeof(float) * THREADS * 2 * NPT);
    static constexpr size_t OFF_RDT = OFF_RU + align128(RAW_ACT);
    static constexpr size_t OFF_RZ = OFF_RDT + align128(RAW_ACT);
    static constexpr size_t OFF_RB = OFF_RZ + align128(RAW_ACT);
    static constexpr size_t OFF_RC = OFF_RB + align128(RAW_BC);
    static constexpr size_t OFF_BAR = OFF_RC + align128(RAW_BC);
    static constexpr size_t SMEM = OFF_BAR + 128;
    static_assert(NPT == 2 || NPT == 4, "two or four states per lane");
    static_assert(TS % TPC == 0, "segments hold whole token groups");
    static_assert((CH * sizeof(T)) % 16 == 0, "TMA rows are whole 16-byte units");
    static_assert(THREADS % 32 == 0 && THREADS <= 1024, "block size");
};

template <class K, typename T>
__global__ void __launch_bounds__(K::THREADS)
scan_ts_kernel(const Params p, const __grid_constant__ Maps m, const int has_z)
{
    constexpr int NPT = K::NPT, NP = K::NP, TPC = K::TPC, SEG = K::SEG, TS = K::TS;
    constexpr int CH = K::CH, TCH = K::TCH, LANES = K::LANES, THREADS = K::THREADS;
    constexpr int ROW2 = K::ROW2, PV = K::PV;
    extern __shared__ __align__(128) unsigned char smem[];
    float2 *sDX = reinterpret_cast<float2 *>(smem + K::OFF_DX);
    float2 *sUG = reinterpret_cast<float2 *>(smem + K::OFF_UG);
    float *sB = reinterpret_cast<float *>(smem + K::OFF_B);
    float *sC = reinterpret_cast<float *>(smem + K::OFF_C);
    float *sXF = reinterpret_cast<float *>(smem + K::OFF_XF);
    T *rU = reinterpret_cast<T *>(smem + K::OFF_RU);
    T *rDT = reinterpret_cast<T *>(smem + K::OFF_RDT);
    T *rZ = reinterpret_cast<T *>(smem + K::OFF_RZ);
    T *rB = reinterpret_cast<T *>(smem + K::OFF_RB);
    T *rC = reinterpret_cast<T *>(smem + K::OFF_RC);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);

    const int tid = threadIdx.x;
    const int seg = tid / LANES, r = tid % LANES;
    const int cl = r / TPC, sub = r % TPC;
    const int64_t cbase = (int64_t)blockIdx.x * CH;
    const int64_t c0 = cbase + cl;
    const bool cvalid = c0 < p.D;
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
    const int mycol = col2(cl);
    const uint32_t tx_bytes = (uint32_t)((has_z ? 3 : 2) * K::RAW_ACT + 2 * K::RAW_BC);

    if (tid == 0) mbar_init(bar);
    __syncthreads();
    auto issue = [&](int64_t t0) {
        mbar_expect_tx(bar, tx_bytes);
        const int x = (int)cbase, y = (int)t0;
        tma_2d(rU, &m.u, bar, x, y);
        tma_2d(rDT, &m.dt, bar, x, y);
        if (has_z) tma_2d(rZ, &m.z, bar, x, y);
        tma_2d(rB, &m.b, bar, 0, y);
        tma_2d(rC, &m.c, bar, 0, y);
    };
    if (tid == 0 && start < end) issue(start);

    // A * log2(e) and the chunk's incoming state (identical in every segment)
    f32x2 A2p[NP], hp[NP];
#pragma unroll
    for (int j = 0; j < NPT; j += 2) {
        const int64_t ai = c0 * kN + sub * NPT + j;
        const int64_t hi = (seq * p.D + c0) * kN + sub * NPT + j;
        A2p[j / 2] = cvalid ? pk2(__ldg(p.A + ai) * kLog2e, __ldg(p.A + ai + 1) * kLog2e) : 0ull;
        hp[j / 2] = (cvalid && p.h0) ? pk2(p.h0[hi], p.h0[hi + 1]) : 0ull;
    }
    const float dsk = (cvalid && p.Dskip) ? __ldg(p.Dskip + c0) : 0.f;

    uint32_t parity = 0;
    bool failed = false;
    for (int64_t t0 = start; t0 < end; t0 += TCH) {
        const int nt = (int)min((int64_t)TCH, end - t0);
        mbar_wait(bar, parity, failed, &g_scan_status, 1);
        parity ^= 1u;

        // ---- pre-pass: items of PV channels of one token ----
#pragma unroll
        for (int i = 0; i < K::IPT; ++i) {
            const int it = tid + i * THREADS;
            if (it < K::ITEMS) {
                const int tl = it / (CH / PV), pc = (it % (CH / PV)) * PV;
                const int64_t cg = cbase + pc;
                const bool live = tl < nt && cg < p.D;
                float fdt[PV], fu[PV], fz[PV], dtb[PV];
#pragma unroll
                for (int e = 0; e < PV; ++e) {
                    fdt[e] = to_f32(rDT[tl * CH + pc + e]);
                    fu[e] = to_f32(rU[tl * CH + pc + e]);
                    fz[e] = has_z ? to_f32(rZ[tl * CH + pc + e]) : 0.f;
                    dtb[e] = (live && p.dt_bias) ? __ldg(p.dt_bias + cg + e) : 0.f;
                }
                prepass_item<PV>(sDX + tl * ROW2 + col2(pc), sUG + tl * ROW2 + col2(pc), live, fdt,
                                 fu, fz, has_z != 0, dtb, p.delta_softplus);
            }
        }
        for (int e = tid; e < K::BCE; e += THREADS) {
            const bool live = e / kN < nt;
            sB[e] = live ? to_f32(rB[e]) : 0.f;
            sC[e] = live ? to_f32(rC[e]) : 0.f;
        }
        __syncthreads();
        if (tid == 0 && t0 + TCH < end) {
            fence_proxy_async();
            issue(t0 + TCH);
        }

        // ---- phase 1: this segment from a zero state ----
        f32x2 dA[TS][NP], bx[TS][NP], hl[NP], P[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            hl[j] = 0ull;
            P[j] = pk2(1.f, 1.f);
        }
#pragma unroll
        for (int t = 0; t < TS; ++t) {
            const int tq = seg * TS + t;
            const float2 v = sDX[tq * ROW2 + mycol];
            const f32x2 dd = pk2(v.x, v.x), xx = pk2(v.y, v.y);
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const float2 b2 = *reinterpret_cast<const float2 *>(sB + tq * kN + sub * NPT + 2 * j);
                float a0, a1;
                upk2(mul2(dd, A2p[j]), a0, a1);
                dA[t][j] = pk2(ex2_approx(a0), ex2_approx(a1));
                bx[t][j] = mul2(xx, pk2(b2.x, b2.y));
                hl[j] = fma2(dA[t][j], hl[j], bx[t][j]);
                P[j] = mul2(P[j], dA[t][j]);
            }
        }
        float *xf = sXF + (size_t)tid * 2 * NPT;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            float a, b;
            upk2(P[j], a, b);
            xf[2 * j] = a;
            xf[2 * j + 1] = b;
            upk2(hl[j], a, b);
            xf[NPT + 2 * j] = a;
            xf[NPT + 2 * j + 1] = b;
        }
        __syncthreads();

        // ---- phase 2: carry across the segments ----
        f32x2 hs[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) hs[j] = hp[j];
#pragma unroll
        for (int v = 0; v < SEG; ++v) {
            if (v == seg) {
#pragma unroll
                for (int j = 0; j < NP; ++j) hs[j] = hp[j];
            }
            const float *src = sXF + (size_t)(v * LANES + r) * 2 * NPT;
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const f32x2 Pv = pk2(src[2 * j], src[2 * j + 1]);
                const f32x2 hv = pk2(src[NPT + 2 * j], src[NPT + 2 * j + 1]);
                hp[j] = fma2(Pv, hp[j], hv);  // after the loop: the chunk's outgoing state
            }
        }

        // ---- phase 3: replay the segment from its true incoming state ----
#pragma unroll
        for (int t = 0; t < TS; t += TPC) {
            float yp[TPC];
#pragma unroll
            for (int q = 0; q < TPC; ++q) {
                const int tq = seg * TS + t + q;
                f32x2 acc = 0ull;
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const float2 c2 = *reinterpret_cast<const float2 *>(sC + tq * kN + sub * NPT + 2 * j);
                    hs[j] = fma2(dA[t + q][j], hs[j], bx[t + q][j]);
                    acc = fma2(pk2(c2.x, c2.y), hs[j], acc);
                }
                float s0, s1;
                upk2(acc, s0, s1);
                yp[q] = s0 + s1;
            }
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
            float2 *q2 = sUG + (seg * TS + t + sub) * ROW2 + mycol;
            const float2 ug = *q2;
            q2->x = (yp[0] + dsk * ug.x) * ug.y;
        }
        __syncthreads();

        // ---- write y ----
        T *Y = static_cast<T *>(p.y);
#pragma unroll
        for (int i = 0; i < K::IPT; ++i) {
            const int it = tid + i * THREADS;
            if (it < K::ITEMS) {
                const int tl = it / (CH / PV), pc = (it % (CH / PV)) * PV;
                const int64_t cg = cbase + pc;
                if (tl < nt && cg < p.D) {
                    float out[PV];
#pragma unroll
                    for (int e = 0; e < PV; ++e) out[e] = sUG[tl * ROW2 + col2(pc) + e].x;
                    store_vec<T, PV>(Y + (t0 + tl) * p.D + cg, out);
                }
            }
        }
        // the next pre-pass rewrites sUG only at this thread's own items
    }
    if (p.h_final && cvalid && seg == 0) {
#pragma unroll
        for (int j = 0; j < NPT; j += 2) {
            float lo, hi;
            upk2(hp[j / 2], lo, hi);
            const int64_t o = (seq * p.D + c0) * kN + sub * NPT + j;
            p.h_final[o] = lo;
            p.h_final[o + 1] = hi;
        }
    }
}

// Longest-first schedule of packed sequences: order[r] = index of the r-th
// longest sequence (ties by index). One block; for S above kSortMax the order
// is the identity.
constexpr int kSortMax = 4096;

__global__ void __launch_bounds__(1024)
order_kernel(const int32_t *__restrict__ cu, int64_t S, int64_t tok, int32_t *__restrict__ order)
{
    __shared__ unsigned long long keys[kSortMax];
    if (S > kSortMax) {
        for (int64_t i = threadIdx.x; i < S; i += blockDim.x) order[i] = (int32_t)i;
        return;
    }
    int P = 1;
    while (P < S) P <<= 1;
    for (int i = threadIdx.x; i < P; i += blockDim.x) {
        unsigned long long k = 0ull;
        if (i < S) {
            const int64_t a = clamp_off(cu[i], tok);
            const int64_t b = max(clamp_off(cu[i + 1], tok), a);
            k = ((unsigned long long)(b - a) << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)i);
        }
        keys[i] = k;
    }
    __syncthreads();
    // bitonic sort, descending
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P; i += blockDim.x) {
                const int l = i ^ j;
                if (l > i) {
                    const bool desc = (i & k) == 0;
                    const unsigned long long a = keys[i], b = keys[l];
                    if (desc ? (a < b) : (a > b)) { keys[i] = b; keys[l] = a; }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < S; i += blockDim.x)
        order[i] = (int32_t)(0xFFFFFFFFu - (unsigned)(keys[i] & 0xFFFFFFFFull));
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <class K, typename T>
cudaError_t run(const Params &p, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_kernel<K, T><<<grid, K::THREADS, K::SMEM, stream>>>(p);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T>
cudaError_t run_tma(const Params &p, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
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
    cudaError_t e = cudaFuncSetAttribute(scan_tma_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_tma_kernel<K, T><<<grid, K::THREADS, K::SMEM, stream>>>(p, m, p.z ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T>
cudaError_t run_staged(const Params &p, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
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
    cudaError_t e = cudaFuncSetAttribute(scan_staged_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM_TMA);
    if (e != cudaSuccess) return e;
    scan_staged_kernel<K, T><<<grid, K::THREADS, K::SMEM_TMA, stream>>>(p, m, p.z ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T>
cudaError_t run_ws(const Params &p, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
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
    cudaError_t e = cudaFuncSetAttribute(scan_ws_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_ws_kernel<K, T><<<grid, K::THREADS, K::SMEM, stream>>>(p, m, p.z ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T>
cudaError_t run_warp(const Params &p, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CPW - 1) / K::CPW), (unsigned)p.S);
    Maps m;
    const bool bf = sizeof(T) == 2;
    const bool aligned = ((uintptr_t)p.A % 16 == 0) &&
                         (!p.h0 || (uintptr_t)p.h0 % 16 == 0) &&
                         (!p.h_final || (uintptr_t)p.h_final % 16 == 0);
    bool ok = aligned && p.tok > 0 &&
              encode_2d(&m.u, p.u, bf, p.D, p.tok, K::CPW, K::TCH) &&
              encode_2d(&m.dt, p.delta, bf, p.D, p.tok, K::CPW, K::TCH) &&
              encode_2d(&m.b, p.B, bf, kN, p.tok, kN, K::TCH) &&
              encode_2d(&m.c, p.C, bf, kN, p.tok, kN, K::TCH);
    if (ok) {
        if (p.z) ok = encode_2d(&m.z, p.z, bf, p.D, p.tok, K::CPW, K::TCH);
        else m.z = m.u;  // never loaded
    }
    if (!ok) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(scan_warp_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_warp_kernel<K, T><<<grid, 32, K::SMEM, stream>>>(p, m, p.z ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
}

template <class K, typename T>
cudaError_t run_ts(const Params &p, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + K::CH - 1) / K::CH), (unsigned)p.S);
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
    cudaError_t e = cudaFuncSetAttribute(scan_ts_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_ts_kernel<K, T><<<grid, K::THREADS, K::SMEM, stream>>>(p, m, p.z ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_pipe(const Params &p, bool bf16, int npt, int sched, cudaStream_t stream,
                             int *launches);

namespace {

int g_forced_npt = 0, g_forced_sched = 0;

// Variants: NPT states per lane; schedule 1: register prefetch, 2: TMA
// staging, 3: TMA staging with time-split chunks; CH channels per CTA, TCH
// tokens per chunk. *piped: set when the pipelined kernels (schedules 9-12)
// ran; they alone write p.ckpt.
template <typename T, int VEC>
cudaError_t dispatch(const Params &p, int npt, int sched, cudaStream_t s, int *n, bool *piped)
{
    if constexpr (VEC == 1) {
        (void)npt; (void)sched; (void)piped;
        return run<Cfg<T, 4, 0, 32, 64, 1>, T>(p, s, n);
    } else {
        if (sched >= 9 && sched <= 12 && p.tok > 0) {
            cudaError_t e = launch_scan_pipe(p, sizeof(T) == 2, npt, sched, s, n);
            if (e != cudaErrorNotSupported) {
                *piped = e == cudaSuccess;
                return e;
            }
        }
        if (sched == 3 && p.tok > 0) {
            cudaError_t e = npt == 2 ? run_ts<TsCfg<T, 2, 4, 8, 8>, T>(p, s, n)
                                     : run_ts<TsCfg<T, 4, 4, 8, 8>, T>(p, s, n);
            if (e != cudaErrorNotSupported) return e;
        }
        if (sched == 6 && p.tok > 0) {
            cudaError_t e;
            if (npt == 16) e = run_ws<WsCfg<T, 16, 64, 8, 64>, T>(p, s, n);
            else if (npt == 8) e = run_ws<WsCfg<T, 8, 64, 8, 64>, T>(p, s, n);
            else if (npt == 2) e = run_ws<WsCfg<T, 2, 16, 16, 64>, T>(p, s, n);
            else e = run_ws<WsCfg<T, 4, 32, 16, 64>, T>(p, s, n);
            if (e != cudaErrorNotSupported) return e;
        }
        if (sched == 8 && p.tok > 0) {
            cudaError_t e;
            if (npt == 16) e = run_staged<Cfg<T, 16, 0, 128, 16, VEC>, T>(p, s, n);
            else if (npt == 8) e = run_staged<Cfg<T, 8, 0, 64, 32, VEC>, T>(p, s, n);
            else if (npt == 2) e = run_staged<Cfg<T, 2, 0, 16, 64, VEC>, T>(p, s, n);
            else e = run_staged<Cfg<T, 4, 0, 32, 32, VEC>, T>(p, s, n);
            if (e != cudaErrorNotSupported) return e;
        }
        if (sched == 7 && p.tok > 0) {
            cudaError_t e;
            if (npt == 16) e = run_warp<WarpCfg<T, 16, 16>, T>(p, s, n);
            else if (npt == 8) e = run_warp<WarpCfg<T, 8, 16>, T>(p, s, n);
            else e = run_warp<WarpCfg<T, 4, 16>, T>(p, s, n);
            if (e != cudaErrorNotSupported) return e;
        }
        if (sched == 4 || sched == 5) {
            // one warp per CTA: a CTA barrier costs next to nothing and warps of
            // different CTAs interleave freely
            cudaError_t e = cudaErrorNotSupported;
            if (p.tok > 0) {
                if (sched == 4) {
                    if (npt == 16) e = run_tma<TmaCfg<T, 16, 32, 32>, T>(p, s, n);
                    else if (npt == 8) e = run_tma<TmaCfg<T, 8, 16, 32>, T>(p, s, n);
                    else e = run_tma<TmaCfg<T, 4, 8, 32>, T>(p, s, n);
                } else {
                    if (npt == 16) e = run_tma<TmaCfg<T, 16, 32, 64>, T>(p, s, n);
                    else if (npt == 8) e = run_tma<TmaCfg<T, 8, 16, 64>, T>(p, s, n);
                    else e = run_tma<TmaCfg<T, 4, 8, 64>, T>(p, s, n);
                }
            }
            if (e != cudaErrorNotSupported) return e;
        }
        if (sched >= 2 && p.tok > 0) {
            cudaError_t e = cudaErrorNotSupported;
            if (npt == 16) e = run_tma<TmaCfg<T, 16, 128, 16>, T>(p, s, n);
            else if (npt == 8) e = run_tma<TmaCfg<T, 8, 64, 16>, T>(p, s, n);
            else if (npt == 2) e = run_tma<TmaCfg<T, 2, 16, 32>, T>(p, s, n);
            else e = run_tma<TmaCfg<T, 4, 32, 16>, T>(p, s, n);
            if (e != cudaErrorNotSupported) return e;
        }
        if (npt == 16) return run<Cfg<T, 16, 0, 128, 32, VEC>, T>(p, s, n);
        if (npt == 8) return run<Cfg<T, 8, 0, 64, 64, VEC>, T>(p, s, n);
        if (npt == 2) return run<Cfg<T, 2, 0, 16, 64, VEC>, T>(p, s, n);
        return run<Cfg<T, 4, 0, 32, 64, VEC>, T>(p, s, n);
    }
}

// SM count of the current device, looked up once per device.
int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        const int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Measured on B200 (exponential rate against the special-function peak):
// with at least two waves of its 128-lane CTAs (three per SM), one lane per
// channel (schedule 12) beats 8 states per lane in the pipelined kernel on
// the packed 65536 x 5120 workload (0.684 against 0.668) and on 32 x 2048 x
// 5120 (0.657 against 0.643). Earlier measurements of the other schedules:
// 8 states per lane with double-buffered TMA staging has the fewest
// instructions per exponential and wins once the GPU holds about 20 warps per
// SM of it (packed 65536 x 5120: 0.60 against 0.52 for the next best); below
// that, latency decides and thinner lanes win: 4 states per lane with register
// prefetch while that still gives about 10 warps per SM (8 x 2048 x 1536:
// 0.366 against 0.356 for 2 states in schedule 8), else 2 states per lane in
// the single-stage TMA layout of schedule 8 (1 x 8192 x 8192: 0.353 against
// 0.31 for 4 states).
void pick_variant(int64_t S, int64_t D, int *npt, int *sched)
{
    const int64_t chains = S * D * kN;            // (sequence, channel, state) recurrences
    const int64_t per_sm = chains / sm_count();
    int npt_auto, sched_auto;
    if (per_sm >= 2 * 3 * 128 * kN) {
        npt_auto = 16;          // one lane per channel: two full waves of 3 CTAs per SM
        sched_auto = 12;
    } else if (per_sm >= 8 * 640) {
        npt_auto = 8;           // about 20 warps per SM of 8-state lanes
        sched_auto = 9;
    } else if (per_sm >= 4 * 128) {
        npt_auto = 4;           // 32-token chunks keep more loads in flight
        // at most two CTAs per SM: the register budget of two
        sched_auto = S * ((D + 31) / 32) <= 2 * (int64_t)sm_count() ? 11 : 10;
    } else {
        npt_auto = 2;           // too few channels to fill the SMs otherwise
        sched_auto = 9;
    }
    *npt = g_forced_npt ? g_forced_npt : npt_auto;
    *sched = g_forced_sched ? g_forced_sched : sched_auto;
}

}  // namespace

void scan_variant_for(int64_t S, int64_t D, int *npt, int *sched) { pick_variant(S, D, npt, sched); }

void set_scan_variant(int npt, int sched)
{
    g_forced_npt = (npt == 2 || npt == 4 || npt == 8 || npt == 16) ? npt : 0;
    g_forced_sched = (sched >= 1 && sched <= 12) ? sched : 0;
    if (g_forced_sched == 12) g_forced_npt = 16;  // one lane per channel, whatever was asked
}

size_t scan_order_bytes(int64_t S) { return (size_t)((S * 4 + 255) / 256) * 256; }

// Longest-first order of packed sequences (as the scan uses it), for the
// library's other kernels over packed sequences.
cudaError_t launch_seq_order(const int32_t *cu, int64_t S, int64_t tok, int32_t *order,
                             cudaStream_t stream)
{
    order_kernel<<<1, 1024, 0, stream>>>(cu, S, tok, order);
    return cudaGetLastError();
}

int device_sm_count() { return sm_count(); }

int read_pipe_status(bool clear);

int read_scan_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_scan_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_scan_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    const int w = read_pipe_status(clear);
    if (w < 0) return -1;
    return v | w;
}

cudaError_t launch_scan(const ScanArgs &a, cudaStream_t stream, int *launches)
{
    Params p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z;
    p.A = a.A; p.Dskip = a.Dskip; p.dt_bias = a.dt_bias; p.h0 = a.h0;
    p.cu = a.cu; p.order = nullptr; p.y = a.y; p.h_final = a.h_final;
    p.S = a.S; p.tok = a.tok; p.D = a.D; p.L = a.cu ? 0 : a.tok / a.S;
    p.delta_softplus = a.delta_softplus;
    p.ckpt = a.ckpt;
    bool piped = false;
    if (a.ckpt_written) *a.ckpt_written = false;
    if (a.cu && a.order && a.S > 1) {
        order_kernel<<<1, 1024, 0, stream>>>(a.cu, a.S, a.tok, a.order);
        ++*launches;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        p.order = a.order;
    }
    int npt, sched;
    pick_variant(a.S, a.D, &npt, &sched);
    cudaError_t e;
    if (a.dtype == DType::BF16) {
        if (a.vec && a.D % 8 == 0) e = dispatch<__nv_bfloat16, 8>(p, npt, sched, stream, launches, &piped);
        else e = dispatch<__nv_bfloat16, 1>(p, npt, sched, stream, launches, &piped);
    } else if (a.vec && a.D % 4 == 0) {
        e = dispatch<float, 4>(p, npt, sched, stream, launches, &piped);
    } else {
        e = dispatch<float, 1>(p, npt, sched, stream, launches, &piped);
    }
    if (a.ckpt_written) *a.ckpt_written = piped;
    return e;
}

}  // namespace ssm

// ---------------------------------------------------------------------------
// Fixed scratch for callers that cannot allocate device memory.
//
// The longest-first schedule of ssm_selective_scan_fwd normally lives in a
// caller-allocated workspace. ssm_selective_scan_fwd_noalloc uses this
// file-scope array instead: every GPU that loads the library holds its 16 KB
// until the process exits, and every call on a device shares it.
// ---------------------------------------------------------------------------
namespace ssm {

constexpr int64_t kNoallocMaxSeqs = 4096;
static __device__ __align__(256) int32_t g_noalloc_order[kNoallocMaxSeqs];

// Device address of g_noalloc_order on the current device. The first request
// on a device looks it up (with that device current) and caches it; later
// requests reuse the cached value.
cudaError_t noalloc_scratch(void **ptr, size_t *bytes)
{
    constexpr int kMaxDevices = 64;
    static void *cached[kMaxDevices] = {};
    static std::mutex lock;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(lock);
    if (!cached[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_order);
        if (e != cudaSuccess) return e;
        cached[dev] = p;
    }
    *ptr = cached[dev];
    *bytes = sizeof(g_noalloc_order);
    return cudaSuccess;
}

int64_t noalloc_max_sequences() { return kNoallocMaxSeqs; }

}  // namespace ssm
