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
// channel) needs N = 16 exponentials against only ~8 bytes of DRAM traffic in
// bf16. The kernel therefore spends as few issue slots as possible on anything
// but the 16 dA exponentials and their 4 FMA-pipe companions:
//
// * A CTA owns one sequence and CH channels. A channel's N = 16 states are split
//   over TPC = 16 / NPT adjacent lanes (NPT states each) so that small batches
//   still fill 148 SMs; h stays in fp32 registers for the whole sequence.
// * The sequence is walked in chunks of TCH tokens. Each chunk's per-(token,
//   channel) work (softplus, delta*u, silu(z), bf16 unpacking) is done ONCE in a
//   cooperative pre-pass into shared memory, from 16-byte loads that were issued
//   one chunk ahead into registers (software prefetch), so the DRAM latency of
//   chunk k+1 hides behind the recurrence of chunk k.
// * In the recurrence each lane reads delta and delta*u (broadcast within the
//   channel) and 4-wide B/C vectors from shared memory, runs NPT exps + FMAs per
//   token, and the TPC partial readouts are combined with a transposed butterfly
//   over shuffles: after log2(TPC) steps lane `sub` holds the full sum of token
//   `sub` of the group, which it gates and writes back in place.
// * Tokens past a sequence's end are padded with delta = 0 (dA = 1, no input),
//   which leaves h unchanged, so the inner loop needs no tail branch.
// * Packed sequences are scheduled longest-first when scratch is supplied.
#include "common.cuh"
#include "internal.h"

namespace ssm {
namespace {

constexpr int kN = 16;

struct Params {
    const void *u, *delta, *B, *C, *z;
    const float *A, *Dskip, *dt_bias, *h0;
    const int32_t *cu;
    const int32_t *order;
    void *y;
    float *h_final;
    int64_t S, tok, D, L;
    int delta_softplus;
};

template <typename T, int NPT_, int CH_, int TCH_, int VEC_>
struct Cfg {
    static constexpr int NPT = NPT_, CH = CH_, TCH = TCH_, VEC = VEC_;
    static constexpr int TPC = kN / NPT;                  // lanes per channel
    static constexpr int THREADS = CH * TPC;
    static constexpr int CV = CH / VEC;                   // channel vectors per row
    static constexpr int ITEMS = TCH * CV;                // (token, vector) items per chunk
    static constexpr int IPT = ITEMS / THREADS;           // items per thread
    static constexpr int SROW = CH + 4;                   // padded smem row, floats
    static constexpr int BCVEC = 16 / sizeof(T);          // B/C elements per 16-byte load
    static constexpr int BCN = TCH * kN / BCVEC;          // 16-byte B (or C) loads per chunk
    static constexpr int BPT = (BCN + THREADS - 1) / THREADS;
    static constexpr size_t SMEM = sizeof(float) * (4 * TCH * SROW + 2 * TCH * kN);
    static_assert(ITEMS % THREADS == 0, "items must divide evenly");
    static_assert(THREADS % CV == 0, "each thread keeps one channel vector");
    static_assert(TCH % TPC == 0, "chunk must hold whole token groups");
    static_assert(THREADS <= 1024 && (THREADS % 32) == 0, "block size");
};

// Raw prefetch register of one (token, vector) item: 16 bytes, or one element.
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

template <class K, typename T>
__global__ void __launch_bounds__(K::THREADS)
scan_kernel(const Params p)
{
    constexpr int NPT = K::NPT, CH = K::CH, TCH = K::TCH, VEC = K::VEC, TPC = K::TPC;
    constexpr int THREADS = K::THREADS, CV = K::CV, IPT = K::IPT, SROW = K::SROW;
    using RawT = typename Raw<T, VEC>::type;

    extern __shared__ __align__(16) float smem[];
    float *sD = smem;                 // delta                [TCH][SROW]
    float *sDX = sD + TCH * SROW;     // delta * u            [TCH][SROW]
    float *sU = sDX + TCH * SROW;     // u, then y in place   [TCH][SROW]
    float *sG = sU + TCH * SROW;      // silu(z) (or 1)       [TCH][SROW]
    float *sB = sG + TCH * SROW;      // B                    [TCH][16]
    float *sC = sB + TCH * kN;        // C                    [TCH][16]

    const int tid = threadIdx.x;
    const int chl = tid / TPC, sub = tid % TPC;
    const int64_t cbase = (int64_t)blockIdx.x * CH;
    const int64_t c = cbase + chl;
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

    const T *U = static_cast<const T *>(p.u);
    const T *DT = static_cast<const T *>(p.delta);
    const T *Z = static_cast<const T *>(p.z);
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    T *Y = static_cast<T *>(p.y);

    // per-lane constants: A * log2(e), the state, Dskip
    float A2[NPT], h[NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
        A2[j] = cvalid ? __ldg(p.A + c * kN + sub * NPT + j) * kLog2e : 0.f;
        h[j] = (cvalid && p.h0) ? p.h0[(seq * p.D + c) * kN + sub * NPT + j] : 0.f;
    }
    const float dsk = (cvalid && p.Dskip) ? __ldg(p.Dskip + c) : 0.f;

    // this thread's channel vector in the pre-pass is fixed (THREADS % CV == 0)
    const int cvl = tid % CV;
    const int64_t cg = cbase + (int64_t)cvl * VEC;
    const bool vvalid = cg < p.D;  // D % VEC == 0 on the vector path
    float dtb[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) dtb[i] = (vvalid && p.dt_bias) ? __ldg(p.dt_bias + cg + i) : 0.f;

    RawT rdt[IPT], ru[IPT], rz[IPT];
    uint4 rb[K::BPT], rc[K::BPT];

    auto prefetch = [&](int64_t t0) {
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            const int tl = (tid + i * THREADS) / CV;
            const int64_t row = t0 + tl;
            if (row < end && vvalid) {
                const int64_t off = row * p.D + cg;
                rdt[i] = ld_raw<T, VEC>(DT + off);
                ru[i] = ld_raw<T, VEC>(U + off);
                if (Z) rz[i] = ld_raw<T, VEC>(Z + off);
            }
        }
#pragma unroll
        for (int i = 0; i < K::BPT; ++i) {
            const int q = tid + i * THREADS;
            const int64_t row = t0 + (q * K::BCVEC) / kN;
            if (q < K::BCN && row < end) {
                const int64_t off = t0 * kN + (int64_t)q * K::BCVEC;
                rb[i] = ldg16(Bp + off);
                rc[i] = ldg16(Cp + off);
            }
        }
    };

    if (start < end) prefetch(start);

    for (int64_t t0 = start; t0 < end; t0 += TCH) {
        const int nt = (int)min((int64_t)TCH, end - t0);

        // ---- pre-pass: per-(token, channel) scalars into shared memory ----
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            const int tl = (tid + i * THREADS) / CV;
            float vd[VEC], vdx[VEC], vu[VEC], vg[VEC];
            if (tl < nt && vvalid) {
                float fdt[VEC], fu[VEC], fz[VEC];
                unpack<T, VEC>(rdt[i], fdt);
                unpack<T, VEC>(ru[i], fu);
                if (Z) unpack<T, VEC>(rz[i], fz);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    float d = fdt[e] + dtb[e];
                    if (p.delta_softplus) d = softplus_f(d);
                    vd[e] = d;
                    vdx[e] = d * fu[e];
                    vu[e] = fu[e];
                    vg[e] = Z ? silu_f(fz[e]) : 1.f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) vd[e] = vdx[e] = vu[e] = vg[e] = 0.f;
            }
            const int so = tl * SROW + cvl * VEC;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                sD[so + e] = vd[e];
                sDX[so + e] = vdx[e];
                sU[so + e] = vu[e];
                sG[so + e] = vg[e];
            }
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

        if (t0 + TCH < end) prefetch(t0 + TCH);

        // ---- recurrence over the chunk ----
        const int ntr = ((nt + TPC - 1) / TPC) * TPC;
        for (int tt = 0; tt < ntr; tt += TPC) {
            float yp[TPC];
#pragma unroll
            for (int q = 0; q < TPC; ++q) {
                const int tq = tt + q;
                const float d = sD[tq * SROW + chl];
                const float dx = sDX[tq * SROW + chl];
                float bv[NPT], cv[NPT];
#pragma unroll
                for (int j = 0; j < NPT; j += 4) {
                    const float4 b4 = *reinterpret_cast<const float4 *>(sB + tq * kN + sub * NPT + j);
                    const float4 c4 = *reinterpret_cast<const float4 *>(sC + tq * kN + sub * NPT + j);
                    bv[j] = b4.x; bv[j + 1] = b4.y; bv[j + 2] = b4.z; bv[j + 3] = b4.w;
                    cv[j] = c4.x; cv[j + 1] = c4.y; cv[j + 2] = c4.z; cv[j + 3] = c4.w;
                }
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < NPT; ++j) {
                    const float dA = ex2_approx(d * A2[j]);
                    h[j] = fmaf(dA, h[j], dx * bv[j]);
                    acc = fmaf(cv[j], h[j], acc);
                }
                yp[q] = acc;
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
            const int tq = tt + sub;
            const float uval = sU[tq * SROW + chl];
            sU[tq * SROW + chl] = (yp[0] + dsk * uval) * sG[tq * SROW + chl];
        }
        __syncthreads();

        // ---- write y (same (token, vector) items as the pre-pass) ----
#pragma unroll
        for (int i = 0; i < IPT; ++i) {
            const int tl = (tid + i * THREADS) / CV;
            if (tl < nt && vvalid) {
                float out[VEC];
                const int so = tl * SROW + cvl * VEC;
#pragma unroll
                for (int e = 0; e < VEC; ++e) out[e] = sU[so + e];
                store_vec<T, VEC>(Y + (t0 + tl) * p.D + cg, out);
            }
        }
        // The next pre-pass rewrites only slots this thread just read (sU) or
        // slots no thread reads after the barrier above, so no barrier here.
    }

    if (cvalid && p.h_final) {
#pragma unroll
        for (int j = 0; j < NPT; ++j) p.h_final[(seq * p.D + c) * kN + sub * NPT + j] = h[j];
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

template <class K, typename T>
cudaError_t run(const Params &p, cudaStream_t stream, int *launches)
{
    const unsigned gx = (unsigned)((p.D + K::CH - 1) / K::CH);
    const unsigned gy = (unsigned)p.S;
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<K, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::SMEM);
    if (e != cudaSuccess) return e;
    scan_kernel<K, T><<<dim3(gx, gy), K::THREADS, K::SMEM, stream>>>(p);
    ++*launches;
    return cudaGetLastError();
}

// Variants: NPT states per lane, CH channels per CTA, TCH tokens per chunk.
template <typename T, int VEC>
cudaError_t dispatch(const Params &p, int npt, cudaStream_t s, int *n)
{
    switch (npt) {
    case 16: return run<Cfg<T, 16, 128, 32, VEC>, T>(p, s, n);
    case 8: return run<Cfg<T, 8, 64, 64, VEC>, T>(p, s, n);
    default: return run<Cfg<T, 4, 32, 64, VEC>, T>(p, s, n);
    }
}

int g_forced_npt = 0;

// States per lane: as many as keep at least ~4 warps per SM sub-partition
// busy (148 SMs x 4 SMSPs); fewer states per lane split a channel over more
// lanes when there are few (sequence, channel) pairs.
int pick_npt(int64_t S, int64_t D)
{
    if (g_forced_npt) return g_forced_npt;
    const int64_t pairs = S * D;
    const int64_t want_warps = 148 * 4 * 4;
    if (pairs / 32 >= want_warps) return 16;
    if (pairs * 2 / 32 >= want_warps) return 8;
    return 4;
}

}  // namespace

void set_scan_npt(int npt) { g_forced_npt = (npt == 4 || npt == 8 || npt == 16) ? npt : 0; }

size_t scan_order_bytes(int64_t S) { return (size_t)((S * 4 + 255) / 256) * 256; }

cudaError_t launch_scan(const ScanArgs &a, cudaStream_t stream, int *launches)
{
    Params p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z;
    p.A = a.A; p.Dskip = a.Dskip; p.dt_bias = a.dt_bias; p.h0 = a.h0;
    p.cu = a.cu; p.order = nullptr; p.y = a.y; p.h_final = a.h_final;
    p.S = a.S; p.tok = a.tok; p.D = a.D; p.L = a.cu ? 0 : a.tok / a.S;
    p.delta_softplus = a.delta_softplus;
    if (a.cu && a.order && a.S > 1) {
        order_kernel<<<1, 1024, 0, stream>>>(a.cu, a.S, a.tok, a.order);
        ++*launches;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        p.order = a.order;
    }
    const int npt = pick_npt(a.S, a.D);
    if (a.dtype == DType::BF16) {
        if (a.vec && a.D % 8 == 0) return dispatch<__nv_bfloat16, 8>(p, npt, stream, launches);
        return dispatch<__nv_bfloat16, 1>(p, npt, stream, launches);
    }
    if (a.vec && a.D % 4 == 0) return dispatch<float, 4>(p, npt, stream, launches);
    return dispatch<float, 1>(p, npt, stream, launches);
}

}  // namespace ssm
