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
#include "common.cuh"
#include "internal.h"
#include "scan_parts.cuh"

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

// The fused kernel: 16-byte channel vectors (4 or 8 states per lane, as the
// scan's variant choice says) where every row is 16-byte aligned, else scalar
// channels with 4 states per lane.
cudaError_t launch_conv_scan(const ConvScanArgs &a, int npt, cudaStream_t stream, int *launches)
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
    if (xb && sb) return by_kw<__nv_bfloat16, __nv_bfloat16>(p, cp, a.K, npt, vec, stream, launches);
    if (xb) return by_kw<__nv_bfloat16, float>(p, cp, a.K, npt, vec, stream, launches);
    if (sb) return by_kw<float, __nv_bfloat16>(p, cp, a.K, npt, vec, stream, launches);
    return by_kw<float, float>(p, cp, a.K, npt, vec, stream, launches);
}

}  // namespace ssm
