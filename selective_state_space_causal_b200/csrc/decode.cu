// decode.cu -- single-token selective state update with cached states (sm_100a).
//
// Follows tp_builder.py (TensorRT-Model-Connect, Mamba family),
// _add_mamba_tp_layer for one token: shift the conv state and append x, conv +
// bias + SiLU, softplus of dt, dA = exp(delta*A), h = dA*h + delta*xc*B,
// y = C.h + D*xc, times silu(z); the updated conv and SSM states are that
// builder's present_conv / present_ssm outputs, written here in place. The
// SSM state is the cache carried from prefill into decode ("Scaling
// State-Space Models on Multiple GPUs with Tensor Parallelism", abstract and
// Fig. 2, component 1).
//
// HBM-bound: each row reads and writes its 16 fp32 states per channel (64 B
// each way), which dwarfs everything else. Two kernels:
// * decode_bulk_kernel (16-byte aligned row slices): rows stream through
//   shared memory in whole blocks by 1-D bulk copies, several rows ahead, and
//   one thread owns all 16 states of a channel (see its comment).
// * decode_kernel (any alignment): two adjacent lanes share a channel, 8
//   states each, loaded as two 16-byte vectors at offsets {0,32} and {16,48}
//   bytes of the channel's 64 B, so every warp-wide load covers whole 32-byte
//   sectors; the per-channel scalars (conv, softplus, gate) are computed by
//   both lanes and the readout is combined with one shuffle.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace ssm {

// Set by a decode kernel whose bounded wait on its bulk copies gave up.
__device__ int g_decode_status = 0;

namespace {

constexpr int kN = 16;
constexpr int kThreads = 256;
constexpr int kChPerBlock = kThreads / 2;

struct Params {
    void *conv_state;
    float *ssm_state;
    const void *x, *dt, *B, *C, *z;
    const float *conv_w, *conv_b, *A, *Dskip, *dt_bias;
    const int32_t *idx;
    void *y;
    int64_t n_slots, D;
    int delta_softplus;
};

// Four consecutive B (or C) entries starting at a multiple of 4.
template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&o)[4])
{
    if constexpr (sizeof(T) == 2) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p));
        const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = to_f32(e[i]);
    } else {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
}

// Rows per thread: the per-channel parameters (A, conv weight and biases) are
// loaded once for R rows, and the loads of all R rows are issued before any
// arithmetic.
constexpr int kRows = 1;

template <typename T, typename TC, int K>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const Params p, const int64_t Bt)
{
    const int tid = threadIdx.x;
    const int sub = tid & 1;
    const int64_t c = (int64_t)blockIdx.x * kChPerBlock + (tid >> 1);
    const int64_t b0 = (int64_t)blockIdx.y * kRows;
    const int64_t D = p.D;
    const bool cvalid = c < D;

    const T *X = static_cast<const T *>(p.x);
    const T *DT = static_cast<const T *>(p.dt);
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    const T *Z = static_cast<const T *>(p.z);
    TC *CS = static_cast<TC *>(p.conv_state);

    // this lane's states: n = sub*4 .. sub*4+3 and 8+sub*4 .. 8+sub*4+3
    float a2[8], wk[K];
    float cb = 0.f, dsk = 0.f, dtb = 0.f;
    if (cvalid) {
        const float4 a0 = __ldg(reinterpret_cast<const float4 *>(p.A + c * kN + sub * 4));
        const float4 a1 = __ldg(reinterpret_cast<const float4 *>(p.A + c * kN + 8 + sub * 4));
        a2[0] = a0.x; a2[1] = a0.y; a2[2] = a0.z; a2[3] = a0.w;
        a2[4] = a1.x; a2[5] = a1.y; a2[6] = a1.z; a2[7] = a1.w;
#pragma unroll
        for (int j = 0; j < 8; ++j) a2[j] *= kLog2e;
        if constexpr (K == 4) {
            const float4 w4 = __ldg(reinterpret_cast<const float4 *>(p.conv_w + c * 4));
            wk[0] = w4.x; wk[1] = w4.y; wk[2] = w4.z; wk[3] = w4.w;
        } else {
#pragma unroll
            for (int k = 0; k < K; ++k) wk[k] = __ldg(p.conv_w + c * K + k);
        }
        cb = p.conv_b ? __ldg(p.conv_b + c) : 0.f;
        dsk = p.Dskip ? __ldg(p.Dskip + c) : 0.f;
        dtb = p.dt_bias ? __ldg(p.dt_bias + c) : 0.f;
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) a2[j] = 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) wk[k] = 0.f;
    }

    // issue every load of the R rows first
    int64_t slot[kRows];
    bool live[kRows];
    float win[kRows][K], dtv[kRows], zv[kRows], bv[kRows][8], cv[kRows][8];
    float4 ha[kRows], hb[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int64_t b = b0 + r;
        const int64_t s = (b < Bt) ? (p.idx ? (int64_t)p.idx[b] : b) : -1;
        slot[r] = s;
        live[r] = cvalid && s >= 0 && s < p.n_slots;
        ha[r] = hb[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (live[r]) {
            const TC *cs = CS + (s * D + c) * (K - 1);
#pragma unroll
            for (int j = 0; j < K - 1; ++j) win[r][j] = to_f32(cs[j]);
            win[r][K - 1] = to_f32(X[b * D + c]);
            dtv[r] = to_f32(DT[b * D + c]);
            zv[r] = Z ? to_f32(Z[b * D + c]) : 0.f;
            const float *hp = p.ssm_state + (s * D + c) * kN;
            ha[r] = *reinterpret_cast<const float4 *>(hp + sub * 4);
            hb[r] = *reinterpret_cast<const float4 *>(hp + 8 + sub * 4);
            float t4[4];
            load4<T>(Bp + b * kN + sub * 4, t4);
#pragma unroll
            for (int i = 0; i < 4; ++i) bv[r][i] = t4[i];
            load4<T>(Bp + b * kN + 8 + sub * 4, t4);
#pragma unroll
            for (int i = 0; i < 4; ++i) bv[r][4 + i] = t4[i];
            load4<T>(Cp + b * kN + sub * 4, t4);
#pragma unroll
            for (int i = 0; i < 4; ++i) cv[r][i] = t4[i];
            load4<T>(Cp + b * kN + 8 + sub * 4, t4);
#pragma unroll
            for (int i = 0; i < 4; ++i) cv[r][4 + i] = t4[i];
        }
    }

#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        float part = 0.f, xcv = 0.f;
        if (live[r]) {
            float acc = cb;
#pragma unroll
            for (int k = 0; k < K; ++k) acc = fmaf(wk[k], win[r][k], acc);
            xcv = silu_f(acc);
            float d = dtv[r] + dtb;
            if (p.delta_softplus) d = softplus_fast(d);
            const float dx = d * xcv;
            float hv[8] = {ha[r].x, ha[r].y, ha[r].z, ha[r].w, hb[r].x, hb[r].y, hb[r].z, hb[r].w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float dA = ex2_approx(d * a2[j]);
                hv[j] = fmaf(dA, hv[j], dx * bv[r][j]);
                part = fmaf(cv[r][j], hv[j], part);
            }
            ha[r] = make_float4(hv[0], hv[1], hv[2], hv[3]);
            hb[r] = make_float4(hv[4], hv[5], hv[6], hv[7]);
        }
        // Both lanes of a channel have read the conv state before this
        // exchange; only afterwards does lane 0 overwrite it.
        const float ysum = part + __shfl_xor_sync(0xffffffffu, part, 1);
        if (live[r]) {
            const int64_t b = b0 + r, s = slot[r];
            float *hp = p.ssm_state + (s * D + c) * kN;
            *reinterpret_cast<float4 *>(hp + sub * 4) = ha[r];
            *reinterpret_cast<float4 *>(hp + 8 + sub * 4) = hb[r];
            if (sub == 0) {
                float yv = ysum + dsk * xcv;
                if (Z) yv *= silu_f(zv[r]);
                static_cast<T *>(p.y)[b * D + c] = from_f32<T>(yv);
                TC *cs = CS + (s * D + c) * (K - 1);
#pragma unroll
                for (int j = 0; j < K - 1; ++j) cs[j] = from_f32<TC>(win[r][j + 1]);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Bulk-staged variant (all row slices 16-byte aligned). A CTA owns kBulkCh
// channels and walks rows gridDim.y apart, so A, the conv weight and the
// per-channel scalars stay in registers. For each of its rows, lane 0 brings
// the row's contiguous state block (kBulkCh x 64 B), conv-state slice and x,
// dt, z slices into shared memory with 1-D bulk copies, kBulkStages rows
// ahead; each thread owns one channel and all 16 of its states, updates them
// in shared memory, and lane 0 writes the state and conv-state blocks back
// with bulk stores. The copies hold no registers, so many rows' bytes are in
// flight per SM, and the state moves in whole 8 KB blocks.
// ---------------------------------------------------------------------------
constexpr int kBulkCh = 128;      // channels (threads) per CTA
constexpr int kBulkStages = 3;    // rows in flight per CTA (measured best of 2..8)

template <typename T, typename TC, int K>
struct BulkTile {
    static constexpr size_t ST = (size_t)kBulkCh * kN * sizeof(float);
    static constexpr size_t CS = ((size_t)kBulkCh * (K - 1) * sizeof(TC) + 15) / 16 * 16;
    static constexpr size_t AC = ((size_t)kBulkCh * sizeof(T) + 15) / 16 * 16;
    static constexpr size_t OFF_CS = ST, OFF_X = OFF_CS + CS, OFF_DT = OFF_X + AC, OFF_Z = OFF_DT + AC;
    static constexpr size_t STAGE = (OFF_Z + AC + 127) / 128 * 128;
    static constexpr size_t SMEM = kBulkStages * STAGE + 8 * kBulkStages;
};

// Four consecutive B (or C) entries starting at a multiple of 4, as two packed pairs.
template <typename T>
__device__ __forceinline__ void load4p(const T *p, f32x2 &lo, f32x2 &hi)
{
    if constexpr (sizeof(T) == 2) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p));
        lo = pk2(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u));
        hi = pk2(__uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
    } else {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        lo = pk2(v.x, v.y);
        hi = pk2(v.z, v.w);
    }
}

template <typename T, typename TC, int K>
__global__ void __launch_bounds__(kBulkCh)
decode_bulk_kernel(const Params p, const int64_t Bt)
{
    using G = BulkTile<T, TC, K>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kBulkStages * G::STAGE);
    const int t = threadIdx.x;
    const int64_t D = p.D;
    const int64_t c0 = (int64_t)blockIdx.x * kBulkCh;
    const int nch = (int)min((int64_t)kBulkCh, D - c0);
    const int64_t c = c0 + t;
    const bool cvalid = t < nch;
    const int64_t rstep = gridDim.y, r0 = blockIdx.y;
    const int nrows = (int)((Bt - r0 + rstep - 1) / rstep);
    const uint32_t st_b = (uint32_t)nch * kN * sizeof(float);
    const uint32_t cs_b = (uint32_t)(nch * (K - 1) * sizeof(TC));
    const uint32_t a_b = (uint32_t)(nch * sizeof(T));
    const int has_z = p.z != nullptr;
    TC *CS = static_cast<TC *>(p.conv_state);

    auto slot = [&](int j) -> int64_t {
        const int64_t b = r0 + (int64_t)j * rstep;
        const int64_t s = p.idx ? (int64_t)p.idx[b] : b;
        return (s >= 0 && s < p.n_slots) ? s : -1;
    };
    auto stage = [&](int st) { return smem + (size_t)st * G::STAGE; };
    auto issue = [&](int j) {  // lane 0 of warp 0 only
        const int st = j % kBulkStages;
        const int64_t s = slot(j);
        if (s < 0) {  // row skipped: complete the phase without data
            mbar_arrive(&bar[st]);
            return;
        }
        const int64_t b = r0 + (int64_t)j * rstep;
        unsigned char *dst = stage(st);
        mbar_expect_tx(&bar[st], st_b + cs_b + (uint32_t)(has_z ? 3 : 2) * a_b);
        bulk_g2s(dst, p.ssm_state + (s * D + c0) * kN, st_b, &bar[st]);
        bulk_g2s(dst + G::OFF_CS, CS + (s * D + c0) * (K - 1), cs_b, &bar[st]);
        bulk_g2s(dst + G::OFF_X, static_cast<const T *>(p.x) + b * D + c0, a_b, &bar[st]);
        bulk_g2s(dst + G::OFF_DT, static_cast<const T *>(p.dt) + b * D + c0, a_b, &bar[st]);
        if (has_z) bulk_g2s(dst + G::OFF_Z, static_cast<const T *>(p.z) + b * D + c0, a_b, &bar[st]);
    };

    if (t == 0) {
        for (int st = 0; st < kBulkStages; ++st) mbar_init_n(&bar[st], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (t == 0)
        for (int j = 0; j < kBulkStages && j < nrows; ++j) issue(j);

    // This thread's 16 states are handled as 4 vectors of 4, visited in an
    // order rotated by rot = (t / 2) mod 4: local vector q is state vector
    // m = (q + rot) mod 4, so the 8 lanes of each shared-memory phase hit 8
    // different bank groups. A, B and C are read in the same rotated order.
    const int rot = (t >> 1) & 3;
    f32x2 A2[8];
    float w[K], cb = 0.f, dtb = 0.f, dsk = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int m = (q + rot) & 3;
        const float4 a4 = cvalid ? __ldg(reinterpret_cast<const float4 *>(p.A + c * kN + 4 * m))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        A2[2 * q] = pk2(a4.x * kLog2e, a4.y * kLog2e);
        A2[2 * q + 1] = pk2(a4.z * kLog2e, a4.w * kLog2e);
    }
#pragma unroll
    for (int k = 0; k < K; ++k) w[k] = cvalid ? __ldg(p.conv_w + c * K + k) : 0.f;
    if (cvalid) {
        cb = p.conv_b ? __ldg(p.conv_b + c) : 0.f;
        dtb = p.dt_bias ? __ldg(p.dt_bias + c) : 0.f;
        dsk = p.Dskip ? __ldg(p.Dskip + c) : 0.f;
    }

    bool failed = false;
    for (int j = 0; j < nrows; ++j) {
        const int st = j % kBulkStages;
        mbar_wait(&bar[st], (uint32_t)((j / kBulkStages) & 1), failed, &g_decode_status, 1);
        const int64_t s = slot(j);
        const int64_t b = r0 + (int64_t)j * rstep;
        unsigned char *sp = stage(st);
        if (s >= 0 && cvalid) {
            float4 *sh = reinterpret_cast<float4 *>(sp) + t * 4;
            float4 hq[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) hq[q] = sh[(q + rot) & 3];
            TC *scs = reinterpret_cast<TC *>(sp + G::OFF_CS) + t * (K - 1);
            float win[K];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) win[k] = to_f32(scs[k]);
            win[K - 1] = to_f32(reinterpret_cast<const T *>(sp + G::OFF_X)[t]);
            float d = to_f32(reinterpret_cast<const T *>(sp + G::OFF_DT)[t]) + dtb;
            float acc = cb;
#pragma unroll
            for (int k = 0; k < K; ++k) acc = fmaf(w[k], win[k], acc);
            const float xcv = silu_f(acc);
            if (p.delta_softplus) d = softplus_fast(d);
            const float dx = d * xcv;
            const f32x2 dd = pk2(d, d), xx = pk2(dx, dx);
            const T *Bp = static_cast<const T *>(p.B) + b * kN;
            const T *Cp = static_cast<const T *>(p.C) + b * kN;
            f32x2 yacc = 0ull;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int m = (q + rot) & 3;
                f32x2 b01, b23, c01, c23;
                load4p<T>(Bp + 4 * m, b01, b23);
                load4p<T>(Cp + 4 * m, c01, c23);
                float4 &h4 = hq[q];
                float e0, e1, e2, e3;
                upk2(mul2(dd, A2[2 * q]), e0, e1);
                upk2(mul2(dd, A2[2 * q + 1]), e2, e3);
                const f32x2 h01 = fma2(pk2(ex2_approx(e0), ex2_approx(e1)), pk2(h4.x, h4.y),
                                       mul2(xx, b01));
                const f32x2 h23 = fma2(pk2(ex2_approx(e2), ex2_approx(e3)), pk2(h4.z, h4.w),
                                       mul2(xx, b23));
                yacc = fma2(c01, h01, yacc);
                yacc = fma2(c23, h23, yacc);
                upk2(h01, h4.x, h4.y);
                upk2(h23, h4.z, h4.w);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) sh[(q + rot) & 3] = hq[q];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) scs[k] = from_f32<TC>(win[k + 1]);
            float y0, y1;
            upk2(yacc, y0, y1);
            float yv = y0 + y1 + dsk * xcv;
            if (has_z) yv *= silu_f(to_f32(reinterpret_cast<const T *>(sp + G::OFF_Z)[t]));
            static_cast<T *>(p.y)[b * D + c] = from_f32<T>(yv);
            // this thread's shared-memory writes, before the bulk store reads them
            fence_proxy_async();
        }
        __syncthreads();
        if (t == 0) {
            if (s >= 0) {
                bulk_s2g(p.ssm_state + (s * D + c0) * kN, sp, st_b);
                bulk_s2g(CS + (s * D + c0) * (K - 1), sp + G::OFF_CS, cs_b);
            }
            bulk_commit();
            // refill the stage of the previous row once its store has read it
            if (j >= 1 && j - 1 + kBulkStages < nrows) {
                bulk_wait_read<1>();
                issue(j - 1 + kBulkStages);
            }
        }
    }
    if (t == 0) bulk_wait<0>();
}

template <typename T, typename TC, int K>
cudaError_t run_bulk(const Params &p, int64_t Bt, cudaStream_t stream, int *launches)
{
    using G = BulkTile<T, TC, K>;
    const uintptr_t mis = (uintptr_t)p.ssm_state | (uintptr_t)p.conv_state | (uintptr_t)p.x |
                          (uintptr_t)p.dt | (uintptr_t)p.z | (uintptr_t)p.B | (uintptr_t)p.C;
    const bool ok = (mis % 16 == 0) && (p.D * (int64_t)sizeof(T)) % 16 == 0 &&
                    (p.D * (K - 1) * (int64_t)sizeof(TC)) % 16 == 0;
    if (!ok) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(decode_bulk_kernel<T, TC, K>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_bulk_kernel<T, TC, K>, kBulkCh,
                                                      G::SMEM) != cudaSuccess)
        return cudaErrorUnknown;
    const int64_t gx = (p.D + kBulkCh - 1) / kBulkCh;
    int64_t gy = ((int64_t)sms * (per_sm > 0 ? per_sm : 1)) / gx;
    gy = gy < 1 ? 1 : (gy > Bt ? Bt : gy);
    if (gy > 65535) gy = 65535;
    decode_bulk_kernel<T, TC, K><<<dim3((unsigned)gx, (unsigned)gy), kBulkCh, G::SMEM, stream>>>(p, Bt);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, typename TC, int K>
cudaError_t run(const Params &p, int64_t Bt, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + kChPerBlock - 1) / kChPerBlock),
                    (unsigned)((Bt + kRows - 1) / kRows));
    decode_kernel<T, TC, K><<<grid, kThreads, 0, stream>>>(p, Bt);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, typename TC, int K>
cudaError_t run_any(const Params &p, int64_t Bt, cudaStream_t s, int *n)
{
    const cudaError_t e = run_bulk<T, TC, K>(p, Bt, s, n);
    if (e != cudaErrorNotSupported) return e;
    return run<T, TC, K>(p, Bt, s, n);
}

template <typename T, typename TC>
cudaError_t by_k(const Params &p, int K, int64_t Bt, cudaStream_t s, int *n)
{
    switch (K) {
    case 2: return run_any<T, TC, 2>(p, Bt, s, n);
    case 3: return run_any<T, TC, 3>(p, Bt, s, n);
    default: return run_any<T, TC, 4>(p, Bt, s, n);
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream, int *launches)
{
    Params p;
    p.conv_state = a.conv_state; p.ssm_state = a.ssm_state;
    p.x = a.x; p.dt = a.dt; p.B = a.B; p.C = a.C; p.z = a.z;
    p.conv_w = a.conv_w; p.conv_b = a.conv_b; p.A = a.A; p.Dskip = a.Dskip;
    p.dt_bias = a.dt_bias; p.idx = a.idx; p.y = a.y;
    p.n_slots = a.n_slots; p.D = a.D; p.delta_softplus = a.delta_softplus;
    if (a.Bt == 0) return cudaSuccess;
    const bool xb = a.dtype == DType::BF16, cb = a.conv_dtype == DType::BF16;
    if (xb && cb) return by_k<__nv_bfloat16, __nv_bfloat16>(p, a.K, a.Bt, stream, launches);
    if (xb) return by_k<__nv_bfloat16, float>(p, a.K, a.Bt, stream, launches);
    if (cb) return by_k<float, __nv_bfloat16>(p, a.K, a.Bt, stream, launches);
    return by_k<float, float>(p, a.K, a.Bt, stream, launches);
}

int read_decode_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_decode_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_decode_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace ssm
