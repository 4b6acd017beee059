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
// each way), which dwarfs everything else. Two adjacent lanes share a channel,
// 8 states each, loaded as two 16-byte vectors at offsets {0,32} and {16,48}
// bytes of the channel's 64 B, so every warp-wide load covers whole 32-byte
// sectors. A thread serves kRows rows of its channel: the channel's
// parameters are loaded once, and all rows' loads are in flight together.
// The per-channel scalars (conv, softplus, gate) are computed by both lanes;
// the readout is combined with one shuffle.
#include "common.cuh"
#include "internal.h"

namespace ssm {
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
            if (p.delta_softplus) d = softplus_f(d);
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

template <typename T, typename TC, int K>
cudaError_t run(const Params &p, int64_t Bt, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + kChPerBlock - 1) / kChPerBlock),
                    (unsigned)((Bt + kRows - 1) / kRows));
    decode_kernel<T, TC, K><<<grid, kThreads, 0, stream>>>(p, Bt);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, typename TC>
cudaError_t by_k(const Params &p, int K, int64_t Bt, cudaStream_t s, int *n)
{
    switch (K) {
    case 2: return run<T, TC, 2>(p, Bt, s, n);
    case 3: return run<T, TC, 3>(p, Bt, s, n);
    default: return run<T, TC, 4>(p, Bt, s, n);
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

}  // namespace ssm
