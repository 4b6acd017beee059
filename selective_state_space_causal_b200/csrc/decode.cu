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
// sectors. The per-channel scalars (conv, softplus, gate) are computed by both
// lanes; the readout is combined with one shuffle.
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

template <typename T, typename TC, int K>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const Params p)
{
    const int tid = threadIdx.x;
    const int sub = tid & 1;
    const int64_t c = (int64_t)blockIdx.x * kChPerBlock + (tid >> 1);
    const int64_t b = blockIdx.y;
    const int64_t s = p.idx ? (int64_t)p.idx[b] : b;
    const bool active = (c < p.D) && (s >= 0) && (s < p.n_slots);
    const int64_t D = p.D;

    const T *X = static_cast<const T *>(p.x);
    const T *DT = static_cast<const T *>(p.dt);
    const T *Bp = static_cast<const T *>(p.B);
    const T *Cp = static_cast<const T *>(p.C);
    const T *Z = static_cast<const T *>(p.z);
    TC *CS = static_cast<TC *>(p.conv_state);

    float win[K];
    float xcv = 0.f, part = 0.f;
    float4 ha = make_float4(0.f, 0.f, 0.f, 0.f), hb = ha;
    float *hp = nullptr;
    if (active) {
        const TC *cs = CS + (s * D + c) * (K - 1);
#pragma unroll
        for (int j = 0; j < K - 1; ++j) win[j] = to_f32(cs[j]);
        win[K - 1] = to_f32(X[b * D + c]);
        float acc = p.conv_b ? __ldg(p.conv_b + c) : 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fmaf(__ldg(p.conv_w + c * K + k), win[k], acc);
        xcv = silu_f(acc);

        float d = to_f32(DT[b * D + c]) + (p.dt_bias ? __ldg(p.dt_bias + c) : 0.f);
        if (p.delta_softplus) d = softplus_f(d);
        const float dx = d * xcv;

        hp = p.ssm_state + (s * D + c) * kN;
        ha = *reinterpret_cast<const float4 *>(hp + sub * 4);
        hb = *reinterpret_cast<const float4 *>(hp + 8 + sub * 4);
        float hv[8] = {ha.x, ha.y, ha.z, ha.w, hb.x, hb.y, hb.z, hb.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int n = (j < 4 ? 0 : 8) + sub * 4 + (j & 3);
            const float a2 = __ldg(p.A + c * kN + n) * kLog2e;
            const float dA = ex2_approx(d * a2);
            hv[j] = fmaf(dA, hv[j], dx * to_f32(Bp[b * kN + n]));
            part = fmaf(to_f32(Cp[b * kN + n]), hv[j], part);
        }
        ha = make_float4(hv[0], hv[1], hv[2], hv[3]);
        hb = make_float4(hv[4], hv[5], hv[6], hv[7]);
    }
    // Both lanes of a channel have read the conv state before this exchange;
    // only afterwards does lane 0 overwrite it.
    const float ysum = part + __shfl_xor_sync(0xffffffffu, part, 1);
    if (active) {
        *reinterpret_cast<float4 *>(hp + sub * 4) = ha;
        *reinterpret_cast<float4 *>(hp + 8 + sub * 4) = hb;
        if (sub == 0) {
            float yv = ysum + (p.Dskip ? __ldg(p.Dskip + c) : 0.f) * xcv;
            if (Z) yv *= silu_f(to_f32(Z[b * D + c]));
            static_cast<T *>(p.y)[b * D + c] = from_f32<T>(yv);
            TC *cs = CS + (s * D + c) * (K - 1);
#pragma unroll
            for (int j = 0; j < K - 1; ++j) cs[j] = from_f32<TC>(win[j + 1]);
        }
    }
}

template <typename T, typename TC, int K>
cudaError_t run(const Params &p, int64_t Bt, cudaStream_t stream, int *launches)
{
    const dim3 grid((unsigned)((p.D + kChPerBlock - 1) / kChPerBlock), (unsigned)Bt);
    decode_kernel<T, TC, K><<<grid, kThreads, 0, stream>>>(p);
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
