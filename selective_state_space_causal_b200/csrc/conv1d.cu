// conv1d.cu -- causal depthwise conv1d + bias + SiLU over packed sequences.
//
// Follows tp_builder.py (TensorRT-Model-Connect, Mamba family),
// _add_mamba_tp_layer: the conv state is shifted by one and the new input
// appended, multiplied elementwise with the (D, K) weight, summed over K, biased
// and passed through SiLU. Here the same window slides over a whole packed
// batch: at every sequence start it is reloaded from that sequence's carried
// state (or zeros), so no input crosses a cu_seqlens boundary ("PackMamba",
// abstract).
//
// HBM-bound: per (token, channel) one input element is read and one output
// element written. Each thread owns a 16-byte vector of channels (8 bf16 or 4
// fp32) and a strip of kStrip consecutive tokens, keeping the K-1 previous
// inputs in registers, so every input is read from DRAM once; the K-1 halo rows
// at a strip's start are re-read from L2. Consecutive threads own consecutive
// channel vectors, so each token row is read and written fully coalesced.
#include "common.cuh"
#include "internal.h"

namespace ssm {
namespace {

constexpr int kStrip = 32;
constexpr int kThreads = 256;

struct Seqs {
    const int32_t *cu;  // nullptr: dense rows of L tokens
    int64_t S, tok, L;

    // Offset of sequence s. The first offset is taken as 0 whatever the array
    // holds, so that every token lies at or after its sequence's start.
    __device__ __forceinline__ int64_t off(int64_t s) const
    {
        if (s == 0) return 0;
        return cu ? clamp_off(cu[s], tok) : s * L;
    }
    // Largest s in [0, S-1] with off(s) <= t.
    __device__ __forceinline__ int64_t find(int64_t t) const
    {
        if (!cu) return min(t / L, S - 1);
        int64_t lo = 0, hi = S - 1;
        while (lo < hi) {
            const int64_t mid = (lo + hi + 1) >> 1;
            if (off(mid) <= t) lo = mid; else hi = mid - 1;
        }
        return lo;
    }
};

template <typename T, typename TS, int VEC, int K>
__global__ void __launch_bounds__(kThreads)
conv1d_kernel(const T *__restrict__ x, T *__restrict__ xc, const float *__restrict__ w,
              const float *__restrict__ bias, Seqs sq, int64_t D,
              const TS *__restrict__ state_in, int apply_silu)
{
    const int64_t nvec = D / VEC;
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t cv = gid % nvec;
    const int64_t t0 = (gid / nvec) * kStrip;
    if (t0 >= sq.tok) return;
    const int64_t t1 = min(t0 + (int64_t)kStrip, sq.tok);
    const int64_t c0 = cv * VEC;

    float wk[K][VEC], bv[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
#pragma unroll
        for (int k = 0; k < K; ++k) wk[k][i] = __ldg(w + (c0 + i) * K + k);
        bv[i] = bias ? __ldg(bias + c0 + i) : 0.f;
    }

    int64_t s = sq.find(t0);
    int64_t s_start = sq.off(s);
    int64_t s_end = max(sq.off(s + 1), s_start);

    // win[j] is the input K-1-j positions before the current token.
    float win[K - 1][VEC];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t pos = t0 - (K - 1) + j;
        if (pos >= s_start) {
            load_vec<T, VEC>(x + pos * D + c0, win[j]);
        } else {
#pragma unroll
            for (int i = 0; i < VEC; ++i)
                win[j][i] = state_in
                    ? to_f32(state_in[(s * D + c0 + i) * (K - 1) + (K - 1) + (pos - s_start)])
                    : 0.f;
        }
    }

    for (int64_t t = t0; t < t1; ++t) {
        if (t >= s_end) {
            // next non-empty sequence: its window starts from its carried state
            while (t >= s_end && s < sq.S - 1) {
                ++s;
                s_start = s_end;
                s_end = max(sq.off(s + 1), s_start);
            }
            if (t >= s_end) break;  // token outside every sequence
#pragma unroll
            for (int j = 0; j < K - 1; ++j)
#pragma unroll
                for (int i = 0; i < VEC; ++i)
                    win[j][i] = state_in ? to_f32(state_in[(s * D + c0 + i) * (K - 1) + j]) : 0.f;
        }
        float xv[VEC], out[VEC];
        load_vec<T, VEC>(x + t * D + c0, xv);
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            float acc = bv[i];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) acc = fmaf(wk[k][i], win[k][i], acc);
            acc = fmaf(wk[K - 1][i], xv[i], acc);
            out[i] = apply_silu ? silu_f(acc) : acc;
        }
        store_vec<T, VEC>(xc + t * D + c0, out);
#pragma unroll
        for (int j = 0; j < K - 2; ++j)
#pragma unroll
            for (int i = 0; i < VEC; ++i) win[j][i] = win[j + 1][i];
#pragma unroll
        for (int i = 0; i < VEC; ++i) win[K - 2][i] = xv[i];
    }
}

// conv_state_out[s, c, :] = last K-1 entries of [conv_state_in[s, c, :] || x_seq[:, c]].
// One thread per (sequence, channel) reads everything it needs before writing,
// so the output may be the same buffer as the input state.
template <typename T, typename TS, int K>
__global__ void __launch_bounds__(kThreads)
conv_state_out_kernel(const T *__restrict__ x, Seqs sq, int64_t D, const TS *state_in,
                      TS *state_out)
{
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (gid >= sq.S * D) return;
    const int64_t s = gid / D, c = gid % D;
    const int64_t s_start = sq.off(s);
    const int64_t len = max(sq.off(s + 1), s_start) - s_start;
    float v[K - 1];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t pos = len - (K - 1) + j;
        v[j] = pos >= 0 ? to_f32(x[(s_start + pos) * D + c])
                        : (state_in ? to_f32(state_in[(s * D + c) * (K - 1) + (K - 1) + pos]) : 0.f);
    }
#pragma unroll
    for (int j = 0; j < K - 1; ++j) state_out[(s * D + c) * (K - 1) + j] = from_f32<TS>(v[j]);
}

template <typename T, typename TS, int K>
cudaError_t run(const ConvArgs &a, cudaStream_t stream, int *launches)
{
    Seqs sq{a.cu, a.S, a.tok, a.cu ? 0 : a.tok / a.S};
    const T *x = static_cast<const T *>(a.x);
    const TS *st_in = static_cast<const TS *>(a.state_in);
    if (a.tok > 0) {
        constexpr int V = 16 / sizeof(T);
        const bool vec = a.vec && (a.D % V == 0);
        const int64_t nvec = vec ? a.D / V : a.D;
        const int64_t threads = nvec * ((a.tok + kStrip - 1) / kStrip);
        const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
        if (vec)
            conv1d_kernel<T, TS, V, K><<<blocks, kThreads, 0, stream>>>(
                x, static_cast<T *>(a.xc), a.w, a.bias, sq, a.D, st_in, a.apply_silu);
        else
            conv1d_kernel<T, TS, 1, K><<<blocks, kThreads, 0, stream>>>(
                x, static_cast<T *>(a.xc), a.w, a.bias, sq, a.D, st_in, a.apply_silu);
        ++*launches;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.state_out) {
        const int64_t n = a.S * a.D;
        const unsigned blocks = (unsigned)((n + kThreads - 1) / kThreads);
        conv_state_out_kernel<T, TS, K><<<blocks, kThreads, 0, stream>>>(
            x, sq, a.D, st_in, static_cast<TS *>(a.state_out));
        ++*launches;
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <typename T, typename TS>
cudaError_t by_k(const ConvArgs &a, cudaStream_t s, int *n)
{
    switch (a.K) {
    case 2: return run<T, TS, 2>(a, s, n);
    case 3: return run<T, TS, 3>(a, s, n);
    default: return run<T, TS, 4>(a, s, n);
    }
}

}  // namespace

cudaError_t launch_conv1d(const ConvArgs &a, cudaStream_t stream, int *launches)
{
    const bool xb = a.x_dtype == DType::BF16, sb = a.state_dtype == DType::BF16;
    if (xb && sb) return by_k<__nv_bfloat16, __nv_bfloat16>(a, stream, launches);
    if (xb) return by_k<__nv_bfloat16, float>(a, stream, launches);
    if (sb) return by_k<float, __nv_bfloat16>(a, stream, launches);
    return by_k<float, float>(a, stream, launches);
}

}  // namespace ssm
