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
// A strip that lies inside one sequence issues all of its loads before any
// arithmetic, which keeps enough bytes in flight to run at HBM speed.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace ssm {

// Set by a conv kernel whose bounded wait on its TMA tile gave up.
__device__ int g_conv_status = 0;

namespace {

constexpr int kStrip = 16;
constexpr int kThreads = 128;

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

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// SiLU as z * 1/(1 + 2^(-z log2 e)) on the special-function unit; every conv
// path (and the packed one below) uses exactly these operations, so a token
// gets the same bits whichever path computes it.
__device__ __forceinline__ float conv_silu(float z)
{
    return z * rcp_approx(ex2_approx(z * -kLog2e) + 1.f);
}

template <typename T, int VEC, int K>
__device__ __forceinline__ void conv_out(const float (&wk)[K][VEC], const float (&bv)[VEC],
                                         const float (&win)[K][VEC], int apply_silu,
                                         float (&out)[VEC])
{
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        float acc = bv[i];
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fmaf(wk[k][i], win[k][i], acc);
        out[i] = apply_silu ? conv_silu(acc) : acc;
    }
}

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

    if constexpr (VEC * sizeof(T) == 16) {
        // Fast path: the strip and its K-1 halo rows lie inside one sequence.
        // All loads are issued before any use, so each thread keeps
        // (kStrip + K - 1) x 16 bytes in flight.
        if (t0 - (K - 1) >= s_start && t0 + kStrip <= s_end) {
            uint4 raw[kStrip + K - 1];
#pragma unroll
            for (int r = 0; r < kStrip + K - 1; ++r)
                raw[r] = ldg16(x + (t0 - (K - 1) + r) * D + c0);
            float win[K][VEC];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) unpack16<T, VEC>(raw[k], win[k]);
#pragma unroll
            for (int t = 0; t < kStrip; ++t) {
                unpack16<T, VEC>(raw[t + K - 1], win[K - 1]);
                float out[VEC];
                conv_out<T, VEC, K>(wk, bv, win, apply_silu, out);
                store_vec<T, VEC>(xc + (t0 + t) * D + c0, out);
#pragma unroll
                for (int k = 0; k < K - 1; ++k)
#pragma unroll
                    for (int i = 0; i < VEC; ++i) win[k][i] = win[k + 1][i];
            }
            return;
        }
    }

    // General path: sequence starts inside the strip or its halo.
    // win[j] is the input K-1-j positions before the current token.
    float win[K][VEC];
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
        load_vec<T, VEC>(x + t * D + c0, win[K - 1]);
        float out[VEC];
        conv_out<T, VEC, K>(wk, bv, win, apply_silu, out);
        store_vec<T, VEC>(xc + t * D + c0, out);
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
#pragma unroll
            for (int i = 0; i < VEC; ++i) win[j][i] = win[j + 1][i];
    }
}

// Packed-pair helpers of the TMA path: 8 bytes of channels (4 bf16 or 2 fp32)
// as VEC/2 fp32x2 pairs, the K-tap window in packed FFMA and conv_silu per half.
template <typename T, int VEC>
__device__ __forceinline__ void unpack8_pk(const uint2 &raw, f32x2 (&o)[VEC / 2])
{
    static_assert(VEC * sizeof(T) == 8, "8-byte vectors");
    if constexpr (sizeof(T) == 2) {
        o[0] = pk2(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u));
        o[1] = pk2(__uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
    } else {
        o[0] = pk2(__uint_as_float(raw.x), __uint_as_float(raw.y));
    }
}

template <typename T, int VEC>
__device__ __forceinline__ void store8_pk(T *p, const f32x2 (&v)[VEC / 2])
{
    uint2 raw;
    if constexpr (sizeof(T) == 2) {
        float a, b, c, d;
        upk2(v[0], a, b);
        upk2(v[1], c, d);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
        raw.x = *reinterpret_cast<const uint32_t *>(&lo);
        raw.y = *reinterpret_cast<const uint32_t *>(&hi);
    } else {
        float a, b;
        upk2(v[0], a, b);
        raw.x = __float_as_uint(a);
        raw.y = __float_as_uint(b);
    }
    *reinterpret_cast<uint2 *>(p) = raw;
}

template <int VEC, int K>
__device__ __forceinline__ void conv_out_pk(const f32x2 (&wk)[K][VEC / 2], const f32x2 (&bv)[VEC / 2],
                                            const f32x2 (&win)[K][VEC / 2], int apply_silu,
                                            f32x2 (&out)[VEC / 2])
{
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) {
        f32x2 acc = bv[i];
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fma2(wk[k][i], win[k][i], acc);
        if (apply_silu) {  // conv_silu on both halves
            float a0, a1;
            upk2(mul2(acc, pk2(-kLog2e, -kLog2e)), a0, a1);
            float d0, d1;
            upk2(add2(pk2(ex2_approx(a0), ex2_approx(a1)), pk2(1.f, 1.f)), d0, d1);
            acc = mul2(acc, pk2(rcp_approx(d0), rcp_approx(d1)));
        }
        out[i] = acc;
    }
}

// conv_state_out[s, c, :] = last K-1 entries of [conv_state_in[s, c, :] || x_seq[:, c]].
// One thread per (sequence, channel) reads everything it needs before writing,
// so the output may be the same buffer as the input state.
template <typename T, typename TS, int K>
__device__ __forceinline__ void state_out_one(const T *__restrict__ x, const Seqs &sq, int64_t D,
                                              const TS *state_in, TS *state_out, int64_t s,
                                              int64_t c)
{
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
__global__ void __launch_bounds__(kThreads)
conv_state_out_kernel(const T *__restrict__ x, Seqs sq, int64_t D, const TS *state_in,
                      TS *state_out)
{
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (gid >= sq.S * D) return;
    state_out_one<T, TS, K>(x, sq, D, state_in, state_out, gid / D, gid % D);
}

// ---------------------------------------------------------------------------
// TMA-tiled variant (16-byte aligned rows). A CTA owns kTileT tokens x one
// 128-byte row of channels: one TMA box of kTileT + K - 1 rows (the K - 1 halo
// rows may start before token 0 or run past the last token; those read zeros)
// lands in shared memory, then each thread slides the K-tap window over its
// kTileG tokens of one 8-byte channel vector and writes 8-byte outputs (a warp
// still writes whole 128-byte rows). 8-byte vectors keep the weights and window
// in few registers, so many CTAs fit per SM and overlap one CTA's load with
// another's arithmetic. When the conv-state output does not overlap the input
// state, CTAs past the n_tiles token tiles of each channel row write it (one
// (sequence, channel) per thread), which saves a launch.
// ---------------------------------------------------------------------------
constexpr int kTileT = 128;      // tokens per CTA
constexpr int kTileG = 16;       // tokens per thread
constexpr int kTileThreads = 128;

template <typename T, typename TS, int K>
__global__ void __launch_bounds__(kTileThreads)
conv1d_tma_kernel(const __grid_constant__ CUtensorMap xmap, T *__restrict__ xc,
                  const float *__restrict__ w, const float *__restrict__ bias, Seqs sq, int64_t D,
                  const TS *__restrict__ state_in, int apply_silu, const T *__restrict__ x,
                  TS *__restrict__ state_out, unsigned n_tiles)
{
    constexpr int VEC = 8 / sizeof(T);         // channels per 8-byte vector
    constexpr int CW = 128 / sizeof(T);        // channels per tile row (128 bytes)
    constexpr int NV = CW / VEC;               // vectors per row
    constexpr int ROWS = kTileT + K - 1;
    static_assert(NV * (kTileT / kTileG) == kTileThreads, "one thread per (vector, token group)");
    __shared__ __align__(128) T tile[ROWS * CW];
    __shared__ __align__(8) uint64_t bar;

    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * kTileT;
    const int64_t cbase = (int64_t)blockIdx.y * CW;
    if (blockIdx.x >= n_tiles) {  // conv-state output of this channel row
        const int64_t idx = (int64_t)(blockIdx.x - n_tiles) * kTileThreads + tid;
        const int64_t ss = idx / CW, cc = cbase + idx % CW;
        if (ss < sq.S && cc < D) state_out_one<T, TS, K>(x, sq, D, state_in, state_out, ss, cc);
        return;
    }
    if (tid == 0) mbar_init(&bar);
    __syncthreads();
    if (tid == 0) {
        mbar_expect_tx(&bar, (uint32_t)(ROWS * CW * sizeof(T)));
        tma_2d(tile, &xmap, &bar, (int)cbase, (int)(t0 - (K - 1)));
    }

    const int v = tid % NV, g = tid / NV;
    const int64_t c0 = cbase + (int64_t)v * VEC;
    const int64_t ta = t0 + (int64_t)g * kTileG;
    const bool active = c0 < D && ta < sq.tok;
    float wk[K][VEC], bv[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
#pragma unroll
        for (int k = 0; k < K; ++k) wk[k][i] = active ? __ldg(w + (c0 + i) * K + k) : 0.f;
        bv[i] = (active && bias) ? __ldg(bias + c0 + i) : 0.f;
    }
    f32x2 wk2[K][VEC / 2], bv2[VEC / 2];
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) {
#pragma unroll
        for (int k = 0; k < K; ++k) wk2[k][i] = pk2(wk[k][2 * i], wk[k][2 * i + 1]);
        bv2[i] = pk2(bv[2 * i], bv[2 * i + 1]);
    }
    // every thread waits, so no thread leaves while the copy is in flight
    bool failed = false;
    mbar_wait(&bar, 0, failed, &g_conv_status, 1);
    if (!active) return;

    const int64_t tb = min(ta + (int64_t)kTileG, sq.tok);
    int64_t s = sq.find(ta);
    int64_t s_start = sq.off(s);
    int64_t s_end = max(sq.off(s + 1), s_start);
    // tile row of token position pos
    auto row = [&](int64_t pos) { return (int)(pos - (t0 - (K - 1))); };

    if (ta - (K - 1) >= s_start && ta + kTileG <= s_end) {
        f32x2 win[K][VEC / 2];
#pragma unroll
        for (int k = 0; k < K - 1; ++k)
            unpack8_pk<T, VEC>(*reinterpret_cast<const uint2 *>(tile + row(ta - (K - 1) + k) * CW + v * VEC), win[k]);
        T *dst = xc + ta * D + c0;
#pragma unroll
        for (int t = 0; t < kTileG; ++t) {
            unpack8_pk<T, VEC>(*reinterpret_cast<const uint2 *>(tile + row(ta + t) * CW + v * VEC), win[K - 1]);
            f32x2 out[VEC / 2];
            conv_out_pk<VEC, K>(wk2, bv2, win, apply_silu, out);
            store8_pk<T, VEC>(dst, out);
            dst += D;
#pragma unroll
            for (int k = 0; k < K - 1; ++k)
#pragma unroll
                for (int i = 0; i < VEC / 2; ++i) win[k][i] = win[k + 1][i];
        }
        return;
    }

    // tokens near a sequence boundary: rebuild the window for every token
    for (int64_t t = ta; t < tb; ++t) {
        while (t >= s_end && s < sq.S - 1) {
            ++s;
            s_start = s_end;
            s_end = max(sq.off(s + 1), s_start);
        }
        if (t >= s_end) break;  // token outside every sequence
        float win[K][VEC];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t pos = t - (K - 1) + k;
            if (pos >= s_start) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) win[k][i] = to_f32(tile[row(pos) * CW + v * VEC + i]);
            } else {
#pragma unroll
                for (int i = 0; i < VEC; ++i)
                    win[k][i] = state_in
                        ? to_f32(state_in[(s * D + c0 + i) * (K - 1) + (K - 1) + (pos - s_start)])
                        : 0.f;
            }
        }
        float out[VEC];
        conv_out<T, VEC, K>(wk, bv, win, apply_silu, out);
        store_vec<T, VEC>(xc + t * D + c0, out);
    }
}

template <typename T, typename TS, int K>
cudaError_t run(const ConvArgs &a, cudaStream_t stream, int *launches)
{
    Seqs sq{a.cu, a.S, a.tok, a.cu ? 0 : a.tok / a.S};
    const T *x = static_cast<const T *>(a.x);
    const TS *st_in = static_cast<const TS *>(a.state_in);
    bool state_done = false;  // the state output rode along with the tile kernel
    if (a.tok > 0) {
        constexpr int V = 16 / sizeof(T);
        const bool vec = a.vec && (a.D % V == 0);
        const int64_t nvec = vec ? a.D / V : a.D;
        const int64_t threads = nvec * ((a.tok + kStrip - 1) / kStrip);
        const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
        CUtensorMap map;
        if (vec && encode_2d(&map, a.x, sizeof(T) == 2, a.D, a.tok, 128 / sizeof(T),
                             kTileT + K - 1)) {
            // the state output rides along unless it overlaps the input state,
            // whose reads by the tile CTAs must all come first
            const size_t sbytes = (size_t)a.S * a.D * (K - 1) * sizeof(TS);
            const char *si = static_cast<const char *>(a.state_in);
            const char *so = static_cast<const char *>(a.state_out);
            const bool ride = a.state_out && (!si || si + sbytes <= so || so + sbytes <= si);
            constexpr int CW = 128 / sizeof(T);
            const unsigned n_tiles = (unsigned)((a.tok + kTileT - 1) / kTileT);
            const unsigned extra =
                ride ? (unsigned)((a.S * CW + kTileThreads - 1) / kTileThreads) : 0u;
            const dim3 grid(n_tiles + extra, (unsigned)((a.D * sizeof(T) + 127) / 128));
            conv1d_tma_kernel<T, TS, K><<<grid, kTileThreads, 0, stream>>>(
                map, static_cast<T *>(a.xc), a.w, a.bias, sq, a.D, st_in, a.apply_silu, x,
                static_cast<TS *>(a.state_out), n_tiles);
            state_done = ride;
        } else if (vec)
            conv1d_kernel<T, TS, V, K><<<blocks, kThreads, 0, stream>>>(
                x, static_cast<T *>(a.xc), a.w, a.bias, sq, a.D, st_in, a.apply_silu);
        else
            conv1d_kernel<T, TS, 1, K><<<blocks, kThreads, 0, stream>>>(
                x, static_cast<T *>(a.xc), a.w, a.bias, sq, a.D, st_in, a.apply_silu);
        ++*launches;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.state_out && !state_done) {
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

int read_conv_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_conv_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_conv_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace ssm
