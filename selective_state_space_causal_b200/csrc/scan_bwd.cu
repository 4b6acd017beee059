// scan_bwd.cu -- gradients of the selective scan over packed sequences (sm_100a).
//
// The training backward pass that PackMamba's packed sequences need ("PackMamba:
// Efficient Processing of Variable-Length Sequences in Mamba training",
// abstract): nothing flows across a cu_seqlens boundary in either direction.
// The forward is the one of tp_builder.py (TensorRT-Model-Connect, Mamba
// family), _add_mamba_tp_layer: D_t = softplus(dt_t + dt_bias),
// a_t = exp(D_t A), h_t = a_t h_{t-1} + D_t u_t B_t,
// y_t = (C_t . h_t + Dskip u_t) silu(z_t). With G_t = dL/dh_t (carried
// backwards: G_t = dq_t C_t + a_{t+1} G_{t+1}, dq_t = dy_t silu(z_t)):
//   du_t = dq_t Dskip + D_t sum_n G_t B_t;   dC_t += dq_t h_t;   dB_t += G_t D_t u_t;
//   dD_t = sum_n G_t (u_t B_t + A a_t h_{t-1});   ddt_t = dD_t softplus'(v_t);
//   dA += G_t D_t a_t h_{t-1};   dz_t = dy_t (C_t . h_t + Dskip u_t) silu'(z_t);
//   dh0 = a_{t0} G_{t0}.
//
// One CTA owns one sequence and kCh channels; a channel's 16 states are split
// over 4 adjacent lanes (4 states each, two packed fp32x2 registers), as in the
// forward's register-prefetch schedule. Two phases:
//   A (forward): walk the sequence in kTS-token chunks and write the state at
//     each chunk start to the workspace (4 bytes per token and channel);
//   B (reverse): for each chunk, last first: a cooperative pre-pass stages the
//     chunk's per-(token, channel) values (delta, softplus', u, dy silu(z),
//     dy silu'(z)) and fp32 B and C rows in shared memory; each lane recomputes
//     its states for the chunk into registers from the checkpoint, then walks
//     the chunk backwards carrying G in registers.
// Sums over a channel's 4 lanes use butterflies; dB and dC, summed over
// channels, go through a transposed shuffle over the warp's 8 channels, a
// shared-memory sum over the CTA's warps, and one fp32 atomic per (token,
// state) and CTA. dA, dDskip and ddt_bias (summed over sequences) take one
// atomic per CTA and channel. The atomics make the last bits of those sums
// depend on the order in which CTAs finish; everything else is deterministic.
#include "common.cuh"

namespace ssm {

namespace {

constexpr int kN = 16;
constexpr int kNPT = 4;               // states per lane
constexpr int kTPC = kN / kNPT;       // lanes per channel
constexpr int kCh = 32;               // channels per CTA
constexpr int kThreads = kCh * kTPC;  // 128
constexpr int kWarps = kThreads / 32;
constexpr int kTS = 16;               // tokens per chunk (one checkpoint each)

struct BwdParams {
    const void *u, *dt, *B, *C, *z, *dy;
    const float *A, *Dskip, *dt_bias, *h0, *dh_final;
    const int32_t *cu;
    void *du, *ddt, *dz;
    float *dB, *dC, *dA, *dDskip, *ddt_bias, *dh0;
    float *ckpt;  // workspace: (tok / kTS + S + 1, D, 16)
    int64_t S, tok, D, L;
    int softplus;
};

// Shared memory of one CTA.
struct Smem {
    float d[kTS][kCh];     // delta
    float dsp[kTS][kCh];   // softplus'(v) (1 without the softplus)
    float u[kTS][kCh];
    float dq[kTS][kCh];    // dy * silu(z)
    float dzf[kTS][kCh];   // dy * silu'(z)
    float B[kTS][kN];
    float C[kTS][kN];
    float red[kWarps][kTS][32];  // dB / dC partial sums of each warp's 8 channels
    float out[3][kTS][kCh];      // du, ddt, dz of the chunk
};

// Raw chunk inputs as they sit in global memory, copied in one chunk ahead.
template <typename T>
struct RawChunk {
    T act[4][kTS][kCh];  // dt, u, z, dy
    T bc[2][kTS][kN];    // B, C
};

// 16-byte asynchronous copy from global to shared memory (completion through
// the issuing thread's cp.async groups).
__device__ __forceinline__ void cp16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :: "r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

// Issue the copies of chunk [t0, t0 + nt): dt and u (and z, dy when `full`)
// rows of the CTA's channels, and the B (and C) rows. Needs D * sizeof(T) and
// every base a multiple of 16 bytes (the host checks).
template <typename T>
__device__ __forceinline__ void issue_chunk(const BwdParams &p, RawChunk<T> &r, int64_t t0, int nt,
                                            int64_t cbase, int nch, bool full)
{
    constexpr int V = 16 / sizeof(T), VR = kCh / V, VB = kN / V;
    const T *src_act[4] = {static_cast<const T *>(p.dt), static_cast<const T *>(p.u),
                           static_cast<const T *>(p.z), static_cast<const T *>(p.dy)};
    const int narr = full ? 4 : 2, nvr = nch / V;
    for (int e = threadIdx.x; e < narr * kTS * VR; e += kThreads) {
        const int arr = e / (kTS * VR), rem = e % (kTS * VR), tl = rem / VR, v = rem % VR;
        if (tl >= nt || v >= nvr || src_act[arr] == nullptr) continue;
        cp16(&r.act[arr][tl][v * V], src_act[arr] + (t0 + tl) * p.D + cbase + v * V);
    }
    const T *src_bc[2] = {static_cast<const T *>(p.B), static_cast<const T *>(p.C)};
    for (int e = threadIdx.x; e < (full ? 2 : 1) * kTS * VB; e += kThreads) {
        const int arr = e / (kTS * VB), rem = e % (kTS * VB), tl = rem / VB, v = rem % VB;
        if (tl >= nt) continue;
        cp16(&r.bc[arr][tl][v * V], src_bc[arr] + (t0 + tl) * kN + v * V);
    }
}

__device__ __forceinline__ float sigmoid_f(float v) { return __fdividef(1.0f, 1.0f + __expf(-v)); }

template <typename T>
__device__ __forceinline__ float ld1(const T *p) { return to_f32(*p); }

// Stage the chunk [t0, t0 + nt) of sequence positions: per-(token, channel)
// values and the fp32 B and C rows. Threads walk (token, channel) items with
// channels fastest, so each warp reads 32 consecutive channels of one token.
template <typename T>
__device__ __forceinline__ void stage_chunk(const BwdParams &p, Smem &sm, int64_t t0, int nt,
                                            int64_t cbase, bool full)
{
    const int tid = threadIdx.x;
    const T *U = static_cast<const T *>(p.u), *DT = static_cast<const T *>(p.dt);
    const T *Z = static_cast<const T *>(p.z), *DY = static_cast<const T *>(p.dy);
    for (int e = tid; e < kTS * kCh; e += kThreads) {
        const int tl = e / kCh, cl = e % kCh;
        const int64_t c = cbase + cl;
        float d = 0.f, dsp = 0.f, u = 0.f, dq = 0.f, dzf = 0.f;
        if (tl < nt && c < p.D) {
            const int64_t o = (t0 + tl) * p.D + c;
            const float v = ld1(DT + o) + (p.dt_bias ? __ldg(p.dt_bias + c) : 0.f);
            d = p.softplus ? softplus_fast(v) : v;
            dsp = p.softplus ? sigmoid_f(v) : 1.f;
            u = ld1(U + o);
            if (full) {
                const float dy = ld1(DY + o);
                float g = 1.f, dg = 0.f;
                if (Z) {
                    const float zt = ld1(Z + o), sg = sigmoid_f(zt);
                    g = zt * sg;
                    dg = sg * (1.f + zt * (1.f - sg));
                }
                dq = dy * g;
                dzf = dy * dg;
            }
        }
        sm.d[tl][cl] = d;
        sm.dsp[tl][cl] = dsp;
        sm.u[tl][cl] = u;
        sm.dq[tl][cl] = dq;
        sm.dzf[tl][cl] = dzf;
    }
    const T *Bp = static_cast<const T *>(p.B), *Cp = static_cast<const T *>(p.C);
    for (int e = tid; e < kTS * kN; e += kThreads) {
        const int tl = e / kN, n = e % kN;
        const bool live = tl < nt;
        sm.B[tl][n] = live ? ld1(Bp + (t0 + tl) * kN + n) : 0.f;
        sm.C[tl][n] = live ? ld1(Cp + (t0 + tl) * kN + n) : 0.f;
    }
}

// The same staging from the raw shared-memory copy of the chunk.
template <typename T>
__device__ __forceinline__ void stage_from_raw(const BwdParams &p, Smem &sm, const RawChunk<T> &r,
                                               int nt, int64_t cbase, bool full)
{
    const int tid = threadIdx.x;
    const bool has_z = p.z != nullptr;
    for (int e = tid; e < kTS * kCh; e += kThreads) {
        const int tl = e / kCh, cl = e % kCh;
        const int64_t c = cbase + cl;
        float d = 0.f, dsp = 0.f, u = 0.f, dq = 0.f, dzf = 0.f;
        if (tl < nt && c < p.D) {
            const float v = to_f32(r.act[0][tl][cl]) + (p.dt_bias ? __ldg(p.dt_bias + c) : 0.f);
            d = p.softplus ? softplus_fast(v) : v;
            dsp = p.softplus ? sigmoid_f(v) : 1.f;
            u = to_f32(r.act[1][tl][cl]);
            if (full) {
                const float dy = to_f32(r.act[3][tl][cl]);
                float g = 1.f, dg = 0.f;
                if (has_z) {
                    const float zt = to_f32(r.act[2][tl][cl]), sg = sigmoid_f(zt);
                    g = zt * sg;
                    dg = sg * (1.f + zt * (1.f - sg));
                }
                dq = dy * g;
                dzf = dy * dg;
            }
        }
        sm.d[tl][cl] = d;
        sm.dsp[tl][cl] = dsp;
        sm.u[tl][cl] = u;
        sm.dq[tl][cl] = dq;
        sm.dzf[tl][cl] = dzf;
    }
    for (int e = tid; e < kTS * kN; e += kThreads) {
        const int tl = e / kN, n = e % kN;
        const bool live = tl < nt;
        sm.B[tl][n] = live ? to_f32(r.bc[0][tl][n]) : 0.f;
        if (full) sm.C[tl][n] = live ? to_f32(r.bc[1][tl][n]) : 0.f;
    }
}

// h <- a * h + (d u) * B for this lane's 4 states; returns a.
__device__ __forceinline__ void fwd_token(f32x2 (&h)[2], const f32x2 (&A2)[2], float d, float u,
                                          const float *Bn, f32x2 (&a)[2])
{
    const f32x2 dd = pk2(d, d), xx = pk2(d * u, d * u);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        float e0, e1;
        upk2(mul2(dd, A2[j]), e0, e1);
        a[j] = pk2(ex2_approx(e0), ex2_approx(e1));
        h[j] = fma2(a[j], h[j], mul2(xx, pk2(Bn[2 * j], Bn[2 * j + 1])));
    }
}

template <typename T, bool ASYNC>
__global__ void __launch_bounds__(kThreads)
scan_bwd_kernel(const BwdParams p)
{
    __shared__ Smem sm;
    __shared__ __align__(16) RawChunk<T> raw[ASYNC ? 2 : 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = tid % kTPC, cl = tid / kTPC;
    const int64_t cbase = (int64_t)blockIdx.x * kCh, c = cbase + cl;
    const int nch = (int)min((int64_t)kCh, p.D - cbase);
    const bool cvalid = c < p.D;
    const int64_t s = blockIdx.y;
    int64_t start, end;
    if (p.cu) {
        start = clamp_off(p.cu[s], p.tok);
        end = max(clamp_off(p.cu[s + 1], p.tok), start);
    } else {
        start = s * p.L;
        end = start + p.L;
    }
    const int64_t len = end - start;
    const int64_t nchunks = (len + kTS - 1) / kTS;
    // checkpoint slots of this sequence: floor(start / kTS) + s + k never collide
    float *ck = p.ckpt + ((start / kTS + s) * p.D + c) * kN + sub * kNPT;

    f32x2 A2[2], Aln[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int n = sub * kNPT + 2 * j;
        const float a0 = cvalid ? __ldg(p.A + c * kN + n) : 0.f;
        const float a1 = cvalid ? __ldg(p.A + c * kN + n + 1) : 0.f;
        A2[j] = pk2(a0 * kLog2e, a1 * kLog2e);
        Aln[j] = pk2(a0, a1);
    }
    const float dsk = (cvalid && p.Dskip) ? __ldg(p.Dskip + c) : 0.f;

    // ---- phase A: forward, checkpoint at every chunk start ----------------
    f32x2 h[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int64_t o = (s * p.D + c) * kN + sub * kNPT + 2 * j;
        h[j] = (cvalid && p.h0) ? pk2(p.h0[o], p.h0[o + 1]) : 0ull;
    }
    if (ASYNC && nchunks > 0) {
        issue_chunk<T>(p, raw[0], start, (int)min((int64_t)kTS, len), cbase, nch, false);
        cp_commit();
    }
    for (int64_t k = 0; k < nchunks; ++k) {
        const int64_t t0 = start + k * kTS;
        const int nt = (int)min((int64_t)kTS, end - t0);
        if (cvalid) {
            float4 v;
            upk2(h[0], v.x, v.y);
            upk2(h[1], v.z, v.w);
            *reinterpret_cast<float4 *>(ck + k * p.D * kN) = v;
        }
        if constexpr (ASYNC) {
            // the next chunk's copies go out before this one is staged; the
            // buffer they fill was last read before the previous barrier
            if (k + 1 < nchunks) {
                const int64_t t1 = t0 + kTS;
                issue_chunk<T>(p, raw[(k + 1) & 1], t1, (int)min((int64_t)kTS, end - t1), cbase,
                               nch, false);
                cp_commit();
                cp_wait<1>();
            } else {
                cp_wait<0>();
            }
            __syncthreads();  // every thread's copies have landed; the previous chunk is done
            stage_from_raw<T>(p, sm, raw[k & 1], nt, cbase, false);
        } else {
            __syncthreads();  // the previous chunk's values are no longer read
            stage_chunk<T>(p, sm, t0, nt, cbase, false);
        }
        __syncthreads();
        for (int tl = 0; tl < nt; ++tl) {
            f32x2 a[2];
            fwd_token(h, A2, sm.d[tl][cl], sm.u[tl][cl], &sm.B[tl][sub * kNPT], a);
        }
    }

    // ---- phase B: reverse ---------------------------------------------------
    f32x2 G[2], dAacc[2] = {0ull, 0ull};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int64_t o = (s * p.D + c) * kN + sub * kNPT + 2 * j;
        G[j] = (cvalid && p.dh_final) ? pk2(p.dh_final[o], p.dh_final[o + 1]) : 0ull;
    }
    float dDsk = 0.f, ddtb = 0.f;
    T *DU = static_cast<T *>(p.du), *DDT = static_cast<T *>(p.ddt), *DZ = static_cast<T *>(p.dz);
    __syncthreads();  // phase A's last chunk is no longer read
    if (ASYNC && nchunks > 0) {
        const int64_t tl0 = start + (nchunks - 1) * kTS;
        issue_chunk<T>(p, raw[0], tl0, (int)(end - tl0), cbase, nch, true);
        cp_commit();
    }
    for (int64_t k = nchunks - 1; k >= 0; --k) {
        const int64_t t0 = start + k * kTS;
        const int nt = (int)min((int64_t)kTS, end - t0);
        const int buf = (int)((nchunks - 1 - k) & 1);
        if constexpr (ASYNC) {
            if (k > 0) {
                issue_chunk<T>(p, raw[buf ^ 1], t0 - kTS, kTS, cbase, nch, true);
                cp_commit();
                cp_wait<1>();
            } else {
                cp_wait<0>();
            }
            __syncthreads();  // copies landed; the previous chunk's shared values are no longer read
            stage_from_raw<T>(p, sm, raw[buf], nt, cbase, true);
        } else {
            __syncthreads();  // the previous chunk's shared values are no longer read
            stage_chunk<T>(p, sm, t0, nt, cbase, true);
        }
        __syncthreads();
        // recompute this lane's states over the chunk from its checkpoint
        f32x2 hc[2], hist[kTS][2];
        if (cvalid) {
            const float4 v = *reinterpret_cast<const float4 *>(ck + k * p.D * kN);
            hc[0] = pk2(v.x, v.y);
            hc[1] = pk2(v.z, v.w);
        } else {
            hc[0] = hc[1] = 0ull;
        }
        {
            f32x2 hr[2] = {hc[0], hc[1]};
#pragma unroll
            for (int tl = 0; tl < kTS; ++tl) {
                if (tl < nt) {
                    f32x2 a[2];
                    fwd_token(hr, A2, sm.d[tl][cl], sm.u[tl][cl], &sm.B[tl][sub * kNPT], a);
                }
                hist[tl][0] = hr[0];
                hist[tl][1] = hr[1];
            }
        }
        // walk the chunk backwards
#pragma unroll
        for (int tl = kTS - 1; tl >= 0; --tl) {
            float pb[2 * kNPT];  // this lane's dB then dC terms of token tl
            if (tl < nt) {
                const float d = sm.d[tl][cl], u = sm.u[tl][cl], dq = sm.dq[tl][cl];
                const float *Bn = &sm.B[tl][sub * kNPT], *Cn = &sm.C[tl][sub * kNPT];
                const f32x2 dd = pk2(d, d), dqq = pk2(dq, dq);
                f32x2 qp = 0ull, dup = 0ull, ddp = 0ull;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const f32x2 b2 = pk2(Bn[2 * j], Bn[2 * j + 1]);
                    const f32x2 c2 = pk2(Cn[2 * j], Cn[2 * j + 1]);
                    const f32x2 hp = tl > 0 ? hist[tl - 1][j] : hc[j];
                    float e0, e1;
                    upk2(mul2(dd, A2[j]), e0, e1);
                    const f32x2 a = pk2(ex2_approx(e0), ex2_approx(e1));
                    G[j] = fma2(dqq, c2, G[j]);                       // G_t = dq C + a_{t+1} G_{t+1}
                    qp = fma2(c2, hist[tl][j], qp);                   // C . h_t
                    dup = fma2(G[j], b2, dup);                        // G . B
                    const f32x2 aAh = mul2(mul2(a, Aln[j]), hp);      // A a h_{t-1}
                    ddp = fma2(G[j], fma2(pk2(u, u), b2, aAh), ddp);  // G (u B + A a h_{t-1})
                    dAacc[j] = fma2(mul2(G[j], dd), mul2(a, hp), dAacc[j]);
                    float g0, g1, h0_, h1_;
                    upk2(mul2(G[j], pk2(d * u, d * u)), g0, g1);     // dB terms
                    upk2(mul2(dqq, hist[tl][j]), h0_, h1_);           // dC terms
                    pb[2 * j] = g0;
                    pb[2 * j + 1] = g1;
                    pb[kNPT + 2 * j] = h0_;
                    pb[kNPT + 2 * j + 1] = h1_;
                    G[j] = mul2(a, G[j]);                             // towards h_{t-1}
                }
                // sums over the channel's 4 lanes
                float q0, q1, u0, u1, x0, x1;
                upk2(qp, q0, q1);
                upk2(dup, u0, u1);
                upk2(ddp, x0, x1);
                float qs = q0 + q1, us = u0 + u1, xs = x0 + x1;
#pragma unroll
                for (int w = 1; w < kTPC; w <<= 1) {
                    qs += __shfl_xor_sync(0xffffffffu, qs, w);
                    us += __shfl_xor_sync(0xffffffffu, us, w);
                    xs += __shfl_xor_sync(0xffffffffu, xs, w);
                }
                if (sub == 0) {
                    const float ddt = xs * sm.dsp[tl][cl];
                    sm.out[0][tl][cl] = dq * dsk + d * us;
                    sm.out[1][tl][cl] = ddt;
                    sm.out[2][tl][cl] = sm.dzf[tl][cl] * (qs + dsk * u);
                    dDsk += dq * u;
                    ddtb += ddt;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 2 * kNPT; ++i) pb[i] = 0.f;
            }
            if (!cvalid) {
#pragma unroll
                for (int i = 0; i < 2 * kNPT; ++i) pb[i] = 0.f;
            }
            // dB / dC: transposed sum over the warp's 8 channels (lane bits 2..4);
            // afterwards lane (chl, sub) holds the sum of term chl of its sub
#pragma unroll
            for (int w = 16, half = kNPT; w >= 4; w >>= 1, half >>= 1) {
                const bool upper = (lane & w) != 0;
#pragma unroll
                for (int i = 0; i < half; ++i) {
                    const float send = upper ? pb[i] : pb[i + half];
                    const float keep = upper ? pb[i + half] : pb[i];
                    pb[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
                }
            }
            // term index held by this lane: bits (16, 8, 4) of the lane pick
            // halves (4, 2, 1) of the 8 terms
            const int term = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
            sm.red[warp][tl][term * kTPC + sub] = pb[0];
        }
        __syncthreads();
        // dB / dC of the chunk: sum over warps, one atomic per (token, state)
        for (int e = tid; e < kTS * 2 * kN; e += kThreads) {
            const int tl = e / (2 * kN), r = e % (2 * kN);  // r = term * 4 + sub
            if (tl >= nt) continue;
            const int term = r / kTPC, sb = r % kTPC;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += sm.red[w][tl][r];
            const int n = sb * kNPT + (term % kNPT);
            float *dst = term < kNPT ? p.dB : p.dC;
            atomicAdd(dst + (t0 + tl) * kN + n, v);
        }
        // du, ddt, dz of the chunk, channels contiguous
        for (int e = tid; e < kTS * kCh; e += kThreads) {
            const int tl = e / kCh, cc = e % kCh;
            const int64_t ch = cbase + cc;
            if (tl < nt && ch < p.D) {
                const int64_t o = (t0 + tl) * p.D + ch;
                DU[o] = from_f32<T>(sm.out[0][tl][cc]);
                DDT[o] = from_f32<T>(sm.out[1][tl][cc]);
                if (DZ) DZ[o] = from_f32<T>(p.z ? sm.out[2][tl][cc] : 0.f);
            }
        }
    }
    if (cvalid) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int n = sub * kNPT + 2 * j;
            float g0, g1, a0, a1;
            upk2(G[j], g0, g1);
            upk2(dAacc[j], a0, a1);
            if (p.dh0) {
                p.dh0[(s * p.D + c) * kN + n] = g0;
                p.dh0[(s * p.D + c) * kN + n + 1] = g1;
            }
            atomicAdd(p.dA + c * kN + n, a0);
            atomicAdd(p.dA + c * kN + n + 1, a1);
        }
        if (sub == 0) {
            if (p.dDskip) atomicAdd(p.dDskip + c, dDsk);
            if (p.ddt_bias) atomicAdd(p.ddt_bias + c, ddtb);
        }
    }
}

__global__ void zero_kernel(float *a, int64_t na, float *b, int64_t nb)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = i; j < na; j += stride) a[j] = 0.f;
    if (b)
        for (int64_t j = i; j < nb; j += stride) b[j] = 0.f;
}

}  // namespace

struct ScanBwdArgs {
    const void *u, *dt, *B, *C, *z, *dy;
    const float *A, *Dskip, *dt_bias, *h0, *dh_final;
    const int32_t *cu;
    int64_t S;
    void *du, *ddt, *dz;
    float *dB, *dC, *dA, *dDskip, *ddt_bias, *dh0;
    float *ckpt;
    int64_t tok, D;
    int softplus;
    bool bf16;
};

size_t scan_bwd_ckpt_floats(int64_t tok, int64_t D, int64_t S)
{
    return (size_t)(tok / kTS + S + 1) * (size_t)D * kN;
}

cudaError_t launch_scan_bwd(const ScanBwdArgs &a, cudaStream_t stream, int *launches)
{
    // the sums that CTAs add into start from zero
    {
        const int64_t n1 = a.tok * kN, n2 = a.tok * kN;
        zero_kernel<<<592, 256, 0, stream>>>(a.dB, n1, a.dC, n2);
        ++*launches;
        zero_kernel<<<64, 256, 0, stream>>>(a.dA, a.D * kN, nullptr, 0);
        ++*launches;
        if (a.dDskip || a.ddt_bias) {
            if (a.dDskip) {
                zero_kernel<<<8, 256, 0, stream>>>(a.dDskip, a.D, nullptr, 0);
                ++*launches;
            }
            if (a.ddt_bias) {
                zero_kernel<<<8, 256, 0, stream>>>(a.ddt_bias, a.D, nullptr, 0);
                ++*launches;
            }
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.S == 0) return cudaSuccess;
    BwdParams p;
    p.u = a.u; p.dt = a.dt; p.B = a.B; p.C = a.C; p.z = a.z; p.dy = a.dy;
    p.A = a.A; p.Dskip = a.Dskip; p.dt_bias = a.dt_bias; p.h0 = a.h0; p.dh_final = a.dh_final;
    p.cu = a.cu; p.du = a.du; p.ddt = a.ddt; p.dz = a.dz;
    p.dB = a.dB; p.dC = a.dC; p.dA = a.dA; p.dDskip = a.dDskip; p.ddt_bias = a.ddt_bias;
    p.dh0 = a.dh0; p.ckpt = a.ckpt;
    p.S = a.S; p.tok = a.tok; p.D = a.D; p.L = a.cu ? 0 : a.tok / a.S; p.softplus = a.softplus;
    const dim3 grid((unsigned)((a.D + kCh - 1) / kCh), (unsigned)a.S);
    const size_t es = a.bf16 ? 2 : 4;
    const uintptr_t mis = (uintptr_t)a.u | (uintptr_t)a.dt | (uintptr_t)a.z | (uintptr_t)a.dy |
                          (uintptr_t)a.B | (uintptr_t)a.C;
    const bool async_ok = (mis % 16 == 0) && ((size_t)a.D * es) % 16 == 0;
    if (a.bf16) {
        if (async_ok) scan_bwd_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, stream>>>(p);
        else scan_bwd_kernel<__nv_bfloat16, false><<<grid, kThreads, 0, stream>>>(p);
    } else {
        if (async_ok) scan_bwd_kernel<float, true><<<grid, kThreads, 0, stream>>>(p);
        else scan_bwd_kernel<float, false><<<grid, kThreads, 0, stream>>>(p);
    }
    ++*launches;
    return cudaGetLastError();
}

}  // namespace ssm
