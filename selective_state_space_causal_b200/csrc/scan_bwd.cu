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
// Two kernels compute the same gradients; the host picks one by problem size
// (scan_bwd_variant_for). Both recompute the forward states from checkpoints
// rather than store them, and both run packed sequences longest first.
//
// scan_bwd_kernel (lane-split, for small S * D): one CTA owns one sequence and
// kCh channels; a channel's 16 states are split over 4 adjacent lanes (4 states
// each, two packed fp32x2 registers), as in the forward's register-prefetch
// schedule. Two phases:
//   A (forward): walk the sequence in kTS-token chunks and write the state at
//     each chunk start to the workspace (4 bytes per token and channel);
//   B (reverse): for each chunk, last first: a cooperative pre-pass stages the
//     chunk's per-(token, channel) values (delta, softplus', u, dy silu(z),
//     dy silu'(z)) and fp32 B and C rows in shared memory; each lane recomputes
//     its states for the chunk into registers from the checkpoint, then walks
//     the chunk backwards carrying G in registers.
// Sums over a channel's 4 lanes wait for a group of 4 tokens and take a
// transposed butterfly that leaves one token's sums in each lane; dB and dC,
// summed over channels, go through a per-warp shared buffer a token pair at a
// time (each lane sums one pair of values over the warp's 8 channels), a
// shared-memory sum over the CTA's warps, and one fp32 atomic per (token,
// state) and CTA. dA, dDskip and ddt_bias (summed over sequences) take one
// atomic per CTA and channel. The atomics make the last bits of those sums
// depend on the order in which CTAs finish; everything else is deterministic.
//
// scan_bwd_ckpt_kernel + scan_bwd_wide_kernel (thread-per-channel, for large
// S * D): one thread per channel with all 16 states, 8-token chunks; the first
// kernel writes the checkpoints, the second walks back, with dB and dC summed
// over channels from shared memory; described above the kernels.
#include <atomic>
#include <type_traits>

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
constexpr int kFwdCk = 8;             // tokens per checkpoint when the forward wrote them

struct BwdParams {
    const void *u, *dt, *B, *C, *z, *dy;
    const float *A, *Dskip, *dt_bias, *h0, *dh_final;
    const int32_t *cu;
    void *du, *ddt, *dz;
    float *dB, *dC, *dA, *dDskip, *ddt_bias, *dh0;
    float *ckpt;  // workspace: one state per chunk start of each sequence and channel
    const int32_t *order;  // longest-first sequence order, or NULL
    int64_t S, tok, D, L;
    int softplus;
    int vec_atomics;  // dB and dC are 16-byte aligned: sums go out as float4 atomics
    // the workspace already holds the state before every 8th token of each
    // sequence (written by the forward pass): no checkpointing pass here
    int have_ckpt;
};

// The sequence of this CTA row (blockIdx.y; the longest-first order when one
// is given) and its token range, with the offsets clamped into [0, tok].
__device__ __forceinline__ void bwd_sequence(const BwdParams &p, int64_t &s, int64_t &start,
                                             int64_t &end)
{
    s = p.order ? (int64_t)p.order[blockIdx.y] : (int64_t)blockIdx.y;
    if (p.cu) {
        start = clamp_off(p.cu[s], p.tok);
        end = max(clamp_off(p.cu[s + 1], p.tok), start);
    } else {
        start = s * p.L;
        end = start + p.L;
    }
}

// Shared memory of one CTA.
struct Smem {
    float d[kTS][kCh];     // delta
    float dsp[kTS][kCh];   // softplus'(v) (1 without the softplus)
    float u[kTS][kCh];
    float dq[kTS][kCh];    // dy * silu(z)
    float dzf[kTS][kCh];   // dy * silu'(z)
    float B[kTS][kN];
    float C[kTS][kN];
    float red[kWarps][kTS][32];  // dB (states 0..15) then dC (16..31) sums of each warp's 8 channels
    float out[3][kTS][kCh];      // du, ddt, dz of the chunk
    float wbuf[kWarps][2][8][32];  // a token pair's dB / dC terms of each warp's 8 channels
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
    const T *DT = static_cast<const T *>(p.dt), *U = static_cast<const T *>(p.u);
    const T *Z = static_cast<const T *>(p.z), *DY = static_cast<const T *>(p.dy);
    const int narr = full ? 4 : 2, nvr = nch / V;
    for (int e = threadIdx.x; e < narr * kTS * VR; e += kThreads) {
        const int arr = e / (kTS * VR), rem = e % (kTS * VR), tl = rem / VR, v = rem % VR;
        const T *src = arr == 0 ? DT : arr == 1 ? U : arr == 2 ? Z : DY;  // selects: no local array
        if (tl >= nt || v >= nvr || src == nullptr) continue;
        cp16(&r.act[arr][tl][v * V], src + (t0 + tl) * p.D + cbase + v * V);
    }
    for (int e = threadIdx.x; e < (full ? 2 : 1) * kTS * VB; e += kThreads) {
        const int arr = e / (kTS * VB), rem = e % (kTS * VB), tl = rem / VB, v = rem % VB;
        if (tl >= nt) continue;
        const T *src = static_cast<const T *>(arr ? p.C : p.B);
        cp16(&r.bc[arr][tl][v * V], src + (t0 + tl) * kN + v * V);
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
    // dynamic: with fp32 inputs and copies in flight it is above 48 KB
    extern __shared__ __align__(16) unsigned char l_smem[];
    Smem &sm = *reinterpret_cast<Smem *>(l_smem);
    RawChunk<T> *raw = reinterpret_cast<RawChunk<T> *>(l_smem + sizeof(Smem));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = tid % kTPC, cl = tid / kTPC;
    const int64_t cbase = (int64_t)blockIdx.x * kCh, c = cbase + cl;
    const int nch = (int)min((int64_t)kCh, p.D - cbase);
    const bool cvalid = c < p.D;
    int64_t s, start, end;
    bwd_sequence(p, s, start, end);
    const int64_t len = end - start;
    const int64_t nchunks = (len + kTS - 1) / kTS;
    // checkpoint slots of this sequence: floor(start / kTS) + s + k never
    // collide; the forward's 8-token checkpoints sit at floor(start / 8) + s
    // + 2k
    float *ck = p.ckpt + ((start / (p.have_ckpt ? kFwdCk : kTS) + s) * p.D + c) * kN + sub * kNPT;
    const int64_t ck_step = (p.have_ckpt ? kTS / kFwdCk : 1) * p.D * kN;

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
    if (!p.have_ckpt) {
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
                *reinterpret_cast<float4 *>(ck + k * ck_step) = v;
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
            const float4 v = *reinterpret_cast<const float4 *>(ck + k * ck_step);
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
        // walk the chunk backwards. Sums over a channel's 4 lanes wait for a
        // group of kTPC tokens and then take a transposed butterfly that leaves
        // token tl + sub's sums in lane `sub`, which writes that token's
        // outputs; dB / dC terms go through the warp's buffer a token pair at a
        // time and are summed over the warp's 8 channels from there.
        float Pq[kTPC], Pu[kTPC], Px[kTPC];  // C.h, G.B, G.(u B + A a h_{t-1}) of my states
        const int cw = lane >> 2;            // channel within the warp
#pragma unroll
        for (int tl = kTS - 1; tl >= 0; --tl) {
            float pb[2 * kNPT];  // this lane's dB then dC terms of token tl
            float q = 0.f, us = 0.f, xs = 0.f;
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
                float q0, q1, u0, u1, x0, x1;
                upk2(qp, q0, q1);
                upk2(dup, u0, u1);
                upk2(ddp, x0, x1);
                q = q0 + q1;
                us = u0 + u1;
                xs = x0 + x1;
            } else {
#pragma unroll
                for (int i = 0; i < 2 * kNPT; ++i) pb[i] = 0.f;
            }
            if (!cvalid) {
#pragma unroll
                for (int i = 0; i < 2 * kNPT; ++i) pb[i] = 0.f;
            }
            Pq[tl % kTPC] = q;
            Pu[tl % kTPC] = us;
            Px[tl % kTPC] = xs;
            float *wb = &sm.wbuf[warp][tl & 1][cw][0];
            *reinterpret_cast<float4 *>(wb + sub * kNPT) = make_float4(pb[0], pb[1], pb[2], pb[3]);
            *reinterpret_cast<float4 *>(wb + kN + sub * kNPT) = make_float4(pb[4], pb[5], pb[6], pb[7]);
            if ((tl & 1) == 0) {
                // tokens tl and tl + 1: lane L sums values 2 (L % 16), +1 of token
                // tl + L / 16 over the warp's 8 channels
                __syncwarp();
                const int sl = lane >> 4, vv = 2 * (lane & 15);
                f32x2 acc = 0ull;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const float2 v = *reinterpret_cast<const float2 *>(&sm.wbuf[warp][sl][ch][vv]);
                    acc = add2(acc, pk2(v.x, v.y));
                }
                float r0, r1;
                upk2(acc, r0, r1);
                *reinterpret_cast<float2 *>(&sm.red[warp][tl + sl][vv]) = make_float2(r0, r1);
                __syncwarp();
            }
            if (tl % kTPC == 0) {
                // the group tl .. tl + 3 is complete: transposed butterfly over
                // the channel's lanes (xor 2, then 1)
#pragma unroll
                for (int w = kTPC / 2; w >= 1; w >>= 1) {
                    const bool upper = (sub & w) != 0;
#pragma unroll
                    for (int i = 0; i < w; ++i) {
                        const float sq = upper ? Pq[i] : Pq[i + w], kq = upper ? Pq[i + w] : Pq[i];
                        const float su = upper ? Pu[i] : Pu[i + w], ku = upper ? Pu[i + w] : Pu[i];
                        const float sx = upper ? Px[i] : Px[i + w], kx = upper ? Px[i + w] : Px[i];
                        Pq[i] = kq + __shfl_xor_sync(0xffffffffu, sq, w);
                        Pu[i] = ku + __shfl_xor_sync(0xffffffffu, su, w);
                        Px[i] = kx + __shfl_xor_sync(0xffffffffu, sx, w);
                    }
                }
                const int tg = tl + sub;  // the token whose sums this lane now holds
                if (tg < nt) {
                    const float d = sm.d[tg][cl], u = sm.u[tg][cl], dq = sm.dq[tg][cl];
                    const float ddt = Px[0] * sm.dsp[tg][cl];
                    sm.out[0][tg][cl] = dq * dsk + d * Pu[0];
                    sm.out[1][tg][cl] = ddt;
                    sm.out[2][tg][cl] = sm.dzf[tg][cl] * (Pq[0] + dsk * u);
                    dDsk += dq * u;
                    ddtb += ddt;
                }
            }
        }
        __syncthreads();
        // dB / dC of the chunk: sum over warps, one atomic per (token, state)
        for (int e = tid; e < kTS * 2 * kN; e += kThreads) {
            const int tl = e / (2 * kN), r = e % (2 * kN);  // r < 16: dB state r, else dC state r - 16
            if (tl >= nt) continue;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += sm.red[w][tl][r];
            float *dst = r < kN ? p.dB : p.dC;
            atomicAdd(dst + (t0 + tl) * kN + (r % kN), v);
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
    }
    // each lane summed its own tokens' dDskip and ddt_bias terms
#pragma unroll
    for (int w = 1; w < kTPC; w <<= 1) {
        dDsk += __shfl_xor_sync(0xffffffffu, dDsk, w);
        ddtb += __shfl_xor_sync(0xffffffffu, ddtb, w);
    }
    if (cvalid && sub == 0) {
        if (p.dDskip) atomicAdd(p.dDskip + c, dDsk);
        if (p.ddt_bias) atomicAdd(p.ddt_bias + c, ddtb);
    }
}

// ---------------------------------------------------------------------------
// Thread-per-channel variant. One thread owns one (sequence, channel) with
// all 16 states in registers (eight packed fp32x2 pairs): sums over states
// take no shuffles, and the CTA's 128 channels share each token's B and C.
// Chunks of kWTS tokens, one checkpoint each. Phase A (the forward pass that
// writes them) runs before, as scan_bwd_ckpt_kernel; this kernel is phase B,
// per chunk, last first:
//   1. recompute the chunk's states from its checkpoint into shared memory,
//      with dz on the way (C . h_t is at hand), keeping each token's delta,
//      delta u, u, dy silu(z) and softplus' in registers;
//   2. dC_t = sum_c dy silu(z) h_t over the CTA's channels, from shared
//      memory (below);
//   3. walk the chunk backwards with G in registers; the states of token t
//      give way to its dB terms G_t delta_t u_t in shared memory;
//   4. dB_t, summed over channels as in 2.
// A channel sum (2, 4) covers the chunk's 4 kWTS (token, 4-state) items: each
// warp takes 8 items, and lane (k, i) = (lane / 8, lane % 8) of warp w adds
// item 8 (w mod kWTS/2) + i over the kWGCh channels of group
// 4 (w div kWTS/2) + k; two shuffles join a warp's four groups, and one
// 16-byte atomic per item and warp adds the result. Rows of the state buffer
// are padded by 16 bytes, so the 8 lanes of a 16-byte load phase, on 8
// consecutive rows, hit 8 different banks; rows of dy silu(z) are padded by 4
// bytes per group and 32 bytes per token, so all 32 lanes' 4-byte loads do
// too.
// ---------------------------------------------------------------------------
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kWCh = 128;              // channels (= threads) per CTA
constexpr int kWTS = 8;                // tokens per chunk and per checkpoint
constexpr int kWMinCtas = kWTS == 4 ? 3 : 2;  // CTAs per SM the shared memory allows
constexpr int kWRow = kWCh + 1;        // float4 per padded state row
constexpr int kWQRow = 136;            // floats per padded dy silu(z) row

constexpr int kWItemWarps = kWTS / 2;  // warps that cover the chunk's items once
constexpr int kWGCh = 4 * kWTS;        // channels per group of a channel sum
static_assert(kWTS == 4 || kWTS == 8, "chunk of 4 or 8 tokens");
static_assert((kWCh / kWGCh - 1) * (kWGCh + 1) + kWGCh <= kWQRow, "dy silu(z) row");

template <typename T>
struct WRaw {
    T act[4][kWTS][kWCh];  // dt, u, z, dy
    T bc[2][kWTS][kN];     // B, C
};

struct WSmem {
    // row (slot * 4 + q): states 4q .. 4q + 3 of every channel; slot 0 holds
    // the checkpoint, slot tl + 1 the states after token tl, later its dB terms
    float4 hist[(kWTS + 1) * 4][kWRow];
    float dq[kWTS][kWQRow];
    float B[kWTS][kN];
    float C[kWTS][kN];
};

__device__ __forceinline__ int wq_col(int c) { return (c / kWGCh) * (kWGCh + 1) + c % kWGCh; }

template <typename T, int NT = kWCh>  // NT: threads of the CTA that share the copies
__device__ __forceinline__ void w_issue(const BwdParams &p, WRaw<T> &r, int64_t t0, int nt,
                                        int64_t cbase, int nch, bool full)
{
    constexpr int V = 16 / sizeof(T), VR = kWCh / V, VB = kN / V;
    const T *DT = static_cast<const T *>(p.dt), *U = static_cast<const T *>(p.u);
    const T *Z = static_cast<const T *>(p.z), *DY = static_cast<const T *>(p.dy);
    const int narr = full ? 4 : 2, nvr = nch / V;
    for (int e = threadIdx.x; e < narr * kWTS * VR; e += NT) {
        const int arr = e / (kWTS * VR), rem = e % (kWTS * VR), tl = rem / VR, v = rem % VR;
        const T *src = arr == 0 ? DT : arr == 1 ? U : arr == 2 ? Z : DY;  // selects: no local array
        if (tl >= nt || v >= nvr || src == nullptr) continue;
        cp16(&r.act[arr][tl][v * V], src + (t0 + tl) * p.D + cbase + v * V);
    }
    for (int e = threadIdx.x; e < (full ? 2 : 1) * kWTS * VB; e += NT) {
        const int arr = e / (kWTS * VB), rem = e % (kWTS * VB), tl = rem / VB, v = rem % VB;
        if (tl >= nt) continue;
        const T *src = static_cast<const T *>(arr ? p.C : p.B);
        cp16(&r.bc[arr][tl][v * V], src + (t0 + tl) * kN + v * V);
    }
}

// Sum over the CTA's channels of the chunk's state rows (weighted by dy
// silu(z) when `weighted`), added into dst (tok, 16) at tokens t0 .. t0 + nt.
__device__ __forceinline__ void w_channel_sum(const BwdParams &p, const WSmem &sm, bool weighted,
                                              float *dst, int64_t t0, int nt)
{
    const int lane = threadIdx.x & 31, k = lane >> 3, w = threadIdx.x >> 5;
    const int item = (w % kWItemWarps) * 8 + (lane & 7), tl = item >> 2, q = item & 3;
    const int g = (w / kWItemWarps) * 4 + k;
    f32x2 s01 = 0ull, s23 = 0ull;
    if (tl < nt) {
        const float4 *row = &sm.hist[(tl + 1) * 4 + q][g * kWGCh];
        if (weighted) {
            const float *wt = &sm.dq[tl][g * (kWGCh + 1)];
#pragma unroll 8
            for (int j = 0; j < kWGCh; ++j) {
                const float4 v = row[j];
                const f32x2 c = pk2(wt[j], wt[j]);
                s01 = fma2(c, pk2(v.x, v.y), s01);
                s23 = fma2(c, pk2(v.z, v.w), s23);
            }
        } else {
#pragma unroll 8
            for (int j = 0; j < kWGCh; ++j) {
                const float4 v = row[j];
                s01 = add2(s01, pk2(v.x, v.y));
                s23 = add2(s23, pk2(v.z, v.w));
            }
        }
    }
    float4 acc;
    upk2(s01, acc.x, acc.y);
    upk2(s23, acc.z, acc.w);
#pragma unroll
    for (int m = 8; m <= 16; m <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
    }
    if (k == 0 && tl < nt) {
        float *o = dst + (t0 + tl) * kN + 4 * q;
        if (p.vec_atomics) {
            atomicAdd(reinterpret_cast<float4 *>(o), acc);
        } else {
            atomicAdd(o, acc.x);
            atomicAdd(o + 1, acc.y);
            atomicAdd(o + 2, acc.z);
            atomicAdd(o + 3, acc.w);
        }
    }
}

// Shared memory: the state rows, two raw chunk buffers and, with bf16
// activations, the next chunk's checkpoint block (with fp32 activations it
// would not leave room for two CTAs per SM, so those read it directly).
constexpr size_t kWCkBytes = (size_t)kWCh * kN * sizeof(float);
constexpr size_t w_smem_bytes(size_t raw_bytes, bool ck_async)
{
    return sizeof(WSmem) + 2 * raw_bytes + (ck_async ? kWCkBytes : 0);
}

template <typename T, bool ASYNC>
__global__ void __launch_bounds__(kWCh, kWMinCtas)
scan_bwd_wide_kernel(const BwdParams p)
{
    constexpr int NP = 8, NQ = 4;  // packed state pairs, state quads
    extern __shared__ __align__(128) unsigned char w_smem[];
    WSmem &sm = *reinterpret_cast<WSmem *>(w_smem);
    WRaw<T> *raw = reinterpret_cast<WRaw<T> *>(w_smem + sizeof(WSmem));
    const int tid = threadIdx.x, cl = tid;
    const int64_t cbase = (int64_t)blockIdx.x * kWCh, c = cbase + cl;
    const int nch = (int)min((int64_t)kWCh, p.D - cbase);
    const bool cvalid = c < p.D;
    int64_t s, start, end;
    bwd_sequence(p, s, start, end);
    const int64_t len = end - start;
    const int64_t nchunks = (len + kWTS - 1) / kWTS;
    // checkpoint slots of this sequence: floor(start / kWTS) + s + k never collide
    float *ck = p.ckpt + ((start / kWTS + s) * p.D + c) * kN;
    const int64_t ck_stride = p.D * kN;

    f32x2 A2[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int n = 2 * j;
        const float a0 = cvalid ? __ldg(p.A + c * kN + n) : 0.f;
        const float a1 = cvalid ? __ldg(p.A + c * kN + n + 1) : 0.f;
        A2[j] = pk2(a0 * kLog2e, a1 * kLog2e);
    }
    const float dsk = (cvalid && p.Dskip) ? __ldg(p.Dskip + c) : 0.f;
    const float dtb = (cvalid && p.dt_bias) ? __ldg(p.dt_bias + c) : 0.f;
    const T *DT = static_cast<const T *>(p.dt), *U = static_cast<const T *>(p.u);
    const T *Z = static_cast<const T *>(p.z), *DY = static_cast<const T *>(p.dy);
    const T *Bp = static_cast<const T *>(p.B), *Cp = static_cast<const T *>(p.C);
    const bool has_z = Z != nullptr;

    // the chunk's B (and C) rows in fp32: one (token, state) per thread
    auto fill_bc = [&](const WRaw<T> &r, int64_t t0, int nt, bool with_c) {
        if (tid >= kWTS * kN) return;
        const int tl = tid >> 4, n = tid & 15;
        float b = 0.f, cc = 0.f;
        if (tl < nt) {
            if constexpr (ASYNC) {
                b = to_f32(r.bc[0][tl][n]);
                if (with_c) cc = to_f32(r.bc[1][tl][n]);
            } else {
                b = ld1(Bp + (t0 + tl) * kN + n);
                if (with_c) cc = ld1(Cp + (t0 + tl) * kN + n);
            }
        }
        sm.B[tl][n] = b;
        if (with_c) sm.C[tl][n] = cc;
    };
    // this channel's value of activation `arr` at chunk token tl (channel valid)
    auto act = [&](const WRaw<T> &r, int arr, int tl, int64_t t) -> float {
        if constexpr (ASYNC) {
            return to_f32(r.act[arr][tl][cl]);
        } else {
            const T *src = arr == 0 ? DT : arr == 1 ? U : arr == 2 ? Z : DY;
            return ld1(src + t * p.D + c);
        }
    };
    // this thread's state rows: one base address, constant offsets after
    const float *Bq = &sm.B[0][0], *Cq = &sm.C[0][0];
    float4 *Hq = &sm.hist[0][cl];
    auto bquad = [&](int tl, int qq) { return *reinterpret_cast<const float4 *>(Bq + tl * kN + 4 * qq); };
    auto cquad = [&](int tl, int qq) { return *reinterpret_cast<const float4 *>(Cq + tl * kN + 4 * qq); };
    auto hist = [&](int slot, int qq) -> float4 & { return Hq[(slot * 4 + qq) * kWRow]; };

    // ---- phase B: reverse -----------------------------------------------------
    f32x2 G[NP], dAacc[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int64_t o = (s * p.D + c) * kN + 2 * j;
        G[j] = (cvalid && p.dh_final) ? pk2(p.dh_final[o], p.dh_final[o + 1]) : 0ull;
        dAacc[j] = 0ull;
    }
    float dDsk = 0.f, ddtb = 0.f;
    T *DU = static_cast<T *>(p.du), *DDT = static_cast<T *>(p.ddt), *DZ = static_cast<T *>(p.dz);
    // with bf16 activations, chunk k - 1's checkpoint rows of the CTA's
    // channels (contiguous, 64 bytes per channel) come in while chunk k runs
    constexpr bool kCkAsync = ASYNC && sizeof(T) == 2;
    float4 *ckb = reinterpret_cast<float4 *>(w_smem + sizeof(WSmem) + 2 * sizeof(WRaw<T>));
    auto issue_ck = [&](int64_t kk) {
        const float *src = p.ckpt + ((start / kWTS + s + kk) * p.D + cbase) * kN;
        for (int e = tid; e < nch * 4; e += kWCh) cp16(&ckb[e], src + 4 * e);
    };
    // the checkpoints come from scan_bwd_ckpt_kernel, launched before on the stream
    if (ASYNC && nchunks > 0) {
        const int64_t tl0 = start + (nchunks - 1) * kWTS;
        w_issue<T>(p, raw[0], tl0, (int)(end - tl0), cbase, nch, true);
        if constexpr (kCkAsync) issue_ck(nchunks - 1);
        cp_commit();
    }
    for (int64_t k = nchunks - 1; k >= 0; --k) {
        const int64_t t0 = start + k * kWTS;
        const int nt = (int)min((int64_t)kWTS, end - t0);
        const int buf = (int)((nchunks - 1 - k) & 1);
        f32x2 hc[NP];
        if (!kCkAsync && cvalid) {
            const float4 *src = reinterpret_cast<const float4 *>(ck + k * ck_stride);
#pragma unroll
            for (int qq = 0; qq < NQ; ++qq) {
                const float4 v = src[qq];
                hc[2 * qq] = pk2(v.x, v.y);
                hc[2 * qq + 1] = pk2(v.z, v.w);
            }
        }
        if constexpr (ASYNC) cp_wait<0>();
        __syncthreads();  // chunk k has landed; the previous chunk's dB sum is done
        if (ASYNC && k > 0) {
            w_issue<T>(p, raw[buf ^ 1], t0 - kWTS, kWTS, cbase, nch, true);
            cp_commit();
        }
        fill_bc(raw[buf], t0, nt, true);
        if (kCkAsync && cvalid) {
#pragma unroll
            for (int qq = 0; qq < NQ; ++qq) {
                const float4 v = ckb[cl * 4 + qq];
                hc[2 * qq] = pk2(v.x, v.y);
                hc[2 * qq + 1] = pk2(v.z, v.w);
            }
        }
        if (!cvalid) {
#pragma unroll
            for (int j = 0; j < NP; ++j) hc[j] = 0ull;
        }
#pragma unroll
        for (int qq = 0; qq < NQ; ++qq) {
            float4 v;
            upk2(hc[2 * qq], v.x, v.y);
            upk2(hc[2 * qq + 1], v.z, v.w);
            hist(0, qq) = v;
        }
        __syncthreads();  // B and C rows staged; the checkpoint block has been read
        if (kCkAsync && k > 0) {
            issue_ck(k - 1);
            cp_commit();
        }

        // 1. recompute the chunk's states; dz
        float dr[kWTS], xr[kWTS], ur[kWTS], qr[kWTS], sr[kWTS];
        auto recompute = [&](auto full) {
            constexpr bool kFull = decltype(full)::value;
#pragma unroll
            for (int tl = 0; tl < kWTS; ++tl) {
                // staged values are read for every lane (shared memory holds
                // some value for each) and masked afterwards, so the token
                // loop has no divergent branch; direct loads stay guarded
                const bool live = (kFull || tl < nt) && cvalid;
                float vdt = 0.f, vu = 0.f, vdy = 0.f, vz = 0.f;
                if (ASYNC || live) {
                    vdt = act(raw[buf], 0, tl, t0 + tl);
                    vu = act(raw[buf], 1, tl, t0 + tl);
                    vdy = act(raw[buf], 3, tl, t0 + tl);
                    if (has_z) vz = act(raw[buf], 2, tl, t0 + tl);
                }
                const float v = vdt + dtb;
                float d = p.softplus ? softplus_fast(v) : v;
                float sp = p.softplus ? sigmoid_f(v) : 1.f;
                float g = 1.f, dg = 0.f;
                if (has_z) {
                    const float sg = sigmoid_f(vz);
                    g = vz * sg;
                    dg = sg * (1.f + vz * (1.f - sg));
                }
                d = live ? d : 0.f;
                sp = live ? sp : 0.f;
                const float u = live ? vu : 0.f;
                const float x = d * u;
                const float dq = live ? vdy * g : 0.f;
                const float dzf = live ? vdy * dg : 0.f;
                dr[tl] = d;
                xr[tl] = x;
                ur[tl] = u;
                qr[tl] = dq;
                sr[tl] = sp;
                sm.dq[tl][wq_col(cl)] = dq;
                if (kFull || tl < nt) {
                    const f32x2 dd = pk2(d, d), xx = pk2(x, x);
                    f32x2 qp = 0ull, qp1 = 0ull;
#pragma unroll
                    for (int qq = 0; qq < NQ; ++qq) {
                        const float4 b4 = bquad(tl, qq);
                        const float4 c4 = cquad(tl, qq);
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = 2 * qq + e;
                            float e0, e1;
                            upk2(mul2(dd, A2[j]), e0, e1);
                            const f32x2 a = pk2(ex2_approx(e0), ex2_approx(e1));
                            const f32x2 b2 = e ? pk2(b4.z, b4.w) : pk2(b4.x, b4.y);
                            const f32x2 c2 = e ? pk2(c4.z, c4.w) : pk2(c4.x, c4.y);
                            hc[j] = fma2(a, hc[j], mul2(xx, b2));
                            if (e) qp1 = fma2(c2, hc[j], qp1);
                            else qp = fma2(c2, hc[j], qp);
                        }
                        float4 v;
                        upk2(hc[2 * qq], v.x, v.y);
                        upk2(hc[2 * qq + 1], v.z, v.w);
                        hist(tl + 1, qq) = v;
                    }
                    float q0s, q1s;
                    upk2(add2(qp, qp1), q0s, q1s);
                    const float qs = q0s + q1s;
                    if (cvalid && DZ)
                        DZ[(t0 + tl) * p.D + c] = from_f32<T>(has_z ? dzf * (qs + dsk * u) : 0.f);
                }
            }
        };
        if (nt == kWTS) recompute(std::true_type{});
        else recompute(std::false_type{});
        __syncthreads();  // the chunk's states and dy silu(z) are in shared memory

        // 2. dC over the CTA's channels
        w_channel_sum(p, sm, true, p.dC, t0, nt);
        __syncthreads();  // the states are no longer read by other threads

        // 3. reverse walk
        auto reverse = [&](auto full) {
            constexpr bool kFull = decltype(full)::value;
#pragma unroll
            for (int tl = kWTS - 1; tl >= 0; --tl) {
                if (kFull || tl < nt) {
                    const float d = dr[tl], x = xr[tl], dq = qr[tl];
                    const f32x2 dd = pk2(d, d), xx = pk2(x, x), dqq = pk2(dq, dq);
                    f32x2 dup = 0ull, ddp = 0ull, dup1 = 0ull, ddp1 = 0ull;
#pragma unroll
                    for (int qq = 0; qq < NQ; ++qq) {
                        const float4 b4 = bquad(tl, qq);
                        const float4 c4 = cquad(tl, qq);
                        const float4 hp = hist(tl, qq);  // h_{t-1}
                        float4 gx;
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = 2 * qq + e;
                            float e0, e1;
                            upk2(mul2(dd, A2[j]), e0, e1);
                            const f32x2 a = pk2(ex2_approx(e0), ex2_approx(e1));
                            const f32x2 b2 = e ? pk2(b4.z, b4.w) : pk2(b4.x, b4.y);
                            const f32x2 c2 = e ? pk2(c4.z, c4.w) : pk2(c4.x, c4.y);
                            const f32x2 h2 = e ? pk2(hp.z, hp.w) : pk2(hp.x, hp.y);
                            G[j] = fma2(dqq, c2, G[j]);         // G_t = dq C + a_{t+1} G_{t+1}
                            const f32x2 g2 = mul2(G[j], xx);    // dB terms
                            if (e) {
                                dup1 = fma2(G[j], b2, dup1);    // G . B
                                upk2(g2, gx.z, gx.w);
                            } else {
                                dup = fma2(G[j], b2, dup);
                                upk2(g2, gx.x, gx.y);
                            }
                            G[j] = mul2(a, G[j]);               // a G_t: dL/dh_{t-1} so far
                            const f32x2 gah = mul2(G[j], h2);   // G a h_{t-1}
                            if (e) ddp1 = fma2(gah, A2[j], ddp1);  // G A a h_{t-1} / ln 2
                            else ddp = fma2(gah, A2[j], ddp);
                            dAacc[j] = fma2(gah, dd, dAacc[j]);
                        }
                        hist(tl + 1, qq) = gx;
                    }
                    float u0, u1, x0, x1;
                    upk2(add2(dup, dup1), u0, u1);
                    upk2(add2(ddp, ddp1), x0, x1);
                    const float us = u0 + u1;
                    const float xs = x0 + x1;
                    // the per-token values are zero for a channel beyond D
                    const float ddt = (ur[tl] * us + kLn2 * xs) * sr[tl];
                    dDsk += dq * ur[tl];
                    ddtb += ddt;
                    if (cvalid) {
                        const int64_t o = (t0 + tl) * p.D + c;
                        DU[o] = from_f32<T>(dq * dsk + d * us);
                        DDT[o] = from_f32<T>(ddt);
                    }
                }
            }
        };
        if (nt == kWTS) reverse(std::true_type{});
        else reverse(std::false_type{});
        __syncthreads();  // the chunk's dB terms are in shared memory

        // 4. dB over the CTA's channels
        w_channel_sum(p, sm, false, p.dB, t0, nt);
    }
    if (cvalid) {
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            const int n = 2 * j;
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
        if (p.dDskip) atomicAdd(p.dDskip + c, dDsk);
        if (p.ddt_bias) atomicAdd(p.ddt_bias + c, ddtb);
    }
}

// Phase A of the thread-per-channel backward as a kernel of its own: the
// forward pass over each sequence that writes the state at every kWTS-token
// chunk start (the checkpoint layout scan_bwd_wide_kernel reads). Without the
// state buffer it needs 18 KB of shared memory (bf16) and few registers, so
// several times as many warps per SM run it as would inside the reverse kernel.
// Two adjacent lanes share a channel, 8 states each, which halves each thread's
// serial chain: with packed sequences of mixed lengths the pass is bound by
// its longest sequence.
constexpr int kCkLanes = 2;                   // lanes per channel (4 measured slower)
constexpr int kCkThreads = kCkLanes * kWCh;

template <typename T, bool ASYNC>
__global__ void __launch_bounds__(kCkThreads)
scan_bwd_ckpt_kernel(const BwdParams p)
{
    constexpr int SPL = kN / kCkLanes, NP = SPL / 2, NQ = SPL / 4;  // states, pairs, quads per lane
    extern __shared__ __align__(128) unsigned char c_smem[];
    WRaw<T> *raw = reinterpret_cast<WRaw<T> *>(c_smem);
    float *sB = reinterpret_cast<float *>(c_smem + 2 * sizeof(WRaw<T>));  // [kWTS][kN]
    const int tid = threadIdx.x, cl = tid / kCkLanes, sub = tid % kCkLanes;
    const int64_t cbase = (int64_t)blockIdx.x * kWCh, c = cbase + cl;
    const int nch = (int)min((int64_t)kWCh, p.D - cbase);
    const bool cvalid = c < p.D;
    int64_t s, start, end;
    bwd_sequence(p, s, start, end);
    const int64_t len = end - start;
    const int64_t nchunks = (len + kWTS - 1) / kWTS;
    float *ck = p.ckpt + ((start / kWTS + s) * p.D + c) * kN + SPL * sub;
    const int64_t ck_stride = p.D * kN;
    f32x2 A2[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const float a0 = cvalid ? __ldg(p.A + c * kN + SPL * sub + 2 * j) : 0.f;
        const float a1 = cvalid ? __ldg(p.A + c * kN + SPL * sub + 2 * j + 1) : 0.f;
        A2[j] = pk2(a0 * kLog2e, a1 * kLog2e);
    }
    const float dtb = (cvalid && p.dt_bias) ? __ldg(p.dt_bias + c) : 0.f;
    const T *DT = static_cast<const T *>(p.dt), *U = static_cast<const T *>(p.u);
    const T *Bp = static_cast<const T *>(p.B);
    // the chunk's B rows in fp32: one (token, state) per thread
    auto fill_bc = [&](const WRaw<T> &r, int64_t t0, int nt, bool) {
        if (tid >= kWTS * kN) return;
        const int tl = tid >> 4, n = tid & 15;
        float b = 0.f;
        if (tl < nt) {
            if constexpr (ASYNC) b = to_f32(r.bc[0][tl][n]);
            else b = ld1(Bp + (t0 + tl) * kN + n);
        }
        sB[tl * kN + n] = b;
    };
    // this channel's dt (arr 0) or u (arr 1) at chunk token tl (channel valid)
    auto act = [&](const WRaw<T> &r, int arr, int tl, int64_t t) -> float {
        if constexpr (ASYNC) return to_f32(r.act[arr][tl][cl]);
        else return ld1((arr == 0 ? DT : U) + t * p.D + c);
    };
    auto bquad = [&](int tl, int qq) {
        return *reinterpret_cast<const float4 *>(sB + tl * kN + SPL * sub + 4 * qq);
    };

    f32x2 h[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int64_t o = (s * p.D + c) * kN + SPL * sub + 2 * j;
        h[j] = (cvalid && p.h0) ? pk2(p.h0[o], p.h0[o + 1]) : 0ull;
    }
    if (ASYNC && nchunks > 0) {
        w_issue<T, kCkThreads>(p, raw[0], start, (int)min((int64_t)kWTS, len), cbase, nch, false);
        cp_commit();
    }
    for (int64_t k = 0; k < nchunks; ++k) {
        const int64_t t0 = start + k * kWTS;
        const int nt = (int)min((int64_t)kWTS, end - t0);
        if (cvalid) {
            float4 *dst = reinterpret_cast<float4 *>(ck + k * ck_stride);
#pragma unroll
            for (int qq = 0; qq < NQ; ++qq) {
                float4 v;
                upk2(h[2 * qq], v.x, v.y);
                upk2(h[2 * qq + 1], v.z, v.w);
                dst[qq] = v;
            }
        }
        if constexpr (ASYNC) cp_wait<0>();
        __syncthreads();  // chunk k has landed; chunk k - 1 is no longer read
        if (ASYNC && k + 1 < nchunks) {
            const int64_t t1 = t0 + kWTS;
            w_issue<T, kCkThreads>(p, raw[(k + 1) & 1], t1, (int)min((int64_t)kWTS, end - t1),
                                   cbase, nch, false);
            cp_commit();
        }
        fill_bc(raw[k & 1], t0, nt, false);
        __syncthreads();
        // full chunks take a copy of the token loop without per-token guards,
        // so the compiler can overlap neighbouring tokens' work
        auto walk = [&](auto full) {
            constexpr bool kFull = decltype(full)::value;
#pragma unroll
            for (int tl = 0; tl < kWTS; ++tl) {
                if (kFull || tl < nt) {
                    const float v = act(raw[k & 1], 0, tl, t0 + tl) + dtb;
                    const float d = p.softplus ? softplus_fast(v) : v;
                    const float x = d * act(raw[k & 1], 1, tl, t0 + tl);
                    const f32x2 dd = pk2(d, d), xx = pk2(x, x);
#pragma unroll
                    for (int qq = 0; qq < NQ; ++qq) {
                        const float4 b4 = bquad(tl, qq);
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = 2 * qq + e;
                            float e0, e1;
                            upk2(mul2(dd, A2[j]), e0, e1);
                            const f32x2 a = pk2(ex2_approx(e0), ex2_approx(e1));
                            const f32x2 b2 = e ? pk2(b4.z, b4.w) : pk2(b4.x, b4.y);
                            h[j] = fma2(a, h[j], mul2(xx, b2));
                        }
                    }
                }
            }
        };
        if (cvalid) {
            if (nt == kWTS) walk(std::true_type{});
            else walk(std::false_type{});
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
    bool have_ckpt = false;  // ckpt already holds the forward's 8-token checkpoints
};

cudaError_t launch_seq_order(const int32_t *cu, int64_t S, int64_t tok, int32_t *order,
                             cudaStream_t stream);
int device_sm_count();

// Checkpoint floats of the thread-per-channel kernel (one state per kWTS
// tokens); the lane-split kernel's one per kTS tokens fits in the same area.
static size_t ckpt_floats(int64_t tok, int64_t D, int64_t S)
{
    return (size_t)(tok / kWTS + S + 1) * (size_t)D * kN;
}

static size_t order_offset(int64_t tok, int64_t D, int64_t S)
{
    return (ckpt_floats(tok, D, S) * sizeof(float) + 255) / 256 * 256;
}

size_t scan_bwd_workspace_bytes(int64_t tok, int64_t D, int64_t S)
{
    return order_offset(tok, D, S) + (size_t)((S * 4 + 255) / 256) * 256;
}

static std::atomic<int> g_bwd_forced{0};

void set_scan_bwd_variant(int v) { g_bwd_forced.store(v, std::memory_order_relaxed); }

// 1: four lanes per channel (kTS-token chunks); 2: one thread per channel.
// The thread-per-channel kernel executes about half the instructions per
// (token, channel) (14 against 28 warp instructions, measured) but has a
// quarter of the threads; it is chosen once its CTAs fill every SM twice
// (two CTAs are resident per SM).
int scan_bwd_variant_for(int64_t S, int64_t D)
{
    const int f = g_bwd_forced.load(std::memory_order_relaxed);
    if (f) return f;
    const int64_t ctas = S * ((D + kWCh - 1) / kWCh);
    return ctas >= 2 * (int64_t)device_sm_count() ? 2 : 1;
}

template <typename T, bool ASYNC>
static cudaError_t run_lanes(const BwdParams &p, dim3 grid, cudaStream_t stream)
{
    const size_t smem = sizeof(Smem) + (ASYNC ? 2 : 1) * sizeof(RawChunk<T>);
    cudaError_t e = cudaFuncSetAttribute(scan_bwd_kernel<T, ASYNC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    scan_bwd_kernel<T, ASYNC><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, bool ASYNC>
static cudaError_t run_ckpt(const BwdParams &p, dim3 grid, cudaStream_t stream, int *launches)
{
    const size_t ck_smem = 2 * sizeof(WRaw<T>) + sizeof(float) * kWTS * kN;
    cudaError_t e = cudaFuncSetAttribute(scan_bwd_ckpt_kernel<T, ASYNC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ck_smem);
    if (e != cudaSuccess) return e;
    scan_bwd_ckpt_kernel<T, ASYNC><<<grid, kCkThreads, ck_smem, stream>>>(p);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, bool ASYNC>
static cudaError_t run_wide(const BwdParams &p, dim3 grid, cudaStream_t stream, int *launches)
{
    // the forward pass that writes the checkpoints (unless the forward scan
    // wrote them), then the reverse pass
    cudaError_t e;
    if (!p.have_ckpt) {
        e = run_ckpt<T, ASYNC>(p, grid, stream, launches);
        if (e != cudaSuccess) return e;
    }
    const size_t smem = w_smem_bytes(sizeof(WRaw<T>), ASYNC && sizeof(T) == 2);
    e = cudaFuncSetAttribute(scan_bwd_wide_kernel<T, ASYNC>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    scan_bwd_wide_kernel<T, ASYNC><<<grid, kWCh, smem, stream>>>(p);
    return cudaGetLastError();
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
    p.dh0 = a.dh0; p.ckpt = a.ckpt; p.order = nullptr; p.have_ckpt = a.have_ckpt ? 1 : 0;
    p.S = a.S; p.tok = a.tok; p.D = a.D; p.L = a.cu ? 0 : a.tok / a.S; p.softplus = a.softplus;
    p.vec_atomics = ((uintptr_t)a.dB % 16 == 0) && ((uintptr_t)a.dC % 16 == 0);
    if (a.cu && a.S > 1) {
        // longest sequences first, so the longest chains do not start last
        int32_t *order = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(a.ckpt) +
                                                     order_offset(a.tok, a.D, a.S));
        cudaError_t e = launch_seq_order(a.cu, a.S, a.tok, order, stream);
        ++*launches;
        if (e != cudaSuccess) return e;
        p.order = order;
    }
    const size_t es = a.bf16 ? 2 : 4;
    const uintptr_t mis = (uintptr_t)a.u | (uintptr_t)a.dt | (uintptr_t)a.z | (uintptr_t)a.dy |
                          (uintptr_t)a.B | (uintptr_t)a.C;
    const bool async_ok = (mis % 16 == 0) && ((size_t)a.D * es) % 16 == 0;
    cudaError_t e;
    if (scan_bwd_variant_for(a.S, a.D) == 2) {
        const dim3 grid((unsigned)((a.D + kWCh - 1) / kWCh), (unsigned)a.S);
        if (a.bf16)
            e = async_ok ? run_wide<__nv_bfloat16, true>(p, grid, stream, launches)
                         : run_wide<__nv_bfloat16, false>(p, grid, stream, launches);
        else
            e = async_ok ? run_wide<float, true>(p, grid, stream, launches)
                         : run_wide<float, false>(p, grid, stream, launches);
    } else {
        const dim3 grid((unsigned)((a.D + kCh - 1) / kCh), (unsigned)a.S);
        if (a.bf16)
            e = async_ok ? run_lanes<__nv_bfloat16, true>(p, grid, stream)
                         : run_lanes<__nv_bfloat16, false>(p, grid, stream);
        else
            e = async_ok ? run_lanes<float, true>(p, grid, stream)
                         : run_lanes<float, false>(p, grid, stream);
    }
    ++*launches;
    return e;
}

// The checkpointing forward pass alone (the state before every 8th token of
// each sequence into a.ckpt), for a forward scan whose kernel did not write
// them. Reads u, dt, B, A, dt_bias and h0; sequences in index order.
cudaError_t launch_scan_bwd_ckpt_pass(const ScanBwdArgs &a, cudaStream_t stream, int *launches)
{
    if (a.S == 0 || a.tok == 0) return cudaSuccess;
    BwdParams p{};
    p.u = a.u; p.dt = a.dt; p.B = a.B; p.A = a.A; p.dt_bias = a.dt_bias; p.h0 = a.h0;
    p.cu = a.cu; p.ckpt = a.ckpt; p.order = nullptr;
    p.S = a.S; p.tok = a.tok; p.D = a.D; p.L = a.cu ? 0 : a.tok / a.S; p.softplus = a.softplus;
    const size_t es = a.bf16 ? 2 : 4;
    const uintptr_t mis = (uintptr_t)a.u | (uintptr_t)a.dt | (uintptr_t)a.B;
    const bool async_ok = (mis % 16 == 0) && ((size_t)a.D * es) % 16 == 0;
    const dim3 grid((unsigned)((a.D + kWCh - 1) / kWCh), (unsigned)a.S);
    if (a.bf16)
        return async_ok ? run_ckpt<__nv_bfloat16, true>(p, grid, stream, launches)
                        : run_ckpt<__nv_bfloat16, false>(p, grid, stream, launches);
    return async_ok ? run_ckpt<float, true>(p, grid, stream, launches)
                    : run_ckpt<float, false>(p, grid, stream, launches);
}

}  // namespace ssm
