/*
 * ssm_oracle.c -- plain fp64 CPU oracle of the selective-SSM mixer core.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path never
 * calls it, and it shares no code, header or constant with the CUDA sources.
 *
 * Everything here is written straight from the definitions, with plain loops,
 * in double precision, no blocking, no fusion and no reordering:
 *
 *   conv:     xc_t[c] = silu(bias[c] + sum_k w[c,k] * win_t[c,k]), where the
 *             window holds the K-1 previous inputs of the same sequence (the
 *             carried conv state, or zeros, before the sequence's first token)
 *             followed by x_t; the newest input pairs with w[c,K-1].
 *             Source: tp_builder.py (TensorRT-Model-Connect, Mamba family),
 *             _add_mamba_tp_layer, conv-state shift and depthwise conv step;
 *             "Scaling State-Space Models on Multiple GPUs with Tensor
 *             Parallelism", Fig. 1 (channel-separable 1D convolution).
 *   delta:    D_t[c] = softplus(dt_t[c] + dt_bias[c])   (same builder, dt step,
 *             written there as log(exp(v) + 1)).
 *   scan:     dA = exp(D_t[c] A[c,n]); h_t[c,n] = dA h_{t-1}[c,n] + D_t[c] u_t[c] B_t[n];
 *             y_t[c] = (sum_n C_t[n] h_t[c,n] + Dskip[c] u_t[c]) * silu(z_t[c])
 *             (same builder: discretisation, state update, readout, D skip,
 *             gate; Fig. 1: state update over the sequence, then gating).
 *   packing:  every sequence of a packed batch starts from its own initial
 *             state; nothing flows across a cu_seqlens boundary ("PackMamba:
 *             Efficient Processing of Variable-Length Sequences in Mamba
 *             training", abstract).
 *   decode:   one token per row updates the cached conv and SSM state in place
 *             (tp_builder.py: present_conv / present_ssm outputs; "Scaling
 *             State-Space Models...", abstract: SSM cache across prefill and
 *             decode).
 *   replay:   the SSM state of a slot is kept as a checkpoint plus the SSM
 *             inputs (delta, xc, B) of the tokens since it; outputs come from
 *             unrolling the recurrence from the checkpoint, and the checkpoint
 *             is rewritten once every W tokens; an optional bf16 copy of the
 *             checkpoint serves the outputs of the other steps ("ReplaySSM:
 *             Cache SSM Inputs, Not State", abstract).
 *
 * Channels are independent, so the outer (sequence, channel) loops may run on
 * several OpenMP threads; each (sequence, channel) is computed by one thread in
 * token order, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MAX_N 256
#define ORACLE_MAX_K 64

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* softplus(v) = log(1 + exp(v)), evaluated without overflow. */
static double softplus(double v) { return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v))); }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Value of the conv window for sequence s, channel c at sequence position p
 * (p < 0 reaches into the carried state: position -1 is the newest state
 * entry, stored at index K-2). */
static double window_value(const double *x, const double *state_in, int64_t D, int K,
                           int64_t start, int64_t s, int64_t c, int64_t p)
{
    if (p >= 0) return x[(start + p) * D + c];
    if (state_in == NULL) return 0.0;
    return state_in[(s * D + c) * (K - 1) + (K - 1) + p];
}

/*
 * x, xc: (tok, D). w: (D, K). bias: (D) or NULL. cu: S+1 offsets.
 * state_in, state_out: (S, D, K-1) or NULL; they must not alias.
 */
void oracle_causal_conv1d(const double *x, double *xc, const double *w, const double *bias,
                          int64_t tok, int64_t D, int K, const int64_t *cu, int64_t S,
                          const double *state_in, double *state_out, int apply_silu)
{
    (void)tok;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t s = 0; s < S; ++s) {
        for (int64_t c = 0; c < D; ++c) {
            const int64_t start = cu[s];
            const int64_t len = cu[s + 1] - cu[s];
            for (int64_t t = 0; t < len; ++t) {
                double acc = bias ? bias[c] : 0.0;
                for (int k = 0; k < K; ++k) {
                    const int64_t p = t - (K - 1) + k;
                    acc += w[c * K + k] * window_value(x, state_in, D, K, start, s, c, p);
                }
                xc[(start + t) * D + c] = apply_silu ? silu(acc) : acc;
            }
            if (state_out) {
                for (int j = 0; j < K - 1; ++j) {
                    const int64_t p = len - (K - 1) + j;
                    state_out[(s * D + c) * (K - 1) + j] =
                        window_value(x, state_in, D, K, start, s, c, p);
                }
            }
        }
    }
}

/*
 * u, delta, z, y: (tok, D). A: (D, N). B, C: (tok, N). Dskip, dt_bias: (D) or
 * NULL. h0, h_final: (S, D, N) or NULL (they may be the same array: each
 * (sequence, channel) reads its h0 before writing its h_final). z == NULL
 * means no gate. Tokens of empty sequences do not exist, so nothing is written
 * for them; their h_final is h0 (or zeros).
 */
void oracle_selective_scan(const double *u, const double *delta, const double *A,
                           const double *B, const double *C, const double *Dskip,
                           const double *z, const double *dt_bias, int delta_softplus,
                           const double *h0, const int64_t *cu, int64_t S, int64_t tok,
                           int64_t D, int N, double *y, double *h_final)
{
    (void)tok;
    if (N > ORACLE_MAX_N) return;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t s = 0; s < S; ++s) {
        for (int64_t c = 0; c < D; ++c) {
            double h[ORACLE_MAX_N];
            for (int n = 0; n < N; ++n) h[n] = h0 ? h0[(s * D + c) * N + n] : 0.0;
            for (int64_t t = cu[s]; t < cu[s + 1]; ++t) {
                double d = delta[t * D + c] + (dt_bias ? dt_bias[c] : 0.0);
                if (delta_softplus) d = softplus(d);
                const double ut = u[t * D + c];
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    const double dA = exp(d * A[c * N + n]);
                    h[n] = dA * h[n] + d * ut * B[t * N + n];
                    acc += C[t * N + n] * h[n];
                }
                double yt = acc + (Dskip ? Dskip[c] : 0.0) * ut;
                if (z) yt *= silu(z[t * D + c]);
                y[t * D + c] = yt;
            }
            if (h_final)
                for (int n = 0; n < N; ++n) h_final[(s * D + c) * N + n] = h[n];
        }
    }
}

/*
 * One decode token per row b. Slot s = idx[b] (or b when idx is NULL); rows
 * with s < 0 are skipped and their y row is left untouched. conv_state:
 * (n_slots, D, K-1), ssm_state: (n_slots, D, N); both are updated in place.
 * x, dt, z, y: (Bt, D); B, C: (Bt, N).
 */
void oracle_state_update(double *conv_state, double *ssm_state, const double *x,
                         const double *dt, const double *B, const double *C, const double *z,
                         const double *conv_w, const double *conv_b, const double *A,
                         const double *Dskip, const double *dt_bias, int delta_softplus,
                         const int64_t *idx, int64_t n_slots, double *y, int64_t Bt,
                         int64_t D, int N, int K)
{
    if (N > ORACLE_MAX_N || K > ORACLE_MAX_K) return;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < Bt; ++b) {
        for (int64_t c = 0; c < D; ++c) {
            const int64_t s = idx ? idx[b] : b;
            if (s < 0 || s >= n_slots) continue;
            double win[ORACLE_MAX_K];
            for (int j = 0; j < K - 1; ++j) win[j] = conv_state[(s * D + c) * (K - 1) + j];
            win[K - 1] = x[b * D + c];
            double acc = conv_b ? conv_b[c] : 0.0;
            for (int k = 0; k < K; ++k) acc += conv_w[c * K + k] * win[k];
            const double xcv = silu(acc);
            for (int j = 0; j < K - 1; ++j) conv_state[(s * D + c) * (K - 1) + j] = win[j + 1];

            double d = dt[b * D + c] + (dt_bias ? dt_bias[c] : 0.0);
            if (delta_softplus) d = softplus(d);
            double *h = ssm_state + (s * D + c) * N;
            double sum = 0.0;
            for (int n = 0; n < N; ++n) {
                const double dA = exp(d * A[c * N + n]);
                h[n] = dA * h[n] + d * xcv * B[b * N + n];
                sum += C[b * N + n] * h[n];
            }
            double yt = sum + (Dskip ? Dskip[c] : 0.0) * xcv;
            if (z) yt *= silu(z[b * D + c]);
            y[b * D + c] = yt;
        }
    }
}

/*
 * Round to the nearest bf16 value (8 significant bits), ties to even. The
 * value is split as m * 2^e with 0.5 <= |m| < 1; m * 2^8 is rounded to an
 * integer in the current (round-to-nearest-even) mode and scaled back. Values
 * are assumed inside bf16's normal range.
 */
static double round_bf16(double v)
{
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    const double m = frexp(v, &e);
    return ldexp(nearbyint(ldexp(m, 8)), e - 8);
}

void oracle_round_bf16(const double *in, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(in[i]);
}

/*
 * The state a replay slot stands for, written as the unrolled recurrence
 * (the product of the decays of the tokens after i is the exponential of A
 * times the sum of their deltas):
 *   h[n] = exp(A[n] * sum_{i<len} delta_i) * base[n]
 *        + sum_{i<len} exp(A[n] * sum_{i<r<len} delta_r) * delta_i * xc_i * B_i[n].
 * base: (D, N); bd, bx: (W, D) deltas and conv outputs of the buffered
 * tokens, oldest first; bB: (W, N); out: (D, N).
 */
static void replay_unroll(const double *base, const double *bd, const double *bx,
                          const double *bB, int64_t len, const double *A, int64_t D, int N,
                          int64_t c, double *out_c)
{
    for (int n = 0; n < N; ++n) {
        const double a = A[c * N + n];
        double total = 0.0;
        for (int64_t i = 0; i < len; ++i) total += bd[i * D + c];
        double h = exp(a * total) * base[c * N + n];
        for (int64_t i = 0; i < len; ++i) {
            double after = 0.0;
            for (int64_t r = i + 1; r < len; ++r) after += bd[r * D + c];
            h += exp(a * after) * bd[i * D + c] * bx[i * D + c] * bB[i * N + n];
        }
        out_c[n] = h;
    }
}

/*
 * Materialise the current state of every slot: ck (n_slots, D, N) replayed
 * over the slot's len[s] buffered tokens. bd, bx: (n_slots, W, D);
 * bB: (n_slots, W, N); h: (n_slots, D, N).
 */
void oracle_replay_state(const double *ck, const double *bd, const double *bx, const double *bB,
                         const int64_t *len, const double *A, int64_t n_slots, int W,
                         int64_t D, int N, double *h)
{
    if (N > ORACLE_MAX_N) return;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t s = 0; s < n_slots; ++s)
        for (int64_t c = 0; c < D; ++c)
            replay_unroll(ck + s * D * N, bd + s * W * D, bx + s * W * D, bB + s * W * N, len[s],
                          A, D, N, c, h + (s * D + c) * N);
}

/*
 * One replay decode token per row b, slot s = idx[b] (or b); rows with s < 0
 * or s >= n_slots are skipped (their y row, buffers and checkpoint untouched).
 * With j = len[s] tokens already buffered:
 *   conv exactly as oracle_state_update (the conv state is kept eagerly);
 *   delta = softplus(dt + dt_bias) (flag);
 *   the token's (delta, xc, B) becomes buffered token j (j + 1 tokens now);
 *   if j + 1 == W (a checkpoint step): h = replay of ck over the j + 1 tokens;
 *     ck = h, ck_lo = round_bf16(h) (if kept), len = 0;
 *   else: h = replay of ck_lo (or ck when no copy is kept) over the j + 1
 *     tokens; len = j + 1;
 *   y = (C.h + Dskip*xc) * silu(z).
 * conv_state (n_slots, D, K-1); ck, ck_lo (n_slots, D, N) (ck_lo may be NULL);
 * bd, bx (n_slots, W, D); bB (n_slots, W, N); len (n_slots); all updated in place.
 */
void oracle_replay_step(double *conv_state, double *ck, double *ck_lo, double *bd, double *bx,
                        double *bB, int64_t *len, int W, const double *x, const double *dt,
                        const double *B, const double *C, const double *z, const double *conv_w,
                        const double *conv_b, const double *A, const double *Dskip,
                        const double *dt_bias, int delta_softplus, const int64_t *idx,
                        int64_t n_slots, double *y, int64_t Bt, int64_t D, int N, int K)
{
    if (N > ORACLE_MAX_N || K > ORACLE_MAX_K || W < 1) return;
    /* rows are independent (distinct slots); each row's channels share its buffer length */
    for (int64_t b = 0; b < Bt; ++b) {
        const int64_t s = idx ? idx[b] : b;
        if (s < 0 || s >= n_slots) continue;
        const int64_t j = len[s];
        const int flush = (j + 1 == W);
        double *sbd = bd + s * W * D, *sbx = bx + s * W * D, *sbB = bB + s * W * N;
        for (int n = 0; n < N; ++n) sbB[j * N + n] = B[b * N + n];
#pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < D; ++c) {
            double win[ORACLE_MAX_K];
            for (int i = 0; i < K - 1; ++i) win[i] = conv_state[(s * D + c) * (K - 1) + i];
            win[K - 1] = x[b * D + c];
            double acc = conv_b ? conv_b[c] : 0.0;
            for (int k = 0; k < K; ++k) acc += conv_w[c * K + k] * win[k];
            const double xcv = silu(acc);
            for (int i = 0; i < K - 1; ++i) conv_state[(s * D + c) * (K - 1) + i] = win[i + 1];

            double d = dt[b * D + c] + (dt_bias ? dt_bias[c] : 0.0);
            if (delta_softplus) d = softplus(d);
            sbd[j * D + c] = d;
            sbx[j * D + c] = xcv;

            const double *base = (flush || ck_lo == NULL) ? ck : ck_lo;
            double h[ORACLE_MAX_N];
            replay_unroll(base + s * D * N, sbd, sbx, sbB, j + 1, A, D, N, c, h);
            double sum = 0.0;
            for (int n = 0; n < N; ++n) sum += C[b * N + n] * h[n];
            double yt = sum + (Dskip ? Dskip[c] : 0.0) * xcv;
            if (z) yt *= silu(z[b * D + c]);
            y[b * D + c] = yt;
            if (flush) {
                for (int n = 0; n < N; ++n) {
                    ck[(s * D + c) * N + n] = h[n];
                    if (ck_lo) ck_lo[(s * D + c) * N + n] = round_bf16(h[n]);
                }
            }
        }
        len[s] = flush ? 0 : j + 1;
    }
}

/*
 * Gradients of the selective scan (the training backward pass that PackMamba's
 * packed sequences need: "PackMamba: Efficient Processing of Variable-Length
 * Sequences in Mamba training", abstract), written from the chain rule of the
 * forward definition above, sequence by sequence, with no flow across a
 * cu_seqlens boundary. For each (sequence, channel), with v_t = dt_t + dt_bias,
 * D_t = softplus(v_t) (or v_t), a_t[n] = exp(D_t A[n]), h_t = a_t h_{t-1} +
 * D_t u_t B_t, q_t = sum_n C_t[n] h_t[n] + Dskip u_t, g_t = silu(z_t) (or 1),
 * y_t = q_t g_t, and an upstream gradient dy_t (plus dh_final for the last
 * state):
 *   dq_t = dy_t g_t;  dz_t = dy_t q_t silu'(z_t);  dDskip += dq_t u_t;
 *   G_t[n] = dq_t C_t[n] + a_{t+1}[n] G_{t+1}[n]   (G after the last token =
 *            dh_final, carried backwards; it is dL/dh_t)
 *   dC_t[n] += dq_t h_t[n];   dB_t[n] += G_t[n] D_t u_t;
 *   du_t = dq_t Dskip + sum_n G_t[n] D_t B_t[n];
 *   dD_t = sum_n G_t[n] (u_t B_t[n] + A[n] a_t[n] h_{t-1}[n]);
 *   dA[n] += G_t[n] D_t a_t[n] h_{t-1}[n];
 *   ddt_t = dD_t softplus'(v_t) (= dD_t when the softplus is off);
 *   ddt_bias += ddt_t;   dh0[n] = a_{t0}[n] G_{t0}[n] for the first token t0.
 * The forward states h_t are recomputed and kept for the whole sequence.
 * Outputs: du, ddt, dz (tok, D) (dz only with z); dB, dC (tok, N) summed over
 * channels; dA (D, N), dDskip, ddt_bias (D) summed over sequences; dh0 (S, D, N).
 * Every output array is written (overwritten), not accumulated into.
 */
void oracle_selective_scan_bwd(const double *u, const double *delta, const double *A,
                               const double *B, const double *C, const double *Dskip,
                               const double *z, const double *dt_bias, int delta_softplus,
                               const double *h0, const int64_t *cu, int64_t S, int64_t tok,
                               int64_t D, int N, const double *dy, const double *dh_final,
                               double *du, double *ddt, double *dz, double *dB, double *dC,
                               double *dA, double *dDskip, double *ddt_bias, double *dh0,
                               double *work)
{
    if (N > ORACLE_MAX_N) return;
    /* work: (tok + S) * N doubles of state history, one channel at a time */
    for (int64_t i = 0; i < tok * N; ++i) dB[i] = dC[i] = 0.0;
    for (int64_t i = 0; i < D * N; ++i) dA[i] = 0.0;
    for (int64_t c = 0; c < D; ++c) {
        if (dDskip) dDskip[c] = 0.0;
        if (ddt_bias) ddt_bias[c] = 0.0;
    }
    for (int64_t s = 0; s < S; ++s) {
        const int64_t t0 = cu[s], t1 = cu[s + 1], len = t1 - t0;
        for (int64_t c = 0; c < D; ++c) {
            /* hist[k] = h after k tokens of the sequence (hist[0] = h0) */
            double *hist = work;
            for (int n = 0; n < N; ++n) hist[n] = h0 ? h0[(s * D + c) * N + n] : 0.0;
            for (int64_t k = 0; k < len; ++k) {
                const int64_t t = t0 + k;
                double d = delta[t * D + c] + (dt_bias ? dt_bias[c] : 0.0);
                if (delta_softplus) d = softplus(d);
                for (int n = 0; n < N; ++n)
                    hist[(k + 1) * N + n] = exp(d * A[c * N + n]) * hist[k * N + n] +
                                            d * u[t * D + c] * B[t * N + n];
            }
            double G[ORACLE_MAX_N];
            for (int n = 0; n < N; ++n) G[n] = dh_final ? dh_final[(s * D + c) * N + n] : 0.0;
            for (int64_t k = len - 1; k >= 0; --k) {
                const int64_t t = t0 + k;
                const double v = delta[t * D + c] + (dt_bias ? dt_bias[c] : 0.0);
                const double d = delta_softplus ? softplus(v) : v;
                const double dsp = delta_softplus ? 1.0 / (1.0 + exp(-v)) : 1.0;
                const double ut = u[t * D + c];
                const double *h = hist + (k + 1) * N, *hp = hist + k * N;
                double q = (Dskip ? Dskip[c] : 0.0) * ut;
                for (int n = 0; n < N; ++n) q += C[t * N + n] * h[n];
                double g = 1.0, dg = 0.0;
                if (z) {
                    const double zt = z[t * D + c], sg = 1.0 / (1.0 + exp(-zt));
                    g = zt * sg;
                    dg = sg * (1.0 + zt * (1.0 - sg));
                }
                const double dq = dy[t * D + c] * g;
                if (dz) dz[t * D + c] = z ? dy[t * D + c] * q * dg : 0.0;
                if (dDskip) dDskip[c] += dq * ut;
                double dut = dq * (Dskip ? Dskip[c] : 0.0), dd = 0.0;
                for (int n = 0; n < N; ++n) {
                    const double a = exp(d * A[c * N + n]);
                    G[n] += dq * C[t * N + n];
                    dC[t * N + n] += dq * h[n];
                    dB[t * N + n] += G[n] * d * ut;
                    dut += G[n] * d * B[t * N + n];
                    dd += G[n] * (ut * B[t * N + n] + A[c * N + n] * a * hp[n]);
                    dA[c * N + n] += G[n] * d * a * hp[n];
                    G[n] *= a;
                }
                du[t * D + c] = dut;
                ddt[t * D + c] = dd * dsp;
                if (ddt_bias) ddt_bias[c] += dd * dsp;
            }
            if (dh0)
                for (int n = 0; n < N; ++n) dh0[(s * D + c) * N + n] = G[n];
        }
    }
}
