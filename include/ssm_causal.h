/*
 * ssm_causal.h -- C ABI of the B200 (sm_100a) selective-SSM mixer core.
 *
 * Three operations, each one asynchronous call on a caller-given stream:
 *
 *   ssm_causal_conv1d           causal depthwise conv1d + bias + SiLU over packed
 *                               sequences, with carried conv state in and out
 *   ssm_selective_scan_fwd      selective scan (dA = exp(delta*A),
 *                               h_t = dA*h_{t-1} + delta*u_t*B_t,
 *                               y_t = (C_t.h_t + Dskip*u_t) * silu(z_t)) over packed
 *                               sequences, with optional h0 and final-state output
 *   ssm_selective_state_update  one decode token per row: conv-state shift, conv,
 *                               softplus, state update in place, readout and gate
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller. The library
 *   never allocates, frees or retains memory, and never synchronises the host.
 * - Layouts are row-major and token-major with channels contiguous:
 *   activations (tok, D); B and C (tok, N), one group shared by all channels;
 *   A (D, N); conv weight (D, K); Dskip, dt_bias, conv bias (D);
 *   SSM state (S, D, N) fp32; conv state (S, D, K-1), oldest entry first.
 * - Packed variable-length sequences are described by cu_seqlens, S+1 int32
 *   offsets on the device: sequence s owns tokens [cu[s], cu[s+1]). It must be
 *   non-decreasing with cu[0] = 0 and cu[S] = tok (ssm_check_cu_seqlens checks
 *   a host copy). Nothing flows across a boundary: each sequence starts from
 *   its own initial state. Kernels clamp every offset into [0, tok], so a bad
 *   array gives wrong values but never an out-of-bounds access. Sequences may
 *   be empty. cu_seqlens == NULL means a dense batch of S rows of tok/S tokens.
 * - Floating-point work is fp32 throughout (fp32 state, fp32 accumulation);
 *   bf16 tensors are converted on load and rounded to nearest even on store.
 * - Results are deterministic: no atomics take part in the arithmetic, except
 *   in the channel- and sequence-sums of ssm_selective_scan_bwd (see there).
 * - Every call returns SSM_OK (0) or a negative status and then launches
 *   nothing; ssm_last_error() gives a message for the calling thread.
 *
 * Sources (titles of the pages this follows):
 * - tp_builder.py (TensorRT-Model-Connect, Mamba family), _add_mamba_tp_layer:
 *   the per-token mixer math (conv-state shift, depthwise conv, softplus of dt,
 *   discretisation dA = exp(delta*A) and dB = delta*B, state update, C readout,
 *   D skip, silu(z) gate) and the present_conv / present_ssm state outputs.
 * - "Scaling State-Space Models on Multiple GPUs with Tensor Parallelism"
 *   (Dutt, Shah, Masarani, Gandhi): Fig. 1 (mixer dataflow) and the abstract
 *   (SSM state cache carried across prefill and decode).
 * - "PackMamba: Efficient Processing of Variable-Length Sequences in Mamba
 *   training", abstract: packed sequences with no information passed between
 *   sequences.
 * - The backward pass of the selective scan (ssm_selective_scan_bwd) is the
 *   chain rule of the forward above, for training on packed sequences
 *   (PackMamba abstract).
 * - "ReplaySSM: Cache SSM Inputs, Not State", abstract: decode with the state
 *   kept as a checkpoint plus the SSM inputs of recent tokens
 *   (ssm_replay_state_update, ssm_replay_reset, ssm_replay_flush).
 */
#ifndef SSM_CAUSAL_H
#define SSM_CAUSAL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *ssm_stream_t;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARGUMENT = -1, /* null required pointer, bad size, unsupported N or K */
    SSM_ERR_UNSUPPORTED_DTYPE = -2,
    SSM_ERR_MISALIGNED = -3,       /* a pointer is not aligned to its element size */
    SSM_ERR_BAD_SEQLENS = -4,      /* cu_seqlens rejected (host check) */
    SSM_ERR_WORKSPACE = -5,        /* workspace given but too small */
    SSM_ERR_CUDA = -6              /* a CUDA launch or runtime call failed */
};

/* Message describing the last failing call on this host thread ("" if none). */
const char *ssm_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int ssm_version(void);

/* Number of kernels this library has launched in this process (all calls,
 * all threads). Lets a caller count launches inside a timed region. */
unsigned long long ssm_launch_count(void);

/*
 * Tuning knob for ssm_selective_scan_fwd's kernel variant: states of one
 * channel per lane (2, 4, 8 or 16; 16 / value lanes then share a channel) and
 * the schedule (1: next chunk prefetched into registers; 2: tiles staged by
 * TMA; 3: TMA staging with each chunk split in time over four warps, which
 * combine their segments through a carry step, only 2 or 4 states per lane;
 * 4 and 5: one-warp CTAs with 32- and 64-token chunks; 6: warp-specialised,
 * helper warps run the per-token work beside the recurrence warps;
 * 7: one-warp CTAs that each own their channels and stage their own tiles,
 * 4, 8 or 16 states per lane; 8: the layout of schedule 1 with TMA staging;
 * 9 and 10: the chunk-pipelined kernel, TMA staging four stages deep, the next
 * chunk's per-token work interleaved with this chunk's recurrence, 16- and
 * 32-token chunks, 2, 4 or 8 states per lane; 11: schedule 10 at 4 states
 * per lane with the register budget of two CTAs per SM; 12: one lane per
 * channel with all 16 states, 128-lane CTAs, TMA staging, no shuffles, for
 * shapes with many (sequence, channel) pairs; it takes any states_per_lane
 * value and reports 16; the library's choice).
 * 0 lets the library choose. Applies to the
 * 16-byte vector path; the scalar path always uses 4 states per lane and
 * register prefetch. A variant whose alignment needs the inputs do not meet
 * falls back to schedule 2, then 1. Process-wide; not thread-safe against
 * concurrent scan calls.
 * Returns SSM_OK or SSM_ERR_INVALID_ARGUMENT. Results differ between variants
 * only in the order of the readout sum.
 */
int ssm_set_scan_variant(int states_per_lane, int schedule);

/*
 * Reports the kernel variant ssm_selective_scan_fwd picks on its 16-byte
 * vector path for S sequences of D channels on the current device: states
 * per lane and schedule, as ssm_set_scan_variant names them (a forced
 * variant is reported as forced). A variant whose alignment needs the
 * inputs do not meet still falls back at call time. Host-only; launches
 * nothing. The writes to *states_per_lane and *schedule are the only
 * effects. Returns SSM_OK, or SSM_ERR_INVALID_ARGUMENT for S < 1, D < 1 or
 * a NULL pointer. An introspection call of this library; the method has no
 * counterpart.
 */
int ssm_scan_variant_for(int64_t S, int64_t D, int *states_per_lane, int *schedule);

/*
 * Device-side status of the library's kernels on the current device: 0 while
 * every bounded wait for a TMA tile or bulk copy completed; bit 0 set once a
 * scan kernel's wait gave up, bit 1 once a conv kernel's did, bit 2 once a
 * decode kernel's did, bit 3 once a replay decode kernel's did (the results
 * of that call are then unspecified; the kernel still terminates), bit 4 once
 * ssm_selftest_wait_timeout's wait gave up. Synchronises the device.
 * clear != 0 resets the flags. Returns SSM_ERR_CUDA if the query itself fails.
 */
int ssm_device_status(int clear);

/*
 * Self-test of the bounded device waits (failure detection; the pages have no
 * counterpart). Every kernel that waits for a TMA tile or bulk copy waits on an
 * mbarrier with a bounded number of suspending tries (2^17, about half a
 * second at most) and, when they run out, sets its status bit and returns
 * instead of hanging. This call launches one small kernel whose barrier
 * expects 16 bytes that no copy delivers, with the limit lowered to `tries`
 * (1..131072): its wait runs out, it sets bit 4 of ssm_device_status and
 * returns with nothing in flight, and the context stays usable. Asynchronous on
 * `stream`. Returns SSM_OK, SSM_ERR_INVALID_ARGUMENT or SSM_ERR_CUDA.
 */
int ssm_selftest_wait_timeout(int tries, ssm_stream_t stream);

/*
 * Checks a HOST copy of cu_seqlens (S+1 entries): cu[0] == 0, non-decreasing,
 * cu[S] == tok. Returns SSM_OK or SSM_ERR_BAD_SEQLENS. Touches no device.
 */
int ssm_check_cu_seqlens(const int32_t *cu_seqlens_host, int64_t S, int64_t tok);

/*
 * Causal depthwise conv1d (+ bias, + SiLU) over packed sequences.
 * Follows tp_builder.py, _add_mamba_tp_layer (conv-state shift and conv step):
 *   xc[t,c] = act(bias[c] + sum_{k<K} w[c,k] * win_t[c,k])
 * where win_t holds the K-1 inputs of the same sequence before t (the carried
 * conv state, or zeros, before the sequence's first token) and then x[t,c];
 * the newest input pairs with w[c,K-1]. act is SiLU when apply_silu != 0.
 *
 *   x              (tok, D) of x_dtype; read only
 *   xc             (tok, D) of x_dtype; written; must not overlap x
 *   weight         (D, K) fp32;  bias: (D) fp32 or NULL (= 0)
 *   tok, D         tokens in the call (>= 0) and channels (>= 1)
 *   K              conv width, 2..4
 *   cu_seqlens, S  see the conventions above (S >= 1)
 *   conv_state_in  (S, D, K-1) of state_dtype or NULL (= zeros)
 *   conv_state_out (S, D, K-1) of state_dtype or NULL (= not written): the last
 *                  K-1 entries of [conv_state_in || x_seq] per sequence, so a
 *                  sequence shorter than K-1 keeps part of its carried state.
 *                  May be the same buffer as conv_state_in.
 * Launches 1 kernel, or 2 when conv_state_out is given.
 */
int ssm_causal_conv1d(const void *x, void *xc, const float *weight, const float *bias,
                      int64_t tok, int64_t D, int K, const int32_t *cu_seqlens, int64_t S,
                      const void *conv_state_in, void *conv_state_out, int apply_silu,
                      ssm_dtype x_dtype, ssm_dtype state_dtype, ssm_stream_t stream);

/*
 * Bytes of optional scratch for ssm_selective_scan_fwd with S packed
 * sequences (a longest-first schedule of the sequences). Passing a NULL
 * workspace is always allowed: sequences are then scheduled in index order,
 * except by schedule 12, whose CTAs rank up to 128 sequences by length
 * themselves.
 */
size_t ssm_scan_workspace_size(int64_t tok, int64_t D, int N, int64_t S);

/*
 * Selective scan over packed sequences.
 * Follows tp_builder.py, _add_mamba_tp_layer (dt softplus, dA = exp(delta*A),
 * dBx = delta*B*u, h = dA*h + dBx, y = C.h + D*u, times silu(z)), run over each
 * sequence in order as Fig. 1 of "Scaling State-Space Models on Multiple GPUs
 * with Tensor Parallelism" describes, resetting at every cu_seqlens boundary
 * ("PackMamba", abstract).
 *
 *   u              (tok, D) act_dtype: the conv output xc
 *   delta          (tok, D) act_dtype: raw dt (delta_softplus != 0) or delta
 *   A              (D, N) fp32 (negative reals for a decaying state)
 *   B, C           (tok, N) act_dtype
 *   Dskip          (D) fp32 or NULL (= 0)
 *   z              (tok, D) act_dtype or NULL (= no gate)
 *   dt_bias        (D) fp32 or NULL (= 0), added before the softplus
 *   delta_softplus 1: delta = softplus(dt + dt_bias); 0: delta = dt + dt_bias
 *   h0             (S, D, N) fp32 or NULL (= zeros)
 *   cu_seqlens, S  see the conventions above
 *   y              (tok, D) act_dtype, written; tokens outside every sequence
 *                  are left untouched
 *   h_final        (S, D, N) fp32 or NULL; may be the same buffer as h0
 *   tok, D, N      N must be 16
 *   workspace      NULL or >= ssm_scan_workspace_size() bytes of device
 *                  scratch, 256-byte aligned; its contents are overwritten
 * y must not overlap u, delta, z, B or C.
 */
int ssm_selective_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                           const void *C, const float *Dskip, const void *z,
                           const float *dt_bias, int delta_softplus, const float *h0,
                           const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                           int64_t tok, int64_t D, int N, ssm_dtype act_dtype, void *workspace,
                           size_t workspace_bytes, ssm_stream_t stream);

/*
 * One decode token per row, updating the cached states in place.
 * Follows the whole of tp_builder.py, _add_mamba_tp_layer for one token (its
 * conv_state / ssm_state inputs and present_conv / present_ssm outputs) and
 * the SSM cache of "Scaling State-Space Models...", abstract and Fig. 2 (1).
 * For row b with slot s = state_indices[b] (or b when state_indices is NULL):
 *   win = [conv_state[s] || x[b]]; xc = silu(conv_b + sum_k conv_w[:,k]*win[k]);
 *   conv_state[s] = last K-1 of win; delta = softplus(dt[b] + dt_bias) (flag);
 *   ssm_state[s] = exp(delta*A)*ssm_state[s] + delta*xc*B[b];
 *   y[b] = (C[b].ssm_state[s] + Dskip*xc) * silu(z[b]).
 *
 *   conv_state     (n_slots, D, K-1) of conv_state_dtype, updated in place
 *   ssm_state      (n_slots, D, N) fp32, updated in place
 *   x, dt, z       (Bt, D) act_dtype (z may be NULL = no gate)
 *   B, C           (Bt, N) act_dtype
 *   conv_w (D, K), conv_b (D) or NULL, A (D, N), Dskip (D) or NULL,
 *   dt_bias (D) or NULL: fp32
 *   state_indices  (Bt) int32 or NULL (= identity, needs n_slots >= Bt). A row
 *                  with index -1 (any negative) is skipped and its y row is
 *                  left untouched; an index >= n_slots is skipped as well.
 *                  Two rows naming the same slot race (undefined result).
 *   y              (Bt, D) act_dtype
 *   N must be 16; K in 2..4. ssm_state, A, B, C and (for K = 4) conv_w must be
 *   16-byte aligned, else SSM_ERR_MISALIGNED.
 */
int ssm_selective_state_update(void *conv_state, float *ssm_state, const void *x,
                               const void *dt, const void *B, const void *C, const void *z,
                               const float *conv_w, const float *conv_b, const float *A,
                               const float *Dskip, const float *dt_bias, int delta_softplus,
                               const int32_t *state_indices, int64_t n_slots, void *y,
                               int64_t Bt, int64_t D, int N, int K, ssm_dtype act_dtype,
                               ssm_dtype conv_state_dtype, ssm_stream_t stream);

/*
 * Causal depthwise conv1d + SiLU fused into the selective scan: the result of
 * ssm_causal_conv1d (apply_silu = 1) feeding ssm_selective_scan_fwd as u, in
 * one kernel that never writes the conv output to memory (it stays in fp32,
 * where the two-call path stores it in act_dtype between the calls). Follows
 * the mixer dataflow of "Scaling State-Space Models on Multiple GPUs with
 * Tensor Parallelism", Fig. 1 (conv, then the state update), with the math of
 * tp_builder.py, _add_mamba_tp_layer, over packed sequences (PackMamba,
 * abstract).
 *
 *   x, conv_w, conv_b, conv_state_in, conv_state_out, K, conv_state_dtype:
 *                  as ssm_causal_conv1d (conv_state_out may be conv_state_in)
 *   xc             (tok, D) act_dtype or NULL: if given, the conv output is also
 *                  written there (rounded to act_dtype)
 *   delta, A, B, C, Dskip, z, dt_bias, delta_softplus, h0, cu_seqlens, S, y,
 *   h_final, tok, D, N, act_dtype: as ssm_selective_scan_fwd (u is the conv
 *                  output); y must not overlap x, delta or z
 * Always one kernel. Where ssm_scan_variant_for reports schedule 12 (many
 * sequence-channel pairs) and every row is 16-byte aligned: one lane per
 * channel with the conv window in the lane's registers, sequences longest
 * first when S <= 128 (each CTA ranks the lengths itself; no workspace),
 * else in index order. Otherwise the scan's register-prefetch layout (4 or 8
 * states per lane as ssm_scan_variant_for reports it, 4 when rows are not
 * 16-byte aligned), sequences in index order. The conv output takes the conv
 * kernel's operations in its order, so an xc copy equals ssm_causal_conv1d's
 * output bit for bit. Where the scan alone would pick a TMA schedule the
 * two-call path can be as fast or faster.
 */
int ssm_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_b,
                      const void *conv_state_in, void *conv_state_out, void *xc, int K,
                      ssm_dtype conv_state_dtype, const void *delta, const float *A,
                      const void *B, const void *C, const float *Dskip, const void *z,
                      const float *dt_bias, int delta_softplus, const float *h0,
                      const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                      int64_t tok, int64_t D, int N, ssm_dtype act_dtype, ssm_stream_t stream);

/*
 * Workspace bytes ssm_selective_scan_bwd needs for `tok` packed tokens of D
 * channels in S sequences (N must be 16; 0 for invalid sizes): room for one
 * fp32 state checkpoint per 8 tokens of each sequence and channel (about 8
 * bytes per token and channel) and the sequences' longest-first order.
 */
size_t ssm_scan_bwd_workspace_size(int64_t tok, int64_t D, int N, int64_t S);

/*
 * Tuning knob for ssm_selective_scan_bwd's kernel: 1 splits each channel's
 * 16 states over 4 lanes (16-token chunks, per-token sums over states and
 * channels by shuffles); 2 runs a checkpointing forward pass (two lanes per
 * channel), then a reverse pass that gives each channel one thread with all 16
 * states (8-token chunks whose states are summed over channels from shared
 * memory; about half of variant 1's instructions per token and channel, a
 * quarter of its threads); 0 lets the library choose (2 once
 * S * ceil(D / 128) reaches twice the SM count, else 1). Process-wide; not
 * thread-safe against concurrent backward calls. Returns SSM_OK or
 * SSM_ERR_INVALID_ARGUMENT. The variants differ only in the order of their
 * floating-point sums.
 */
int ssm_set_scan_bwd_variant(int variant);

/*
 * The kernel (1 or 2, as ssm_set_scan_bwd_variant names them) that
 * ssm_selective_scan_bwd uses for S sequences of D channels on the current
 * device, written to *variant. Host-only; launches nothing. Returns SSM_OK,
 * or SSM_ERR_INVALID_ARGUMENT for S < 1, D < 1 or a NULL pointer.
 */
int ssm_scan_bwd_variant_for(int64_t S, int64_t D, int *variant);

/*
 * Backward of ssm_selective_scan_fwd: gradients of the loss L through
 * sum(dy * y) + sum(dh_final * h_final) with respect to every input, for
 * training on packed sequences ("PackMamba: Efficient Processing of
 * Variable-Length Sequences in Mamba training", abstract: no information
 * passes between sequences, forwards or backwards). The forward is the one
 * of ssm_selective_scan_fwd (tp_builder.py, _add_mamba_tp_layer); with
 * G_t = dL/dh_t = dy_t silu(z_t) C_t + exp(delta_{t+1} A) G_{t+1}:
 *   du_t = dy_t silu(z_t) Dskip + delta_t (G_t . B_t)
 *   ddelta_t = [G_t . (u_t B_t + A exp(delta_t A) h_{t-1})] softplus'(dt_t + dt_bias)
 *   dz_t = dy_t (C_t . h_t + Dskip u_t) silu'(z_t)
 *   dB_t = sum_c delta_t u_t G_t,  dC_t = sum_c dy_t silu(z_t) h_t
 *   dA = sum_t G_t delta_t exp(delta_t A) h_{t-1},  dDskip = sum_t dy_t silu(z_t) u_t
 *   ddt_bias = sum_t ddelta_t,  dh0 = exp(delta_{t0} A) G_{t0} (first token t0)
 * (softplus' = 1 and no bias when delta_softplus = 0; silu(z) = 1 and
 * silu' = 0 without z). The forward states are recomputed, not stored.
 *
 *   u, delta, B, C, Dskip, z, dt_bias, delta_softplus, h0, cu_seqlens, S,
 *   tok, D, N, act_dtype: exactly the forward call's arguments
 *   dy             (tok, D) act_dtype: gradient of y
 *   dh_final       (S, D, N) fp32 or NULL (= 0): gradient of h_final
 *   du, ddelta     (tok, D) act_dtype, written; ddelta is the gradient of the
 *                  raw `delta` input (before dt_bias and the softplus)
 *   dz             (tok, D) act_dtype or NULL; written (zeros when z is NULL)
 *   dB, dC         (tok, N) fp32, written (summed over channels)
 *   dA             (D, N) fp32, written (summed over sequences and tokens)
 *   dDskip, ddt_bias (D) fp32 or NULL, written
 *   dh0            (S, D, N) fp32 or NULL, written
 *   workspace      >= ssm_scan_bwd_workspace_size() bytes, 256-byte aligned;
 *                  required; its contents are overwritten
 * dB, dC, dA, dDskip and ddt_bias are sums over CTAs taken with fp32 atomics,
 * so their last bits may differ from run to run; every other output is
 * deterministic. Outputs must not overlap the inputs.
 */
int ssm_selective_scan_bwd(const void *u, const void *delta, const float *A, const void *B,
                           const void *C, const float *Dskip, const void *z,
                           const float *dt_bias, int delta_softplus, const float *h0,
                           const int32_t *cu_seqlens, int64_t S, const void *dy,
                           const float *dh_final, void *du, void *ddelta, void *dz, float *dB,
                           float *dC, float *dA, float *dDskip, float *ddt_bias, float *dh0,
                           int64_t tok, int64_t D, int N, ssm_dtype act_dtype, void *workspace,
                           size_t workspace_bytes, ssm_stream_t stream);

/*
 * Training pair: a forward scan that leaves the backward pass its state
 * checkpoints, and the backward pass that reads them instead of running its
 * own checkpointing forward pass (for a training step's forward, whose inputs
 * the backward sees again).
 *
 * ssm_selective_scan_fwd_ckpt computes exactly what ssm_selective_scan_fwd
 * computes (y and h_final bit for bit, same arguments) and also writes, into
 * bwd_workspace, the fp32 state of every sequence and channel before each
 * 8th token of the sequence (before tokens 0, 8, 16, ...; about 8 bytes per
 * token and channel). The pipelined kernels (schedules 9 to 12) write them as
 * they go; with any other kernel the library adds a checkpointing pass after
 * the scan.
 *   bwd_workspace  >= ssm_scan_bwd_workspace_size(tok, D, N, S) bytes,
 *                  256-byte aligned, required, owned by the caller; must not
 *                  overlap `workspace`
 * Errors: those of ssm_selective_scan_fwd; SSM_ERR_WORKSPACE when
 * bwd_workspace is NULL or too small; SSM_ERR_MISALIGNED when it is not
 * 256-byte aligned; SSM_ERR_INVALID_ARGUMENT when the workspaces overlap.
 *
 * ssm_selective_scan_bwd_ckpt takes ssm_selective_scan_bwd's arguments, with
 * `workspace` the bwd_workspace that ssm_selective_scan_fwd_ckpt filled for
 * the same u, delta, A, B, dt_bias, delta_softplus, h0, cu_seqlens and sizes
 * (on the same stream, or ordered after it), unchanged since. Gradients as
 * ssm_selective_scan_bwd's, except that the states come from the forward's
 * own arithmetic, so results differ from it in the last bits. Checkpoints that
 * do not match the inputs give wrong gradients; nothing checks them.
 */
int ssm_selective_scan_fwd_ckpt(const void *u, const void *delta, const float *A, const void *B,
                                const void *C, const float *Dskip, const void *z,
                                const float *dt_bias, int delta_softplus, const float *h0,
                                const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                                int64_t tok, int64_t D, int N, ssm_dtype act_dtype,
                                void *workspace, size_t workspace_bytes, void *bwd_workspace,
                                size_t bwd_workspace_bytes, ssm_stream_t stream);

int ssm_selective_scan_bwd_ckpt(const void *u, const void *delta, const float *A, const void *B,
                                const void *C, const float *Dskip, const void *z,
                                const float *dt_bias, int delta_softplus, const float *h0,
                                const int32_t *cu_seqlens, int64_t S, const void *dy,
                                const float *dh_final, void *du, void *ddelta, void *dz,
                                float *dB, float *dC, float *dA, float *dDskip, float *ddt_bias,
                                float *dh0, int64_t tok, int64_t D, int N, ssm_dtype act_dtype,
                                void *workspace, size_t workspace_bytes, ssm_stream_t stream);

/*
 * Replay decode: one token per row, with each slot's SSM state kept as a
 * checkpoint plus the SSM inputs of the tokens since it.
 * Follows "ReplaySSM: Cache SSM Inputs, Not State" (abstract): the recurrence
 * is unrolled so that outputs are computed by replaying the buffered inputs
 * from the checkpoint, the checkpoint is rewritten only once every W tokens,
 * and a low-precision copy of the checkpoint serves the outputs of the other
 * steps while the fp32 checkpoint alone feeds the recurrent update. The
 * per-token math is that of ssm_selective_state_update (tp_builder.py,
 * _add_mamba_tp_layer), computed with the same operations in the same order.
 *
 * For row b with slot s = state_indices[b] (or b) and j = buf_len[s] tokens
 * buffered:
 *   conv, conv-state shift, delta exactly as ssm_selective_state_update;
 *   if j + 1 == W (a checkpoint step): h = ckpt[s] replayed over the j
 *     buffered tokens and this one; ckpt[s] = h; ckpt_lo[s] = bf16(h);
 *     buf_len[s] = 0;
 *   else: h = ckpt_lo[s] (or ckpt[s] when ckpt_lo is NULL) replayed over the
 *     j buffered tokens and this one; this token's (delta, delta*xc) becomes
 *     buffer entry j and its B entry j; buf_len[s] = j + 1;
 *   y[b] = (C[b].h + Dskip*xc) * silu(z[b]).
 * Replaying a token is h = exp(delta*A)*h + (delta*xc)*B with that token's
 * values. After a checkpoint step ckpt[s] holds bit-for-bit the state that
 * ssm_selective_state_update would hold after the same tokens.
 *
 *   conv_state     (n_slots, D, K-1) of conv_state_dtype, updated in place
 *   ckpt           (n_slots, D, N) fp32 checkpoint, rewritten on checkpoint steps
 *   ckpt_lo        (n_slots, D, N) bf16 copy of ckpt, or NULL (outputs then read
 *                  ckpt on every step)
 *   buf            (n_slots, W-1, D, 2) fp32: (delta, delta*xc) of buffered
 *                  tokens, oldest first; NULL allowed when W == 1
 *   buf_B          (n_slots, W-1, N) fp32: B of buffered tokens; NULL when W == 1
 *   buf_len        (n_slots) int32: tokens buffered per slot, 0..W-1 (a value
 *                  outside is clamped into that range)
 *   tickets        (n_slots) uint32 scratch: all zero before the first call
 *                  (ssm_replay_reset zeroes them); every call leaves them zero.
 *                  The channel blocks of a row count themselves here, and the
 *                  last one advances buf_len.
 *   W              checkpoint interval, 1..8 (W == 1 is eager decode plus the
 *                  bf16 copy)
 *   x, dt, z, B, C, conv_w, conv_b, A, Dskip, dt_bias, delta_softplus,
 *   state_indices, n_slots, y, Bt, D, N, K, dtypes: as ssm_selective_state_update
 * All of conv_state, ckpt, ckpt_lo, buf, buf_B, x, dt, z, B, C and A must be
 * 16-byte aligned and D * element size of x (and D * (K-1) * element size of
 * the conv state) a multiple of 16 bytes, else SSM_ERR_MISALIGNED. Two rows
 * naming the same slot race (undefined result). Before the first step of a
 * window, ckpt must hold the state and ssm_replay_reset must have run.
 */
int ssm_replay_state_update(void *conv_state, float *ckpt, void *ckpt_lo, float *buf,
                            float *buf_B, int32_t *buf_len, uint32_t *tickets, int W,
                            const void *x, const void *dt, const void *B, const void *C,
                            const void *z, const float *conv_w, const float *conv_b,
                            const float *A, const float *Dskip, const float *dt_bias,
                            int delta_softplus, const int32_t *state_indices, int64_t n_slots,
                            void *y, int64_t Bt, int64_t D, int N, int K, ssm_dtype act_dtype,
                            ssm_dtype conv_state_dtype, ssm_stream_t stream);

/*
 * Starts the replay window of each listed slot at the state held in ckpt
 * (for example a prefill's final state): ckpt_lo[s] = bf16(ckpt[s]) when
 * ckpt_lo is not NULL, buf_len[s] = 0, tickets[s] = 0.
 * ("ReplaySSM: Cache SSM Inputs, Not State", abstract: checkpoint plus input
 * buffer.)
 *   slots  (n) int32 slot numbers, or NULL for slots 0..n-1; entries outside
 *          [0, n_slots) are skipped
 *   ckpt (n_slots, D, N) fp32; ckpt_lo (n_slots, D, N) bf16 or NULL; both
 *   16-byte aligned. N must be 16.
 */
int ssm_replay_reset(const float *ckpt, void *ckpt_lo, int32_t *buf_len, uint32_t *tickets,
                     const int32_t *slots, int64_t n, int64_t n_slots, int64_t D, int N,
                     ssm_stream_t stream);

/*
 * Replays every buffered token of each listed slot into its fp32 checkpoint,
 * refreshes the bf16 copy and empties the buffer (buf_len[s] = 0), with the
 * arithmetic of a checkpoint step. Afterwards ckpt[s] is the slot's current
 * state, as ssm_selective_state_update would hold it; use it to hand a slot
 * back to eager decode or to read its state. Two launches (the lengths are
 * cleared after every channel has read them).
 *   Arguments as ssm_replay_state_update and ssm_replay_reset.
 */
int ssm_replay_flush(float *ckpt, void *ckpt_lo, const float *buf, const float *buf_B,
                     int32_t *buf_len, uint32_t *tickets, const float *A, int W,
                     const int32_t *slots, int64_t n, int64_t n_slots, int64_t D, int N,
                     ssm_stream_t stream);

/*
 * ssm_selective_scan_fwd without a workspace, for callers that cannot
 * allocate device memory when they call it: an inference engine that reserves
 * all of its device memory at start-up and forbids allocation afterwards, or a
 * plugin whose host framework owns the device allocator and hands it no
 * scratch. Not part of the method the pages describe (the paper has no
 * counterpart); it is a packaging of the same scan.
 *
 * Arguments, results and errors are those of ssm_selective_scan_fwd. The
 * longest-first schedule of packed sequences lives in a fixed 16 KB array
 * inside the library instead of a workspace, so a packed call (cu_seqlens
 * given) may name at most 4096 sequences; larger S with cu_seqlens is
 * rejected with SSM_ERR_INVALID_ARGUMENT before anything is launched. Dense
 * calls (cu_seqlens NULL) and single sequences need no schedule and accept any
 * S. The library allocates nothing for this call: every GPU that loads the
 * library holds the array until the process exits. The first packed call on a
 * device looks the array's address up (with that device current) and caches
 * it for the life of the process; make that first call before any stream
 * capture, and do not use this entry point on a device after a
 * cudaDeviceReset (or any other teardown of its primary context) in the same
 * process, since the cached address would then be stale. All calls on a
 * device share the one array and
 * each overwrites it completely before reading it, so nothing needs clearing,
 * but two such calls that run at the same time on one GPU (different streams
 * without ordering between them) race on it and give unspecified results.
 */
int ssm_selective_scan_fwd_noalloc(const void *u, const void *delta, const float *A,
                                   const void *B, const void *C, const float *Dskip,
                                   const void *z, const float *dt_bias, int delta_softplus,
                                   const float *h0, const int32_t *cu_seqlens, int64_t S,
                                   void *y, float *h_final, int64_t tok, int64_t D, int N,
                                   ssm_dtype act_dtype, ssm_stream_t stream);

/*
 * Measurement helpers (not part of the method; the pages have no counterpart).
 * The selective scan's roofline is set by the special-function unit (one ex2
 * per state and token), so its denominator is measured on the device at hand
 * instead of derived from unit counts.
 *
 * ssm_probe_rate launches one throughput probe over every SM (warps_per_sm / 8
 * CTAs of 256 threads on each SM, 8 independent dependency chains per thread;
 * warps_per_sm is 8, 16, ..., 64, and 64 gives the peak) and writes the
 * operations it performs to *ops; time the launch with CUDA events on
 * `stream` and divide. kind: 0 ex2.approx.ftz.f32 (special-function unit;
 * ops = ex2 results), 1 packed fp32x2 FMA (ops = fp32 FMAs, two per
 * instruction), 2 scalar fp32 FMA, 3 the scan recurrence's mix of one ex2 per
 * two packed FMA-pipe operations (ops = ex2 results). `iters` loop steps per
 * thread set the run time (each step is 8 operations per thread, 16 FMAs for
 * kind 1). sink: device fp32 buffer of at least ssm_probe_sink_floats()
 * entries, overwritten with one value per thread. Returns SSM_OK,
 * SSM_ERR_INVALID_ARGUMENT, SSM_ERR_MISALIGNED or SSM_ERR_CUDA.
 */
int64_t ssm_probe_sink_floats(void);
int ssm_probe_rate(int kind, int iters, int warps_per_sm, float *sink, int64_t sink_floats,
                   double *ops, ssm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSM_CAUSAL_H */
