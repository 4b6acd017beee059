// api.cu -- the extern "C" boundary: argument validation, dispatch, errors.
//
// Every entry point validates its arguments on the host before touching the
// device (the tensor-parallel builder this library follows rejects bad shapes
// up front as well: tp_builder.py, _validate_mamba_tp), then launches its
// kernels asynchronously on the caller's stream. Failures return a negative
// status and leave a message in a thread-local buffer.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/ssm_causal.h"
#include "internal.h"

namespace ssm {
void set_scan_variant(int npt, int sched);
void scan_variant_for(int64_t S, int64_t D, int *npt, int *sched);
size_t scan_order_bytes(int64_t S);
int read_scan_status(bool clear);
int read_conv_status(bool clear);
int read_decode_status(bool clear);
cudaError_t noalloc_scratch(void **ptr, size_t *bytes);
int64_t noalloc_max_sequences();
int read_replay_status(bool clear);
int probe_sink_floats();
int read_selftest_status(bool clear);
cudaError_t launch_wait_selftest(unsigned tries, cudaStream_t stream, int *launches);
cudaError_t launch_probe(int kind, int iters, int per_sm, float *sink, double *ops,
                         cudaStream_t stream, int *launches);

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
size_t scan_bwd_workspace_bytes(int64_t tok, int64_t D, int64_t S);
cudaError_t launch_scan_bwd_ckpt_pass(const ScanBwdArgs &a, cudaStream_t stream, int *launches);
void set_scan_bwd_variant(int v);
int scan_bwd_variant_for(int64_t S, int64_t D);

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
cudaError_t launch_conv_scan(const ConvScanArgs &a, int npt, int sched, cudaStream_t stream,
                             int *launches);
int read_conv_scan_status(bool clear);
cudaError_t launch_scan_bwd(const ScanBwdArgs &a, cudaStream_t stream, int *launches);

struct ReplayStepArgs {
    void *conv_state;
    float *ckpt;
    void *ckpt_lo;
    float *buf, *bufB;
    int32_t *len;
    uint32_t *tickets;
    int W;
    const void *x, *dt, *B, *C, *z;
    const float *conv_w, *conv_b, *A, *Dskip, *dt_bias;
    int delta_softplus;
    const int32_t *idx;
    int64_t n_slots;
    void *y;
    int64_t Bt, D;
    int K;
    bool act_bf16, conv_bf16;
};
cudaError_t launch_replay_step(const ReplayStepArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_replay_reset(const float *ckpt, void *ckpt_lo, int32_t *len, uint32_t *tickets,
                                const int32_t *slots, int64_t n, int64_t n_slots, int64_t D,
                                cudaStream_t stream, int *launches);
cudaError_t launch_replay_flush(float *ckpt, void *ckpt_lo, const float *buf, const float *bufB,
                                int32_t *len, uint32_t *tickets, const float *A, int W,
                                const int32_t *slots, int64_t n, int64_t n_slots, int64_t D,
                                cudaStream_t stream, int *launches);
}  // namespace ssm

namespace {

thread_local std::string g_error;
std::atomic<unsigned long long> g_launches{0};

int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_error = buf;
    return code;
}

int ok()
{
    g_error.clear();
    return SSM_OK;
}

size_t esize(ssm_dtype t) { return t == SSM_BF16 ? 2 : 4; }

bool valid_dtype(ssm_dtype t) { return t == SSM_F32 || t == SSM_BF16; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ssm::DType dt(ssm_dtype t) { return t == SSM_BF16 ? ssm::DType::BF16 : ssm::DType::F32; }

int finish(cudaError_t e, int launched, const char *what)
{
    g_launches.fetch_add((unsigned long long)launched, std::memory_order_relaxed);
    if (e != cudaSuccess)
        return fail(SSM_ERR_CUDA, "%s: CUDA error %d (%s)", what, (int)e, cudaGetErrorString(e));
    return ok();
}

// Common checks of the packed-sequence description.
int check_seqs(const char *fn, const int32_t *cu, int64_t S, int64_t tok)
{
    if (S < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: S must be >= 1 (got %lld)", fn, (long long)S);
    if (S > 65535)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: at most 65535 sequences per call (got %lld)", fn,
                    (long long)S);
    if (tok < 0 || tok > (int64_t)INT32_MAX)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: tok out of range (%lld)", fn, (long long)tok);
    if (!cu && tok % S != 0)
        return fail(SSM_ERR_INVALID_ARGUMENT,
                    "%s: without cu_seqlens, tok (%lld) must be a multiple of S (%lld)", fn,
                    (long long)tok, (long long)S);
    if (cu && !aligned(cu, 4)) return fail(SSM_ERR_MISALIGNED, "%s: cu_seqlens misaligned", fn);
    return SSM_OK;
}

}  // namespace

extern "C" {

const char *ssm_last_error(void) { return g_error.c_str(); }

int ssm_version(void) { return 100; }

unsigned long long ssm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ssm_set_scan_variant(int npt, int sched)
{
    const bool npt_ok = npt == 0 || npt == 2 || npt == 4 || npt == 8 || npt == 16;
    const bool sched_ok = sched >= 0 && sched <= 12;
    if (!npt_ok || !sched_ok)
        return fail(SSM_ERR_INVALID_ARGUMENT,
                    "ssm_set_scan_variant: states per lane 0, 2, 4, 8 or 16; schedule 0..12");
    ssm::set_scan_variant(npt, sched);
    return ok();
}

int ssm_scan_variant_for(int64_t S, int64_t D, int *states_per_lane, int *schedule)
{
    if (S < 1 || D < 1 || !states_per_lane || !schedule)
        return fail(SSM_ERR_INVALID_ARGUMENT,
                    "ssm_scan_variant_for: S >= 1, D >= 1 and two output pointers required");
    ssm::scan_variant_for(S, D, states_per_lane, schedule);
    return ok();
}

int ssm_device_status(int clear)
{
    const int a0 = ssm::read_scan_status(clear != 0);
    const int a1 = ssm::read_conv_scan_status(clear != 0);
    const int a = (a0 < 0 || a1 < 0) ? -1 : (a0 | a1);
    const int b = ssm::read_conv_status(clear != 0);
    const int d = ssm::read_decode_status(clear != 0);
    const int r = ssm::read_replay_status(clear != 0);
    const int t = ssm::read_selftest_status(clear != 0);
    if (a < 0 || b < 0 || d < 0 || r < 0 || t < 0)
        return fail(SSM_ERR_CUDA, "ssm_device_status: CUDA query failed");
    g_error.clear();
    return (a ? 1 : 0) | (b ? 2 : 0) | (d ? 4 : 0) | (r ? 8 : 0) | (t ? 16 : 0);
}

int ssm_check_cu_seqlens(const int32_t *cu, int64_t S, int64_t tok)
{
    if (!cu) return fail(SSM_ERR_INVALID_ARGUMENT, "ssm_check_cu_seqlens: null pointer");
    if (S < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "ssm_check_cu_seqlens: S must be >= 1");
    if (cu[0] != 0) return fail(SSM_ERR_BAD_SEQLENS, "cu_seqlens[0] = %d, expected 0", cu[0]);
    for (int64_t i = 0; i < S; ++i)
        if (cu[i + 1] < cu[i])
            return fail(SSM_ERR_BAD_SEQLENS, "cu_seqlens decreases at %lld (%d -> %d)",
                        (long long)i, cu[i], cu[i + 1]);
    if ((int64_t)cu[S] != tok)
        return fail(SSM_ERR_BAD_SEQLENS, "cu_seqlens[S] = %d, expected tok = %lld", cu[S],
                    (long long)tok);
    return ok();
}

int ssm_causal_conv1d(const void *x, void *xc, const float *weight, const float *bias,
                      int64_t tok, int64_t D, int K, const int32_t *cu_seqlens, int64_t S,
                      const void *conv_state_in, void *conv_state_out, int apply_silu,
                      ssm_dtype x_dtype, ssm_dtype state_dtype, ssm_stream_t stream)
{
    const char *fn = "ssm_causal_conv1d";
    if (!valid_dtype(x_dtype) || !valid_dtype(state_dtype))
        return fail(SSM_ERR_UNSUPPORTED_DTYPE, "%s: unknown dtype", fn);
    if (D < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: D must be >= 1", fn);
    if (K < 2 || K > 4) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: K must be 2..4 (got %d)", fn, K);
    if (int r = check_seqs(fn, cu_seqlens, S, tok)) return r;
    if (!weight) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: weight is NULL", fn);
    if (tok > 0 && (!x || !xc)) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: x or xc is NULL", fn);
    if (conv_state_out && S * D > 0 && !x && tok > 0)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: x is NULL", fn);
    const size_t es = esize(x_dtype), ss = esize(state_dtype);
    if (!aligned(x, es) || !aligned(xc, es) || !aligned(weight, 4) || !aligned(bias, 4) ||
        !aligned(conv_state_in, ss) || !aligned(conv_state_out, ss))
        return fail(SSM_ERR_MISALIGNED, "%s: a pointer is not aligned to its element size", fn);
    if (x && xc && tok > 0) {
        const char *a = static_cast<const char *>(x), *b = static_cast<const char *>(xc);
        const size_t bytes = (size_t)tok * D * es;
        if (a < b + bytes && b < a + bytes)
            return fail(SSM_ERR_INVALID_ARGUMENT, "%s: xc overlaps x", fn);
    }
    ssm::ConvArgs a{x, xc, weight, bias, tok, D, K, cu_seqlens, S, conv_state_in,
                    conv_state_out, apply_silu, dt(x_dtype), dt(state_dtype),
                    aligned(x, 16) && aligned(xc, 16)};
    int launched = 0;
    cudaError_t e = ssm::launch_conv1d(a, reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

size_t ssm_scan_workspace_size(int64_t tok, int64_t D, int N, int64_t S)
{
    (void)tok; (void)D; (void)N;
    return S > 1 ? ssm::scan_order_bytes(S) : 0;
}

// The forward scan's checks and launch; with bwd_ws (already checked), the
// state before every 8th token of each sequence also goes there for the
// backward pass.
static int scan_fwd_impl(const char *fn, const void *u, const void *delta, const float *A,
                         const void *B, const void *C, const float *Dskip, const void *z,
                         const float *dt_bias, int delta_softplus, const float *h0,
                         const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                         int64_t tok, int64_t D, int N, ssm_dtype act_dtype, void *workspace,
                         size_t workspace_bytes, void *bwd_ws, ssm_stream_t stream)
{
    if (!valid_dtype(act_dtype)) return fail(SSM_ERR_UNSUPPORTED_DTYPE, "%s: unknown dtype", fn);
    if (N != 16) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: N must be 16 (got %d)", fn, N);
    if (D < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: D must be >= 1", fn);
    if (int r = check_seqs(fn, cu_seqlens, S, tok)) return r;
    if (!A) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: A is NULL", fn);
    if (tok > 0 && (!u || !delta || !B || !C || !y))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: u, delta, B, C and y are required", fn);
    const size_t es = esize(act_dtype);
    if (!aligned(u, es) || !aligned(delta, es) || !aligned(z, es) || !aligned(y, es) ||
        !aligned(A, 4) || !aligned(Dskip, 4) || !aligned(dt_bias, 4) || !aligned(h0, 4) ||
        !aligned(h_final, 4))
        return fail(SSM_ERR_MISALIGNED, "%s: a pointer is not aligned to its element size", fn);
    if (!aligned(B, 16) || !aligned(C, 16))
        return fail(SSM_ERR_MISALIGNED, "%s: B and C must be 16-byte aligned", fn);
    const size_t need = ssm_scan_workspace_size(tok, D, N, S);
    if (workspace && workspace_bytes < need)
        return fail(SSM_ERR_WORKSPACE, "%s: workspace has %zu bytes, needs %zu", fn,
                    workspace_bytes, need);
    if (workspace && !aligned(workspace, 256))
        return fail(SSM_ERR_MISALIGNED, "%s: workspace must be 256-byte aligned", fn);
    if (y && tok > 0) {
        const size_t bytes = (size_t)tok * D * es;
        const void *ins[3] = {u, delta, z};
        for (const void *in : ins) {
            if (!in) continue;
            const char *a = static_cast<const char *>(in), *b = static_cast<const char *>(y);
            if (a < b + bytes && b < a + bytes)
                return fail(SSM_ERR_INVALID_ARGUMENT, "%s: y overlaps an input", fn);
        }
    }
    const bool vec = aligned(u, 16) && aligned(delta, 16) && aligned(y, 16) &&
                     (!z || aligned(z, 16));
    bool written = false;
    ssm::ScanArgs a{u, delta, A, B, C, Dskip, z, dt_bias, delta_softplus, h0, cu_seqlens, S,
                    y, h_final, tok, D, N, dt(act_dtype),
                    workspace ? static_cast<int32_t *>(workspace) : nullptr, vec,
                    static_cast<float *>(bwd_ws), &written};
    int launched = 0;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = ssm::launch_scan(a, st, &launched);
    if (e == cudaSuccess && bwd_ws && !written) {
        // the kernel that ran does not write checkpoints: a pass of its own
        ssm::ScanBwdArgs b{u, delta, B, C, z, nullptr, A, Dskip, dt_bias, h0, nullptr,
                           cu_seqlens, S, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                           nullptr, nullptr, nullptr, static_cast<float *>(bwd_ws), tok, D,
                           delta_softplus, act_dtype == SSM_BF16};
        e = ssm::launch_scan_bwd_ckpt_pass(b, st, &launched);
    }
    return finish(e, launched, fn);
}

int ssm_selective_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                           const void *C, const float *Dskip, const void *z,
                           const float *dt_bias, int delta_softplus, const float *h0,
                           const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                           int64_t tok, int64_t D, int N, ssm_dtype act_dtype, void *workspace,
                           size_t workspace_bytes, ssm_stream_t stream)
{
    return scan_fwd_impl("ssm_selective_scan_fwd", u, delta, A, B, C, Dskip, z, dt_bias,
                         delta_softplus, h0, cu_seqlens, S, y, h_final, tok, D, N, act_dtype,
                         workspace, workspace_bytes, nullptr, stream);
}

int ssm_selective_scan_fwd_ckpt(const void *u, const void *delta, const float *A, const void *B,
                                const void *C, const float *Dskip, const void *z,
                                const float *dt_bias, int delta_softplus, const float *h0,
                                const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                                int64_t tok, int64_t D, int N, ssm_dtype act_dtype,
                                void *workspace, size_t workspace_bytes, void *bwd_workspace,
                                size_t bwd_workspace_bytes, ssm_stream_t stream)
{
    const char *fn = "ssm_selective_scan_fwd_ckpt";
    if (N == 16 && D >= 1 && S >= 0 && tok >= 0) {
        const size_t need = ssm_scan_bwd_workspace_size(tok, D, N, S);
        if (!bwd_workspace || bwd_workspace_bytes < need)
            return fail(SSM_ERR_WORKSPACE, "%s: bwd_workspace has %zu bytes, needs %zu", fn,
                        bwd_workspace ? bwd_workspace_bytes : (size_t)0, need);
        if (!aligned(bwd_workspace, 256))
            return fail(SSM_ERR_MISALIGNED, "%s: bwd_workspace must be 256-byte aligned", fn);
        if (workspace && bwd_workspace) {
            const char *a = static_cast<const char *>(workspace);
            const char *b = static_cast<const char *>(bwd_workspace);
            if (a < b + need && b < a + workspace_bytes)
                return fail(SSM_ERR_INVALID_ARGUMENT, "%s: the two workspaces overlap", fn);
        }
    }
    return scan_fwd_impl(fn, u, delta, A, B, C, Dskip, z, dt_bias, delta_softplus, h0,
                         cu_seqlens, S, y, h_final, tok, D, N, act_dtype, workspace,
                         workspace_bytes, bwd_workspace, stream);
}

int ssm_selective_state_update(void *conv_state, float *ssm_state, const void *x,
                               const void *dt_, const void *B, const void *C, const void *z,
                               const float *conv_w, const float *conv_b, const float *A,
                               const float *Dskip, const float *dt_bias, int delta_softplus,
                               const int32_t *state_indices, int64_t n_slots, void *y,
                               int64_t Bt, int64_t D, int N, int K, ssm_dtype act_dtype,
                               ssm_dtype conv_state_dtype, ssm_stream_t stream)
{
    const char *fn = "ssm_selective_state_update";
    if (!valid_dtype(act_dtype) || !valid_dtype(conv_state_dtype))
        return fail(SSM_ERR_UNSUPPORTED_DTYPE, "%s: unknown dtype", fn);
    if (N != 16) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: N must be 16 (got %d)", fn, N);
    if (K < 2 || K > 4) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: K must be 2..4 (got %d)", fn, K);
    if (D < 1 || Bt < 0 || Bt > 65535 || n_slots < 0)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: bad sizes (D=%lld, Bt=%lld, n_slots=%lld)", fn,
                    (long long)D, (long long)Bt, (long long)n_slots);
    if (!state_indices && n_slots < Bt)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: identity slots need n_slots >= Bt", fn);
    if (Bt > 0 && (!conv_state || !ssm_state || !x || !dt_ || !B || !C || !conv_w || !A || !y))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: a required pointer is NULL", fn);
    const size_t es = esize(act_dtype);
    if (!aligned(x, es) || !aligned(dt_, es) || !aligned(B, es) || !aligned(C, es) ||
        !aligned(z, es) || !aligned(y, es) || !aligned(conv_state, esize(conv_state_dtype)) ||
        !aligned(conv_w, 4) || !aligned(conv_b, 4) || !aligned(A, 4) || !aligned(Dskip, 4) ||
        !aligned(dt_bias, 4) || !aligned(state_indices, 4))
        return fail(SSM_ERR_MISALIGNED, "%s: a pointer is not aligned to its element size", fn);
    if (!aligned(ssm_state, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16) ||
        (K == 4 && !aligned(conv_w, 16)))
        return fail(SSM_ERR_MISALIGNED,
                    "%s: ssm_state, A, B, C (and conv_w when K = 4) must be 16-byte aligned", fn);
    ssm::DecodeArgs a{conv_state, ssm_state, x, dt_, B, C, z, conv_w, conv_b, A, Dskip, dt_bias,
                      delta_softplus, state_indices, n_slots, y, Bt, D, N, K, dt(act_dtype),
                      dt(conv_state_dtype)};
    int launched = 0;
    cudaError_t e = ssm::launch_decode(a, reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

int ssm_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_b,
                      const void *conv_state_in, void *conv_state_out, void *xc, int K,
                      ssm_dtype conv_state_dtype, const void *delta, const float *A,
                      const void *B, const void *C, const float *Dskip, const void *z,
                      const float *dt_bias, int delta_softplus, const float *h0,
                      const int32_t *cu_seqlens, int64_t S, void *y, float *h_final,
                      int64_t tok, int64_t D, int N, ssm_dtype act_dtype, ssm_stream_t stream)
{
    const char *fn = "ssm_conv_scan_fwd";
    if (!valid_dtype(act_dtype) || !valid_dtype(conv_state_dtype))
        return fail(SSM_ERR_UNSUPPORTED_DTYPE, "%s: unknown dtype", fn);
    if (N != 16) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: N must be 16 (got %d)", fn, N);
    if (K < 2 || K > 4) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: K must be 2..4 (got %d)", fn, K);
    if (D < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: D must be >= 1", fn);
    if (int r = check_seqs(fn, cu_seqlens, S, tok)) return r;
    if (!A || !conv_w) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: A and conv_w are required", fn);
    if (tok > 0 && (!x || !delta || !B || !C || !y))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: x, delta, B, C and y are required", fn);
    const size_t es = esize(act_dtype), ss = esize(conv_state_dtype);
    if (!aligned(x, es) || !aligned(delta, es) || !aligned(z, es) || !aligned(y, es) ||
        !aligned(xc, es) || !aligned(conv_state_in, ss) || !aligned(conv_state_out, ss) ||
        !aligned(A, 4) || !aligned(conv_w, 4) || !aligned(conv_b, 4) || !aligned(Dskip, 4) ||
        !aligned(dt_bias, 4) || !aligned(h0, 4) || !aligned(h_final, 4))
        return fail(SSM_ERR_MISALIGNED, "%s: a pointer is not aligned to its element size", fn);
    if (!aligned(B, 16) || !aligned(C, 16))
        return fail(SSM_ERR_MISALIGNED, "%s: B and C must be 16-byte aligned", fn);
    if (tok > 0) {
        const size_t bytes = (size_t)tok * D * es;
        const void *outs[2] = {y, xc};
        const void *ins[4] = {x, delta, z, nullptr};
        for (const void *o : outs) {
            if (!o) continue;
            for (const void *in : ins) {
                if (!in) continue;
                const char *a = static_cast<const char *>(in), *b = static_cast<const char *>(o);
                if (a < b + bytes && b < a + bytes)
                    return fail(SSM_ERR_INVALID_ARGUMENT, "%s: an output overlaps an input", fn);
            }
        }
        if (xc) {
            const char *a = static_cast<const char *>(xc), *b = static_cast<const char *>(y);
            if (a < b + bytes && b < a + bytes)
                return fail(SSM_ERR_INVALID_ARGUMENT, "%s: xc overlaps y", fn);
        }
    }
    int npt = 4, sched = 1;
    ssm::scan_variant_for(S, D, &npt, &sched);
    ssm::ScanArgs sa{x, delta, A, B, C, Dskip, z, dt_bias, delta_softplus, h0, cu_seqlens, S, y,
                     h_final, tok, D, N, dt(act_dtype), nullptr, true};
    ssm::ConvScanArgs a{x, conv_w, conv_b, conv_state_in, conv_state_out, xc, K,
                        dt(conv_state_dtype), sa};
    int launched = 0;
    cudaError_t e = ssm::launch_conv_scan(a, npt == 8 ? 8 : 4, sched,
                                          reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

size_t ssm_scan_bwd_workspace_size(int64_t tok, int64_t D, int N, int64_t S)
{
    if (tok < 0 || D < 1 || N != 16 || S < 1) return 0;
    return ssm::scan_bwd_workspace_bytes(tok, D, S);
}

int ssm_set_scan_bwd_variant(int variant)
{
    if (variant < 0 || variant > 2)
        return fail(SSM_ERR_INVALID_ARGUMENT, "ssm_set_scan_bwd_variant: variant 0, 1 or 2");
    ssm::set_scan_bwd_variant(variant);
    return ok();
}

int ssm_scan_bwd_variant_for(int64_t S, int64_t D, int *variant)
{
    if (S < 1 || D < 1 || !variant)
        return fail(SSM_ERR_INVALID_ARGUMENT,
                    "ssm_scan_bwd_variant_for: S >= 1, D >= 1 and an output pointer required");
    *variant = ssm::scan_bwd_variant_for(S, D);
    return ok();
}

// The backward scan's checks and launch; have_ckpt: the workspace holds the
// forward's checkpoints (ssm_selective_scan_fwd_ckpt).
static int scan_bwd_impl(const char *fn, bool have_ckpt, const void *u, const void *delta,
                         const float *A, const void *B, const void *C, const float *Dskip,
                         const void *z, const float *dt_bias, int delta_softplus,
                         const float *h0, const int32_t *cu_seqlens, int64_t S, const void *dy,
                         const float *dh_final, void *du, void *ddelta, void *dz, float *dB,
                         float *dC, float *dA, float *dDskip, float *ddt_bias, float *dh0,
                         int64_t tok, int64_t D, int N, ssm_dtype act_dtype, void *workspace,
                         size_t workspace_bytes, ssm_stream_t stream)
{
    if (!valid_dtype(act_dtype)) return fail(SSM_ERR_UNSUPPORTED_DTYPE, "%s: unknown dtype", fn);
    if (N != 16) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: N must be 16 (got %d)", fn, N);
    if (D < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: D must be >= 1", fn);
    if (int r = check_seqs(fn, cu_seqlens, S, tok)) return r;
    if (!A || !dA || !dB || !dC) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: A, dA, dB and dC are required", fn);
    if (tok > 0 && (!u || !delta || !B || !C || !dy || !du || !ddelta))
        return fail(SSM_ERR_INVALID_ARGUMENT,
                    "%s: u, delta, B, C, dy, du and ddelta are required", fn);
    const size_t es = esize(act_dtype);
    const void *acts[] = {u, delta, z, dy, du, ddelta, dz, B, C};
    for (const void *q : acts)
        if (!aligned(q, es)) return fail(SSM_ERR_MISALIGNED, "%s: a pointer is not aligned to its element size", fn);
    const void *f32s[] = {A, Dskip, dt_bias, h0, dh_final, dB, dC, dA, dDskip, ddt_bias, dh0};
    for (const void *q : f32s)
        if (!aligned(q, 4)) return fail(SSM_ERR_MISALIGNED, "%s: an fp32 pointer is misaligned", fn);
    const size_t need = ssm_scan_bwd_workspace_size(tok, D, N, S);
    if (!workspace || workspace_bytes < need)
        return fail(SSM_ERR_WORKSPACE, "%s: workspace has %zu bytes, needs %zu", fn,
                    workspace ? workspace_bytes : (size_t)0, need);
    if (!aligned(workspace, 256))
        return fail(SSM_ERR_MISALIGNED, "%s: workspace must be 256-byte aligned", fn);
    if (tok > 0) {
        // (tok, D) activations against (tok, D) inputs and the (tok, N) B, C rows
        const size_t bytes = (size_t)tok * D * es, bc_bytes = (size_t)tok * N * es;
        const void *outs[] = {du, ddelta, dz};
        const void *ins[] = {u, delta, z, dy, B, C};
        const size_t in_bytes[] = {bytes, bytes, bytes, bytes, bc_bytes, bc_bytes};
        for (const void *o : outs) {
            if (!o) continue;
            for (int i = 0; i < 6; ++i) {
                if (!ins[i]) continue;
                const char *a = static_cast<const char *>(o), *b = static_cast<const char *>(ins[i]);
                if (a < b + in_bytes[i] && b < a + bytes)
                    return fail(SSM_ERR_INVALID_ARGUMENT, "%s: a gradient overlaps an input", fn);
            }
        }
    }
    ssm::ScanBwdArgs a{u, delta, B, C, z, dy, A, Dskip, dt_bias, h0, dh_final, cu_seqlens, S,
                       du, ddelta, dz, dB, dC, dA, dDskip, ddt_bias, dh0,
                       static_cast<float *>(workspace), tok, D, delta_softplus,
                       act_dtype == SSM_BF16, have_ckpt};
    int launched = 0;
    cudaError_t e = ssm::launch_scan_bwd(a, reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

int ssm_selective_scan_bwd(const void *u, const void *delta, const float *A, const void *B,
                           const void *C, const float *Dskip, const void *z,
                           const float *dt_bias, int delta_softplus, const float *h0,
                           const int32_t *cu_seqlens, int64_t S, const void *dy,
                           const float *dh_final, void *du, void *ddelta, void *dz, float *dB,
                           float *dC, float *dA, float *dDskip, float *ddt_bias, float *dh0,
                           int64_t tok, int64_t D, int N, ssm_dtype act_dtype, void *workspace,
                           size_t workspace_bytes, ssm_stream_t stream)
{
    return scan_bwd_impl("ssm_selective_scan_bwd", false, u, delta, A, B, C, Dskip, z, dt_bias,
                         delta_softplus, h0, cu_seqlens, S, dy, dh_final, du, ddelta, dz, dB, dC,
                         dA, dDskip, ddt_bias, dh0, tok, D, N, act_dtype, workspace,
                         workspace_bytes, stream);
}

int ssm_selective_scan_bwd_ckpt(const void *u, const void *delta, const float *A, const void *B,
                                const void *C, const float *Dskip, const void *z,
                                const float *dt_bias, int delta_softplus, const float *h0,
                                const int32_t *cu_seqlens, int64_t S, const void *dy,
                                const float *dh_final, void *du, void *ddelta, void *dz,
                                float *dB, float *dC, float *dA, float *dDskip, float *ddt_bias,
                                float *dh0, int64_t tok, int64_t D, int N, ssm_dtype act_dtype,
                                void *workspace, size_t workspace_bytes, ssm_stream_t stream)
{
    return scan_bwd_impl("ssm_selective_scan_bwd_ckpt", true, u, delta, A, B, C, Dskip, z,
                         dt_bias, delta_softplus, h0, cu_seqlens, S, dy, dh_final, du, ddelta,
                         dz, dB, dC, dA, dDskip, ddt_bias, dh0, tok, D, N, act_dtype, workspace,
                         workspace_bytes, stream);
}

// Shared checks of a replay slot list (NULL = slots 0..n-1).
static int check_replay_slots(const char *fn, const int32_t *slots, int64_t n, int64_t n_slots,
                              int64_t D, int N)
{
    if (N != 16) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: N must be 16 (got %d)", fn, N);
    if (D < 1 || n < 0 || n > 65535 || n_slots < 0)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: bad sizes (D=%lld, n=%lld, n_slots=%lld)", fn,
                    (long long)D, (long long)n, (long long)n_slots);
    if (!slots && n > n_slots)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: without a slot list, n must be <= n_slots", fn);
    if (!aligned(slots, 4)) return fail(SSM_ERR_MISALIGNED, "%s: slots misaligned", fn);
    return SSM_OK;
}

int ssm_replay_state_update(void *conv_state, float *ckpt, void *ckpt_lo, float *buf,
                            float *buf_B, int32_t *buf_len, uint32_t *tickets, int W,
                            const void *x, const void *dt_, const void *B, const void *C,
                            const void *z, const float *conv_w, const float *conv_b,
                            const float *A, const float *Dskip, const float *dt_bias,
                            int delta_softplus, const int32_t *state_indices, int64_t n_slots,
                            void *y, int64_t Bt, int64_t D, int N, int K, ssm_dtype act_dtype,
                            ssm_dtype conv_state_dtype, ssm_stream_t stream)
{
    const char *fn = "ssm_replay_state_update";
    if (!valid_dtype(act_dtype) || !valid_dtype(conv_state_dtype))
        return fail(SSM_ERR_UNSUPPORTED_DTYPE, "%s: unknown dtype", fn);
    if (N != 16) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: N must be 16 (got %d)", fn, N);
    if (K < 2 || K > 4) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: K must be 2..4 (got %d)", fn, K);
    if (W < 1 || W > 8) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: W must be 1..8 (got %d)", fn, W);
    if (D < 1 || Bt < 0 || Bt > 65535 || n_slots < 0)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: bad sizes (D=%lld, Bt=%lld, n_slots=%lld)", fn,
                    (long long)D, (long long)Bt, (long long)n_slots);
    if (!state_indices && n_slots < Bt)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: identity slots need n_slots >= Bt", fn);
    if (Bt > 0 && (!conv_state || !ckpt || !buf_len || !tickets || !x || !dt_ || !B || !C ||
                   !conv_w || !A || !y))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: a required pointer is NULL", fn);
    if (Bt > 0 && W > 1 && (!buf || !buf_B))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: W > 1 needs buf and buf_B", fn);
    const size_t es = esize(act_dtype), cs = esize(conv_state_dtype);
    if (!aligned(conv_w, 4) || !aligned(conv_b, 4) || !aligned(Dskip, 4) ||
        !aligned(dt_bias, 4) || !aligned(state_indices, 4) || !aligned(buf_len, 4) ||
        !aligned(tickets, 4) || !aligned(y, es))
        return fail(SSM_ERR_MISALIGNED, "%s: a pointer is not aligned to its element size", fn);
    if (!aligned(conv_state, 16) || !aligned(ckpt, 16) || !aligned(ckpt_lo, 16) ||
        !aligned(buf, 16) || !aligned(buf_B, 16) || !aligned(x, 16) || !aligned(dt_, 16) ||
        !aligned(z, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(A, 16) ||
        (D * (int64_t)es) % 16 != 0 || (D * (K - 1) * (int64_t)cs) % 16 != 0)
        return fail(SSM_ERR_MISALIGNED,
                    "%s: conv_state, ckpt, ckpt_lo, buf, buf_B, x, dt, z, B, C and A must be "
                    "16-byte aligned, and D * element size (and D * (K-1) * conv-state element "
                    "size) multiples of 16 bytes", fn);
    ssm::ReplayStepArgs a{conv_state, ckpt, ckpt_lo, buf, buf_B, buf_len, tickets, W, x, dt_, B,
                          C, z, conv_w, conv_b, A, Dskip, dt_bias, delta_softplus,
                          state_indices, n_slots, y, Bt, D, K, act_dtype == SSM_BF16,
                          conv_state_dtype == SSM_BF16};
    int launched = 0;
    cudaError_t e = ssm::launch_replay_step(a, reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

int ssm_replay_reset(const float *ckpt, void *ckpt_lo, int32_t *buf_len, uint32_t *tickets,
                     const int32_t *slots, int64_t n, int64_t n_slots, int64_t D, int N,
                     ssm_stream_t stream)
{
    const char *fn = "ssm_replay_reset";
    if (int r = check_replay_slots(fn, slots, n, n_slots, D, N)) return r;
    if (n > 0 && (!buf_len || !tickets || (ckpt_lo && !ckpt)))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: a required pointer is NULL", fn);
    if (!aligned(ckpt, 16) || !aligned(ckpt_lo, 16) || !aligned(buf_len, 4) || !aligned(tickets, 4))
        return fail(SSM_ERR_MISALIGNED, "%s: ckpt and ckpt_lo must be 16-byte aligned", fn);
    int launched = 0;
    cudaError_t e = ssm::launch_replay_reset(ckpt, ckpt_lo, buf_len, tickets, slots, n, n_slots,
                                             D, reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

int ssm_replay_flush(float *ckpt, void *ckpt_lo, const float *buf, const float *buf_B,
                     int32_t *buf_len, uint32_t *tickets, const float *A, int W,
                     const int32_t *slots, int64_t n, int64_t n_slots, int64_t D, int N,
                     ssm_stream_t stream)
{
    const char *fn = "ssm_replay_flush";
    if (W < 1 || W > 8) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: W must be 1..8 (got %d)", fn, W);
    if (int r = check_replay_slots(fn, slots, n, n_slots, D, N)) return r;
    if (n > 0 && (!ckpt || !buf_len || !tickets || !A || (W > 1 && (!buf || !buf_B))))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: a required pointer is NULL", fn);
    if (!aligned(ckpt, 16) || !aligned(ckpt_lo, 16) || !aligned(buf, 16) || !aligned(buf_B, 16) ||
        !aligned(A, 16) || !aligned(buf_len, 4) || !aligned(tickets, 4))
        return fail(SSM_ERR_MISALIGNED,
                    "%s: ckpt, ckpt_lo, buf, buf_B and A must be 16-byte aligned", fn);
    int launched = 0;
    cudaError_t e = ssm::launch_replay_flush(ckpt, ckpt_lo, buf, buf_B, buf_len, tickets, A, W,
                                             slots, n, n_slots, D,
                                             reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

// For callers that cannot allocate device memory: the same scan, with its
// schedule scratch in a fixed device array owned by the library instead of a
// caller-allocated workspace. It forwards to ssm_selective_scan_fwd.
int ssm_selective_scan_fwd_noalloc(const void *u, const void *delta, const float *A,
                                   const void *B, const void *C, const float *Dskip,
                                   const void *z, const float *dt_bias, int delta_softplus,
                                   const float *h0, const int32_t *cu_seqlens, int64_t S,
                                   void *y, float *h_final, int64_t tok, int64_t D, int N,
                                   ssm_dtype act_dtype, ssm_stream_t stream)
{
    const char *fn = "ssm_selective_scan_fwd_noalloc";
    if (cu_seqlens && S > ssm::noalloc_max_sequences())
        return fail(SSM_ERR_INVALID_ARGUMENT,
                    "%s: at most %lld packed sequences per call (got %lld); the fixed scratch "
                    "holds one schedule entry per sequence",
                    fn, (long long)ssm::noalloc_max_sequences(), (long long)S);
    // Only packed calls of two or more sequences use the schedule; dense rows
    // and a single sequence run without it, whatever S is.
    void *scratch = nullptr;
    size_t bytes = 0;
    if (cu_seqlens && S > 1) {
        cudaError_t e = ssm::noalloc_scratch(&scratch, &bytes);
        if (e != cudaSuccess)
            return fail(SSM_ERR_CUDA, "%s: looking up the fixed scratch failed: %s", fn,
                        cudaGetErrorString(e));
    }
    return ssm_selective_scan_fwd(u, delta, A, B, C, Dskip, z, dt_bias, delta_softplus, h0,
                                  cu_seqlens, S, y, h_final, tok, D, N, act_dtype, scratch, bytes,
                                  stream);
}

int ssm_selftest_wait_timeout(int tries, ssm_stream_t stream)
{
    const char *fn = "ssm_selftest_wait_timeout";
    if (tries < 1 || tries > (1 << 17))
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: tries must be 1..131072 (got %d)", fn, tries);
    int launched = 0;
    cudaError_t e = ssm::launch_wait_selftest((unsigned)tries,
                                              reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

int64_t ssm_probe_sink_floats(void) { return (int64_t)ssm::probe_sink_floats(); }

int ssm_probe_rate(int kind, int iters, int warps_per_sm, float *sink, int64_t sink_floats,
                   double *ops, ssm_stream_t stream)
{
    const char *fn = "ssm_probe_rate";
    if (kind < 0 || kind > 3)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: kind must be 0..3 (got %d)", fn, kind);
    if (warps_per_sm < 8 || warps_per_sm > 64 || warps_per_sm % 8 != 0)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: warps_per_sm must be 8, 16, ..., 64 (got %d)",
                    fn, warps_per_sm);
    if (iters < 1) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: iters must be >= 1", fn);
    if (!sink || !ops) return fail(SSM_ERR_INVALID_ARGUMENT, "%s: sink and ops are required", fn);
    if (!aligned(sink, 4)) return fail(SSM_ERR_MISALIGNED, "%s: sink misaligned", fn);
    const int64_t need = ssm_probe_sink_floats();
    if (sink_floats < need)
        return fail(SSM_ERR_INVALID_ARGUMENT, "%s: sink holds %lld floats, needs %lld", fn,
                    (long long)sink_floats, (long long)need);
    int launched = 0;
    cudaError_t e = ssm::launch_probe(kind, iters, warps_per_sm / 8, sink, ops,
                                      reinterpret_cast<cudaStream_t>(stream), &launched);
    return finish(e, launched, fn);
}

}  // extern "C"
