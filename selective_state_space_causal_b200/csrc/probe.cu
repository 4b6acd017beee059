// probe.cu -- throughput probes of the units the scan's roofline is set by.
//
// The scan's bound is the special-function unit (one ex2 per state and
// token); its roofline denominator is measured here rather than derived from
// unit counts: a kernel that keeps every SM's special-function units busy
// with independent ex2.approx.ftz.f32 chains, and, for comparison, the same
// for the FMA pipe with packed fp32x2 and scalar fp32 FMAs, and a mix of one
// ex2 per two packed FMA-pipe operations (the recurrence's per-state mix).
// The caller times a launch with CUDA events and divides the operation count
// it is given by the elapsed time.
#include <cuda_runtime.h>

#include "common.cuh"
#include "tma.cuh"

namespace ssm {

// Set by the wait self-test when its bounded wait gives up (as it must).
__device__ int g_selftest_status = 0;

namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeBlocksPerSM = 8;  // 2048 threads: every warp slot of an SM
constexpr int kChains = 8;            // independent dependency chains per thread

__global__ void __launch_bounds__(kProbeThreads)
probe_ex2_kernel(float *sink, int iters)
{
    float x[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) x[k] = 0.5f + 0.01f * k + 1e-6f * threadIdx.x;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < kChains; ++k) x[k] = ex2_approx(-x[k]);  // stays in [0.5, 1]
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += x[k];
    sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void __launch_bounds__(kProbeThreads)
probe_ffma2_kernel(float *sink, int iters)
{
    f32x2 x[kChains];
    const f32x2 a = pk2(0.999f, 0.998f), b = pk2(1e-3f, 2e-3f);
#pragma unroll
    for (int k = 0; k < kChains; ++k) x[k] = pk2(0.5f + 0.01f * k, 1e-6f * threadIdx.x);
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < kChains; ++k) x[k] = fma2(x[k], a, b);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) {
        float lo, hi;
        upk2(x[k], lo, hi);
        s += lo + hi;
    }
    sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void __launch_bounds__(kProbeThreads)
probe_ffma_kernel(float *sink, int iters)
{
    float x[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) x[k] = 0.5f + 0.01f * k + 1e-6f * threadIdx.x;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < kChains; ++k) x[k] = fmaf(x[k], 0.999f, 1e-3f);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += x[k];
    sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

// Per state pair and step: one packed FMA-pipe operation that forms the two
// exponent arguments (a chain of its own, as delta * A does not depend on the
// state), two ex2, a packed multiply for the input term and two packed FMAs
// (state update and readout): the recurrence's instruction mix.
__global__ void __launch_bounds__(kProbeThreads)
probe_mix_kernel(float *sink, int iters)
{
    constexpr int P = kChains / 2;
    f32x2 arg[P], h[P], acc[P];
    const f32x2 dd = pk2(0.5f, 0.25f), bb = pk2(-0.01f, -0.02f), cc = pk2(0.5f, 0.25f);
#pragma unroll
    for (int k = 0; k < P; ++k) {
        arg[k] = pk2(-0.01f * (k + 1), -1e-6f * threadIdx.x);
        h[k] = pk2(0.5f + 0.01f * k, 1e-6f * threadIdx.x);
        acc[k] = 0ull;
    }
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < P; ++k) {
            arg[k] = fma2(arg[k], dd, bb);  // converges to about -0.02 and -0.027
            float a0, a1;
            upk2(arg[k], a0, a1);
            const f32x2 e = pk2(ex2_approx(a0), ex2_approx(a1));
            h[k] = fma2(e, h[k], mul2(arg[k], cc));
            acc[k] = fma2(cc, h[k], acc[k]);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < P; ++k) {
        float lo, hi;
        upk2(add2(h[k], acc[k]), lo, hi);
        s += lo + hi;
    }
    sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

// Self-test of the bounded mbarrier wait every TMA-staged kernel uses: the
// barrier expects 16 transaction bytes that no copy ever delivers, so the
// wait runs out after `tries` suspending tries, sets the status bit and the
// kernel returns. Nothing is in flight when it exits.
__global__ void wait_selftest_kernel(unsigned tries)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) mbar_init(&bar);
    __syncthreads();
    if (threadIdx.x == 0) mbar_expect_tx(&bar, 16);
    bool failed = false;
    mbar_wait(&bar, 0u, failed, &g_selftest_status, 1, tries);
}

}  // namespace

int device_sm_count();

int read_selftest_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_selftest_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_selftest_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

cudaError_t launch_wait_selftest(unsigned tries, cudaStream_t stream, int *launches)
{
    wait_selftest_kernel<<<1, 32, 0, stream>>>(tries);
    ++*launches;
    return cudaGetLastError();
}

int probe_sink_floats() { return device_sm_count() * kProbeBlocksPerSM * kProbeThreads; }

// Launches probe `kind` (0 ex2, 1 packed fp32x2 FMA, 2 scalar fp32 FMA, 3 the
// recurrence mix) with `per_sm` CTAs of 8 warps per SM (1..8) and returns the
// operations it performs (ex2 results for 0 and 3, FMAs for 1 and 2) in *ops.
cudaError_t launch_probe(int kind, int iters, int per_sm, float *sink, double *ops,
                         cudaStream_t stream, int *launches)
{
    const int blocks = device_sm_count() * per_sm;
    const double lanes = (double)blocks * kProbeThreads * iters;
    switch (kind) {
    case 0:
        probe_ex2_kernel<<<blocks, kProbeThreads, 0, stream>>>(sink, iters);
        *ops = lanes * kChains;
        break;
    case 1:
        probe_ffma2_kernel<<<blocks, kProbeThreads, 0, stream>>>(sink, iters);
        *ops = lanes * kChains * 2;
        break;
    case 2:
        probe_ffma_kernel<<<blocks, kProbeThreads, 0, stream>>>(sink, iters);
        *ops = lanes * kChains;
        break;
    default:
        probe_mix_kernel<<<blocks, kProbeThreads, 0, stream>>>(sink, iters);
        *ops = lanes * kChains;
        break;
    }
    ++*launches;
    return cudaGetLastError();
}

}  // namespace ssm
