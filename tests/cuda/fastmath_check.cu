// Accuracy of the library's FMA-pipe exp2, softplus and silu (common.cuh)
// against fp64 references and CUDA's exp2f, over dense sweeps. Prints one line
// per function: max relative error and the worst input. Every index stays
// inside its buffer.
#include <cmath>
#include <cstdio>
#include <vector>

#include "common.cuh"

using namespace ssm;

__global__ void run(const float *x, int n, float *e2, float *e2ref, float *sp, float *sp1, float *si)
{
    int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 >= n) return;
    float a, b;
    exp2_fma2(x[i], x[i + 1], a, b);
    e2[i] = a; e2[i + 1] = b;
    e2ref[i] = exp2f(x[i]); e2ref[i + 1] = exp2f(x[i + 1]);
    softplus2(x[i], x[i + 1], a, b);
    sp[i] = a; sp[i + 1] = b;
    sp1[i] = softplus_fast(x[i]); sp1[i + 1] = softplus_fast(x[i + 1]);
    silu2(x[i], x[i + 1], a, b);
    si[i] = a; si[i + 1] = b;
}

int main()
{
    const int n = 1 << 22;
    std::vector<float> hx(n);
    for (int i = 0; i < n; ++i) hx[i] = -90.0f + 180.0f * (float)i / (float)n;  // [-90, 90)
    float *dx, *d[5];
    cudaMalloc(&dx, n * sizeof(float));
    for (auto &p : d) cudaMalloc(&p, n * sizeof(float));
    cudaMemcpy(dx, hx.data(), n * sizeof(float), cudaMemcpyHostToDevice);
    run<<<n / 2 / 256, 256>>>(dx, n, d[0], d[1], d[2], d[3], d[4]);
    std::vector<float> h[5];
    for (int k = 0; k < 5; ++k) {
        h[k].resize(n);
        cudaMemcpy(h[k].data(), d[k], n * sizeof(float), cudaMemcpyDeviceToHost);
    }
    double e_exp = 0, e_exp_cuda = 0, e_sp = 0, e_sp1 = 0, e_si = 0, e_sp20 = 0, e_si20 = 0;
    float w_exp = 0, w_sp = 0, w_si = 0;
    for (int i = 0; i < n; ++i) {
        const double x = hx[i];
        if (x >= -125.0 && x <= 125.0) {   // normal range of the result
            const double r = std::exp2(x);
            const double e = std::fabs(h[0][i] - r) / r;
            if (e > e_exp) { e_exp = e; w_exp = hx[i]; }
            e_exp_cuda = std::fmax(e_exp_cuda, std::fabs(h[1][i] - r) / r);
        }
        // results below the normal fp32 range (x < -85) are not compared
        const double spr = (x > 0 ? x : 0.0) + std::log1p(std::exp(-std::fabs(x)));
        if (x >= -85.0) {
            const double e = std::fabs(h[2][i] - spr) / spr;
            if (e > e_sp) { e_sp = e; w_sp = hx[i]; }
            if (std::fabs(x) <= 20.0) e_sp20 = std::fmax(e_sp20, e);
            e_sp1 = std::fmax(e_sp1, std::fabs(h[3][i] - spr) / spr);
        }
        const double sir = x / (1.0 + std::exp(-x));
        const double scale = std::fabs(sir);
        if (x >= -80.0 && scale > 0.0) {
            const double e = std::fabs(h[4][i] - sir) / scale;
            if (e > e_si) { e_si = e; w_si = hx[i]; }
            if (std::fabs(x) <= 20.0) e_si20 = std::fmax(e_si20, e);
        }
    }
    printf("exp2_fma2 max_rel %.3e at %.6f (CUDA exp2f max_rel %.3e)\n", e_exp, w_exp, e_exp_cuda);
    printf("softplus2 max_rel %.3e at %.6f (softplus_fast max_rel %.3e)\n", e_sp, w_sp, e_sp1);
    printf("silu2 max_rel %.3e at %.6f\n", e_si, w_si);
    printf("softplus2_core max_rel %.3e\n", e_sp20);
    printf("silu2_core max_rel %.3e\n", e_si20);
    cudaError_t st = cudaDeviceSynchronize();
    printf("status %s\n", cudaGetErrorString(st));
    return st == cudaSuccess ? 0 : 1;
}
