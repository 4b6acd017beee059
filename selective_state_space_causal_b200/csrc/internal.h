// internal.h -- launchers behind the C ABI (host side, C++ only).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

enum class DType { F32 = 0, BF16 = 1 };

struct ConvArgs {
    const void *x;
    void *xc;
    const float *w;
    const float *bias;
    int64_t tok, D;
    int K;
    const int32_t *cu;  // nullptr: dense rows of tok / S
    int64_t S;
    const void *state_in;
    void *state_out;
    int apply_silu;
    DType x_dtype, state_dtype;
    bool vec;  // 16-byte vector path allowed (alignment checked by the caller)
};

struct ScanArgs {
    const void *u, *delta;
    const float *A;
    const void *B, *C;
    const float *Dskip;
    const void *z;
    const float *dt_bias;
    int delta_softplus;
    const float *h0;
    const int32_t *cu;
    int64_t S;
    void *y;
    float *h_final;
    int64_t tok, D;
    int N;
    DType dtype;
    int32_t *order;  // nullptr: sequences in index order; else S entries of scratch
    bool vec;
    // the state before every 8th token of each sequence, for the backward
    // pass, or nullptr; *ckpt_written reports whether the kernel that ran wrote
    // them (the pipelined kernel does, the other schedules do not)
    float *ckpt = nullptr;
    bool *ckpt_written = nullptr;
};

struct DecodeArgs {
    void *conv_state;
    float *ssm_state;
    const void *x, *dt, *B, *C, *z;
    const float *conv_w, *conv_b, *A, *Dskip, *dt_bias;
    int delta_softplus;
    const int32_t *idx;
    int64_t n_slots;
    void *y;
    int64_t Bt, D;
    int N, K;
    DType dtype, conv_dtype;
};

// Each returns cudaSuccess or the launch error.
cudaError_t launch_conv1d(const ConvArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_scan(const ScanArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream, int *launches);

}  // namespace ssm
