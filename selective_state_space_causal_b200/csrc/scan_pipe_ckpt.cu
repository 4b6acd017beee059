// scan_pipe_ckpt.cu -- the chunk-pipelined selective scan that also writes,
// for the backward pass, the fp32 state before every 8th token of each
// sequence (ssm_selective_scan_fwd_ckpt; the kernels are in scan_pipe.cuh).
// A translation unit of its own so that the plain forward kernels compile
// without the checkpoint stores and both compile in parallel.
#include "scan_pipe.cuh"

namespace ssm {

int read_pipe_ckpt_status(bool clear) { return read_tu_pipe_status(clear); }

cudaError_t launch_scan_pipe_ckpt(const Params &p, bool bf16, int npt, int sched,
                                  cudaStream_t stream, int *launches)
{
    return launch_pipe_cfg<true>(p, bf16, npt, sched, stream, launches);
}

}  // namespace ssm
