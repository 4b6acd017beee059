// scan_pipe.cu -- the chunk-pipelined selective scan as the forward calls it
// (schedules 9 to 11; the kernels are in scan_pipe.cuh).
#include "scan_pipe.cuh"

namespace ssm {

int read_pipe_ckpt_status(bool clear);
cudaError_t launch_scan_pipe_ckpt(const Params &p, bool bf16, int npt, int sched,
                                  cudaStream_t stream, int *launches);

int read_pipe_status(bool clear)
{
    const int a = read_tu_pipe_status(clear), b = read_pipe_ckpt_status(clear);
    return (a < 0 || b < 0) ? -1 : (a | b);
}

// Schedules 9 and 10 (16- and 32-token chunks), 11 (schedule 10 at 4 states
// per lane with up to 255 registers, two CTAs per SM; for bf16) and 12 (one
// lane per channel with all 16 states, 128-lane CTAs) for 16-byte
// aligned rows (D a multiple of 8 for bf16, of 4 for fp32);
// cudaErrorNotSupported when the tensor maps cannot be encoded. CTAs of four
// warps. With p.ckpt the kernels that also write the backward pass's
// checkpoints run instead.
cudaError_t launch_scan_pipe(const Params &p, bool bf16, int npt, int sched, cudaStream_t stream,
                             int *launches)
{
    if (p.ckpt) return launch_scan_pipe_ckpt(p, bf16, npt, sched, stream, launches);
    return launch_pipe_cfg<false>(p, bf16, npt, sched, stream, launches);
}

}  // namespace ssm
