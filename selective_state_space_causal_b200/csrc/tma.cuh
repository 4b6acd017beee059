// tma.cuh -- TMA tile loads, mbarrier waits and tensor-map encoding (sm_100a).
//
// Loads are plain per-CTA tile copies (cp.async.bulk.tensor, no multicast) of
// this GPU's own memory into the calling CTA's shared memory; completion is
// tracked by an mbarrier with an expected transaction byte count.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// Bounded waits: each try suspends the thread in hardware until the phase
// completes or about kSuspendNs nanoseconds pass, so a waiting warp takes no
// issue slots; after kWaitTries tries (about half a second) the wait gives up.
constexpr unsigned kWaitTries = 1u << 17;
constexpr uint32_t kSuspendNs = 4096;

__device__ __forceinline__ uint32_t saddr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(saddr(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Barrier expecting `count` arrivals per phase (no fence; the caller fences).
__device__ __forceinline__ void mbar_init_n(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(saddr(bar)), "r"(count) : "memory");
}

// Plain arrival (release semantics for this thread's earlier shared-memory writes).
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(saddr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(saddr(bar)), "r"(bytes) : "memory");
}

// 2-D tile load: box at (x = inner coordinate, y = row) into dst.
__device__ __forceinline__ void tma_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x,
                                       int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        :: "r"(saddr(dst)), "l"(map), "r"(x), "r"(y), "r"(saddr(bar)) : "memory");
}

// 1-D bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from this GPU's global memory into this CTA's shared memory, completing on
// `bar` with `bytes` transaction bytes. No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(saddr(dst)), "l"(src), "r"(bytes), "r"(saddr(bar)) : "memory");
}

// 1-D bulk copy from this CTA's shared memory to global memory, tracked by the
// issuing thread's bulk-async groups (commit, then wait).
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(dst), "r"(saddr(src)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's committed groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(N) : "memory");
}

// Wait until at most N of this thread's committed groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait()
{
    asm volatile("cp.async.bulk.wait_group %0;" :: "n"(N) : "memory");
}

// Order earlier generic-proxy reads of shared memory before later TMA writes.
__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Waits for phase `parity` of the barrier with a bounded number of
// suspending tries (kWaitTries unless a smaller count is given). On timeout it
// sets bit `code` of *status and marks `failed`, after which this thread no
// longer waits at all, so a kernel always terminates.
__device__ __forceinline__ void mbar_wait(uint64_t *bar, uint32_t parity, bool &failed,
                                          int *status, int code, unsigned tries = kWaitTries)
{
    if (failed) return;
    for (unsigned i = 0; i < tries; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done) : "r"(saddr(bar)), "r"(parity), "r"(kSuspendNs) : "memory");
        if (done) return;
    }
    failed = true;
    atomicOr(status, code);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess || q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

// 2-D tile map over a row-major (rows, inner) tensor of bf16 or fp32;
// out-of-range reads fill zeros. Returns false if the map cannot be encoded.
inline bool encode_2d(CUtensorMap *map, const void *base, bool bf16, uint64_t inner, uint64_t rows,
                      uint32_t box_inner, uint32_t box_rows)
{
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    const uint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * es};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ssm
