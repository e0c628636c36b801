// diag.cu -- a diagnostic of the tensor-core kernels' bounded waits.
//
// The projection form's tcgen05 kernels wait for their MMAs on mbarriers with an iteration
// limit; a wait that runs out sets the workspace's error word, frees the kernel's tensor
// memory and returns, so the context stays usable and ss2d_device_status reports
// SS2D_ERR_DEVICE.  This kernel runs that path on purpose: it allocates tensor memory, waits on
// an mbarrier that nothing arrives at with the caller's limit, records the timeout in the
// error word exactly as the GEMM kernels do, frees the tensor memory and returns.
#include <stdint.h>

#include "ss2d.h"
#include "tcgen05.cuh"

namespace ss2d {
namespace {

__global__ void bounded_wait_probe_kernel(int *err, long long limit)
{
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(&mbar)), "r"(1));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc::smem_u32(&tmem_slot)),
                     "r"(32));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = tmem_slot;
    // no arrival is ever made: the wait runs out after `limit` polls
    const bool ok = tc::mbar_wait(tc::smem_u32(&mbar), 0u, limit);
    if (__syncthreads_or(ok ? 0 : 1)) {
        if (threadIdx.x == 0)
            atomicExch(err, 1);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(32));
}

}  // namespace
}  // namespace ss2d

extern "C" int ss2d_diag_bounded_wait(int *error_word, long long spin_limit, void *stream)
{
    if (!error_word || spin_limit < 1 || spin_limit > (1LL << 20))  // at most about 4 s of polling
        return SS2D_ERR_INVALID_ARG;
    ss2d::bounded_wait_probe_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(error_word, spin_limit);
    return cudaGetLastError() == cudaSuccess ? SS2D_OK : SS2D_ERR_CUDA;
}
