// launch_util.h -- host helpers shared by the kernel launchers (internal).
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace ss2d {

constexpr int kMaxDevices = 128;

// Serialises the raising of shared-memory limits across host threads.
inline std::mutex g_configure_smem_mutex;

// Raises a kernel's dynamic shared-memory limit to `bytes` and asks for the largest
// shared-memory carveout, once per device and size (configured[] is per kernel and holds
// the limit set so far on each device).  Safe to call from several host threads: the
// limit only grows, so a call never lowers it under another thread's larger launch.
template <class K>
cudaError_t configure_smem(K kernel, int bytes, int *configured)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    if (bytes <= __atomic_load_n(&configured[dev], __ATOMIC_ACQUIRE))
        return cudaSuccess;
    std::lock_guard<std::mutex> lock(g_configure_smem_mutex);
    if (bytes <= __atomic_load_n(&configured[dev], __ATOMIC_ACQUIRE))
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
        return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    __atomic_store_n(&configured[dev], bytes, __ATOMIC_RELEASE);
    return cudaSuccess;
}

}  // namespace ss2d
