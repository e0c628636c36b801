// launch_util.h -- host helpers shared by the kernel launchers (internal).
#pragma once

#include <cuda_runtime.h>

namespace ss2d {

constexpr int kMaxDevices = 128;

// Raises a kernel's dynamic shared-memory limit to `bytes` and asks for the largest
// shared-memory carveout, once per device and size (configured[] is per kernel).
template <class K>
cudaError_t configure_smem(K kernel, int bytes, int *configured)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    if (bytes <= configured[dev])
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
        return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    configured[dev] = bytes;
    return cudaSuccess;
}

}  // namespace ss2d
