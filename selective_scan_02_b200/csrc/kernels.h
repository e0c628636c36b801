// kernels.h -- host-side launchers of the libss2d kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

struct ScanArgs;

cudaError_t launch_cross_scan(const void *x, bool bf16, void *xs, int B, int D, int H, int W, cudaStream_t s);
cudaError_t launch_cross_merge(const float *ys, float *y, int B, int D, int H, int W, cudaStream_t s);
cudaError_t launch_fill_zero(float *p, size_t n, cudaStream_t s);

// mode: 0 standalone scan, 1 fused core (u gathered from x, output merged into y).
cudaError_t launch_scan(const ScanArgs &a, int N, int mode, cudaStream_t s);

}  // namespace ss2d
