// xproj.h -- the projection path of the fused core (x_proj on tensor cores,
// then the scan with dt_proj fused).  Internal.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

// 0 if the projection path supports this shape, else a nonzero reason code.
int xproj_supported(int B, int D, int H, int W, int N, int R);

// True when the scan fuses dt_proj for this dt_rank; otherwise dts is materialised in the
// workspace and only channels-first x and y are supported.
bool xproj_dt_fused(int R);

// Bytes of workspace the projection path needs.
size_t xproj_workspace_bytes(int B, int D, int H, int W, int N, int R, bool ch_last);

// The x_proj GEMM alone: x_dbl (B, 4, R+2N, L) fp32, each direction's rows in its scan
// order, from channels-first bf16 x and the bf16 weights (4, R+2N, D).  err points at
// xproj_header_bytes() of scratch holding the error word of the kernel's bounded waits; the
// kernel only ever sets it, so the caller clears it (launch_clear_error_word) once per call.
cudaError_t launch_xproj_gemm(const void *x_cf, const void *x_proj_weight, float *xdbl, int *err, int B, int D, int H,
                              int W, int N, int R, cudaStream_t s);
size_t xproj_header_bytes();

// Zeroes the xproj_header_bytes() header that holds the error word.
cudaError_t launch_clear_error_word(int *err, cudaStream_t s);

// The projection form of the fused core.  The workspace starts with the error-word header;
// clear_err zeroes it first (a caller running the batch in slices clears it once, so a wait
// that ran out in any slice stays visible).  y (B, D, L) fp32 receives the four directions'
// atomic adds and is zeroed here first: inside the plane transpose of x when the scan reads
// that copy, else by its own launch.
cudaError_t launch_core_with_projections(const void *x, const void *x_proj_weight, const float *dt_projs_weight,
                                         const float *A_logs, const float *Ds, const float *dt_bias, bool softplus,
                                         float *y, void *workspace, int B, int D, int H, int W, int N, int R,
                                         bool ch_last, bool clear_err, cudaStream_t s);

}  // namespace ss2d
