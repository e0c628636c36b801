// proj_bwd.h -- launchers of the projection form's backward (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

// The gradient of x_dbl (B, 4, R+2N, L), scan order, held as three arrays: rows 0..R-1
// (dt_low) in d_dtlow (B, 4, R, L), rows R..R+N-1 in dB and R+N..R+2N-1 in dC (B, 4, N, L).
struct ProjGradRows {
    float *d_dtlow;
    const float *dB;
    const float *dC;
    int R, N;
};

// True when the projection backward supports dt_rank R at state size N with D channels
// (1 <= R <= 64, D % 16 == 0).
bool proj_bwd_supported(int N, int R, int D, int W);

// x_proj's adjoints on the tensor cores (16 <= D <= 256, D % 16 == 0, W % 8 == 0).
bool xproj_bwd_tc_supported(int D, int W);
// Bytes of the partial sums of dWx that launch_xproj_bwd needs.
size_t xproj_bwd_partial_bytes(int N, int R, int D, int W);
// x_proj's adjoints: on the tensor cores (launch_xproj_bwd_tc) where they tile the shape
// (xproj_bwd_tc_supported and 4(R + 2N) <= 256), otherwise on the CUDA cores in fp32.
cudaError_t launch_xproj_bwd(const ProjGradRows &g, const void *Wx, const void *x, float *dx, float *dWx, float *part,
                             int *err, int B, int D, int H, int W, cudaStream_t s);
// dx (B, D, H, W) += Wx^T dP and dWx (4, R+2N, D) = sum over pixels of dP x^T, with dP the
// gradient of x_dbl held in g, x (B, D, H, W) and Wx (4, R+2N, D) bf16; part holds
// xproj_bwd_partial_bytes, err the error word of the kernels' bounded waits.
cudaError_t launch_xproj_bwd_tc(const ProjGradRows &g, const void *Wx, const void *x, float *dx, float *dWx,
                                float *part, int *err, int B, int D, int H, int W, cudaStream_t s);

// dts (B, 4D, L) fp32, scan order: dts[b,k*D+d,l] = sum_r Wdt[k,d,r] xdbl[b,k,r,l].
cudaError_t launch_dtproj_expand(const float *xdbl, const float *Wdt, float *dts, int B, int D, int L, int R, int N,
                                 cudaStream_t s);

// Given ddts (B, 4D, L), dB and dC (in g), and the forward's xdbl, bf16 x and weights:
// writes g.d_dtlow, adds dt_proj's weight gradient into dWdt (4, D, R) (zeroed by the
// caller) and x_proj's adjoint into dx (B, D, H, W), and writes x_proj's weight gradient
// dWx (4, R+2N, D).  part and err as for launch_xproj_bwd_tc.
cudaError_t launch_proj_bwd(const ProjGradRows &g, const float *ddts, const float *xdbl, const float *Wdt,
                            const void *Wx, const void *x, float *dx, float *dWdt, float *dWx, float *part, int *err,
                            int B, int D, int H, int W, cudaStream_t s);

}  // namespace ss2d
