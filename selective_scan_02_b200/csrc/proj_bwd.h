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

// True when the projection backward supports dt_rank R at state size N (R <= 16, R + 2N <= 48).
bool proj_bwd_supported(int N, int R);

// dts (B, 4D, L) fp32, scan order: dts[b,k*D+d,l] = sum_r Wdt[k,d,r] xdbl[b,k,r,l].
cudaError_t launch_dtproj_expand(const float *xdbl, const float *Wdt, float *dts, int B, int D, int L, int R, int N,
                                 cudaStream_t s);

// Given ddts (B, 4D, L), dB and dC (in g), and the forward's xdbl and weights: writes
// g.d_dtlow, adds dt_proj's weight gradient into dWdt (4, D, R), x_proj's adjoint into dx
// (B, D, H, W) and x_proj's weight gradient into dWx (4, R+2N, D).  x32 is x (B, D, H, W) in
// fp32 and xT32 the same with transposed planes (B, D, W, H).  dWdt and dWx must be zeroed
// by the caller.
cudaError_t launch_proj_bwd(const ProjGradRows &g, const float *ddts, const float *xdbl, const float *Wdt,
                            const void *Wx, const float *x32, const float *xT32, float *dx, float *dWdt, float *dWx,
                            int B, int D, int H, int W, cudaStream_t s);

}  // namespace ss2d
