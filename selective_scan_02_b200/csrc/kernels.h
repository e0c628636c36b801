// kernels.h -- host-side launchers of the libss2d kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ss2d {

struct ScanArgs;
struct BwdArgs;

cudaError_t launch_cross_scan(const void *x, bool bf16, void *xs, int B, int D, int H, int W, cudaStream_t s);
cudaError_t launch_cross_merge(const float *ys, float *y, int B, int D, int H, int W, cudaStream_t s);
cudaError_t launch_fill_zero(float *p, size_t n, cudaStream_t s);
// y = ((y + y2) + y1) + y3 element-wise (the page-order merge of four per-direction outputs).
cudaError_t launch_page_order_sum(float *y, const float *y1, const float *y2, const float *y3, size_t n,
                                  cudaStream_t s);
// dst[i] = src[i] rounded to nearest-even bf16, for n fp32 values.
cudaError_t launch_f32_to_bf16(const float *src, void *dst, size_t n, cudaStream_t s);
// dst[i] = src[i] for n bf16 values widened to fp32.
cudaError_t launch_bf16_to_f32(const void *src, float *dst, size_t n, cudaStream_t s);
// xT[plane, w*H + h] = x[plane, h*W + w] for `planes` planes of (H, W) elements.
cudaError_t launch_transpose_planes(const void *x, bool bf16, void *xT, int planes, int H, int W, cudaStream_t s);
// The same for bf16 planes with H and W even, setting the fp32 planes y_zero (same shape) to
// zero in the same kernel.
bool transpose_planes_can_zero(bool bf16, int H, int W);
cudaError_t launch_transpose_planes_zero(const void *x, void *xT, float *y_zero, int planes, int H, int W,
                                         cudaStream_t s);

// True when the fused scan of these arguments reads u of the column-major orders from a
// transposed copy of x (ScanArgs::uT, (B, D, W, H)) instead of gathering it from x:
// the N = 16 kernel (whole or segmented sequences), with rows of L elements 16-byte aligned.
bool scan_reads_transposed_u(int N, int mode, int u_bf16, int delta_bf16, int softplus, int L);

// mode: 0 standalone scan, 1 fused core (u gathered from x, output merged into y),
// 2 fused core with projections.  Scans whole sequences (a.nseg <= 1).
cudaError_t launch_scan(const ScanArgs &a, int N, int mode, cudaStream_t s);

// Segmented fused scan for long sequences with few channels (few images): splits each
// sequence into *nseg segments of *seg_len steps (nseg = 1 when splitting does not pay).
// Planned for the N = 16 kernel in modes 1 and 2.
void plan_segments(int B, int G, int per_group, int L, int N, int mode, int u_bf16, int delta_bf16, int softplus,
                   int *nseg, int *seg_len);
size_t segment_workspace_bytes(int B, int C, int nseg, int N);
// Checkpoint pass of the backward of the fused N = 16 scan (bf16 or fp32 u and delta, softplus
// on): the state before every 16th step of every channel into ckpt, laid out as
// ScanArgs::ckpt describes.
cudaError_t launch_scan_checkpoints(const ScanArgs &a, float *ckpt, cudaStream_t s);
// The same, segmented (a.nseg > 1, a.seg_len a multiple of 32): first pass, carry, then the
// checkpoint pass from the carried states; seg_ws holds segment_workspace_bytes.
cudaError_t launch_scan_checkpoints_segmented(const ScanArgs &a, float *ckpt, float *seg_ws, cudaStream_t s);

// First pass, carry and second pass of a segmented fused scan, mode 1 (dts given) or 2
// (delta from dt_low) (a.nseg, a.seg_len set, seg_len a multiple of 32; seg_ws holds
// segment_workspace_bytes).
cudaError_t launch_scan_segmented(const ScanArgs &a, int N, int mode, float *seg_ws, cudaStream_t s);

}  // namespace ss2d

namespace ss2d {

// True when the backward of the fused core supports these arguments: N = 16, u and delta
// both bf16 or both fp32, softplus on.  bf16 inputs are widened to fp32 before the backward
// scan runs.
bool scan_bwd_supported(int N, int u_bf16, int delta_bf16, int softplus, int L);
// The backward walk's segment plan for B images of D channels and L steps: *nseg = 1 (whole
// sequences) when the 16-channel items of all four directions fill a wave of
// scan_bwd_kernel CTAs, when L < 256 or when L % 4 != 0; else segments of *seg_len steps (a
// multiple of 32, at least 128) chosen to fill the walk's waves.
int scan_bwd_ctas_per_sm();
void plan_bwd_segments(int B, int D, int L, int *nseg, int *seg_len);
// The backward scan kernel on fp32 x and dts (checkpoints, transposed x and dy in place).
cudaError_t launch_scan_bwd(const BwdArgs &a, cudaStream_t s);

}  // namespace ss2d
