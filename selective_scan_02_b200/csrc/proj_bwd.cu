// proj_bwd.cu -- gradient of the two projections of the core's projection form.
//
// In the projection form (section 3.2 of the VMamba SS2D article) the scan's inputs
// are made from x by two linear maps:
//   x_dbl[b,k,c,l] = sum_d Wx[k,c,d] xs[b,k,d,l]        (x_proj; xs = CrossScan(x))
//   dts[b,k,d,l]   = sum_r Wdt[k,d,r] x_dbl[b,k,r,l]    (dt_proj on the first R rows)
//   B, C           = rows R..R+N-1 and R+N..R+2N-1 of x_dbl.
// Their adjoints are the transposed contractions.  dt_proj's (R multiply-adds per element)
// run here in fp32 on the CUDA cores once the scan's backward has produced ddts, dBs and
// dCs (all in scan order):
//   dtproj_expand_kernel   dts from x_dbl (the forward's dt_proj, materialised for the
//                          backward scan, in the forward's order of operations);
//   dtproj_dgrad_kernel    d_dtlow[b,k,r,l] = sum_d Wdt[k,d,r] ddts[b,k,d,l];
//   dtproj_wgrad_kernel    dWdt[k,d,r] = sum_{b,l} ddts[b,k,d,l] x_dbl[b,k,r,l];
// and then x_proj's adjoints, dx += Wx^T dP and dWx = sum dP x^T, on the tensor cores
// (xproj_bwd.cu), where dP is x_dbl's gradient (d_dtlow, dBs, dCs stacked).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "launch_util.h"
#include "proj_bwd.h"
#include "scan.cuh"

namespace ss2d {

namespace {


__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Thread = step l of one (image, direction): its R dt_low values stay in registers while it
// walks the direction's D channels, whose dt_proj weights (D, R) sit in shared memory.
constexpr int kDtThreads = 128;

__host__ __device__ inline int dt_smem_bytes(int D, int R) { return D * R * (int)sizeof(float); }

__device__ __forceinline__ void load_dt_weights(float *sw, const float *Wdt, int k, int D, int R)
{
    for (int i = threadIdx.x; i < D * R; i += blockDim.x)
        sw[i] = __ldg(Wdt + (size_t)k * D * R + i);
    __syncthreads();
}

__global__ void __launch_bounds__(kDtThreads) dtproj_expand_kernel(const float *__restrict__ xdbl,
                                                                  const float *__restrict__ Wdt,
                                                                  float *__restrict__ dts, int D, int L, int R,
                                                                  int Cp)
{
    extern __shared__ float sw[];
    const int bk = blockIdx.y, k = bk & 3;
    load_dt_weights(sw, Wdt, k, D, R);
    const int l = blockIdx.x * kDtThreads + threadIdx.x;
    if (l >= L)
        return;
    float t[kMaxR];
    const float *src = xdbl + (size_t)bk * Cp * L + l;
#pragma unroll
    for (int r = 0; r < kMaxR; ++r)
        t[r] = r < R ? __ldg(src + (size_t)r * L) : 0.0f;
    float *dst = dts + (size_t)bk * D * L + l;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
        float z = 0.0f;  // the forward's order: r = 0, 1, ..., R-1 from zero
#pragma unroll
        for (int r = 0; r < kMaxR; ++r)
            if (r < R)
                z = fmaf(sw[d * R + r], t[r], z);
        dst[(size_t)d * L] = z;
    }
}

__global__ void __launch_bounds__(kDtThreads) dtproj_dgrad_kernel(const float *__restrict__ ddts,
                                                                 const float *__restrict__ Wdt,
                                                                 float *__restrict__ d_dtlow, int D, int L, int R)
{
    extern __shared__ float sw[];
    const int bk = blockIdx.y, k = bk & 3;
    load_dt_weights(sw, Wdt, k, D, R);
    const int l = blockIdx.x * kDtThreads + threadIdx.x;
    if (l >= L)
        return;
    float acc[kMaxR];
#pragma unroll
    for (int r = 0; r < kMaxR; ++r)
        acc[r] = 0.0f;
    const float *src = ddts + (size_t)bk * D * L + l;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
        const float v = __ldg(src + (size_t)d * L);
#pragma unroll
        for (int r = 0; r < kMaxR; ++r)
            if (r < R)
                acc[r] = fmaf(sw[d * R + r], v, acc[r]);
    }
    float *dst = d_dtlow + (size_t)bk * R * L + l;
#pragma unroll
    for (int r = 0; r < kMaxR; ++r)
        if (r < R)
            dst[(size_t)r * L] = acc[r];
}

// The same two kernels for dt_ranks above kMaxR, or weights (D x R) too large for shared
// memory at once: each (image, direction)'s weights pass through shared memory 64 channels
// at a time, and a thread keeps up to kMaxRLarge values.  The expansion sums r = 0 .. R-1
// from zero like the forward's dtproj_fwd_kernel and the scan's fused dt_proj, so its dts is
// the forward's delta input bit for bit.
constexpr int kDtChunk = 64;
bool dt_chunked(int D, int R) { return R > kMaxR || dt_smem_bytes(D, R) > 96 * 1024; }

__global__ void __launch_bounds__(kDtThreads) dtproj_expand_chunked_kernel(const float *__restrict__ xdbl,
                                                                          const float *__restrict__ Wdt,
                                                                          float *__restrict__ dts, int D, int L,
                                                                          int R, int Cp)
{
    __shared__ float sw[kDtChunk * kMaxRLarge];
    const int bk = blockIdx.y, k = bk & 3;
    const int l = blockIdx.x * kDtThreads + threadIdx.x;
    float t[kMaxRLarge];
    const float *src = xdbl + (size_t)bk * Cp * L + (l < L ? l : 0);
#pragma unroll
    for (int r = 0; r < kMaxRLarge; ++r)
        t[r] = (r < R && l < L) ? __ldg(src + (size_t)r * L) : 0.0f;
    float *dst = dts + (size_t)bk * D * L + l;
    for (int d0 = 0; d0 < D; d0 += kDtChunk) {
        const int nd = min(kDtChunk, D - d0);
        __syncthreads();
        for (int e = threadIdx.x; e < nd * R; e += kDtThreads)
            sw[e] = __ldg(Wdt + ((size_t)k * D + d0) * R + e);
        __syncthreads();
        if (l < L) {
            for (int d = 0; d < nd; ++d) {
                float z = 0.0f;  // the forward's order: r = 0, 1, ..., R-1 from zero
#pragma unroll
                for (int r = 0; r < kMaxRLarge; ++r)
                    if (r < R)
                        z = fmaf(sw[d * R + r], t[r], z);
                dst[(size_t)(d0 + d) * L] = z;
            }
        }
    }
}

__global__ void __launch_bounds__(kDtThreads) dtproj_dgrad_chunked_kernel(const float *__restrict__ ddts,
                                                                         const float *__restrict__ Wdt,
                                                                         float *__restrict__ d_dtlow, int D, int L,
                                                                         int R)
{
    __shared__ float sw[kDtChunk * kMaxRLarge];
    const int bk = blockIdx.y, k = bk & 3;
    const int l = blockIdx.x * kDtThreads + threadIdx.x;
    float acc[kMaxRLarge];
#pragma unroll
    for (int r = 0; r < kMaxRLarge; ++r)
        acc[r] = 0.0f;
    const float *src = ddts + (size_t)bk * D * L + (l < L ? l : 0);
    for (int d0 = 0; d0 < D; d0 += kDtChunk) {
        const int nd = min(kDtChunk, D - d0);
        __syncthreads();
        for (int e = threadIdx.x; e < nd * R; e += kDtThreads)
            sw[e] = __ldg(Wdt + ((size_t)k * D + d0) * R + e);
        __syncthreads();
        if (l < L) {
            for (int d = 0; d < nd; ++d) {
                const float v = __ldg(src + (size_t)(d0 + d) * L);
#pragma unroll
                for (int r = 0; r < kMaxRLarge; ++r)
                    if (r < R)
                        acc[r] = fmaf(sw[d * R + r], v, acc[r]);
            }
        }
    }
    if (l >= L)
        return;
    float *dst = d_dtlow + (size_t)bk * R * L + l;
#pragma unroll
    for (int r = 0; r < kMaxRLarge; ++r)
        if (r < R)
            dst[(size_t)r * L] = acc[r];
}

// Block: direction k, TILE consecutive channels, a slice of the batch; each thread strides
// over the steps, reusing its R dt_low values for the tile's channels.
constexpr int kWgThreads = 256;

template <int RM, int TILE>
__global__ void __launch_bounds__(kWgThreads) dtproj_wgrad_kernel(const float *__restrict__ ddts,
                                                                 const float *__restrict__ xdbl,
                                                                 float *__restrict__ dWdt, int B, int D, int L,
                                                                 int R, int Cp, int b_per_block)
{
    constexpr int kWgTile = TILE;
    __shared__ float red[kWgTile * RM][kWgThreads / 32];
    const int nt = (D + kWgTile - 1) / kWgTile;
    const int k = blockIdx.x / nt, d0 = (blockIdx.x % nt) * kWgTile;
    const int b0 = blockIdx.y * b_per_block, b1 = min(B, b0 + b_per_block);
    float acc[kWgTile][RM];
#pragma unroll
    for (int i = 0; i < kWgTile; ++i)
#pragma unroll
        for (int r = 0; r < RM; ++r)
            acc[i][r] = 0.0f;
    for (int b = b0; b < b1; ++b) {
        const float *g = ddts + ((size_t)b * 4 * D + (size_t)k * D + d0) * L;
        const float *t = xdbl + ((size_t)b * 4 + k) * Cp * L;
#pragma unroll 2
        for (int l = threadIdx.x; l < L; l += kWgThreads) {
            float tv[RM];
#pragma unroll
            for (int r = 0; r < RM; ++r)
                tv[r] = r < R ? __ldg(t + (size_t)r * L + l) : 0.0f;
#pragma unroll
            for (int i = 0; i < kWgTile; ++i) {
                if (d0 + i < D) {
                    const float v = __ldg(g + (size_t)i * L + l);
#pragma unroll
                    for (int r = 0; r < RM; ++r)
                        if (r < R)
                            acc[i][r] = fmaf(v, tv[r], acc[i][r]);
                }
            }
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < kWgTile; ++i)
#pragma unroll
        for (int r = 0; r < RM; ++r) {
            if (r < R) {
                const float v = warp_sum(acc[i][r]);
                if (lane == 0)
                    red[i * RM + r][warp] = v;
            }
        }
    __syncthreads();
    for (int o = threadIdx.x; o < kWgTile * RM; o += kWgThreads) {
        const int i = o / RM, r = o % RM;
        if (r < R && d0 + i < D) {
            float sum = 0.0f;
#pragma unroll
            for (int w = 0; w < kWgThreads / 32; ++w)
                sum += red[o][w];
            atomicAdd(dWdt + ((size_t)k * D + d0 + i) * R + r, sum);
        }
    }
}

int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return sms;
}

}  // namespace

bool proj_bwd_supported(int N, int R, int D, int W)
{
    (void)N;
    (void)W;
    return R >= 1 && R <= kMaxRLarge && D % 16 == 0 && D >= 16;
}

cudaError_t launch_dtproj_expand(const float *xdbl, const float *Wdt, float *dts, int B, int D, int L, int R, int N,
                                 cudaStream_t s)
{
    if (B < 1 || B * 4 > 65535)
        return cudaErrorInvalidValue;
    const dim3 grid((L + kDtThreads - 1) / kDtThreads, B * 4);
    if (dt_chunked(D, R)) {
        dtproj_expand_chunked_kernel<<<grid, kDtThreads, 0, s>>>(xdbl, Wdt, dts, D, L, R, R + 2 * N);
        return cudaGetLastError();
    }
    static int configured[kMaxDevices] = {};
    const int smem = dt_smem_bytes(D, R);
    cudaError_t e = configure_smem(dtproj_expand_kernel, smem, configured);
    if (e != cudaSuccess)
        return e;
    dtproj_expand_kernel<<<grid, kDtThreads, smem, s>>>(xdbl, Wdt, dts, D, L, R, R + 2 * N);
    return cudaGetLastError();
}

cudaError_t launch_proj_bwd(const ProjGradRows &g, const float *ddts, const float *xdbl, const float *Wdt,
                            const void *Wx, const void *x, float *dx, float *dWdt, float *dWx, float *part, int *err,
                            int B, int D, int H, int W, cudaStream_t s)
{
    const int L = H * W, R = g.R, Cp = g.R + 2 * g.N;
    if (B < 1 || B * 4 > 65535)
        return cudaErrorInvalidValue;
    // d_dtlow, then dWdt
    cudaError_t e = cudaSuccess;
    const dim3 dt_grid((L + kDtThreads - 1) / kDtThreads, B * 4);
    if (dt_chunked(D, R)) {
        dtproj_dgrad_chunked_kernel<<<dt_grid, kDtThreads, 0, s>>>(ddts, Wdt, g.d_dtlow, D, L, R);
    } else {
        static int configured_dt[kMaxDevices] = {};
        const int dsm = dt_smem_bytes(D, R);
        e = configure_smem(dtproj_dgrad_kernel, dsm, configured_dt);
        if (e != cudaSuccess)
            return e;
        dtproj_dgrad_kernel<<<dt_grid, kDtThreads, dsm, s>>>(ddts, Wdt, g.d_dtlow, D, L, R);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int tile = R <= 16 ? 4 : (R <= 32 ? 2 : 1);
    const int nt = (D + tile - 1) / tile;
    int bpb = 1;
    while (bpb < B && (long long)4 * nt * ((B + 2 * bpb - 1) / (2 * bpb)) >= 16LL * sm_count())
        bpb *= 2;
    const dim3 wg_grid(4 * nt, (B + bpb - 1) / bpb);
    if (R <= 8)
        dtproj_wgrad_kernel<8, 4><<<wg_grid, kWgThreads, 0, s>>>(ddts, xdbl, dWdt, B, D, L, R, Cp, bpb);
    else if (R <= 16)
        dtproj_wgrad_kernel<16, 4><<<wg_grid, kWgThreads, 0, s>>>(ddts, xdbl, dWdt, B, D, L, R, Cp, bpb);
    else if (R <= 32)
        dtproj_wgrad_kernel<32, 2><<<wg_grid, kWgThreads, 0, s>>>(ddts, xdbl, dWdt, B, D, L, R, Cp, bpb);
    else
        dtproj_wgrad_kernel<64, 1><<<wg_grid, kWgThreads, 0, s>>>(ddts, xdbl, dWdt, B, D, L, R, Cp, bpb);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    // x_proj's adjoints: tensor cores where they tile the shape, else the CUDA cores
    return launch_xproj_bwd(g, Wx, x, dx, dWx, part, err, B, D, H, W, s);
}

}  // namespace ss2d
