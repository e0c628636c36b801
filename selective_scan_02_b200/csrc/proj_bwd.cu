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
//                          backward scan, in the forward's order of operations;
//                          dtproj_expand4_kernel does four steps per thread when L % 4 == 0);
//   dtproj_dgrad_kernel    d_dtlow[b,k,r,l] = sum_d Wdt[k,d,r] ddts[b,k,d,l];
//   dtproj_wgrad_kernel    dWdt[k,d,r] = sum_{b,l} ddts[b,k,d,l] x_dbl[b,k,r,l];
//   dtproj_adj_kernel      both adjoints from one shared-memory copy of each ddts tile, where
//                          the weights and a 64-step tile of every channel fit (D <= 256,
//                          R <= 16, L % 4 == 0); the two kernels above elsewhere;
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

// The same expansion, four steps per thread (L % 4 == 0): the dt_low values and the stores
// are 16 bytes wide, and each weight read from shared memory serves four steps.  Every step
// keeps the order r = 0, 1, ..., R-1 from zero, so the result is dtproj_expand_kernel's.
__global__ void __launch_bounds__(kDtThreads) dtproj_expand4_kernel(const float *__restrict__ xdbl,
                                                                   const float *__restrict__ Wdt,
                                                                   float *__restrict__ dts, int D, int L, int R,
                                                                   int Cp)
{
    extern __shared__ float sw[];
    const int bk = blockIdx.y, k = bk & 3;
    load_dt_weights(sw, Wdt, k, D, R);
    const int l = (blockIdx.x * kDtThreads + threadIdx.x) * 4;
    if (l >= L)
        return;
    float4 t[kMaxR];
    const float *src = xdbl + (size_t)bk * Cp * L + l;
#pragma unroll
    for (int r = 0; r < kMaxR; ++r)
        t[r] = r < R ? __ldg(reinterpret_cast<const float4 *>(src + (size_t)r * L)) : make_float4(0.f, 0.f, 0.f, 0.f);
    float *dst = dts + (size_t)bk * D * L + l;
#pragma unroll 2
    for (int d = 0; d < D; ++d) {
        float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kMaxR; ++r) {
            if (r < R) {
                const float w = sw[d * R + r];
                z.x = fmaf(w, t[r].x, z.x);
                z.y = fmaf(w, t[r].y, z.y);
                z.z = fmaf(w, t[r].z, z.z);
                z.w = fmaf(w, t[r].w, z.w);
            }
        }
        *reinterpret_cast<float4 *>(dst + (size_t)d * L) = z;
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

// dt_proj's two adjoints in one pass over ddts (R <= 16, D <= 256, L % 4 == 0).  A CTA keeps
// one direction k and walks tiles of 64 steps of that direction's images.  Each tile of ddts
// (D x 64) and of dt_low (R x 64) is copied once into shared memory, and both contractions
// read it there:
//   d_dtlow[b,k,r,l] = sum_d Wdt[k,d,r] ddts[b,k,d,l]: thread = (step, quarter of the
//                      channels); the four partial sums are added in a fixed order;
//   dWdt[k,d,r]     += sum_l ddts[b,k,d,l] dt_low[b,k,r,l]: thread = channel; each tile's
//                      64 products are summed in two interleaved halves and added to a register
//                      total over the CTA's tiles, then one atomic add per entry at the end.
// The two separate kernels above read ddts twice and the dt_low rows once per channel tile.
constexpr int kAdjThreads = 256, kAdjLT = 64, kAdjLP = kAdjLT + 4, kAdjMaxD = 256;

// Shared memory (floats): ddts tile (D, kAdjLP), dt_low tile (RM, kAdjLP), Wdt[k] (D, RM),
// partial sums (4, RM, kAdjLT).  The row pitch of 68 floats keeps 16-byte rows aligned and
// makes the channel-per-thread float4 reads conflict-free (17 16-byte units per row).
__host__ __device__ inline int adj_smem_bytes(int D, int RM)
{
    return (D * kAdjLP + RM * kAdjLP + D * RM + 4 * RM * kAdjLT) * (int)sizeof(float);
}

template <int RM>
__global__ void __launch_bounds__(kAdjThreads) dtproj_adj_kernel(const float *__restrict__ ddts,
                                                                const float *__restrict__ xdbl,
                                                                const float *__restrict__ Wdt,
                                                                float *__restrict__ d_dtlow,
                                                                float *__restrict__ dWdt, int B, int D, int L,
                                                                int R, int Cp)
{
    extern __shared__ __align__(16) float adj_smem[];
    float *sg = adj_smem;
    float *st = sg + D * kAdjLP;
    float *sw = st + RM * kAdjLP;
    float *sred = sw + D * RM;
    const int k = blockIdx.y, tid = threadIdx.x;
    for (int i = tid; i < D * RM; i += kAdjThreads) {
        const int d = i / RM, r = i % RM;
        sw[i] = r < R ? __ldg(Wdt + ((size_t)k * D + d) * R + r) : 0.0f;
    }
    for (int i = R * kAdjLP + tid; i < RM * kAdjLP; i += kAdjThreads)
        st[i] = 0.0f;  // dt_low rows R..RM-1 stay zero
    float acc[RM];
#pragma unroll
    for (int r = 0; r < RM; ++r)
        acc[r] = 0.0f;
    const int nlt = (L + kAdjLT - 1) / kAdjLT;
    const long long ntiles = (long long)B * nlt;
    const int s = tid & (kAdjLT - 1), q = tid / kAdjLT;  // d_dtlow: step and channel quarter
    for (long long j = blockIdx.x; j < ntiles; j += gridDim.x) {
        const int b = (int)(j / nlt), l0 = (int)(j % nlt) * kAdjLT;
        const float *g = ddts + ((size_t)b * 4 + k) * D * L;
        const float *t = xdbl + ((size_t)b * 4 + k) * Cp * L;
        __syncthreads();  // the previous tile's readers are done with sg, st and sred
        for (int p = tid; p < (D + R) * (kAdjLT / 4); p += kAdjThreads) {
            const int row = p / (kAdjLT / 4), c = (p % (kAdjLT / 4)) * 4;
            const int bytes = l0 + c < L ? 16 : 0;  // L % 4 == 0: a piece is whole or past the end
            const size_t off = bytes ? (size_t)l0 + c : 0;
            if (row < D)
                cp_async16(sg + row * kAdjLP + c, g + (size_t)row * L + off, bytes);
            else
                cp_async16(st + (row - D) * kAdjLP + c, t + (size_t)(row - D) * L + off, bytes);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        float a[RM];
#pragma unroll
        for (int r = 0; r < RM; ++r)
            a[r] = 0.0f;
#pragma unroll 4
        for (int d = q; d < D; d += kAdjThreads / kAdjLT) {
            const float v = sg[d * kAdjLP + s];
            const float4 *w4 = reinterpret_cast<const float4 *>(sw + d * RM);
#pragma unroll
            for (int r4 = 0; r4 < RM / 4; ++r4) {
                if (4 * r4 < R) {
                    const float4 w = w4[r4];
                    a[4 * r4] = fmaf(w.x, v, a[4 * r4]);
                    a[4 * r4 + 1] = fmaf(w.y, v, a[4 * r4 + 1]);
                    a[4 * r4 + 2] = fmaf(w.z, v, a[4 * r4 + 2]);
                    a[4 * r4 + 3] = fmaf(w.w, v, a[4 * r4 + 3]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RM; ++r)
            if (r < R)
                sred[(q * RM + r) * kAdjLT + s] = a[r];
        __syncthreads();
        for (int o = tid; o < R * kAdjLT; o += kAdjThreads) {
            const int r = o / kAdjLT, so = o % kAdjLT;
            if (l0 + so < L) {
                const float v = ((sred[r * kAdjLT + so] + sred[(RM + r) * kAdjLT + so]) +
                                 sred[(2 * RM + r) * kAdjLT + so]) +
                                sred[(3 * RM + r) * kAdjLT + so];
                d_dtlow[(((size_t)b * 4 + k) * R + r) * L + l0 + so] = v;
            }
        }
        if (tid < D) {
            // the tile's sum in two halves of 32 steps (even and odd pairs), then into the total
            float p0[RM], p1[RM];
#pragma unroll
            for (int r = 0; r < RM; ++r) {
                p0[r] = 0.0f;
                p1[r] = 0.0f;
            }
            const float4 *gr = reinterpret_cast<const float4 *>(sg + tid * kAdjLP);
#pragma unroll 4
            for (int s4 = 0; s4 < kAdjLT / 4; ++s4) {
                const float4 gv = gr[s4];
#pragma unroll
                for (int r = 0; r < RM; ++r) {
                    if (r < R) {
                        const float4 tv = reinterpret_cast<const float4 *>(st + r * kAdjLP)[s4];
                        p0[r] = fmaf(gv.x, tv.x, p0[r]);
                        p1[r] = fmaf(gv.y, tv.y, p1[r]);
                        p0[r] = fmaf(gv.z, tv.z, p0[r]);
                        p1[r] = fmaf(gv.w, tv.w, p1[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RM; ++r)
                acc[r] += p0[r] + p1[r];
        }
    }
    if (tid < D) {
#pragma unroll
        for (int r = 0; r < RM; ++r)
            if (r < R)
                atomicAdd(dWdt + ((size_t)k * D + tid) * R + r, acc[r]);
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
    const int smem = dt_smem_bytes(D, R);
    if (L % 4 == 0 && (((uintptr_t)xdbl | (uintptr_t)dts) & 15) == 0) {
        static int configured4[kMaxDevices] = {};
        cudaError_t e = configure_smem(dtproj_expand4_kernel, smem, configured4);
        if (e != cudaSuccess)
            return e;
        const dim3 grid4((L / 4 + kDtThreads - 1) / kDtThreads, B * 4);
        dtproj_expand4_kernel<<<grid4, kDtThreads, smem, s>>>(xdbl, Wdt, dts, D, L, R, R + 2 * N);
        return cudaGetLastError();
    }
    static int configured[kMaxDevices] = {};
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
    cudaError_t e = cudaSuccess;
    if (!dt_chunked(D, R) && D <= kAdjMaxD && L % 4 == 0 && (((uintptr_t)ddts | (uintptr_t)xdbl) & 15) == 0) {
        // both adjoints in one pass over ddts; a grid of one wave, each CTA keeping one direction
        const int rm = R <= 8 ? 8 : 16;
        const int smem = adj_smem_bytes(D, rm);
        int per_sm = (228 * 1024) / (smem + 1024);
        per_sm = per_sm < 1 ? 1 : (per_sm > 2048 / kAdjThreads ? 2048 / kAdjThreads : per_sm);
        const long long ntiles = (long long)B * ((L + kAdjLT - 1) / kAdjLT);
        long long gx = (long long)sm_count() * per_sm / 4;
        gx = gx < 1 ? 1 : (gx > ntiles ? ntiles : gx);
        const dim3 grid((unsigned)gx, 4);
        if (rm == 8) {
            static int configured_a8[kMaxDevices] = {};
            e = configure_smem(dtproj_adj_kernel<8>, smem, configured_a8);
            if (e != cudaSuccess)
                return e;
            dtproj_adj_kernel<8><<<grid, kAdjThreads, smem, s>>>(ddts, xdbl, Wdt, g.d_dtlow, dWdt, B, D, L, R, Cp);
        } else {
            static int configured_a16[kMaxDevices] = {};
            e = configure_smem(dtproj_adj_kernel<16>, smem, configured_a16);
            if (e != cudaSuccess)
                return e;
            dtproj_adj_kernel<16><<<grid, kAdjThreads, smem, s>>>(ddts, xdbl, Wdt, g.d_dtlow, dWdt, B, D, L, R, Cp);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
        return launch_xproj_bwd(g, Wx, x, dx, dWx, part, err, B, D, H, W, s);
    }
    // d_dtlow, then dWdt
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
