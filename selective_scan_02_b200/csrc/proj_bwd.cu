// proj_bwd.cu -- gradient of the two projections of the core's projection form.
//
// In the projection form (section 3.2 of the VMamba SS2D article) the scan's inputs
// are made from x by two linear maps:
//   x_dbl[b,k,c,l] = sum_d Wx[k,c,d] xs[b,k,d,l]        (x_proj; xs = CrossScan(x))
//   dts[b,k,d,l]   = sum_r Wdt[k,d,r] x_dbl[b,k,r,l]    (dt_proj on the first R rows)
//   B, C           = rows R..R+N-1 and R+N..R+2N-1 of x_dbl.
// Their adjoints are the transposed contractions, computed here in fp32 on the CUDA
// cores once the scan's backward has produced ddts, dBs and dCs (all in scan order):
//   dtproj_expand_kernel   dts from x_dbl (the forward's dt_proj, materialised for the
//                          backward scan, in the forward's order of operations);
//   dtproj_dgrad_kernel    d_dtlow[b,k,r,l] = sum_d Wdt[k,d,r] ddts[b,k,d,l];
//   dtproj_wgrad_kernel    dWdt[k,d,r] = sum_{b,l} ddts[b,k,d,l] x_dbl[b,k,r,l];
//   xproj_dgrad_kernel     dx[b,d,p] += sum_{k,c} Wx[k,c,d] dP[b,k,c,l_k(p)], where dP is
//                          x_dbl's gradient (d_dtlow, dBs, dCs stacked) and l_k(p) the step
//                          at which direction k visits pixel p (CrossScan's adjoint is
//                          CrossMerge);
//   xproj_wgrad_kernel     dWx[k,c,d] = sum_{b,l} dP[b,k,c,l] xs[b,k,d,l], with xs read as
//                          rows of x (directions 0/2) or of x with transposed planes (1/3),
//                          forwards or backwards.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "proj_bwd.h"
#include "scan.cuh"

namespace ss2d {

namespace {

constexpr int kMaxCp = kMaxR + 32;  // rows of x_dbl at N = 16

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Row c of direction k of x_dbl's gradient for image b: d_dtlow, dBs or dCs.
__device__ __forceinline__ const float *dp_row(const ProjGradRows &g, int b, int k, int c, int L)
{
    const size_t bk = (size_t)b * 4 + k;
    if (c < g.R)
        return g.d_dtlow + (bk * g.R + c) * L;
    if (c < g.R + g.N)
        return g.dB + (bk * g.N + (c - g.R)) * L;
    return g.dC + (bk * g.N + (c - g.R - g.N)) * L;
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

// Block: direction k, kWgTile consecutive channels, a slice of the batch; each thread
// strides over the steps, reusing its R dt_low values for the tile's channels.
constexpr int kWgThreads = 256;
constexpr int kWgTile = 4;

__global__ void __launch_bounds__(kWgThreads) dtproj_wgrad_kernel(const float *__restrict__ ddts,
                                                                 const float *__restrict__ xdbl,
                                                                 float *__restrict__ dWdt, int B, int D, int L,
                                                                 int R, int Cp, int b_per_block)
{
    __shared__ float red[kWgTile * kMaxR][kWgThreads / 32];
    const int nt = (D + kWgTile - 1) / kWgTile;
    const int k = blockIdx.x / nt, d0 = (blockIdx.x % nt) * kWgTile;
    const int b0 = blockIdx.y * b_per_block, b1 = min(B, b0 + b_per_block);
    float acc[kWgTile][kMaxR];
#pragma unroll
    for (int i = 0; i < kWgTile; ++i)
#pragma unroll
        for (int r = 0; r < kMaxR; ++r)
            acc[i][r] = 0.0f;
    for (int b = b0; b < b1; ++b) {
        const float *g = ddts + ((size_t)b * 4 * D + (size_t)k * D + d0) * L;
        const float *t = xdbl + ((size_t)b * 4 + k) * Cp * L;
        for (int l = threadIdx.x; l < L; l += kWgThreads) {
            float tv[kMaxR];
#pragma unroll
            for (int r = 0; r < kMaxR; ++r)
                tv[r] = r < R ? __ldg(t + (size_t)r * L + l) : 0.0f;
#pragma unroll
            for (int i = 0; i < kWgTile; ++i) {
                if (d0 + i < D) {
                    const float v = __ldg(g + (size_t)i * L + l);
#pragma unroll
                    for (int r = 0; r < kMaxR; ++r)
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
        for (int r = 0; r < kMaxR; ++r) {
            if (r < R) {
                const float v = warp_sum(acc[i][r]);
                if (lane == 0)
                    red[i * kMaxR + r][warp] = v;
            }
        }
    __syncthreads();
    for (int o = threadIdx.x; o < kWgTile * kMaxR; o += kWgThreads) {
        const int i = o / kMaxR, r = o % kMaxR;
        if (r < R && d0 + i < D) {
            float sum = 0.0f;
#pragma unroll
            for (int w = 0; w < kWgThreads / 32; ++w)
                sum += red[o][w];
            atomicAdd(dWdt + ((size_t)k * D + d0 + i) * R + r, sum);
        }
    }
}

// ---- dx += x_proj's adjoint ------------------------------------------------------------
// Block: an 8 x 8 pixel tile of one image and 96 channels; thread (dq, pq) owns channels
// 6dq..6dq+5 and pixels 4pq..4pq+3 of the tile.  Shared memory holds the tile's column of
// dP for all 4*Cp rows (gathered at each direction's scan index of the pixels) and the
// matching 96-channel slice of Wx, both fp32.
constexpr int kDgTile = 8;
constexpr int kDgPix = kDgTile * kDgTile;
constexpr int kDgCh = 96;
constexpr int kDgThreads = 256;

__host__ __device__ inline int dgrad_smem_bytes(int Cp) { return 4 * Cp * (kDgPix + kDgCh) * (int)sizeof(float); }

__global__ void __launch_bounds__(kDgThreads) xproj_dgrad_kernel(const ProjGradRows g,
                                                                const __nv_bfloat16 *__restrict__ Wx,
                                                                float *__restrict__ dx, int D, int H, int W,
                                                                int tiles_w, int tiles_h)
{
    extern __shared__ __align__(16) float sm[];
    const int Cp = g.R + 2 * g.N, NP = 4 * Cp, L = H * W;
    float *sP = sm;                        // [NP][kDgPix]
    float *sW = sm + (size_t)NP * kDgPix;  // [NP][kDgCh]
    int t = blockIdx.x;
    const int tw = t % tiles_w;
    t /= tiles_w;
    const int th = t % tiles_h;
    const int b = t / tiles_h;
    const int d0 = blockIdx.y * kDgCh;
    const int h0 = th * kDgTile, w0 = tw * kDgTile;

    {
        // thread = one pixel of the tile (j) and every fourth row; for the column-major
        // directions the pixels are enumerated column by column, so that consecutive
        // threads read consecutive steps
        const int j = threadIdx.x % kDgPix, c0 = threadIdx.x / kDgPix;
        constexpr int kRowStep = kDgThreads / kDgPix;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int hl = (k & 1) ? (j & 7) : (j >> 3), wl = (k & 1) ? (j >> 3) : (j & 7);
            const int h = h0 + hl, w = w0 + wl;
            const bool inside = h < H && w < W;
            const int pk = (k & 1) ? w * H + h : h * W + w;
            const int l = inside ? ((k & 2) ? L - 1 - pk : pk) : 0;
            float *dst = sP + (size_t)(k * Cp) * kDgPix + hl * kDgTile + wl;
            for (int c = c0; c < Cp; c += kRowStep)
                dst[c * kDgPix] = inside ? __ldg(dp_row(g, b, k, c, L) + l) : 0.0f;
        }
    }
    for (int idx = threadIdx.x; idx < NP * kDgCh; idx += kDgThreads) {
        const int n = idx / kDgCh, dl = idx % kDgCh;
        const int d = d0 + dl;
        sW[idx] = d < D ? __bfloat162float(Wx[(size_t)n * D + d]) : 0.0f;
    }
    __syncthreads();

    const int dq = threadIdx.x / 16, pq = threadIdx.x % 16;
    float acc[6][4];
#pragma unroll
    for (int i = 0; i < 6; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.0f;
    for (int n = 0; n < NP; ++n) {
        const float4 p = *reinterpret_cast<const float4 *>(sP + n * kDgPix + 4 * pq);
        const float2 w01 = *reinterpret_cast<const float2 *>(sW + n * kDgCh + 6 * dq);
        const float2 w23 = *reinterpret_cast<const float2 *>(sW + n * kDgCh + 6 * dq + 2);
        const float2 w45 = *reinterpret_cast<const float2 *>(sW + n * kDgCh + 6 * dq + 4);
        const float pv[4] = {p.x, p.y, p.z, p.w}, wv[6] = {w01.x, w01.y, w23.x, w23.y, w45.x, w45.y};
#pragma unroll
        for (int i = 0; i < 6; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc[i][j] = fmaf(wv[i], pv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 6; ++i) {
        const int d = d0 + 6 * dq + i;
        if (d >= D)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = 4 * pq + j;
            const int h = h0 + p / kDgTile, w = w0 + p % kDgTile;
            if (h < H && w < W) {
                float *o = dx + (((size_t)b * D + d) * H + h) * W + w;
                *o += acc[i][j];
            }
        }
    }
}

// ---- dWx = sum over pixels of dP xs^T ------------------------------------------------------
// Block: one direction k, 64 channels, and a slice of the (image, 32-step chunk) pairs;
// thread (cq, dq) owns rows 4cq..4cq+3 of x_dbl and channels 4dq..4dq+3.  Each chunk
// stages dP rows and xs rows transposed ([step][row]) so the inner loop reads float4s.
constexpr int kWxSteps = 32;
constexpr int kWxCh = 64;
constexpr int kWxRows = kMaxCp;                    // rows of x_dbl held (Cp <= 48)
constexpr int kWxThreads = (kWxRows / 4) * (kWxCh / 4);  // 12 x 16 = 192
static_assert(kWxThreads % kWxSteps == 0, "staging assigns whole steps to threads");

__global__ void __launch_bounds__(kWxThreads) xproj_wgrad_kernel(const ProjGradRows g, const float *__restrict__ x32,
                                                                const float *__restrict__ xT32,
                                                                float *__restrict__ dWx, int B, int D, int L,
                                                                int chunks_per_block)
{
    // row pitches padded by 4 floats: the staging writes (step fastest) then hit 4-way bank
    // conflicts at most, and the float4 reads stay 16-byte aligned
    __shared__ __align__(16) float sG[kWxSteps][kWxRows + 4];
    __shared__ __align__(16) float sX[kWxSteps][kWxCh + 4];
    const int Cp = g.R + 2 * g.N;
    const int nd = (D + kWxCh - 1) / kWxCh;
    const int k = blockIdx.x / nd;
    const int d0 = (blockIdx.x % nd) * kWxCh;
    const int nlc = (L + kWxSteps - 1) / kWxSteps;
    const long long total = (long long)B * nlc;
    const long long ch0 = (long long)blockIdx.y * chunks_per_block;
    const long long ch1 = min(total, ch0 + chunks_per_block);
    const bool rev = (k & 2) != 0;
    const float *xsrc = (k & 1) ? xT32 : x32;
    const int cq = threadIdx.x / (kWxCh / 4), dq = threadIdx.x % (kWxCh / 4);

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.0f;

    for (long long chunk = ch0; chunk < ch1; ++chunk) {
        const int b = (int)(chunk / nlc);
        const int l0 = (int)(chunk % nlc) * kWxSteps;
        __syncthreads();
        {
            // thread = one step (s) and every sixth row: consecutive threads read consecutive steps
            constexpr int kRowStep = kWxThreads / kWxSteps;
            const int s = threadIdx.x % kWxSteps, r0 = threadIdx.x / kWxSteps;
            const int l = l0 + s;
            const bool ok = l < L;
            for (int c = r0; c < kWxRows; c += kRowStep)
                sG[s][c] = (c < Cp && ok) ? __ldg(dp_row(g, b, k, c, L) + l) : 0.0f;
            const float *xrow = xsrc + ((size_t)b * D + d0) * L + (ok ? (rev ? L - 1 - l : l) : 0);
            for (int dl = r0; dl < kWxCh; dl += kRowStep)
                sX[s][dl] = (ok && d0 + dl < D) ? __ldg(xrow + (size_t)dl * L) : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < kWxSteps; ++s) {
            const float4 gv = *reinterpret_cast<const float4 *>(&sG[s][4 * cq]);
            const float4 xv = *reinterpret_cast<const float4 *>(&sX[s][4 * dq]);
            const float ga[4] = {gv.x, gv.y, gv.z, gv.w}, xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(ga[i], xa[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int c = 4 * cq + i;
        if (c >= Cp)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int d = d0 + 4 * dq + j;
            if (d < D)
                atomicAdd(dWx + ((size_t)k * Cp + c) * D + d, acc[i][j]);
        }
    }
}

int g_sms = 0;

int sm_count()
{
    if (g_sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            g_sms = 148;
    }
    return g_sms;
}

}  // namespace

bool proj_bwd_supported(int N, int R) { return R >= 1 && R <= kMaxR && R + 2 * N <= kMaxCp; }

// Opt in to more than 48 KB of dynamic shared memory for kernel f once per device.
template <class F>
cudaError_t allow_smem(F f, int bytes, int *configured)
{
    if (bytes <= 48 * 1024 || bytes <= *configured)
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        *configured = bytes;
    return e;
}

cudaError_t launch_dtproj_expand(const float *xdbl, const float *Wdt, float *dts, int B, int D, int L, int R, int N,
                                 cudaStream_t s)
{
    if (B < 1 || B * 4 > 65535)
        return cudaErrorInvalidValue;
    static int configured = 0;
    const int smem = dt_smem_bytes(D, R);
    cudaError_t e = allow_smem(dtproj_expand_kernel, smem, &configured);
    if (e != cudaSuccess)
        return e;
    dtproj_expand_kernel<<<dim3((L + kDtThreads - 1) / kDtThreads, B * 4), kDtThreads, smem, s>>>(xdbl, Wdt, dts, D,
                                                                                               L, R, R + 2 * N);
    return cudaGetLastError();
}

cudaError_t launch_proj_bwd(const ProjGradRows &g, const float *ddts, const float *xdbl, const float *Wdt,
                            const void *Wx, const float *x32, const float *xT32, float *dx, float *dWdt, float *dWx,
                            int B, int D, int H, int W, cudaStream_t s)
{
    const int L = H * W, R = g.R, Cp = g.R + 2 * g.N;
    if (B < 1 || B * 4 > 65535)
        return cudaErrorInvalidValue;
    // d_dtlow, then dWdt
    static int configured_dt = 0;
    const int dsm = dt_smem_bytes(D, R);
    cudaError_t e = allow_smem(dtproj_dgrad_kernel, dsm, &configured_dt);
    if (e != cudaSuccess)
        return e;
    dtproj_dgrad_kernel<<<dim3((L + kDtThreads - 1) / kDtThreads, B * 4), kDtThreads, dsm, s>>>(ddts, Wdt,
                                                                                              g.d_dtlow, D, L, R);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int nt = (D + kWgTile - 1) / kWgTile;
    int bpb = 1;
    while (bpb < B && (long long)4 * nt * ((B + 2 * bpb - 1) / (2 * bpb)) >= 4LL * sm_count())
        bpb *= 2;
    dtproj_wgrad_kernel<<<dim3(4 * nt, (B + bpb - 1) / bpb), kWgThreads, 0, s>>>(ddts, xdbl, dWdt, B, D, L, R, Cp,
                                                                                 bpb);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;

    // dx += x_proj's adjoint
    const int smem = dgrad_smem_bytes(Cp);
    static int configured = 0;
    e = allow_smem(xproj_dgrad_kernel, smem, &configured);
    if (e != cudaSuccess)
        return e;
    const int tiles_h = (H + kDgTile - 1) / kDgTile, tiles_w = (W + kDgTile - 1) / kDgTile;
    const long long tiles = (long long)B * tiles_h * tiles_w;
    if (tiles > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    xproj_dgrad_kernel<<<dim3((unsigned)tiles, (D + kDgCh - 1) / kDgCh), kDgThreads, smem, s>>>(
        g, static_cast<const __nv_bfloat16 *>(Wx), dx, D, H, W, tiles_w, tiles_h);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;

    // dWx: about four blocks per SM in all
    const int nd = (D + kWxCh - 1) / kWxCh;
    const long long total = (long long)B * ((L + kWxSteps - 1) / kWxSteps);
    long long slices = (4LL * sm_count() + 4 * nd - 1) / (4 * nd);
    if (slices > total)
        slices = total;
    if (slices > 65535)
        slices = 65535;
    const int cpb = (int)((total + slices - 1) / slices);
    slices = (total + cpb - 1) / cpb;
    xproj_wgrad_kernel<<<dim3(4 * nd, (unsigned)slices), kWxThreads, 0, s>>>(g, x32, xT32, dWx, B, D, L, cpb);
    return cudaGetLastError();
}

}  // namespace ss2d
