// xproj_bwd.cu -- the adjoints of x_proj on the 5th-generation tensor cores.
//
// x_proj (section 3.2 of the VMamba SS2D article) is, per image, one GEMM over the
// channels: x_dbl[b,k,c,l_k(p)] = sum_d Wx[k,c,d] x[b,d,p].  With n = k*Cp + c running
// over the rows of all four directions and dP the gradient of x_dbl gathered at each
// direction's scan index of a pixel, its two adjoints are GEMMs again:
//   dx[b,d,p]  += sum_n Wx[n,d] dP[b,n,p]            (K = the 4*Cp rows)
//   dWx[n,d]    = sum_{b,p} dP[b,n,p] x[b,d,p]        (K = every pixel of the batch)
// Both run as tcgen05.mma (kind::f16, bf16 operands, fp32 accumulators in tensor memory)
// on tiles of 128 pixels (8 image rows x 16 columns).  dP is fp32; it enters the MMA as
// two bf16 parts, dP ~ hi + lo with hi = bf16(dP) and lo = bf16(dP - hi), so each product
// keeps about 16 bits of dP (x and Wx are bf16 already and enter exactly).
//   xproj_dgrad_tc_kernel  D = dP_tile (M = 128 pixels, K = 4Cp) x Wx^T (N = D), then
//                          dx += D at the tile's pixels;
//   xproj_wgrad_tc_kernel  per CTA, over its tiles: D += x_tile^T (M = 128 channels, twice
//                          for D > 128) x dP_tile (N = 4Cp), then one partial sum per CTA;
//   wx_reduce_kernel       dWx = sum of the partial sums (fixed order: deterministic).
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "launch_util.h"
#include "proj_bwd.h"
#include "tcgen05.cuh"

namespace ss2d {

namespace {

constexpr int kTH = 8, kTW = 16, kTM = kTH * kTW;  // pixel tile = MMA M (dx) or K (dWx)
constexpr int kTcThreads = 256;                    // a thread per pixel / TMEM lane, two warps per lane quarter
constexpr int kPartCtas = 148;                     // CTAs of the weight-gradient kernel
constexpr int kMaxD = 256;                         // channels: one MMA N (dx), two M blocks (dWx)

__host__ __device__ inline int kpad(int NP) { return (NP + 15) / 16 * 16; }
// one operand tile of 128 pixels x KP rows, canonical no-swizzle layout
__host__ __device__ inline int ptile_bytes(int KP) { return (KP / 8) * 2048; }

// Row c of direction k of x_dbl's gradient for image b: d_dtlow, dB or dC.
__device__ __forceinline__ const float *grad_row(const ProjGradRows &g, int b, int k, int c, int L)
{
    const size_t bk = (size_t)b * 4 + k;
    if (c < g.R)
        return g.d_dtlow + (bk * g.R + c) * L;
    if (c < g.R + g.N)
        return g.dB + (bk * g.N + (c - g.R)) * L;
    return g.dC + (bk * g.N + (c - g.R - g.N)) * L;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// The dP tile of the 128 pixels at (h0, w0) of image b, as hi and lo bf16 parts, each with
// element (m, n) at (n/8)*2048 + (m/8)*128 + (n%8)*16 + (m%8)*2 (m = hl*16 + wl).  Item =
// (row n, tile row hl, 8-column group wg): 8 pixels, one 16-byte store per part.  The
// column-major directions give consecutive threads consecutive rows, so that their loads
// walk consecutive steps; W % 8 == 0 keeps every 8-column group wholly inside or outside.
// A thread loads kGatherBatch items before it converts and stores any of them, so that
// their global loads are in flight together.
constexpr int kGatherBatch = 4;

__device__ __forceinline__ void load_dp_item(const ProjGradRows &g, int b, int h0, int w0, int H, int W, int Cp,
                                             int it, float (&v)[8])
{
    const int L = H * W;
    const int n = it / 16, q = it % 16;
    const int k = n / Cp, c = n % Cp;
    const int hl = (k & 1) ? (q & 7) : (q >> 1), wg = (k & 1) ? (q >> 3) : (q & 1);
    const int h = h0 + hl, w = w0 + 8 * wg;
    if (h < H && w < W) {
        const float *row = grad_row(g, b, k, c, L);
        if (!(k & 1)) {
            const int pk = h * W + w;
            if (!(k & 2)) {
                const float4 a0 = __ldg(reinterpret_cast<const float4 *>(row + pk));
                const float4 a1 = __ldg(reinterpret_cast<const float4 *>(row + pk + 4));
                v[0] = a0.x, v[1] = a0.y, v[2] = a0.z, v[3] = a0.w;
                v[4] = a1.x, v[5] = a1.y, v[6] = a1.z, v[7] = a1.w;
            } else {
                // pixel pk + i sits at step L - 1 - pk - i: the 8 steps from L - 8 - pk, reversed
                const float4 a0 = __ldg(reinterpret_cast<const float4 *>(row + L - 8 - pk));
                const float4 a1 = __ldg(reinterpret_cast<const float4 *>(row + L - 4 - pk));
                v[7] = a0.x, v[6] = a0.y, v[5] = a0.z, v[4] = a0.w;
                v[3] = a1.x, v[2] = a1.y, v[1] = a1.z, v[0] = a1.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pk = (w + i) * H + h;
                v[i] = __ldg(row + ((k & 2) ? L - 1 - pk : pk));
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = 0.0f;
    }
}

__device__ __forceinline__ void store_dp_item(int Cp, int it, const float (&v)[8], unsigned char *sHi,
                                              unsigned char *sLo)
{
    const int n = it / 16, q = it % 16;
    const int k = n / Cp;
    const int hl = (k & 1) ? (q & 7) : (q >> 1), wg = (k & 1) ? (q >> 3) : (q & 1);
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        r[i] = v[i] - __bfloat162float(__float2bfloat16_rn(v[i]));
    const uint4 hi = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                pack_bf16(v[6], v[7]));
    const uint4 lo = make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]), pack_bf16(r[4], r[5]),
                                pack_bf16(r[6], r[7]));
    const int off = (n / 8) * 2048 + (hl * 2 + wg) * 128 + (n % 8) * 16;
    *reinterpret_cast<uint4 *>(sHi + off) = hi;
    *reinterpret_cast<uint4 *>(sLo + off) = lo;
}

__device__ void gather_dp_tile(const ProjGradRows &g, int b, int h0, int w0, int H, int W, int Cp,
                               unsigned char *sHi, unsigned char *sLo)
{
    const int total = 4 * Cp * 16;
    for (int base = threadIdx.x; base < total; base += kGatherBatch * blockDim.x) {
        float v[kGatherBatch][8];
#pragma unroll
        for (int j = 0; j < kGatherBatch; ++j) {
            const int it = base + j * (int)blockDim.x;
            if (it < total)
                load_dp_item(g, b, h0, w0, H, W, Cp, it, v[j]);
        }
#pragma unroll
        for (int j = 0; j < kGatherBatch; ++j) {
            const int it = base + j * (int)blockDim.x;
            if (it < total)
                store_dp_item(Cp, it, v[j], sHi, sLo);
        }
    }
}

// Rows NP..KP-1 of a dP tile (the K padding) are zero.
__device__ void zero_dp_padding(int NP, int KP, unsigned char *sHi, unsigned char *sLo)
{
    for (int it = threadIdx.x; it < (KP - NP) * 16; it += blockDim.x) {
        const int n = NP + it / 16, mg = it % 16;
        const int off = (n / 8) * 2048 + mg * 128 + (n % 8) * 16;
        *reinterpret_cast<uint4 *>(sHi + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sLo + off) = make_uint4(0, 0, 0, 0);
    }
}

__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc::smem_u32(slot)),
                 "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
}

__device__ __forceinline__ void tmem_dealloc(uint32_t tmem, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(cols));
}

__device__ __forceinline__ void mbar_init(uint64_t *mbar)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar)), "r"(1));
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mb)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mb)
                 : "memory");
}

struct XbArgs {
    ProjGradRows g;
    const __nv_bfloat16 *Wx;  // (4*Cp, D)
    const __nv_bfloat16 *x;   // (B, D, H, W)
    float *dx;                // (B, D, H, W), accumulated
    float *part;              // (kPartCtas, 4*Cp, D) partial sums of dWx
    int *err;                 // set to nonzero if a bounded wait runs out
    int B, D, H, W, tiles_h, tiles_w, ntiles;
};

__device__ __forceinline__ void tile_origin(const XbArgs &a, int t, int &b, int &h0, int &w0)
{
    const int tw = t % a.tiles_w;
    const int rest = t / a.tiles_w;
    h0 = (rest % a.tiles_h) * kTH;
    b = rest / a.tiles_h;
    w0 = tw * kTW;
}

__global__ void __launch_bounds__(kTcThreads, 1) xproj_dgrad_tc_kernel(const XbArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int Cp = a.g.R + 2 * a.g.N, NP = 4 * Cp, KP = kpad(NP), D = a.D;
    const uint32_t SBO_W = (uint32_t)(KP / 8) * 128u;
    unsigned char *sW = smem;                           // Wx^T: (d, n) at (d/8)*SBO_W + (n/8)*128 + (d%8)*16 + (n%8)*2
    unsigned char *sHi = smem + (size_t)D * KP * 2;
    unsigned char *sLo = sHi + ptile_bytes(KP);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sLo + ptile_bytes(KP));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Wx^T: item = (channel d, 8 consecutive rows n), one 16-byte core-matrix row; consecutive
    // threads take consecutive channels, so each of the 8 loads is coalesced
    for (int it = tid; it < D * (KP / 8); it += kTcThreads) {
        const int ng = it / D, d = it % D;
        uint32_t wv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n0 = ng * 8 + 2 * i;
            const unsigned short lo = n0 < NP ? __bfloat16_as_ushort(a.Wx[(size_t)n0 * D + d]) : 0;
            const unsigned short hi = n0 + 1 < NP ? __bfloat16_as_ushort(a.Wx[(size_t)(n0 + 1) * D + d]) : 0;
            wv[i] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        *reinterpret_cast<uint4 *>(sW + (d / 8) * SBO_W + ng * 128 + (d % 8) * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    zero_dp_padding(NP, KP, sHi, sLo);
    if (tid == 0)
        mbar_init(mbar);
    if (warp == 0)
        tmem_alloc(tmem_slot, 256);
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    // kind::f16: fp32 accumulate, bf16 A and B, A MN-major (pixels contiguous), B K-major
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(D >> 3) << 17) |
                           ((uint32_t)(kTM >> 4) << 24);
    const uint32_t wBase = tc::smem_u32(sW), hiBase = tc::smem_u32(sHi), loBase = tc::smem_u32(sLo);
    const uint32_t mb = tc::smem_u32(mbar);
    uint32_t phase = 0;

    for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
        int b, h0, w0;
        tile_origin(a, t, b, h0, w0);
        gather_dp_tile(a.g, b, h0, w0, a.H, a.W, Cp, sHi, sLo);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
            for (int j = 0; j < KP / 16; ++j) {
                const uint64_t bd = tc::smem_desc(wBase + j * 256u, 128u, SBO_W);
                tc::mma_bf16(tmem, tc::smem_desc(hiBase + j * 4096u, 2048u, 128u), bd, idesc, j > 0 ? 1u : 0u);
                tc::mma_bf16(tmem, tc::smem_desc(loBase + j * 4096u, 2048u, 128u), bd, idesc, 1u);
            }
            mma_commit(mb);
        }
        const bool ok_wait = tc::mbar_wait(mb, phase);
        phase ^= 1u;
        if (__syncthreads_or(ok_wait ? 0 : 1)) {
            if (tid == 0)
                atomicExch(a.err, 1);
            break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        // epilogue: thread = pixel m (TMEM lane); warps w and w + 4 share lane quarter w and
        // take alternate 32-channel chunks
        const int quarter = warp & 3;
        const int m = quarter * 32 + lane;
        const int h = h0 + m / kTW, w = w0 + m % kTW;
        const bool inside = h < a.H && w < a.W;
        float *o = a.dx + ((size_t)b * D * a.H + h) * a.W + w;
        const size_t plane = (size_t)a.H * a.W;
        for (int cc = warp >> 2; cc < (D + 31) / 32; cc += kTcThreads / 128) {
            uint32_t v[32];
            tc::tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cc * 32), v);
            if (inside) {
                // all 32 loads first, then the stores: the rows are distinct
                float cur[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    cur[i] = cc * 32 + i < D ? o[(size_t)(cc * 32 + i) * plane] : 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (cc * 32 + i < D)
                        o[(size_t)(cc * 32 + i) * plane] = cur[i] + __uint_as_float(v[i]);
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
        __syncthreads();
    }
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, 256);
}

__global__ void __launch_bounds__(kTcThreads, 1) xproj_wgrad_tc_kernel(const XbArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int Cp = a.g.R + 2 * a.g.N, NP = 4 * Cp, KP = kpad(NP), D = a.D;
    const int nmc = (D + 127) / 128;                     // 128-channel M blocks
    unsigned char *sX = smem;                           // x tile: (d, m) at (d/8)*2048 + (m/8)*128 + (d%8)*16 + (m%8)*2
    unsigned char *sHi = smem + kMaxD * 256;
    unsigned char *sLo = sHi + ptile_bytes(KP);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sLo + ptile_bytes(KP));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // channel rows D..nmc*128-1 of the x tile stay zero
    for (int it = tid; it < (nmc * 128 - D) * 16; it += kTcThreads) {
        const int d = D + it / 16, mg = it % 16;
        *reinterpret_cast<uint4 *>(sX + (d / 8) * 2048 + mg * 128 + (d % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    zero_dp_padding(NP, KP, sHi, sLo);
    if (tid == 0)
        mbar_init(mbar);
    if (warp == 0)
        tmem_alloc(tmem_slot, 512);
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    // kind::f16: fp32 accumulate, bf16 A and B, both K-major (pixels contiguous), M = 128, N = KP
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(KP >> 3) << 17) |
                           ((uint32_t)(kTM >> 4) << 24);
    const uint32_t xBase = tc::smem_u32(sX), hiBase = tc::smem_u32(sHi), loBase = tc::smem_u32(sLo);
    const uint32_t mb = tc::smem_u32(mbar);
    uint32_t phase = 0;
    bool first = true;
    bool failed = false;

    for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
        int b, h0, w0;
        tile_origin(a, t, b, h0, w0);
        // x tile with cp.async: item (d, tile row hl, 8-column group wg), 16 bytes
        for (int it = tid; it < D * 16; it += kTcThreads) {
            const int d = it / 16, hl = (it % 16) >> 1, wg = it & 1;
            const int h = h0 + hl, w = w0 + 8 * wg;
            const bool ok = h < a.H && w < a.W;
            const __nv_bfloat16 *src = a.x + (((size_t)b * D + d) * a.H + (ok ? h : 0)) * a.W + (ok ? w : 0);
            cp_async16(sX + (d / 8) * 2048 + (hl * 2 + wg) * 128 + (d % 8) * 16, src, ok ? 16 : 0);
        }
        cp_async_commit();
        gather_dp_tile(a.g, b, h0, w0, a.H, a.W, Cp, sHi, sLo);
        cp_async_wait<0>();
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
            for (int mc = 0; mc < nmc; ++mc) {
                for (int j = 0; j < kTM / 16; ++j) {
                    const uint64_t ad = tc::smem_desc(xBase + mc * 32768u + j * 256u, 128u, 2048u);
                    const uint32_t acc = (first && j == 0) ? 0u : 1u;
                    tc::mma_bf16(tmem + (uint32_t)(mc * KP), ad, tc::smem_desc(hiBase + j * 256u, 128u, 2048u), idesc,
                                 acc);
                    tc::mma_bf16(tmem + (uint32_t)(mc * KP), ad, tc::smem_desc(loBase + j * 256u, 128u, 2048u), idesc,
                                 1u);
                }
            }
            mma_commit(mb);
        }
        first = false;
        const bool ok_wait = tc::mbar_wait(mb, phase);
        phase ^= 1u;
        if (__syncthreads_or(ok_wait ? 0 : 1)) {
            if (tid == 0)
                atomicExch(a.err, 1);
            failed = true;
            break;
        }
    }
    if (!failed) {
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        // thread = channel d of M block mc (TMEM lane), 32 rows n per load; warps w and w + 4
        // share lane quarter w and take alternate 32-row chunks
        float *out = a.part + (size_t)blockIdx.x * NP * D;
        const int quarter = warp & 3;
        for (int mc = 0; mc < nmc; ++mc) {
            const int d = mc * 128 + quarter * 32 + lane;
            for (int cc = warp >> 2; cc < (KP + 31) / 32; cc += kTcThreads / 128) {
                uint32_t v[32];
                tc::tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mc * KP + cc * 32), v);
                if (d < D) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = cc * 32 + i;
                        if (n < NP)
                            out[(size_t)n * D + d] = __uint_as_float(v[i]);
                    }
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, 512);
}

__global__ void wx_reduce_kernel(const float *__restrict__ part, float *__restrict__ dWx, int nparts, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        float s = 0.0f;
        for (int p = 0; p < nparts; ++p)
            s += __ldg(part + (size_t)p * n + i);
        dWx[i] = s;
    }
}


// ---------------------------------------------------------------------------------------
// The same two adjoints on the CUDA cores in fp32, for the shapes the tensor-core kernels
// above do not tile (widths that are not multiples of 8, more than 256 channels, more than
// 256 rows of x_dbl: the other VMamba stages).  Both are tiled 64 x 64 outputs per
// 256-thread block, 4 x 4 per thread, 16 reduction values per shared-memory stage.
constexpr int kCcT = 64, kCcK = 16, kCcThreads = 256;

// scan index of pixel p in direction k
__device__ __forceinline__ int scan_index(int k, int p, int H, int W, int L)
{
    const int h = p / W, w = p - h * W;
    const int pk = (k & 1) ? w * H + h : p;
    return (k & 2) ? L - 1 - pk : pk;
}

// dx[b, d, p] += sum_n Wx[n, d] dP[b, n, p]; block = (64 pixels, 64 channels, image b)
__global__ void __launch_bounds__(kCcThreads) xproj_dgrad_cc_kernel(const ProjGradRows g,
                                                                   const __nv_bfloat16 *__restrict__ Wx,
                                                                   float *__restrict__ dx, int D, int H, int W)
{
    __shared__ float sP[kCcK][kCcT + 4];
    __shared__ float sW[kCcK][kCcT + 4];
    const int L = H * W, Cp = g.R + 2 * g.N, NP = 4 * Cp;
    const int p0 = blockIdx.x * kCcT, d0 = blockIdx.y * kCcT, b = blockIdx.z;
    const int tid = threadIdx.x, tp = tid & 15, td = tid >> 4;
    float acc[4][4] = {};
    for (int n0 = 0; n0 < NP; n0 += kCcK) {
        for (int e = tid; e < kCcK * kCcT; e += kCcThreads) {
            const int nn = e / kCcT, pp = e % kCcT, n = n0 + nn, p = p0 + pp;
            float v = 0.0f;
            if (n < NP && p < L) {
                const int k = n / Cp, c = n - k * Cp;
                v = grad_row(g, b, k, c, L)[scan_index(k, p, H, W, L)];
            }
            sP[nn][pp] = v;
            const int d = d0 + pp;
            sW[nn][pp] = (n < NP && d < D) ? __bfloat162float(Wx[(size_t)n * D + d]) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int nn = 0; nn < kCcK; ++nn) {
            float pv[4], wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pv[i] = sP[nn][tp * 4 + i];
                wv[i] = sW[nn][td * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(pv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int d = d0 + td * 4 + j;
        if (d >= D)
            continue;
        float *row = dx + ((size_t)b * D + d) * L;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int p = p0 + tp * 4 + i;
            if (p < L)
                row[p] += acc[i][j];
        }
    }
}

// Partial sums of dWx[n, d] = sum_{b, p} dP[b, n, p] x[b, d, p] over split z of the batch's
// pixels; block = (64 rows n, 64 channels d, split z), part (nsplit, 4 Cp, D)
__global__ void __launch_bounds__(kCcThreads) xproj_wgrad_cc_kernel(const ProjGradRows g,
                                                                   const __nv_bfloat16 *__restrict__ x,
                                                                   float *__restrict__ part, int B, int D, int H,
                                                                   int W, int nsplit)
{
    __shared__ float sP[kCcK][kCcT + 4];
    __shared__ float sX[kCcK][kCcT + 4];
    const int L = H * W, Cp = g.R + 2 * g.N, NP = 4 * Cp;
    const int n0 = blockIdx.x * kCcT, d0 = blockIdx.y * kCcT, z = blockIdx.z;
    const long long P = (long long)B * L;
    const long long q_begin = P * z / nsplit, q_end = P * (z + 1) / nsplit;
    const int tid = threadIdx.x, tn = tid & 15, td = tid >> 4;
    float acc[4][4] = {};
    for (long long q0 = q_begin; q0 < q_end; q0 += kCcK) {
        for (int e = tid; e < kCcK * kCcT; e += kCcThreads) {
            const int qq = e / kCcT, rr = e % kCcT;
            const long long q = q0 + qq;
            float pv = 0.0f, xv = 0.0f;
            if (q < q_end) {
                const int b = (int)(q / L), p = (int)(q - (long long)b * L);
                const int n = n0 + rr, d = d0 + rr;
                if (n < NP) {
                    const int k = n / Cp, c = n - k * Cp;
                    pv = grad_row(g, b, k, c, L)[scan_index(k, p, H, W, L)];
                }
                if (d < D)
                    xv = __bfloat162float(x[((size_t)b * D + d) * L + p]);
            }
            sP[qq][rr] = pv;
            sX[qq][rr] = xv;
        }
        __syncthreads();
#pragma unroll
        for (int qq = 0; qq < kCcK; ++qq) {
            float pv[4], xv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pv[i] = sP[qq][tn * 4 + i];
                xv[i] = sX[qq][td * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(pv[i], xv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = n0 + tn * 4 + i;
        if (n >= NP)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int d = d0 + td * 4 + j;
            if (d < D)
                part[((size_t)z * NP + n) * D + d] = acc[i][j];
        }
    }
}

constexpr int kCcSplits = 16;  // pixel splits of the CUDA-core weight gradient (its partial sums)

size_t dgrad_smem(int D, int KP) { return (size_t)D * KP * 2 + 2 * (size_t)ptile_bytes(KP) + 16; }
size_t wgrad_smem(int KP) { return (size_t)kMaxD * 256 + 2 * (size_t)ptile_bytes(KP) + 16; }

}  // namespace

bool xproj_bwd_tc_supported(int D, int W) { return D % 16 == 0 && D >= 16 && D <= kMaxD && W % 8 == 0; }

static bool use_tc(int N, int R, int D, int W) { return xproj_bwd_tc_supported(D, W) && kpad(4 * (R + 2 * N)) <= 256; }

size_t xproj_bwd_partial_bytes(int N, int R, int D, int W)
{
    const int parts = use_tc(N, R, D, W) ? kPartCtas : kCcSplits;
    return (size_t)parts * 4 * (R + 2 * N) * D * sizeof(float);
}

cudaError_t launch_xproj_bwd(const ProjGradRows &g, const void *Wx, const void *x, float *dx, float *dWx, float *part,
                             int *err, int B, int D, int H, int W, cudaStream_t s)
{
    if (use_tc(g.N, g.R, D, W))
        return launch_xproj_bwd_tc(g, Wx, x, dx, dWx, part, err, B, D, H, W, s);
    if (B < 1 || B > 65535)
        return cudaErrorInvalidValue;
    const int L = H * W, NP = 4 * (g.R + 2 * g.N);
    xproj_dgrad_cc_kernel<<<dim3((L + kCcT - 1) / kCcT, (D + kCcT - 1) / kCcT, B), kCcThreads, 0, s>>>(
        g, static_cast<const __nv_bfloat16 *>(Wx), dx, D, H, W);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    xproj_wgrad_cc_kernel<<<dim3((NP + kCcT - 1) / kCcT, (D + kCcT - 1) / kCcT, kCcSplits), kCcThreads, 0, s>>>(
        g, static_cast<const __nv_bfloat16 *>(x), part, B, D, H, W, kCcSplits);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int n = NP * D;
    wx_reduce_kernel<<<(n + 255) / 256, 256, 0, s>>>(part, dWx, kCcSplits, n);
    return cudaGetLastError();
}

cudaError_t launch_xproj_bwd_tc(const ProjGradRows &g, const void *Wx, const void *x, float *dx, float *dWx,
                                float *part, int *err, int B, int D, int H, int W, cudaStream_t s)
{
    if (!xproj_bwd_tc_supported(D, W) || B < 1)
        return cudaErrorInvalidValue;
    const int Cp = g.R + 2 * g.N, NP = 4 * Cp, KP = kpad(NP);
    if (KP > 256 || 2 * KP > 512)
        return cudaErrorInvalidValue;
    XbArgs a{};
    a.g = g;
    a.Wx = static_cast<const __nv_bfloat16 *>(Wx);
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.dx = dx;
    a.part = part;
    a.err = err;
    a.B = B;
    a.D = D;
    a.H = H;
    a.W = W;
    a.tiles_h = (H + kTH - 1) / kTH;
    a.tiles_w = (W + kTW - 1) / kTW;
    a.ntiles = B * a.tiles_h * a.tiles_w;

    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const size_t sd = dgrad_smem(D, KP), sw = wgrad_smem(KP);
    static int conf_d[kMaxDevices] = {}, conf_w[kMaxDevices] = {};
    e = configure_smem(xproj_dgrad_tc_kernel, (int)sd, conf_d);
    if (e == cudaSuccess)
        e = configure_smem(xproj_wgrad_tc_kernel, (int)sw, conf_w);
    if (e != cudaSuccess)
        return e;
    const int gd = a.ntiles < sms ? a.ntiles : sms;
    xproj_dgrad_tc_kernel<<<gd, kTcThreads, sd, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int gw = a.ntiles < kPartCtas ? a.ntiles : kPartCtas;
    xproj_wgrad_tc_kernel<<<gw, kTcThreads, sw, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int n = NP * D;
    wx_reduce_kernel<<<(n + 255) / 256, 256, 0, s>>>(part, dWx, gw, n);
    return cudaGetLastError();
}

}  // namespace ss2d
