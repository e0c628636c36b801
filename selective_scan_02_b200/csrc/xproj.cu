// xproj.cu -- the projection path of the fused core.
//
// x_proj (SS2D article, section 3.2): x_dbl[b,k,c,l] = sum_d W[k,c,d] xs[b,k,d,l].
// Because xs[b,k,:,l] is x[b,:,pi_k(l)], the product is one GEMM per image,
// P[p, n] = sum_d x[b,d,p] Wcat[n,d] with n = k*Cp + c over all four
// directions, whose rows are then written to x_dbl in each direction's scan
// order.  It runs on the 5th-generation tensor cores:
//   - a CTA owns a tile of 128 pixels (8 image rows x 16 columns) of one
//     image; the bf16 x tile is copied to shared memory with cp.async into
//     the canonical MN-major layout (8 pixels x 8 channels core matrices),
//     the bf16 weights of all directions stay resident in the K-major layout;
//   - one thread issues tcgen05.mma (kind::f16, M = 128, N = 4*Cp rounded up
//     to 32, K = 16 per instruction) accumulating fp32 in tensor memory;
//   - tcgen05.commit signals an mbarrier; every warp then reads its 32 TMEM
//     lanes (one pixel per thread) and writes the 4*Cp values to x_dbl at the
//     scan index of that pixel in each direction.
// The scan kernel then reads dt_low / B / C rows of x_dbl and computes
// dt_proj (R multiply-adds per element) in its prepass.
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "launch_util.h"
#include "scan.cuh"
#include "tcgen05.cuh"
#include "xproj.h"

namespace ss2d {

namespace {

constexpr int kTileH = 8;
constexpr int kTileW = 16;
constexpr int kTileM = kTileH * kTileW;  // 128 pixels = MMA M
constexpr int kThreads = 128;
constexpr int kResThreads = 256;  // the resident-weight kernel: two warps per TMEM lane quarter
constexpr int kTmemCols = 256;
constexpr size_t kWsHeader = 256;         // error word and padding at the start of the workspace

struct XprojArgs {
    const __nv_bfloat16 *x;  // (B, D, H, W)
    const __nv_bfloat16 *w;  // (4, Cp, D)
    float *xdbl;             // (B, 4, Cp, L)
    int *err;                // set to nonzero if a bounded wait runs out
    int B, D, H, W, L, Cp, NP, tiles_h, tiles_w, ntiles;
    int n_base;              // chunked kernel: first of this launch's output columns n = k*Cp + c
};

__host__ __device__ inline size_t a_bytes(int D) { return (size_t)D * 256; }                        // D/8 K-groups x 16 MN core matrices x 128 B
__host__ __device__ inline size_t b_bytes(int D, int NP) { return (size_t)(NP / 8) * (D / 8) * 128; }  // NP/8 N-groups x D/8 K core matrices
__host__ __device__ inline size_t smem_bytes(int D, int NP) { return a_bytes(D) + b_bytes(D, NP) + 16; }

__global__ void __launch_bounds__(kResThreads, 1) xproj_kernel(const XprojArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int D = a.D;
    unsigned char *sA = smem;
    unsigned char *sB = smem + a_bytes(D);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sB + b_bytes(D, a.NP));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ncp = 4 * a.Cp;
    const uint32_t SBO_B = (uint32_t)(D / 8) * 128u;

    // Weights of all four directions, K-major core matrices: element (n, d) at
    // (n/8)*SBO_B + (d/8)*128 + (n%8)*16 + (d%8)*2.  Rows n >= 4*Cp are zero.
    for (int p = tid; p < a.NP * (D / 8); p += kResThreads) {
        const int n = p / (D / 8), kc = p % (D / 8);
        const __nv_bfloat16 *src = a.w + (size_t)min(n, ncp - 1) * D + kc * 8;
        cp_async16(sB + (n / 8) * SBO_B + kc * 128 + (n % 8) * 16, src, n < ncp ? 16 : 0);
    }
    cp_async_commit();
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar)), "r"(1));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc::smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    // kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, A MN-major, B K-major.
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(a.NP >> 3) << 17) |
                           ((uint32_t)(kTileM >> 4) << 24);
    const uint32_t aBase = tc::smem_u32(sA), bBase = tc::smem_u32(sB), mb = tc::smem_u32(mbar);
    uint32_t phase = 0;
    const int L = a.L;

    // x tile of tile t, MN-major core matrices: element (m, d) at
    // (d/8)*2048 + (m/8)*128 + (d%8)*16 + (m%8)*2; out-of-image pixels are zero.  Pixel
    // order m = wg*64 + hl*8 + (wl % 8) with wg = wl / 8: each warp of the epilogue (32
    // consecutive m) covers 4 rows x 8 columns, so its stores of a row-major direction
    // land as 4 runs of 8 steps and those of a column-major one as 8 runs of 4.
    auto stage_tile = [&](int t) {
        const int tw = t % a.tiles_w;
        const int rest = t / a.tiles_w;
        const int th = rest % a.tiles_h;
        const int b = rest / a.tiles_h;
        const int h0 = th * kTileH, w0 = tw * kTileW;
        for (int p = tid; p < D * 16; p += kResThreads) {
            const int d = p >> 4, rem = p & 15, hl = rem >> 1, wg = rem & 1;
            const int h = h0 + hl, w = w0 + 8 * wg;
            const bool ok = h < a.H && w < a.W;
            const __nv_bfloat16 *src = a.x + (((size_t)b * D + d) * a.H + (ok ? h : 0)) * a.W + (ok ? w : 0);
            cp_async16(sA + (d >> 3) * 2048 + (wg * 8 + hl) * 128 + (d & 7) * 16, src, ok ? 16 : 0);
        }
        cp_async_commit();
    };

    if (blockIdx.x < a.ntiles)
        stage_tile(blockIdx.x);
    for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
        const int tw = t % a.tiles_w;
        const int rest = t / a.tiles_w;
        const int th = rest % a.tiles_h;
        const int b = rest / a.tiles_h;
        const int h0 = th * kTileH, w0 = tw * kTileW;

        cp_async_wait<0>();
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncthreads();

        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
            for (int j = 0; j < D / 16; ++j) {
                const uint64_t ad = tc::smem_desc(aBase + j * 4096u, 2048u, 128u);
                const uint64_t bd = tc::smem_desc(bBase + j * 256u, 128u, SBO_B);
                tc::mma_bf16(tmem, ad, bd, idesc, j > 0 ? 1u : 0u);
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mb)
                         : "memory");
        }
        const bool ok_wait = tc::mbar_wait(mb, phase);
        phase ^= 1u;
        const int failed = __syncthreads_or(ok_wait ? 0 : 1);
        if (failed) {
            if (tid == 0)
                atomicExch(a.err, 1);
            break;
        }
        // the MMAs have read the x tile: load the next one while this tile's epilogue runs
        if (t + (int)gridDim.x < a.ntiles)
            stage_tile(t + gridDim.x);
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");

        // Epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (thread = pixel m) of every
        // second 32-column chunk, starting at chunk w / 4.  Column n = k * Cp + c goes to
        // x_dbl[b, k, c, l_k] with l_k this pixel's step in direction k; (k, c) and the
        // destination pointer advance with n, one division per chunk.
        const int lq = warp & 3;
        const int m = lq * 32 + lane;
        const int h = h0 + ((m >> 3) & 7), w = w0 + (m >> 6) * 8 + (m & 7);
        const bool inside = h < a.H && w < a.W;
        const int prow = h * a.W + w, pcol = w * a.H + h;
        // steps of this pixel in directions 0..3, and the change from direction k - 1 to k
        const int l0 = prow, l1 = pcol, l2 = L - 1 - prow, l3 = L - 1 - pcol;
        float *outb = a.xdbl + (size_t)b * 4 * a.Cp * L;
        for (int cc = warp >> 2; cc < a.NP / 32; cc += kResThreads / 128) {
            uint32_t v[32];
            tc::tmem_ld32(tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(cc * 32), v);
            if (inside) {
                const int n0 = cc * 32;
                int k = n0 / a.Cp, c = n0 - k * a.Cp;
                float *dst = outb + (size_t)n0 * L + (k == 0 ? l0 : k == 1 ? l1 : k == 2 ? l2 : l3);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (n0 + i < ncp)
                        *dst = __uint_as_float(v[i]);
                    dst += L;
                    if (++c == a.Cp && k < 3) {  // next direction: move to its step of this pixel
                        c = 0;
                        ++k;
                        dst += k == 1 ? l1 - l0 : k == 2 ? l2 - l1 : l3 - l2;
                    }
                }
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
        __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
}

int round_np(int Cp) { return ((4 * Cp + 31) / 32) * 32; }

// ---------------------------------------------------------------------------------------
// The same GEMM for any image width and channel count (the other VMamba stages: 28x28
// D = 384, 14x14 D = 768, 7x7 D = 1536).  A tile is 128 consecutive pixels of one image in
// row-major order, so any W works; the reduction over channels runs in chunks of kKC
// channels through a two-deep shared-memory ring (x tile and weight chunk per stage), so any
// D works; rows whose length is not a multiple of 8 pixels are staged element by element.
// The MMAs of chunk k run while chunk k + 1 is copied in.
constexpr int kKC = 64;  // channels per reduction chunk

__host__ __device__ inline size_t gen_a_bytes() { return (size_t)kKC * 256; }  // kKC/8 K-groups x 16 core matrices
__host__ __device__ inline size_t gen_b_bytes(int NP) { return (size_t)NP * kKC * 2; }
__host__ __device__ inline size_t gen_stage_bytes(int NP) { return gen_a_bytes() + gen_b_bytes(NP); }
__host__ __device__ inline size_t gen_smem_bytes(int NP) { return 2 * gen_stage_bytes(NP) + 64; }

__global__ void __launch_bounds__(kThreads, 1) xproj_gen_kernel(const XprojArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int D = a.D, L = a.L, NP = a.NP;
    const size_t stage_bytes = gen_stage_bytes(NP);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + 2 * stage_bytes);  // one per ring stage
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ncp = min(4 * a.Cp - a.n_base, NP);       // columns n_base .. n_base + ncp of this launch
    const __nv_bfloat16 *wrows = a.w + (size_t)a.n_base * D;
    const uint32_t SBO_B = (uint32_t)(kKC / 8) * 128u;  // bytes between N groups of the weight chunk
    const int nk = (D + kKC - 1) / kKC;                  // D % 16 == 0: the last chunk holds kcn(k) channels
    const int tiles_img = (L + kTileM - 1) / kTileM;
    const int ntiles = a.B * tiles_img;
    const bool rows16 = (L & 7) == 0;  // 8-pixel pieces of x rows are 16-byte aligned

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar)), "r"(1));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar + 1)), "r"(1));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc::smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(NP >> 3) << 17) |
                           ((uint32_t)(kTileM >> 4) << 24);

    // chunk kc of tile (b, p0) into ring stage st
    auto stage = [&](int b, int p0, int kc, int st) {
        unsigned char *sA = smem + st * stage_bytes;
        unsigned char *sB = sA + gen_a_bytes();
        const int d0 = kc * kKC, kcn = min(kKC, D - d0);
        // weights of all four directions, channels d0 .. d0 + kcn: element (n, d) at
        // (n/8)*SBO_B + (d/8)*128 + (n%8)*16 + (d%8)*2; rows n >= 4*Cp are zero
        for (int pc = tid; pc < NP * (kcn / 8); pc += kThreads) {
            const int n = pc / (kcn / 8), kg = pc % (kcn / 8);
            const __nv_bfloat16 *src = wrows + (size_t)min(n, ncp - 1) * D + d0 + kg * 8;
            cp_async16(sB + (n / 8) * SBO_B + kg * 128 + (n % 8) * 16, src, n < ncp ? 16 : 0);
        }
        // x: pixels p0 .. p0 + 127, channels d0 .. d0 + kcn: element (m, d) at
        // (d/8)*2048 + (m/8)*128 + (d%8)*16 + (m%8)*2; pixels past the image are zero
        const __nv_bfloat16 *xb = a.x + ((size_t)b * D + d0) * L;
        if (rows16) {
            for (int pc = tid; pc < kcn * 16; pc += kThreads) {
                const int d = pc >> 4, mg = pc & 15, p = p0 + mg * 8;
                const int nv = max(0, min(8, L - p));
                cp_async16(sA + (d >> 3) * 2048 + mg * 128 + (d & 7) * 16, nv > 0 ? xb + (size_t)d * L + p : xb,
                           nv * 2);
            }
        } else {
            const unsigned short *xs = reinterpret_cast<const unsigned short *>(xb);
            for (int e = tid; e < kcn * kTileM; e += kThreads) {
                const int d = e / kTileM, m = e % kTileM, p = p0 + m;
                const unsigned short v = p < L ? __ldg(xs + (size_t)d * L + p) : (unsigned short)0;
                *reinterpret_cast<unsigned short *>(sA + (d >> 3) * 2048 + (m >> 3) * 128 + (d & 7) * 16 + (m & 7) * 2) = v;
            }
        }
        cp_async_commit();
    };
    // every thread waits for the commit that completes the given phase of stage st's barrier;
    // false in every thread if any thread's wait ran out
    uint32_t phase[2] = {0u, 0u};
    auto wait_stage = [&](int st) -> bool {
        const bool ok = tc::mbar_wait(tc::smem_u32(mbar + st), phase[st]);
        phase[st] ^= 1u;
        return __syncthreads_or(ok ? 0 : 1) == 0;
    };

    bool good = true;
    for (int t = blockIdx.x; t < ntiles && good; t += gridDim.x) {
        const int b = t / tiles_img, p0 = (t - b * tiles_img) * kTileM;
        stage(b, p0, 0, 0);
        for (int kc = 0; kc < nk && good; ++kc) {
            const int st = kc & 1;
            cp_async_wait<0>();
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            __syncthreads();
            if (tid == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
                const uint32_t aB = tc::smem_u32(smem + st * stage_bytes), bB = aB + (uint32_t)gen_a_bytes();
                const int kcn = min(kKC, D - kc * kKC);
                for (int j = 0; j < kcn / 16; ++j) {
                    const uint64_t ad = tc::smem_desc(aB + j * 4096u, 2048u, 128u);
                    const uint64_t bd = tc::smem_desc(bB + j * 256u, 128u, SBO_B);
                    tc::mma_bf16(tmem, ad, bd, idesc, (kc > 0 || j > 0) ? 1u : 0u);
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                                 tc::smem_u32(mbar + st))
                             : "memory");
            }
            if (kc + 1 < nk) {
                // chunk kc + 1 goes to the other stage, last read by the MMAs of chunk kc - 1
                if (kc >= 1)
                    good = wait_stage(st ^ 1);
                if (good)
                    stage(b, p0, kc + 1, st ^ 1);
            }
        }
        // the tile's last two commits (MMAs complete in order; both phases are consumed)
        if (good && nk >= 2)
            good = wait_stage((nk - 2) & 1);
        if (good)
            good = wait_stage((nk - 1) & 1);
        if (!good) {
            if (tid == 0)
                atomicExch(a.err, 1);
            break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");

        // Epilogue: thread = pixel m (TMEM lane), 32 columns per load.
        const int m = warp * 32 + lane, p = p0 + m;
        const bool inside = p < L;
        const int h = inside ? p / a.W : 0, w = inside ? p - h * a.W : 0;
        const int prow = p, pcol = w * a.H + h;
        // steps of this pixel in directions 0..3; (k, c) and the destination advance with the
        // column, one division per 32-column chunk
        const int l0 = prow, l1 = pcol, l2 = L - 1 - prow, l3 = L - 1 - pcol;
        float *outb = a.xdbl + (size_t)b * 4 * a.Cp * L;
        for (int cc = 0; cc < NP / 32; ++cc) {
            uint32_t v[32];
            tc::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cc * 32), v);
            if (inside) {
                const int ng0 = a.n_base + cc * 32;
                int k = ng0 / a.Cp, c = ng0 - k * a.Cp;
                float *dst = outb + (size_t)ng0 * L + (k == 0 ? l0 : k == 1 ? l1 : k == 2 ? l2 : l3);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (cc * 32 + i < ncp)
                        *dst = __uint_as_float(v[i]);
                    dst += L;
                    if (++c == a.Cp && k < 3) {
                        c = 0;
                        ++k;
                        dst += k == 1 ? l1 - l0 : k == 2 ? l2 - l1 : l3 - l2;
                    }
                }
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
        __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
}

// dt_proj for dt_ranks above what the scan fuses (kMaxR): dts[b,k,d,l] = sum_r W[k,d,r]
// dt_low[b,k,r,l] (SS2D article section 3.2), materialised in fp32 in scan order for the
// direct-form scan.  Thread = step l of one (image, direction), its R dt_low values in
// registers; the direction's weights pass through shared memory 64 channels at a time.
constexpr int kDtpThreads = 128;
constexpr int kDtpChunk = 64;

__global__ void __launch_bounds__(kDtpThreads) dtproj_fwd_kernel(const float *__restrict__ xdbl,
                                                               const float *__restrict__ Wdt, float *__restrict__ dts,
                                                               int D, int L, int R, int Cp)
{
    __shared__ float sw[kDtpChunk * kMaxRLarge];
    const int bk = blockIdx.y, k = bk & 3;
    const int l = blockIdx.x * kDtpThreads + threadIdx.x;
    float t[kMaxRLarge];
    const float *src = xdbl + (size_t)bk * Cp * L + (l < L ? l : 0);
#pragma unroll
    for (int r = 0; r < kMaxRLarge; ++r)
        t[r] = (r < R && l < L) ? __ldg(src + (size_t)r * L) : 0.0f;
    float *dst = dts + (size_t)bk * D * L + l;
    for (int d0 = 0; d0 < D; d0 += kDtpChunk) {
        const int nd = min(kDtpChunk, D - d0);
        __syncthreads();
        for (int e = threadIdx.x; e < nd * R; e += kDtpThreads)
            sw[e] = __ldg(Wdt + ((size_t)k * D + d0) * R + e);
        __syncthreads();
        if (l < L) {
            for (int d = 0; d < nd; ++d) {
                float z = 0.0f;
#pragma unroll
                for (int r = 0; r < kMaxRLarge; ++r)
                    if (r < R)
                        z = fmaf(sw[d * R + r], t[r], z);
                dst[(size_t)(d0 + d) * L] = z;
            }
        }
    }
}

// The resident-weight kernel covers widths that are multiples of 8 and channel counts whose
// weights fit in shared memory next to one x tile; the chunked kernel covers the rest.
bool xproj_resident_ok(int D, int W, int NP) { return NP <= 256 && W % 8 == 0 && smem_bytes(D, NP) <= 200 * 1024; }

}  // namespace

int xproj_supported(int B, int D, int H, int W, int N, int R)
{
    (void)B;
    (void)H;
    (void)W;
    (void)N;
    if (R < 1 || R > kMaxRLarge)
        return 1;
    if (D % 16 != 0)
        return 2;
    if (R > kMaxR && (long long)B * 4 > 65535)
        return 3;  // dtproj_fwd_kernel puts each (image, direction) in the grid's y dimension
    return 0;
}

bool xproj_dt_fused(int R) { return R <= kMaxR; }

// Bytes of x with transposed planes the scan reads for the column-major orders (0 if unused).
// The workspace is sized for the softplus case; without softplus the copy is not made.
static size_t transposed_bytes(int B, int D, int H, int W, int N, int R, bool softplus = true)
{
    if (!xproj_dt_fused(R) || !scan_reads_transposed_u(N, kFusedProj, 1, 0, softplus ? 1 : 0, H * W))
        return 0;
    return (size_t)B * D * H * W * sizeof(__nv_bfloat16);
}

// Segments of the projection form's scan (few images: long sequences split so the GPU fills).
static void proj_segments(int B, int D, int L, int N, bool softplus, int *nseg, int *seg_len)
{
    plan_segments(B, 4, D, L, N, kFusedProj, 1, 0, softplus ? 1 : 0, nseg, seg_len);
}

// Bytes of x_dbl plus the copy of x that follows it (see xproj_workspace_bytes).
static size_t xdbl_and_copy_bytes(int B, int D, int H, int W, int N, int R, bool ch_last)
{
    const size_t extra = ch_last ? (size_t)B * D * H * W * sizeof(__nv_bfloat16) : transposed_bytes(B, D, H, W, N, R);
    // dt_ranks the scan does not fuse: dts (B, 4, D, L) fp32 made by dtproj_fwd_kernel
    const size_t dts = xproj_dt_fused(R) ? 0 : (size_t)B * 4 * D * H * W * sizeof(float);
    return (size_t)B * 4 * (R + 2 * N) * H * W * sizeof(float) + extra + dts;
}

// Workspace: error-word header, x_dbl (B, 4, R+2N, L) fp32, then either (channels-first x,
// when used) x with its planes transposed, (B, D, W, H) bf16, or (channels-last x) x in
// channels-first order, (B, D, H, W) bf16, for the GEMM; then, when the scan is segmented,
// the segment states.  Sized for softplus on (without it the scan is neither segmented nor
// reads the transposed copy).
size_t xproj_workspace_bytes(int B, int D, int H, int W, int N, int R, bool ch_last)
{
    int nseg = 1, seg_len = H * W;
    if (xproj_dt_fused(R))
        proj_segments(B, D, H * W, N, true, &nseg, &seg_len);
    return kWsHeader + xdbl_and_copy_bytes(B, D, H, W, N, R, ch_last) + segment_workspace_bytes(B, 4 * D, nseg, N);
}

cudaError_t launch_xproj_gemm(const void *x_cf, const void *x_proj_weight, float *xdbl, int *err, int B, int D, int H,
                              int W, int N, int R, cudaStream_t s)
{
    const int Cp = R + 2 * N;
    XprojArgs xa{};
    xa.x = static_cast<const __nv_bfloat16 *>(x_cf);
    xa.w = static_cast<const __nv_bfloat16 *>(x_proj_weight);
    xa.xdbl = xdbl;
    xa.err = err;
    xa.B = B;
    xa.D = D;
    xa.H = H;
    xa.W = W;
    xa.L = H * W;
    xa.Cp = Cp;
    xa.NP = round_np(Cp);
    xa.n_base = 0;
    xa.tiles_h = (H + kTileH - 1) / kTileH;
    xa.tiles_w = (W + kTileW - 1) / kTileW;
    xa.ntiles = B * xa.tiles_h * xa.tiles_w;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    if (xproj_resident_ok(D, W, xa.NP)) {
        const size_t smem = smem_bytes(D, xa.NP);
        static int configured[kMaxDevices] = {};
        e = configure_smem(xproj_kernel, (int)smem, configured);
        if (e != cudaSuccess)
            return e;
        const int grid = xa.ntiles < 2 * sms ? xa.ntiles : 2 * sms;
        xproj_kernel<<<grid, kResThreads, smem, s>>>(xa);
        return cudaGetLastError();
    }
    // at most 256 output columns per launch (the MMA's N and the tensor-memory accumulator)
    const long long ntiles = (long long)B * ((xa.L + kTileM - 1) / kTileM);
    const int grid = (int)(ntiles < 2LL * sms ? ntiles : 2LL * sms);
    static int configured_gen[kMaxDevices] = {};
    for (int nb = 0; nb < 4 * Cp; nb += 256) {
        XprojArgs pa = xa;
        pa.n_base = nb;
        pa.NP = ((std::min(256, 4 * Cp - nb) + 31) / 32) * 32;
        const size_t smem = gen_smem_bytes(pa.NP);
        e = configure_smem(xproj_gen_kernel, (int)gen_smem_bytes(256), configured_gen);
        if (e != cudaSuccess)
            return e;
        xproj_gen_kernel<<<grid, kThreads, smem, s>>>(pa);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

size_t xproj_header_bytes() { return kWsHeader; }

cudaError_t launch_clear_error_word(int *err, cudaStream_t s)
{
    return launch_fill_zero(reinterpret_cast<float *>(err), kWsHeader / sizeof(float), s);
}

cudaError_t launch_core_with_projections(const void *x, const void *x_proj_weight, const float *dt_projs_weight,
                                         const float *A_logs, const float *Ds, const float *dt_bias, bool softplus,
                                         float *y, void *workspace, int B, int D, int H, int W, int N, int R,
                                         bool ch_last, bool clear_err, cudaStream_t s)
{
    const int Cp = R + 2 * N;
    const int L = H * W;
    int *err = static_cast<int *>(workspace);
    float *xdbl = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWsHeader);
    void *after_xdbl = reinterpret_cast<char *>(xdbl) + (size_t)B * 4 * Cp * L * sizeof(float);
    // the GEMM reads channels-first x: a channels-last x (B, L, D) is transposed per image first
    // (its pair kernel also zeroes y, which has as many elements, where L and D are even)
    const void *x_cf = x;
    const bool zero_in_cl_transpose = ch_last && transpose_planes_can_zero(true, L, D);
    if (ch_last) {
        cudaError_t e = zero_in_cl_transpose ? launch_transpose_planes_zero(x, after_xdbl, y, B, L, D, s)
                                             : launch_transpose_planes(x, true, after_xdbl, B, L, D, s);
        if (e != cudaSuccess)
            return e;
        x_cf = after_xdbl;
    }
    // y starts at zero: zeroed by a plane transpose of x where the scan reads that copy (below)
    // or the GEMM does (above) and the pair kernel can (bf16 x, even sides), else here
    const bool transposed = !ch_last && xproj_dt_fused(R) && transposed_bytes(B, D, H, W, N, R, softplus) > 0;
    const bool zero_in_transpose = (transposed && transpose_planes_can_zero(true, H, W)) || zero_in_cl_transpose;
    cudaError_t e = clear_err ? launch_clear_error_word(err, s) : cudaSuccess;
    if (e == cudaSuccess && !zero_in_transpose)
        e = launch_fill_zero(y, (size_t)B * D * L, s);
    if (e == cudaSuccess)
        e = launch_xproj_gemm(x_cf, x_proj_weight, xdbl, err, B, D, H, W, N, R, s);
    if (e != cudaSuccess)
        return e;

    ScanArgs sa{};
    sa.u = x;
    sa.ch_last = ch_last ? 1 : 0;
    if (!xproj_dt_fused(R)) {
        // dt_proj materialised (dts in scan order after x_dbl), then the direct-form scan with
        // B and C read from x_dbl's rows; channels-first only (checked by the caller)
        float *dts = reinterpret_cast<float *>(after_xdbl);
        dim3 grid((L + kDtpThreads - 1) / kDtpThreads, (unsigned)B * 4);
        dtproj_fwd_kernel<<<grid, kDtpThreads, 0, s>>>(xdbl, dt_projs_weight, dts, D, L, R, Cp);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
        sa.delta = dts;
        sa.A_log = A_logs;
        sa.Bm = xdbl + (size_t)R * L;
        sa.Cm = xdbl + (size_t)(R + N) * L;
        sa.gs = (long long)Cp * L;
        sa.Dv = Ds;
        sa.bias = dt_bias;
        sa.y = y;
        sa.B = B;
        sa.C = 4 * D;
        sa.G = 4;
        sa.L = L;
        sa.per_group = D;
        sa.W = W;
        sa.divH = {H, 1.0f / (float)H};
        sa.u_bf16 = 1;
        sa.delta_bf16 = 0;
        sa.softplus = softplus ? 1 : 0;
        sa.delta_bytes = (size_t)B * 4 * D * L * sizeof(float);
        return launch_scan(sa, N, kFused, s);
    }
    if (transposed) {
        e = zero_in_transpose ? launch_transpose_planes_zero(x, after_xdbl, y, B * D, H, W, s)
                              : launch_transpose_planes(x, true, after_xdbl, B * D, H, W, s);
        if (e != cudaSuccess)
            return e;
        sa.uT = after_xdbl;
    }
    sa.delta = nullptr;
    sa.A_log = A_logs;
    sa.Bm = xdbl + (size_t)R * L;
    sa.Cm = xdbl + (size_t)(R + N) * L;
    sa.dtl = xdbl;
    sa.Wdt = dt_projs_weight;
    sa.Dv = Ds;
    sa.bias = dt_bias;
    sa.y = y;
    sa.gs = (long long)Cp * L;
    sa.B = B;
    sa.C = 4 * D;
    sa.G = 4;
    sa.L = L;
    sa.per_group = D;
    sa.W = W;
    sa.divH = {H, 1.0f / (float)H};
    sa.R = R;
    sa.u_bf16 = 1;
    sa.delta_bf16 = 0;
    sa.softplus = softplus ? 1 : 0;
    sa.delta_bytes = 0;
    int nseg, seg_len;
    proj_segments(B, D, L, N, softplus, &nseg, &seg_len);
    if (nseg > 1) {
        sa.nseg = nseg;
        sa.seg_len = seg_len;
        float *seg_ws = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWsHeader +
                                                  xdbl_and_copy_bytes(B, D, H, W, N, R, ch_last));
        return launch_scan_segmented(sa, N, kFusedProj, seg_ws, s);
    }
    return launch_scan(sa, N, kFusedProj, s);
}

}  // namespace ss2d
