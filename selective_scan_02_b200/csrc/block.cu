// block.cu -- the SS2D block around the fused core (SS2D article, section 1: input
// projection, depthwise convolution, cross scan + selective scan, output projection; VMamba
// overview page, section 2.2: SiLU activation, d_conv = 3, a learnable gate):
//
//   xz  = x @ W_in^T (+ b_in)                      rowgemm_kernel, tcgen05, bf16 out
//   x_c = SiLU(dwconv(xz[:, :D]) + b_conv)         dwconv_silu_kernel, channels-last in,
//                                                  bf16 out in the core's layout
//   y   = core(x_c)                                ss2d_forward_core, projection form
//   g   = LayerNorm_D(y) * SiLU(xz[:, D:])         norm_gate_cl_kernel / norm_gate_kernel,
//                                                  bf16 out
//   out = g @ W_out^T (+ b_out)                    rowgemm_kernel, fp32 or bf16 out
//
// x, xz, g and out are channels last, (B, H, W, C) flattened to (B*H*W, C) rows.  x_c and y
// are channels-last too where the core's channels-last form covers the shape (N = 16,
// dt_rank <= 16) and D <= 768; else they are channel-first, which the core's projection path
// reads without a transposed copy.  bf16 storage between the steps, fp32 arithmetic inside
// them.
#include <cuda_bf16.h>
#include <stdarg.h>
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "api_internal.h"
#include "common.cuh"
#include "launch_util.h"
#include "ss2d.h"
#include "tcgen05.cuh"

namespace ss2d {
namespace {

// ---------------------------------------------------------------------------------------
// Row-major GEMM on the 5th-generation tensor cores: C[m, n] = sum_k A[m, k] W[n, k] (+ bias[n])
// with A (M, K) and W (Nout, K) bf16 row-major (K contiguous, K % 16 == 0), fp32
// accumulation in tensor memory and a bf16 or fp32 row-major C.
//   - work item = (128-row tile, pass of up to 256 output columns); consecutive items share
//     a tile, so a pass after the first reads its A rows from L2;
//   - the reduction runs in chunks of 64 through a two-deep shared-memory ring (A chunk and
//     W chunk per stage, both in the K-major canonical layout: element (r, k) at
//     (r/8)*1024 + (k/8)*128 + (r%8)*16 + (k%8)*2), copied with cp.async; the MMAs of chunk
//     c run while chunk c + 1 is copied;
//   - one thread issues tcgen05.mma (kind::f16, M = 128, N = the pass's columns, K = 16);
//     tcgen05.commit signals the stage's mbarrier (bounded waits);
//   - epilogue: thread = row (TMEM lane), 32 columns per tcgen05.ld, bias added, stored as
//     16-byte vectors along the row.
// Shared memory is sized for two CTAs per SM, so one CTA's epilogue overlaps the other's
// MMAs and copies, and two 256-column TMEM allocations fill the SM's 512 columns exactly.
constexpr int kGThreads = 128;
constexpr int kGM = 128;
constexpr int kGKC = 64;
constexpr int kGNmax = 256;
constexpr uint32_t kGSbo = (kGKC / 8) * 128;  // bytes between 8-row groups of a chunk

__host__ __device__ constexpr size_t g_a_bytes() { return (size_t)kGM * kGKC * 2; }
__host__ __device__ constexpr size_t g_b_bytes() { return (size_t)kGNmax * kGKC * 2; }
__host__ __device__ constexpr size_t g_stage_bytes() { return g_a_bytes() + g_b_bytes(); }
__host__ __device__ constexpr size_t g_smem_bytes() { return 2 * g_stage_bytes() + 64; }

// two floats rounded to bf16 (nearest, ties to even), the first in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

struct GemmArgs {
    const __nv_bfloat16 *A;  // (M, lda) rows, the first K columns used
    const __nv_bfloat16 *Wt; // (Nout, K)
    const float *bias;       // (Nout) or null
    void *C;                 // (M, ldc) rows, columns 0 .. Nout
    int *err;                // set to nonzero if a bounded wait runs out
    long long M;
    int K, Nout, lda, ldc;
    int np;                  // columns per pass: a multiple of 16, at most 256
    int npass;               // ceil(Nout / np)
    long long mtiles;        // ceil(M / 128)
    int c_bf16;              // C is bf16 (else fp32)
};

__global__ void __launch_bounds__(kGThreads, 1) rowgemm_kernel(const GemmArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + 2 * g_stage_bytes());
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = a.K, np = a.np;
    const int nk = (K + kGKC - 1) / kGKC;

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar)), "r"(1));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar + 1)), "r"(1));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc::smem_u32(tmem_slot)),
                     "r"(kGNmax));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    // kind::f16: fp32 accumulate, bf16 A and B, both K-major, N = np, M = 128
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(np >> 3) << 17) |
                           ((uint32_t)(kGM >> 4) << 24);

    // chunk kc of item (m0, n0) into ring stage st; rows past M and columns past Nout are zero
    auto stage = [&](long long m0, int n0, int kc, int st) {
        unsigned char *sA = smem + st * g_stage_bytes();
        unsigned char *sB = sA + g_a_bytes();
        const int k0 = kc * kGKC, nkg = min(kGKC, K - k0) / 8;
        // piece index: (r % 8) fastest, then the 8-element group along K, then r / 8, so each
        // 8 consecutive threads fill one 128-byte run of shared memory
        for (int pc = tid; pc < kGM * nkg; pc += kGThreads) {
            const int r8 = pc & 7, kg = (pc >> 3) % nkg, rg = (pc >> 3) / nkg;
            const long long m = m0 + rg * 8 + r8;
            const bool ok = m < a.M;
            const __nv_bfloat16 *src = a.A + (ok ? m : 0) * (long long)a.lda + k0 + kg * 8;
            cp_async16(sA + rg * kGSbo + kg * 128 + r8 * 16, src, ok ? 16 : 0);
        }
        for (int pc = tid; pc < np * nkg; pc += kGThreads) {
            const int r8 = pc & 7, kg = (pc >> 3) % nkg, rg = (pc >> 3) / nkg;
            const int n = n0 + rg * 8 + r8;
            const bool ok = n < a.Nout;
            const __nv_bfloat16 *src = a.Wt + (size_t)(ok ? n : 0) * K + k0 + kg * 8;
            cp_async16(sB + rg * kGSbo + kg * 128 + r8 * 16, src, ok ? 16 : 0);
        }
        cp_async_commit();
    };
    uint32_t phase[2] = {0u, 0u};
    auto wait_stage = [&](int st) -> bool {
        const bool ok = tc::mbar_wait(tc::smem_u32(mbar + st), phase[st]);
        phase[st] ^= 1u;
        return __syncthreads_or(ok ? 0 : 1) == 0;
    };

    bool good = true;
    const long long items = a.mtiles * a.npass;
    for (long long it = blockIdx.x; it < items && good; it += gridDim.x) {
        const long long tile = it / a.npass;
        const int pass = (int)(it - tile * a.npass);
        const long long m0 = tile * kGM;
        const int n0 = pass * np;
        stage(m0, n0, 0, 0);
        for (int kc = 0; kc < nk && good; ++kc) {
            const int st = kc & 1;
            cp_async_wait<0>();
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            __syncthreads();
            if (tid == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
                const uint32_t aB = tc::smem_u32(smem + st * g_stage_bytes()), bB = aB + (uint32_t)g_a_bytes();
                const int kcn = min(kGKC, K - kc * kGKC);
                for (int j = 0; j < kcn / 16; ++j) {
                    const uint64_t ad = tc::smem_desc(aB + j * 256u, 128u, kGSbo);
                    const uint64_t bd = tc::smem_desc(bB + j * 256u, 128u, kGSbo);
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
                    stage(m0, n0, kc + 1, st ^ 1);
            }
        }
        // the item's last two commits (MMAs complete in order; every commit is waited once)
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

        // Epilogue: thread = row m (TMEM lane), 32 columns per load.
        const long long m = m0 + warp * 32 + lane;
        const bool row_ok = m < a.M;
        const int ncols = min(np, a.Nout - n0);
        for (int cc = 0; cc * 32 < ncols; ++cc) {
            uint32_t v[32];
            tc::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cc * 32), v);
            if (!row_ok)
                continue;
            const int c0 = n0 + cc * 32, cn = min(32, a.Nout - c0);
            float f[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                f[i] = __uint_as_float(v[i]) + ((a.bias && i < cn) ? __ldg(a.bias + c0 + i) : 0.0f);
            if (a.c_bf16) {
                __nv_bfloat16 *row = static_cast<__nv_bfloat16 *>(a.C) + m * (long long)a.ldc + c0;
                if (cn == 32) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 pk;
                        pk.x = pack_bf16x2(f[8 * q + 0], f[8 * q + 1]);
                        pk.y = pack_bf16x2(f[8 * q + 2], f[8 * q + 3]);
                        pk.z = pack_bf16x2(f[8 * q + 4], f[8 * q + 5]);
                        pk.w = pack_bf16x2(f[8 * q + 6], f[8 * q + 7]);
                        reinterpret_cast<uint4 *>(row)[q] = pk;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < cn)
                            row[i] = __float2bfloat16_rn(f[i]);
                }
            } else {
                float *row = static_cast<float *>(a.C) + m * (long long)a.ldc + c0;
                if (cn == 32) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        reinterpret_cast<float4 *>(row)[q] = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2],
                                                                         f[4 * q + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < cn)
                            row[i] = f[i];
                }
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
        __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kGNmax));
}

// ---------------------------------------------------------------------------------------
// The same GEMM with the whole weight matrix resident in shared memory (Nout * K * 2 bytes next
// to the A ring) and up to 512 output columns in one tensor-memory accumulator: the input and
// output projections of VMamba-T stage 1 (K = 96, N = 384 and K = 192, N = 96).  Persistent
// CTAs, one per SM, walk 128-row tiles; the A tiles of the next STAGES - 1 tiles (STAGES = 3,
// or 2 where three do not fit) are in
// flight (cp.async groups) while the current tile's MMAs and epilogue run, so the loads, the
// MMAs and the stores of consecutive tiles overlap.  Per tile: wait for its A group, one
// thread issues the MMAs (N split into instructions of at most 256 columns), the loads of a
// later tile are issued into the stage the previous tile's MMAs released, then the epilogue
// reads tensor memory (thread = row; four warps per 32-row quarter, each on every fourth
// 32-column chunk) and stores the tile.
constexpr int kResThreads = 512;  // 16 warps: all of them copy A tiles and share the epilogue
constexpr int kResWarps = kResThreads / 32;

// per-warp staging of one 32-row x 32-column output chunk, rows padded by 16 bytes
__host__ __device__ constexpr size_t res_stage_pitch(int esz) { return (size_t)32 * esz + 16; }
__host__ __device__ constexpr size_t res_w_bytes(int K, int Nout) { return (size_t)((Nout + 7) / 8) * 8 * K * 2; }
__host__ __device__ constexpr size_t res_a_bytes(int K) { return (size_t)kGM * K * 2; }
__host__ __device__ constexpr size_t res_smem_bytes(int K, int Nout, int esz, int stages)
{
    return res_w_bytes(K, Nout) + stages * res_a_bytes(K) + kResWarps * 32 * res_stage_pitch(esz) + 64;
}

__host__ __device__ constexpr uint32_t tmem_cols_for(int n)
{
    return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : n <= 256 ? 256u : 512u;
}

template <int STAGES>
__global__ void __launch_bounds__(kResThreads, 1) rowgemm_res_kernel(const GemmArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int K = a.K, Nout = a.Nout;
    const int NP = ((Nout + 15) / 16) * 16;  // MMA columns (rows of W past Nout are zero)
    const int esz = a.c_bf16 ? 2 : 4;
    const int pitch = (int)res_stage_pitch(esz);
    unsigned char *sW = smem;
    unsigned char *sA0 = smem + res_w_bytes(K, NP);
    unsigned char *sOut = sA0 + STAGES * res_a_bytes(K);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sOut + kResWarps * 32 * res_stage_pitch(esz));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nkg = K / 8;
    const uint32_t SBO = (uint32_t)nkg * 128u;  // bytes between 8-row groups (A and W)
    const uint32_t tcols = tmem_cols_for(NP);

    // resident weights: element (n, k) at (n/8)*SBO + (k/8)*128 + (n%8)*16 + (k%8)*2
    for (int pc = tid; pc < NP * nkg; pc += kResThreads) {
        const int r8 = pc & 7, kg = (pc >> 3) % nkg, rg = (pc >> 3) / nkg;
        const int n = rg * 8 + r8;
        const bool ok = n < Nout;
        cp_async16(sW + rg * SBO + kg * 128 + r8 * 16, a.Wt + (size_t)(ok ? n : 0) * K + kg * 8, ok ? 16 : 0);
    }
    cp_async_commit();
    // A tile of the i-th tile of this CTA into ring stage i % STAGES (an empty group past the end).
    // Piece pc = (row group rg, K group kg, row r8) with (pc >> 3) = rg * nkg + kg; the thread's
    // (rg, kg) start once per CTA and advance by a fixed step, without a division per piece.
    const long long ntile = a.mtiles;
    const int kg_first = (tid >> 3) % nkg, rg_first = (tid >> 3) / nkg;
    const int kg_step = (kResThreads >> 3) % nkg, rg_step = (kResThreads >> 3) / nkg;
    auto load_a = [&](long long i) {
        const long long t = blockIdx.x + i * gridDim.x;
        if (t < ntile) {
            unsigned char *sA = sA0 + (size_t)(i % STAGES) * res_a_bytes(K);
            const long long m0 = t * kGM;
            int kg = kg_first, rg = rg_first;
            for (int pc = tid; pc < kGM * nkg; pc += kResThreads) {
                const int r8 = pc & 7;
                const long long m = m0 + rg * 8 + r8;
                const bool ok = m < a.M;
                cp_async16(sA + rg * SBO + kg * 128 + r8 * 16, a.A + (ok ? m : 0) * (long long)a.lda + kg * 8,
                           ok ? 16 : 0);
                kg += kg_step;
                rg += rg_step;
                if (kg >= nkg) {
                    kg -= nkg;
                    ++rg;
                }
            }
        }
        cp_async_commit();
    };
    for (int i = 0; i < STAGES - 1; ++i)
        load_a(i);

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tc::smem_u32(mbar)), "r"(1));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc::smem_u32(tmem_slot)),
                     "r"(tcols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const uint32_t n0cols = NP < 256 ? (uint32_t)NP : 256u;  // first MMA's columns, then the rest
    const uint32_t idesc0 = (1u << 4) | (1u << 7) | (1u << 10) | ((n0cols >> 3) << 17) | ((uint32_t)(kGM >> 4) << 24);
    const uint32_t idesc1 = (1u << 4) | (1u << 7) | (1u << 10) | (((uint32_t)(NP - (int)n0cols) >> 3) << 17) |
                            ((uint32_t)(kGM >> 4) << 24);
    const uint32_t mb = tc::smem_u32(mbar);
    uint32_t phase = 0;
    unsigned char *stg = sOut + (size_t)warp * 32 * pitch;  // this warp's staging chunk

    for (long long i = 0;; ++i) {
        const long long t = blockIdx.x + i * gridDim.x;
        if (t >= ntile)
            break;
        cp_async_wait<STAGES - 2>();  // this tile's group (and the weights) have landed
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
            const uint32_t aB = tc::smem_u32(sA0 + (size_t)(i % STAGES) * res_a_bytes(K));
            const uint32_t wB = tc::smem_u32(sW);
            for (int j = 0; j < K / 16; ++j) {
                const uint64_t ad = tc::smem_desc(aB + j * 256u, 128u, SBO);
                tc::mma_bf16(tmem, ad, tc::smem_desc(wB + j * 256u, 128u, SBO), idesc0, j > 0 ? 1u : 0u);
                if (NP > 256)
                    tc::mma_bf16(tmem + 256u, ad, tc::smem_desc(wB + 32u * SBO + j * 256u, 128u, SBO), idesc1,
                                 j > 0 ? 1u : 0u);
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mb)
                         : "memory");
        }
        // the stage of tile i - 1 is free (its MMAs completed before its epilogue)
        load_a(i + STAGES - 1);
        const bool ok_wait = tc::mbar_wait(mb, phase);
        phase ^= 1u;
        if (__syncthreads_or(ok_wait ? 0 : 1)) {
            if (tid == 0)
                atomicExch(a.err, 1);
            break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");

        // Epilogue.  Warp w reads TMEM lanes 32 (w % 4) .. + 31 (thread = row) of every fourth
        // 32-column chunk, starting at chunk w / 4.  Each chunk goes through the warp's staging
        // area so that the global stores run along the rows: a 16-byte store per lane covers
        // 8 rows x 64 bytes (bf16) or 4 rows x 128 bytes (fp32) per instruction.
        const int lq = warp & 3;
        const long long mrow0 = t * kGM + lq * 32;
        for (int cc = warp >> 2; cc * 32 < Nout; cc += kResWarps / 4) {
            uint32_t v[32];
            tc::tmem_ld32(tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(cc * 32), v);
            const int c0 = cc * 32, cn = min(32, Nout - c0);
            float f[32];
#pragma unroll
            for (int q = 0; q < 32; ++q)
                f[q] = __uint_as_float(v[q]) + ((a.bias && q < cn) ? __ldg(a.bias + c0 + q) : 0.0f);
            unsigned char *myrow = stg + lane * pitch;
            if (a.c_bf16) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 pk;
                    pk.x = pack_bf16x2(f[8 * q + 0], f[8 * q + 1]);
                    pk.y = pack_bf16x2(f[8 * q + 2], f[8 * q + 3]);
                    pk.z = pack_bf16x2(f[8 * q + 4], f[8 * q + 5]);
                    pk.w = pack_bf16x2(f[8 * q + 6], f[8 * q + 7]);
                    *reinterpret_cast<uint4 *>(myrow + q * 16) = pk;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4 *>(myrow + q * 16) =
                        make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
            }
            __syncwarp();
            // row r of the chunk = 16-byte pieces; lanes take consecutive pieces of consecutive rows
            const int lp = esz == 2 ? 2 : 3;  // log2 of the pieces per row: 4 (bf16) or 8 (fp32)
            const int pieces = 1 << lp;
            const int cn_pieces = (cn * esz + 15) / 16;
            for (int e = lane; e < 32 * pieces; e += 32) {
                const int r = e >> lp, pc = e & (pieces - 1);
                const long long m = mrow0 + r;
                if (m < a.M && pc < cn_pieces) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(stg + r * pitch + pc * 16);
                    unsigned char *dstp = static_cast<unsigned char *>(a.C) + (m * (long long)a.ldc + c0) * esz + pc * 16;
                    if ((pc + 1) * 16 <= cn * esz) {
                        *reinterpret_cast<uint4 *>(dstp) = val;
                    } else {  // the ragged last piece of the last chunk: element by element
                        const unsigned char *srcp = stg + r * pitch + pc * 16;
                        for (int bb = 0; bb < cn * esz - pc * 16; ++bb)
                            dstp[bb] = srcp[bb];
                    }
                }
            }
            __syncwarp();
        }
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
        __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(tcols));
}

// ---------------------------------------------------------------------------------------
// Depthwise convolution + bias + SiLU.  CTA = kCvTH output rows x 32 output columns x 64
// channels of one image.  The kCvTH + KS - 1 input rows it needs (32 + KS - 1 pixels each,
// zero outside the image) are copied from the channels-last xz rows into shared memory, 33
// 32-bit words per pixel (64 bf16 and one pad word, so that the 32 lanes, one per output
// column, read 32 different banks); the copy issues its 16-byte loads four at a time before
// storing them.  Thread = output column (lane) and channel pairs (warp + 8 i).  For KS <= 3
// the pair's weights stay in registers and a KS x KS window of input words slides down the
// kCvTH output rows, so each output row loads KS new words; larger kernels read every tap from
// shared memory.  Results are rounded to bf16 and stored channel-first, 32 consecutive columns
// per warp store, or (CLO) channels-last, the pair's two channels as one 4-byte store per pixel.
constexpr int kCvThreads = 256;
constexpr int kCvTW = 32;
constexpr int kCvTH = 4;
constexpr int kCvTC = 64;
constexpr int kCvRow = kCvTC / 2 + 1;

__host__ __device__ constexpr size_t cv_smem_bytes(int ks)
{
    return (size_t)(kCvTH + ks - 1) * (kCvTW + ks - 1) * kCvRow * 4 + (size_t)(kCvTC / 2) * ks * ks * 8 +
           (size_t)(kCvTC / 2) * 8;
}

struct ConvArgs {
    const __nv_bfloat16 *xz;  // (B*H*W, ldx) rows; channels 0 .. D - 1 are the scan branch
    const float *w;           // (D, KS, KS)
    const float *bias;        // (D) or null
    __nv_bfloat16 *xc;        // (B, D, H, W), or (B, H, W, D) when cl_out is set
    int B, D, H, W, ldx, tiles_h, tiles_w, tiles_c;
    int cl_out;
};

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// SiLU with the hardware exponential and reciprocal (five instructions; relative error of a
// few units in the last fp32 place, far below the bf16 rounding that follows; v / inf = -0
// for very negative v)
__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

template <int KS, bool CLO>
__global__ void __launch_bounds__(kCvThreads) dwconv_silu_kernel(const ConvArgs a)
{
    constexpr int R = (KS - 1) / 2, PW = kCvTW + KS - 1, NR = kCvTH + KS - 1;
    constexpr int NPIECE = NR * PW * (kCvTC / 8);
    extern __shared__ __align__(16) unsigned char cv_smem[];
    uint32_t *sx = reinterpret_cast<uint32_t *>(cv_smem);               // [NR][PW][kCvRow]
    float2 *sw = reinterpret_cast<float2 *>(sx + NR * PW * kCvRow);     // [pair][KS * KS]
    float2 *sb = sw + (kCvTC / 2) * KS * KS;                            // [pair]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    long long blk = blockIdx.x;
    const int tcn = (int)(blk % a.tiles_c);
    blk /= a.tiles_c;
    const int tw = (int)(blk % a.tiles_w);
    blk /= a.tiles_w;
    const int th = (int)(blk % a.tiles_h);
    const int b = (int)(blk / a.tiles_h);
    const int d0 = tcn * kCvTC, w0 = tw * kCvTW, h0 = th * kCvTH;
    const int nch = min(kCvTC, a.D - d0);  // a multiple of 16

    for (int i = tid; i < (nch / 2) * KS * KS; i += kCvThreads) {
        const int p = i / (KS * KS), t = i - p * KS * KS;
        sw[i] = make_float2(__ldg(a.w + (size_t)(d0 + 2 * p) * KS * KS + t),
                            __ldg(a.w + (size_t)(d0 + 2 * p + 1) * KS * KS + t));
    }
    for (int p = tid; p < nch / 2; p += kCvThreads)
        sb[p] = a.bias ? make_float2(__ldg(a.bias + d0 + 2 * p), __ldg(a.bias + d0 + 2 * p + 1)) : make_float2(0.f, 0.f);
    for (int base = tid; base < NPIECE; base += 4 * kCvThreads) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * kCvThreads;
            const int piece = i & 7, pix = i >> 3, r = pix / PW, c = pix - r * PW;
            const int hh = h0 + r - R, ww = w0 + c - R;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < NPIECE && hh >= 0 && hh < a.H && ww >= 0 && ww < a.W && piece * 8 < nch)
                v[u] = __ldg(reinterpret_cast<const uint4 *>(a.xz + ((long long)(b * a.H + hh) * a.W + ww) * a.ldx +
                                                             d0 + piece * 8));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * kCvThreads;
            if (i < NPIECE) {
                uint32_t *dst = sx + (i >> 3) * kCvRow + (i & 7) * 4;
                dst[0] = v[u].x;
                dst[1] = v[u].y;
                dst[2] = v[u].z;
                dst[3] = v[u].w;
            }
        }
    }
    __syncthreads();

    const long long plane = (long long)a.H * a.W;
    if constexpr (CLO && KS <= 3) {
        // channels-last out: lane = channel pair, warp = (output row, 16-column half).  The
        // pair's weights stay in registers and a KS x KS window slides along the row (KS new
        // words per output, lanes on consecutive words); each store writes one pixel's pairs,
        // 128 consecutive bytes per warp.  Same order of operations as the channel-first path.
        const int p = lane, oh = warp & 3, cb = (warp >> 2) * (kCvTW / 2);
        const int h = h0 + oh;
        if (p < nch / 2 && h < a.H) {
            const float2 bb = sb[p];
            float2 wt[KS * KS];
#pragma unroll
            for (int t = 0; t < KS * KS; ++t)
                wt[t] = sw[p * KS * KS + t];
            float2 win[KS][KS];  // win[r][c % KS]: input word of (row oh + r, column cb + c)
#pragma unroll
            for (int r = 0; r < KS; ++r)
#pragma unroll
                for (int c = 0; c < KS - 1; ++c)
                    win[r][c] = unpack_bf16x2(sx[((oh + r) * PW + cb + c) * kCvRow + p]);
            uint32_t *o = reinterpret_cast<uint32_t *>(a.xc + (((long long)b * a.H + h) * a.W + w0 + cb) * a.D + d0) + p;
#pragma unroll
            for (int oc = 0; oc < kCvTW / 2; ++oc) {
#pragma unroll
                for (int r = 0; r < KS; ++r)
                    win[r][(oc + KS - 1) % KS] = unpack_bf16x2(sx[((oh + r) * PW + cb + oc + KS - 1) * kCvRow + p]);
                float2 acc = bb;
#pragma unroll
                for (int r = 0; r < KS; ++r)
#pragma unroll
                    for (int c = 0; c < KS; ++c)
                        acc = __ffma2_rn(wt[r * KS + c], win[r][(oc + c) % KS], acc);
                if (w0 + cb + oc < a.W)
                    o[(long long)oc * (a.D / 2)] = pack_bf16x2(silu_fast(acc.x), silu_fast(acc.y));
            }
        }
    } else if constexpr (KS <= 3) {
        // lane = (channel pair of two, column pair): half-warp h takes pair 2 pp + h, lane l % 16
        // the output columns 2 (l % 16) and 2 (l % 16) + 1, so that its KS x (KS + 1) window of
        // input words serves both and each channel's two outputs go out as one bf16 pair
        const int half = lane >> 4, cw = 2 * (lane & 15);
        const int ow = w0 + cw;
        const bool pairs_out = (a.W & 1) == 0;  // (h W + ow) is even: 4-byte stores
        for (int pp = warp; pp < nch / 4; pp += kCvThreads / 32) {
            const int p = 2 * pp + half;
            const float2 bb = sb[p];
            float2 wt[KS * KS];
#pragma unroll
            for (int t = 0; t < KS * KS; ++t)
                wt[t] = sw[p * KS * KS + t];
            __nv_bfloat16 *dst = a.xc + ((long long)b * a.D + d0 + 2 * p) * plane + ow;
            float2 win[KS][KS + 1];  // win[row % KS][c]: input word of (row, cw + c)
#pragma unroll
            for (int r = 0; r < KS - 1; ++r)
#pragma unroll
                for (int c = 0; c <= KS; ++c)
                    win[r][c] = unpack_bf16x2(sx[(r * PW + cw + c) * kCvRow + p]);
#pragma unroll
            for (int oh = 0; oh < kCvTH; ++oh) {
#pragma unroll
                for (int c = 0; c <= KS; ++c)
                    win[(oh + KS - 1) % KS][c] = unpack_bf16x2(sx[((oh + KS - 1) * PW + cw + c) * kCvRow + p]);
                float2 acc0 = bb, acc1 = bb;  // columns ow and ow + 1, both channels of the pair
#pragma unroll
                for (int r = 0; r < KS; ++r)
#pragma unroll
                    for (int c = 0; c < KS; ++c) {
                        acc0 = __ffma2_rn(wt[r * KS + c], win[(oh + r) % KS][c], acc0);
                        acc1 = __ffma2_rn(wt[r * KS + c], win[(oh + r) % KS][c + 1], acc1);
                    }
                const int h = h0 + oh;
                if (h < a.H && ow < a.W) {
                    const float s00 = silu_fast(acc0.x), s01 = silu_fast(acc1.x);
                    const float s10 = silu_fast(acc0.y), s11 = silu_fast(acc1.y);
                    __nv_bfloat16 *d = dst + (long long)h * a.W;
                    if (pairs_out && ow + 1 < a.W) {
                        *reinterpret_cast<uint32_t *>(d) = pack_bf16x2(s00, s01);
                        *reinterpret_cast<uint32_t *>(d + plane) = pack_bf16x2(s10, s11);
                    } else {
                        d[0] = __float2bfloat16_rn(s00);
                        d[plane] = __float2bfloat16_rn(s10);
                        if (ow + 1 < a.W) {
                            d[1] = __float2bfloat16_rn(s01);
                            d[plane + 1] = __float2bfloat16_rn(s11);
                        }
                    }
                }
            }
        }
    } else {
        const int ow = w0 + lane;
        for (int p = warp; p < nch / 2; p += kCvThreads / 32) {
            const float2 bb = sb[p];
            __nv_bfloat16 *dst = a.xc + ((long long)b * a.D + d0 + 2 * p) * plane + ow;
            for (int oh = 0; oh < kCvTH; ++oh) {
                float2 acc = bb;
#pragma unroll
                for (int r = 0; r < KS; ++r)
#pragma unroll
                    for (int c = 0; c < KS; ++c)
                        acc = __ffma2_rn(sw[p * KS * KS + r * KS + c],
                                         unpack_bf16x2(sx[((oh + r) * PW + lane + c) * kCvRow + p]), acc);
                if (ow < a.W && h0 + oh < a.H) {
                    if constexpr (CLO) {
                        *reinterpret_cast<uint32_t *>(a.xc + (((long long)b * a.H + h0 + oh) * a.W + ow) * a.D + d0 +
                                                      2 * p) = pack_bf16x2(silu_fast(acc.x), silu_fast(acc.y));
                    } else {
                        dst[(long long)(h0 + oh) * a.W] = __float2bfloat16_rn(silu_fast(acc.x));
                        dst[plane + (long long)(h0 + oh) * a.W] = __float2bfloat16_rn(silu_fast(acc.y));
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Output normalisation and gate: g[p, d] = bf16(((y[d, p] - mean_p) * rstd_p * gamma[d] +
// beta[d]) * SiLU(z[p, d])), mean and biased variance over the D channels of pixel p.
// CTA = 32 consecutive pixels of one image, 256 threads:
//   stage   y (channel-first) is read along the pixels (128 bytes per channel, 16-byte loads)
//           into a [D/2][33] tile of channel pairs (float2), and (D <= kNgMaxDZ) the pixels' z
//           rows into a second tile, every load issued before the first use;
//   stats   thread = (pixel, one of 8 groups of channel pairs): partial sums over the group,
//           added up per pixel by one warp, first for the mean, then for the variance;
//   output  warp = pixel, lane = channel pair: y, gamma, beta and z are read as pairs and g is
//           written as bf16 pairs, 128 bytes per warp instruction.
constexpr int kNgThreads = 256;
constexpr int kNgP = 32;
constexpr int kNgGroups = kNgThreads / kNgP;  // channel-pair groups of the statistics

struct NormArgs {
    const float *y;             // (B, D, L); (B*L, D) rows for norm_gate_cl_kernel
    const __nv_bfloat16 *z;     // (B*L, ldz) rows
    const float *gamma, *beta;  // (D)
    __nv_bfloat16 *g;           // (B*L, D)
    float eps;
    int B, D, L, ldz, tiles_l;
};

// y tile, gamma and beta, partial sums, mean and rstd; with ZS also the z tile (16-byte
// aligned: D is a multiple of 16)
__host__ __device__ constexpr size_t ng_smem_bytes(int D, bool zs)
{
    return ((size_t)D * (kNgP + 1 + 2) + (size_t)(kNgGroups + 2) * kNgP) * sizeof(float) +
           (zs ? (size_t)kNgP * D * 2 : 0);
}
constexpr int kNgMaxDZ = 1120;  // largest D whose z tile fits next to the y tile

template <bool ZS>
__global__ void __launch_bounds__(kNgThreads) norm_gate_kernel(const NormArgs a)
{
    extern __shared__ float sy[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int D = a.D, P = D / 2;
    float2 *st = reinterpret_cast<float2 *>(sy);  // [P][kNgP + 1]: channels 2p, 2p + 1 of each pixel
    float *sgam = sy + D * (kNgP + 1), *sbet = sgam + D;
    float *spart = sbet + D, *smean = spart + kNgGroups * kNgP, *srstd = smean + kNgP;
    __nv_bfloat16 *sz = reinterpret_cast<__nv_bfloat16 *>(srstd + kNgP);
    const long long blk = blockIdx.x;
    const int b = (int)(blk / a.tiles_l);
    const int p0 = (int)(blk - (long long)b * a.tiles_l) * kNgP;
    const float *yb = a.y + (long long)b * D * a.L + p0;
    for (int d = tid; d < D; d += kNgThreads) {
        sgam[d] = __ldg(a.gamma + d);
        sbet[d] = __ldg(a.beta + d);
    }
    // z rows of the 32 pixels (16-byte pieces; D % 16 == 0), loaded with the y tile so that the
    // gated output reads z from shared memory (wide D reads z from global memory instead)
    if constexpr (ZS) {
        const int zp = D / 8, nz = kNgP * zp;
        for (int base = tid; base < nz; base += 4 * kNgThreads) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = base + u * kNgThreads, j = i / zp, k = i - j * zp;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (i < nz && p0 + j < a.L)
                    v[u] = __ldg(reinterpret_cast<const uint4 *>(a.z + ((long long)b * a.L + p0 + j) * a.ldz) + k);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = base + u * kNgThreads;
                if (i < nz)
                    reinterpret_cast<uint4 *>(sz)[i] = v[u];
            }
        }
    }
    // y tile: item i = (channel d = i / 8, pixels 4q .. 4q + 3 with q = i % 8); a 16-byte load
    // where the four pixels are inside the image and 16-byte aligned (L % 4 == 0), else four
    // guarded loads.  Four items in flight per thread.  Channel d lands in component d % 2 of
    // pair row d / 2.
    const int n4 = D * (kNgP / 4);
    const bool vec = (a.L & 3) == 0 && p0 + kNgP <= a.L;
    for (int base = tid; base < n4; base += 4 * kNgThreads) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * kNgThreads, d = i >> 3, q = i & 7;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < n4) {
                const float *src = yb + (long long)d * a.L + 4 * q;
                if (vec) {
                    v[u] = __ldg(reinterpret_cast<const float4 *>(src));
                } else {
                    const int pl = p0 + 4 * q;
                    v[u].x = pl < a.L ? __ldg(src) : 0.f;
                    v[u].y = pl + 1 < a.L ? __ldg(src + 1) : 0.f;
                    v[u].z = pl + 2 < a.L ? __ldg(src + 2) : 0.f;
                    v[u].w = pl + 3 < a.L ? __ldg(src + 3) : 0.f;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * kNgThreads;
            if (i < n4) {
                const int d = i >> 3;
                float *dst = sy + ((d >> 1) * (kNgP + 1) + 4 * (i & 7)) * 2 + (d & 1);
                dst[0] = v[u].x;
                dst[2] = v[u].y;
                dst[4] = v[u].z;
                dst[6] = v[u].w;
            }
        }
    }
    __syncthreads();

    // statistics: thread = (pixel jp = lane, group grp = warp of channel pairs grp, grp + 8, ...)
    {
        const int jp = lane, grp = warp;
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 4
        for (int p = grp; p < P; p += kNgGroups) {
            const float2 v = st[p * (kNgP + 1) + jp];
            s0 += v.x;
            s1 += v.y;
        }
        spart[grp * kNgP + jp] = s0 + s1;
        __syncthreads();
        if (warp == 0) {
            float t = 0.0f;
#pragma unroll
            for (int k = 0; k < kNgGroups; ++k)
                t += spart[k * kNgP + lane];
            smean[lane] = t / (float)D;
        }
        __syncthreads();
        const float mean = smean[jp];
        float q0 = 0.0f, q1 = 0.0f;
#pragma unroll 4
        for (int p = grp; p < P; p += kNgGroups) {
            const float2 v = st[p * (kNgP + 1) + jp];
            const float e0 = v.x - mean, e1 = v.y - mean;
            q0 = fmaf(e0, e0, q0);
            q1 = fmaf(e1, e1, q1);
        }
        spart[grp * kNgP + jp] = q0 + q1;  // every read of the mean sums ended at the barrier above
        __syncthreads();
        if (warp == 0) {
            float t = 0.0f;
#pragma unroll
            for (int k = 0; k < kNgGroups; ++k)
                t += spart[k * kNgP + lane];
            srstd[lane] = 1.0f / sqrtf(t / (float)D + a.eps);
        }
        __syncthreads();
    }

    // gated output: warp = pixel, lane = channel pair lane + 32 k (the tile's 8-byte reads are
    // conflict-free: a half-warp covers 16 consecutive pair rows of pitch 33 pairs)
    const float2 *sg2 = reinterpret_cast<const float2 *>(sgam), *sb2 = reinterpret_cast<const float2 *>(sbet);
    for (int j = warp; j < kNgP; j += kNgThreads / 32) {
        const int p = p0 + j;
        if (p >= a.L)
            break;
        const float mean = smean[j], rstd = srstd[j];
        const long long row = (long long)b * a.L + p;
        const uint32_t *zr = reinterpret_cast<const uint32_t *>(ZS ? sz + j * D : a.z + row * a.ldz);
        uint32_t *gr = reinterpret_cast<uint32_t *>(a.g + row * D);
        for (int c = lane; c < P; c += 32) {
            const float2 v = st[c * (kNgP + 1) + j], gm = sg2[c], bt = sb2[c];
            const float2 zz = unpack_bf16x2(ZS ? zr[c] : __ldg(zr + c));
            const float o0 = fmaf((v.x - mean) * rstd, gm.x, bt.x) * silu_fast(zz.x);
            const float o1 = fmaf((v.y - mean) * rstd, gm.y, bt.y) * silu_fast(zz.y);
            gr[c] = pack_bf16x2(o0, o1);
        }
    }
}

// The same normalisation and gate on channels-last y, (B*L, D) rows: warp = pixel, lane =
// channel pairs lane + 32 j (j < NPL), held in registers; the mean, then the biased variance
// about it, are warp sums.  Same formula and output layout as norm_gate_kernel.
constexpr int kNgClMaxPairs = 12;  // pairs per lane: D <= 768

template <int NPL>
__global__ void __launch_bounds__(kNgThreads) norm_gate_cl_kernel(const NormArgs a)
{
    const int lane = threadIdx.x & 31;
    const long long pix = (long long)blockIdx.x * (kNgThreads / 32) + (threadIdx.x >> 5);
    if (pix >= (long long)a.B * a.L)
        return;
    const int D = a.D, P = D / 2;
    const float2 *yr = reinterpret_cast<const float2 *>(a.y + pix * D);
    const uint32_t *zr = reinterpret_cast<const uint32_t *>(a.z + pix * a.ldz);
    float2 v[NPL];
    uint32_t zw[NPL];  // the gate's z pairs, loaded with y so that both are in flight together
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int c = lane + 32 * j;
        v[j] = c < P ? __ldg(yr + c) : make_float2(0.f, 0.f);
        zw[j] = c < P ? __ldg(zr + c) : 0u;
    }
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < NPL; ++j)
        s += v[j].x + v[j].y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)D;
    float q = 0.0f;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        if (lane + 32 * j < P) {
            const float e0 = v[j].x - mean, e1 = v[j].y - mean;
            q = fmaf(e0, e0, q);
            q = fmaf(e1, e1, q);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = 1.0f / sqrtf(q / (float)D + a.eps);
    uint32_t *gr = reinterpret_cast<uint32_t *>(a.g + pix * D);
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int c = lane + 32 * j;
        if (c < P) {
            const float2 gm = make_float2(__ldg(a.gamma + 2 * c), __ldg(a.gamma + 2 * c + 1));
            const float2 bt = make_float2(__ldg(a.beta + 2 * c), __ldg(a.beta + 2 * c + 1));
            const float2 zz = unpack_bf16x2(zw[j]);
            const float o0 = fmaf((v[j].x - mean) * rstd, gm.x, bt.x) * silu_fast(zz.x);
            const float o1 = fmaf((v[j].y - mean) * rstd, gm.y, bt.y) * silu_fast(zz.y);
            gr[c] = pack_bf16x2(o0, o1);
        }
    }
}

// ---------------------------------------------------------------------------------------
// Host side.

constexpr int kNgMaxD = 1648;  // [D][33] fp32 tile, gamma and beta within 227 KB of shared memory
constexpr size_t kHdr = 256;   // the block kernels' error word, then padding

int block_sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return 148;
    return sms;
}

int bfail(int status, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    return set_last_error(status, buf);
}

int bcuda(cudaError_t e, const char *what)
{
    return bfail(SS2D_ERR_CUDA, "ss2d_block_forward: %s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t r256(size_t n) { return (n + 255) & ~(size_t)255; }

cudaError_t launch_rowgemm(const __nv_bfloat16 *A, int lda, const __nv_bfloat16 *Wt, const float *bias, void *C,
                           int ldc, bool c_bf16, long long M, int K, int Nout, int *err, cudaStream_t s)
{
    static int configured[kMaxDevices];
    GemmArgs g{};
    g.A = A;
    g.Wt = Wt;
    g.bias = bias;
    g.C = C;
    g.err = err;
    g.M = M;
    g.K = K;
    g.Nout = Nout;
    g.lda = lda;
    g.ldc = ldc;
    g.np = Nout <= kGNmax ? ((Nout + 15) / 16) * 16 : kGNmax;
    g.npass = (Nout + g.np - 1) / g.np;
    g.mtiles = (M + kGM - 1) / kGM;
    g.c_bf16 = c_bf16 ? 1 : 0;
    // weights resident when they fit next to the A ring (three stages, else two) and the
    // staging chunks, and the columns fit one accumulator
    const int NPr = ((Nout + 15) / 16) * 16, esz = c_bf16 ? 2 : 4;
    const size_t limit = 220 * 1024;
    if (Nout <= 512 && K % 16 == 0 && res_smem_bytes(K, NPr, esz, 2) <= limit) {
        const int grid = (int)(g.mtiles < block_sm_count() ? g.mtiles : block_sm_count());
        cudaError_t e;
        if (res_smem_bytes(K, NPr, esz, 3) <= limit) {
            static int configured_res3[kMaxDevices];
            const size_t smem = res_smem_bytes(K, NPr, esz, 3);
            e = configure_smem(rowgemm_res_kernel<3>, (int)smem, configured_res3);
            if (e != cudaSuccess)
                return e;
            rowgemm_res_kernel<3><<<grid, kResThreads, smem, s>>>(g);
        } else {
            static int configured_res2[kMaxDevices];
            const size_t smem = res_smem_bytes(K, NPr, esz, 2);
            e = configure_smem(rowgemm_res_kernel<2>, (int)smem, configured_res2);
            if (e != cudaSuccess)
                return e;
            rowgemm_res_kernel<2><<<grid, kResThreads, smem, s>>>(g);
        }
        return cudaGetLastError();
    }
    cudaError_t e = configure_smem(rowgemm_kernel, (int)g_smem_bytes(), configured);
    if (e != cudaSuccess)
        return e;
    const long long items = g.mtiles * g.npass;
    const int grid = (int)(items < 2LL * block_sm_count() ? items : 2LL * block_sm_count());
    rowgemm_kernel<<<grid, kGThreads, g_smem_bytes(), s>>>(g);
    return cudaGetLastError();
}

template <int KS, bool CLO>
cudaError_t launch_dwconv_ks(const ConvArgs &c, cudaStream_t s)
{
    static int configured[kMaxDevices];
    const size_t smem = cv_smem_bytes(KS);
    cudaError_t e = configure_smem(dwconv_silu_kernel<KS, CLO>, (int)smem, configured);
    if (e != cudaSuccess)
        return e;
    const long long blocks = (long long)c.B * c.tiles_h * c.tiles_w * c.tiles_c;
    dwconv_silu_kernel<KS, CLO><<<(unsigned)blocks, kCvThreads, smem, s>>>(c);
    return cudaGetLastError();
}

template <bool CLO>
cudaError_t launch_dwconv_layout(const ConvArgs &c, int k, cudaStream_t s)
{
    switch (k) {
    case 1: return launch_dwconv_ks<1, CLO>(c, s);
    case 3: return launch_dwconv_ks<3, CLO>(c, s);
    case 5: return launch_dwconv_ks<5, CLO>(c, s);
    case 7: return launch_dwconv_ks<7, CLO>(c, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dwconv(const ConvArgs &c, int k, cudaStream_t s)
{
    return c.cl_out ? launch_dwconv_layout<true>(c, k, s) : launch_dwconv_layout<false>(c, k, s);
}

template <int NPL>
cudaError_t launch_norm_gate_cl_t(const NormArgs &n, cudaStream_t s)
{
    const long long pixels = (long long)n.B * n.L;
    const long long grid = (pixels + kNgThreads / 32 - 1) / (kNgThreads / 32);
    norm_gate_cl_kernel<NPL><<<(unsigned)grid, kNgThreads, 0, s>>>(n);
    return cudaGetLastError();
}

// Channels-last y: (B*L, D) rows, D <= 2 * 32 * kNgClMaxPairs.
cudaError_t launch_norm_gate_cl(const NormArgs &n, cudaStream_t s)
{
    const int npl = (n.D / 2 + 31) / 32;
    if (npl <= 1)
        return launch_norm_gate_cl_t<1>(n, s);
    if (npl <= 2)
        return launch_norm_gate_cl_t<2>(n, s);
    if (npl <= 3)
        return launch_norm_gate_cl_t<3>(n, s);
    if (npl <= 4)
        return launch_norm_gate_cl_t<4>(n, s);
    if (npl <= 6)
        return launch_norm_gate_cl_t<6>(n, s);
    if (npl <= 8)
        return launch_norm_gate_cl_t<8>(n, s);
    if (npl <= kNgClMaxPairs)
        return launch_norm_gate_cl_t<kNgClMaxPairs>(n, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_norm_gate(const NormArgs &n, cudaStream_t s)
{
    const unsigned grid = (unsigned)((long long)n.B * n.tiles_l);
    if (n.D <= kNgMaxDZ) {
        static int configured[kMaxDevices];
        const size_t smem = ng_smem_bytes(n.D, true);
        cudaError_t e = configure_smem(norm_gate_kernel<true>, (int)smem, configured);
        if (e != cudaSuccess)
            return e;
        norm_gate_kernel<true><<<grid, kNgThreads, smem, s>>>(n);
    } else {
        static int configured[kMaxDevices];
        const size_t smem = ng_smem_bytes(n.D, false);
        cudaError_t e = configure_smem(norm_gate_kernel<false>, (int)smem, configured);
        if (e != cudaSuccess)
            return e;
        norm_gate_kernel<false><<<grid, kNgThreads, smem, s>>>(n);
    }
    return cudaGetLastError();
}

// Where the core runs channels-last inside the block: x_c and y then stay in the pixel-major
// order of the projections, so the convolution stores pixel rows, the normalisation reads them
// and the core's column orders read x_c's channel runs.  That needs the core's channels-last
// form (N = 16, dt_rank <= 16 fused in the scan, one launch of at most 65535 32x32 tiles for the
// GEMM's transposed copy) and D <= 768 for the normalisation's registers; elsewhere the block
// runs channel-first.
bool block_channels_last(const ss2d_block_args *a)
{
    const long long tiles = (((long long)a->H * a->W + 31) / 32) * ((a->D + 31) / 32);
    return a->N == 16 && a->R >= 1 && a->R <= 16 && a->D <= 64 * kNgClMaxPairs && tiles <= 65535;
}

// The core's arguments for the block's x_c (bf16) and y (fp32), in the block's layout.
ss2d_core_args core_args_of(const ss2d_block_args *a, const void *xc, float *y)
{
    ss2d_core_args c;
    memset(&c, 0, sizeof(c));
    c.struct_size = sizeof(ss2d_core_args);
    c.B = a->B;
    c.D = a->D;
    c.H = a->H;
    c.W = a->W;
    c.N = a->N;
    c.R = a->R;
    c.x = xc;
    c.x_dtype = SS2D_BF16;
    c.A_logs = a->A_logs;
    c.Ds = a->Ds;
    c.dt_bias = a->dt_projs_bias;
    c.delta_softplus = 1;
    c.x_proj_weight = a->x_proj_weight;
    c.dt_projs_weight = a->dt_projs_weight;
    c.y = y;
    c.layout = block_channels_last(a) ? SS2D_CHANNELS_LAST : SS2D_CHANNELS_FIRST;
    c.y_dtype = SS2D_F32;
    c.merge_order = SS2D_MERGE_ATOMIC;
    return c;
}

struct BlockLayout {
    size_t core_off, core_bytes, xz_off, xc_off, y_off, total;
};

// Workspace: error word | the core's workspace | xz (M, 2D) bf16 | x_c (B, D, L) bf16, later g
// (M, D) bf16 | y (B, D, L) fp32, each part 256-byte aligned.
BlockLayout block_layout(const ss2d_block_args *a, size_t core_bytes)
{
    const size_t M = (size_t)a->B * a->H * a->W, D = a->D;
    BlockLayout l{};
    l.core_off = kHdr;
    l.core_bytes = core_bytes;
    l.xz_off = l.core_off + r256(core_bytes);
    l.xc_off = l.xz_off + r256(M * 2 * D * 2);
    l.y_off = l.xc_off + r256(M * D * 2);
    l.total = l.y_off + r256(M * D * 4);
    return l;
}

struct Span2 {
    const void *p;
    size_t n;
};

bool overlap2(Span2 x, Span2 y)
{
    if (!x.p || !y.p || !x.n || !y.n)
        return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x.p), b0 = reinterpret_cast<uintptr_t>(y.p);
    return a0 < b0 + y.n && b0 < a0 + x.n;
}

// Host checks of the block's arguments; on success *core_bytes is the core's workspace.
int check_block(const ss2d_block_args *a, bool check_out, size_t *core_bytes)
{
    if (!a)
        return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: args is null");
    if (a->struct_size != sizeof(ss2d_block_args))
        return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: struct_size %zu is not %zu", a->struct_size,
                     sizeof(ss2d_block_args));
    if (a->B <= 0 || a->H <= 0 || a->W <= 0 || a->d_model <= 0 || a->D <= 0 || a->N <= 0 || a->R <= 0 ||
        a->d_conv <= 0)
        return bfail(SS2D_ERR_INVALID_ARG,
                     "ss2d_block_forward: sizes must be positive (B=%d H=%d W=%d d_model=%d D=%d N=%d R=%d d_conv=%d)",
                     a->B, a->H, a->W, a->d_model, a->D, a->N, a->R, a->d_conv);
    if (a->d_conv % 2 == 0)
        return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: d_conv=%d must be odd", a->d_conv);
    if (!a->x || !a->in_proj_weight || !a->conv_weight || !a->x_proj_weight || !a->dt_projs_weight || !a->A_logs ||
        !a->out_norm_weight || !a->out_norm_bias || !a->out_proj_weight || (check_out && !a->out))
        return bfail(SS2D_ERR_INVALID_ARG,
                     "ss2d_block_forward: x, in_proj_weight, conv_weight, x_proj_weight, dt_projs_weight, A_logs, "
                     "out_norm_weight, out_norm_bias, out_proj_weight and out must be non-null");
    if (!(a->out_norm_eps > 0.0f) || a->out_norm_eps > 1e30f)
        return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: out_norm_eps must be positive and finite");
    if (a->out_dtype != SS2D_F32 && a->out_dtype != SS2D_BF16)
        return bfail(SS2D_ERR_UNSUPPORTED, "ss2d_block_forward: out_dtype %d is not SS2D_F32 or SS2D_BF16",
                     a->out_dtype);
    if (a->d_conv > 7)
        return bfail(SS2D_ERR_UNSUPPORTED, "ss2d_block_forward: d_conv=%d; 1, 3, 5 and 7 are built", a->d_conv);
    if (a->d_model % 16 != 0 || a->D % 16 != 0)
        return bfail(SS2D_ERR_UNSUPPORTED, "ss2d_block_forward: d_model=%d and D=%d must be multiples of 16",
                     a->d_model, a->D);
    if (a->D > kNgMaxD)
        return bfail(SS2D_ERR_UNSUPPORTED, "ss2d_block_forward: D=%d; the normalisation tile takes D <= %d", a->D,
                     kNgMaxD);
    if (a->N != 16)
        return bfail(SS2D_ERR_UNSUPPORTED, "ss2d_block_forward: N=%d; the block is built for N = 16", a->N);
    const long long M = (long long)a->B * a->H * a->W;
    const long long conv_blocks = (long long)a->B * ((a->H + kCvTH - 1) / kCvTH) * ((a->W + kCvTW - 1) / kCvTW) *
                                  ((a->D + kCvTC - 1) / kCvTC);
    const long long norm_blocks = (long long)a->B * ((a->H * (long long)a->W + kNgP - 1) / kNgP);
    if (M > 0x7fffffffLL || conv_blocks > 0x7fffffffLL || norm_blocks > 0x7fffffffLL)
        return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: problem too large");
    // the core's own checks, with x standing in for x_c (same type and alignment)
    ss2d_core_args c = core_args_of(a, a->x, nullptr);
    const int st = validate_core_args(&c, false);
    if (st != SS2D_OK)
        return st;
    const size_t cw = ss2d_forward_core_workspace(&c);
    if (cw == (size_t)-1)
        return bfail(SS2D_ERR_UNSUPPORTED, "ss2d_block_forward: the core rejects this shape");
    *core_bytes = cw;
    const void *ptrs[] = {a->x, a->in_proj_weight, a->in_proj_bias, a->conv_weight, a->conv_bias, a->x_proj_weight,
                          a->dt_projs_weight, a->dt_projs_bias, a->A_logs, a->Ds, a->out_norm_weight,
                          a->out_norm_bias, a->out_proj_weight, a->out_proj_bias, a->out};
    for (const void *p : ptrs)
        if (p && !al16(p))
            return bfail(SS2D_ERR_MISALIGNED, "ss2d_block_forward: every tensor must be 16-byte aligned");
    if (check_out) {
        const size_t D = a->D, dm = a->d_model, N = a->N, R = a->R, k = a->d_conv;
        const Span2 out{a->out, (size_t)M * dm * (a->out_dtype == SS2D_BF16 ? 2 : 4)};
        const Span2 ins[] = {{a->x, (size_t)M * dm * 2},
                             {a->in_proj_weight, 2 * D * dm * 2},
                             {a->in_proj_bias, a->in_proj_bias ? 2 * D * 4 : 0},
                             {a->conv_weight, D * k * k * 4},
                             {a->conv_bias, a->conv_bias ? D * 4 : 0},
                             {a->x_proj_weight, 4 * (R + 2 * N) * D * 2},
                             {a->dt_projs_weight, 4 * D * R * 4},
                             {a->dt_projs_bias, a->dt_projs_bias ? 4 * D * 4 : 0},
                             {a->A_logs, 4 * D * N * 4},
                             {a->Ds, a->Ds ? 4 * D * 4 : 0},
                             {a->out_norm_weight, D * 4},
                             {a->out_norm_bias, D * 4},
                             {a->out_proj_weight, dm * D * 2},
                             {a->out_proj_bias, a->out_proj_bias ? dm * 4 : 0}};
        for (const Span2 &s : ins)
            if (overlap2(s, out))
                return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: out overlaps an input");
    }
    return SS2D_OK;
}

}  // namespace
}  // namespace ss2d

extern "C" size_t ss2d_block_forward_workspace(const ss2d_block_args *args)
{
    ss2d::set_last_error(SS2D_OK, "");
    size_t core_bytes = 0;
    if (ss2d::check_block(args, false, &core_bytes) != SS2D_OK)
        return (size_t)-1;
    return ss2d::block_layout(args, core_bytes).total;
}

extern "C" int ss2d_block_forward(const ss2d_block_args *args, void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace ss2d;
    set_last_error(SS2D_OK, "");
    size_t core_bytes = 0;
    int st = check_block(args, true, &core_bytes);
    if (st != SS2D_OK)
        return st;
    const ss2d_block_args &a = *args;
    const BlockLayout lay = block_layout(args, core_bytes);
    const long long M = (long long)a.B * a.H * a.W;
    const int L = a.H * a.W, D = a.D;
    if (!workspace || workspace_bytes < lay.total)
        return bfail(SS2D_ERR_WORKSPACE, "ss2d_block_forward: workspace of %zu bytes needed, %zu given", lay.total,
                     workspace_bytes);
    if (!al16(workspace))
        return bfail(SS2D_ERR_MISALIGNED, "ss2d_block_forward: workspace must be 16-byte aligned");
    if (overlap2({workspace, lay.total}, {a.out, (size_t)M * a.d_model * (a.out_dtype == SS2D_BF16 ? 2 : 4)}))
        return bfail(SS2D_ERR_INVALID_ARG, "ss2d_block_forward: workspace overlaps out");
    char *ws = static_cast<char *>(workspace);
    int *err = reinterpret_cast<int *>(ws);
    void *core_ws = ws + lay.core_off;
    __nv_bfloat16 *xz = reinterpret_cast<__nv_bfloat16 *>(ws + lay.xz_off);
    __nv_bfloat16 *xc = reinterpret_cast<__nv_bfloat16 *>(ws + lay.xc_off);
    __nv_bfloat16 *g = xc;  // x_c is dead once the core has run
    float *y = reinterpret_cast<float *>(ws + lay.y_off);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
    if (e != cudaSuccess)
        return bcuda(e, "clearing the error word");
    // 1. input projection: xz = x W_in^T (+ b_in), bf16
    e = launch_rowgemm(static_cast<const __nv_bfloat16 *>(a.x), a.d_model,
                       static_cast<const __nv_bfloat16 *>(a.in_proj_weight), a.in_proj_bias, xz, 2 * D, true, M,
                       a.d_model, 2 * D, err, s);
    if (e != cudaSuccess)
        return bcuda(e, "input projection launch");
    // 2. depthwise convolution + SiLU of the scan branch, bf16, in the block's layout
    const bool cl = block_channels_last(args);
    ConvArgs cv{};
    cv.xz = xz;
    cv.w = a.conv_weight;
    cv.bias = a.conv_bias;
    cv.xc = xc;
    cv.B = a.B;
    cv.D = D;
    cv.H = a.H;
    cv.W = a.W;
    cv.ldx = 2 * D;
    cv.tiles_h = (a.H + kCvTH - 1) / kCvTH;
    cv.tiles_w = (a.W + kCvTW - 1) / kCvTW;
    cv.tiles_c = (D + kCvTC - 1) / kCvTC;
    cv.cl_out = cl ? 1 : 0;
    e = launch_dwconv(cv, a.d_conv, s);
    if (e != cudaSuccess)
        return bcuda(e, "convolution launch");
    // 3. the core, projection form, fp32 y in the block's layout
    ss2d_core_args c = core_args_of(args, xc, y);
    st = ss2d_forward_core(&c, core_ws, lay.core_bytes, stream);
    if (st != SS2D_OK)
        return st;
    // 4. LayerNorm over D, gated by SiLU(z), bf16
    NormArgs nm{};
    nm.y = y;
    nm.z = xz + D;
    nm.gamma = a.out_norm_weight;
    nm.beta = a.out_norm_bias;
    nm.g = g;
    nm.eps = a.out_norm_eps;
    nm.B = a.B;
    nm.D = D;
    nm.L = L;
    nm.ldz = 2 * D;
    nm.tiles_l = (L + kNgP - 1) / kNgP;
    e = cl ? launch_norm_gate_cl(nm, s) : launch_norm_gate(nm, s);
    if (e != cudaSuccess)
        return bcuda(e, "normalisation launch");
    // 5. output projection
    e = launch_rowgemm(g, D, static_cast<const __nv_bfloat16 *>(a.out_proj_weight), a.out_proj_bias, a.out,
                       a.d_model, a.out_dtype == SS2D_BF16, M, D, a.d_model, err, s);
    if (e != cudaSuccess)
        return bcuda(e, "output projection launch");
    return SS2D_OK;
}

extern "C" int ss2d_block_device_status(const ss2d_block_args *args, const void *workspace, void *stream)
{
    using namespace ss2d;
    set_last_error(SS2D_OK, "");
    size_t core_bytes = 0;
    int st = check_block(args, false, &core_bytes);
    if (st != SS2D_OK)
        return st;
    if (!workspace)
        return bfail(SS2D_ERR_WORKSPACE, "ss2d_block_device_status: workspace is null");
    const BlockLayout lay = block_layout(args, core_bytes);
    // the core's word (its own status call synchronises the stream)
    ss2d_core_args c = core_args_of(args, args->x, nullptr);
    st = ss2d_device_status(&c, static_cast<const char *>(workspace) + lay.core_off, 0, stream);
    if (st != SS2D_OK)
        return st;
    int word = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return bcuda(e, "reading the error word");
    if (word != 0)
        return bfail(SS2D_ERR_DEVICE, "ss2d_block_forward: a tensor-core kernel's bounded wait ran out; out is not valid");
    return SS2D_OK;
}
