// Host emulation of the CUDA features the kernels use: one std::thread per lane,
// warp-synchronous operations on a per-warp barrier, __syncthreads on a per-CTA barrier,
// cp.async as checked immediate copies.
#pragma once
#include <atomic>
#include <barrier>
#include <cassert>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <memory>
#include <thread>
#include <type_traits>
#include <vector>
#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __align__(n) alignas(n)
struct dim3e { unsigned x, y, z; };
inline thread_local dim3e threadIdx, blockIdx, blockDim, gridDim;
struct float2 { float x, y; };
struct alignas(16) float4 { float x, y, z, w; };
struct int2 { int x, y; };
struct uint2 { unsigned x, y; };
inline float2 make_float2(float a, float b) { return {a, b}; }
inline float4 make_float4(float a, float b, float c, float d) { return {a, b, c, d}; }
struct __nv_bfloat16 { uint16_t v; };
inline float __bfloat162float(__nv_bfloat16 b) { uint32_t u = (uint32_t)b.v << 16; float f; memcpy(&f, &u, 4); return f; }
inline float __uint_as_float(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
inline uint32_t __float_as_uint(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
inline float __fdividef(float a, float b) { return a / b; }
inline float2 __fmul2_rn(float2 a, float2 b) { return {a.x * b.x, a.y * b.y}; }
inline float2 __fadd2_rn(float2 a, float2 b) { return {a.x + b.x, a.y + b.y}; }
inline float2 __ffma2_rn(float2 a, float2 b, float2 c) { return {fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y)}; }
template <class T> inline T __ldg(const T *p) { return *p; }
using std::min; using std::max;
inline float atomicAdd(float *p, float v) { return std::atomic_ref<float>(*p).fetch_add(v); }

// per-CTA warp context
struct WarpCtx {
    std::barrier<> bar{32};
    float slot[32];
    unsigned char *smem;
    size_t smem_bytes;
};
inline thread_local WarpCtx *g_warp;
inline thread_local int g_lane;
inline void __syncwarp(unsigned = 0xffffffffu) { g_warp->bar.arrive_and_wait(); }
inline float __shfl_xor_sync(unsigned mask, float v, int d)
{
    if (mask != 0xffffffffu) { fprintf(stderr, "shfl with partial mask\n"); abort(); }
    g_warp->slot[g_lane] = v;
    g_warp->bar.arrive_and_wait();
    float r = g_warp->slot[g_lane ^ d];
    g_warp->bar.arrive_and_wait();
    return r;
}
// per-CTA context of a kernel with more than one warp (the warps share the CTA's shared memory)
struct BlockCtx {
    std::barrier<> bar;
    explicit BlockCtx(int threads) : bar(threads) {}
};
inline thread_local BlockCtx *g_block;
inline void __syncthreads() { g_block->bar.arrive_and_wait(); }
inline bool in_smem(const void *p, size_t n)
{
    const unsigned char *c = (const unsigned char *)p;
    return c >= g_warp->smem && c + n <= g_warp->smem + g_warp->smem_bytes;
}
// prmt (byte permute): byte i of the result is byte s_i of the 8-byte value {b, a} (a is bytes
// 0-3), where s_i is the low 3 bits of nibble i of the selector.
inline uint32_t __byte_perm(uint32_t a, uint32_t b, uint32_t s)
{
    const uint64_t v = ((uint64_t)b << 32) | a;
    uint32_t r = 0;
    for (int i = 0; i < 4; ++i)
        r |= (uint32_t)((v >> (8 * ((s >> (4 * i)) & 7))) & 0xff) << (8 * i);
    return r;
}
// Runs fn() as every thread of a (gx, gy) grid of CTAs of `threads` threads (a multiple of 32)
// that share `smem_bytes` of shared memory per CTA, one CTA after another.
template <class F>
void emu_grid(unsigned gx, unsigned gy, int threads, size_t smem_bytes, F fn)
{
    for (unsigned by = 0; by < gy; ++by)
        for (unsigned bx = 0; bx < gx; ++bx) {
            BlockCtx blk(threads);
            const int nw = threads / 32;
            std::unique_ptr<WarpCtx[]> warps(new WarpCtx[nw]);
            std::vector<unsigned char> smem(smem_bytes + 16);
            unsigned char *base = smem.data() + (16 - ((uintptr_t)smem.data() & 15)) % 16;
            memset(base, 0xCD, smem_bytes);
            for (int w = 0; w < nw; ++w) {
                warps[w].smem = base;
                warps[w].smem_bytes = smem_bytes;
            }
            std::vector<std::thread> th;
            for (int t = 0; t < threads; ++t)
                th.emplace_back([&, t] {
                    threadIdx = {(unsigned)t, 0, 0};
                    blockIdx = {bx, by, 0};
                    blockDim = {(unsigned)threads, 1, 1};
                    gridDim = {gx, gy, 1};
                    g_block = &blk;
                    g_warp = &warps[t / 32];
                    g_lane = t % 32;
                    fn();
                });
            for (auto &t : th) t.join();
        }
}
