// Host versions of the device helpers of common.cuh used by the kernels (same arithmetic
// formulas; exp2/log2 from the C library in place of the hardware units).
#pragma once
#include "cuda_emu.h"
namespace ss2d {
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
inline float ex2_approx(float x) { return exp2f(x); }
inline float lg2_approx(float x) { return log2f(x); }
inline float log1p_unit_f32(float e)
{
    float r = fmaf(-0.008561575785279274f, e, 0.04416891559958458f);
    r = fmaf(r, e, -0.10779239237308502f); r = fmaf(r, e, 0.17752929031848907f);
    r = fmaf(r, e, -0.24498216807842255f); r = fmaf(r, e, 0.3327595293521881f);
    r = fmaf(r, e, -0.4999743700027466f); r = fmaf(r, e, 0.9999998211860657f);
    return e * r;
}
inline float softplus_f32(float z) { const float e = ex2_approx(-fabsf(z) * kLog2e); return fmaxf(z, 0.0f) + log1p_unit_f32(e); }
inline void softplus_sigmoid_f32(float z, float &sp, float &sig)
{
    const float e = ex2_approx(-fabsf(z) * kLog2e);
    sp = fmaxf(z, 0.0f) + log1p_unit_f32(e);
    sig = __fdividef(z >= 0.0f ? 1.0f : e, 1.0f + e);
}
inline uint64_t l2_policy_evict_first() { return 1; }
inline uint64_t l2_policy_evict_last() { return 2; }
inline void cp_async_copy(void *smem, const void *gmem, int n, int bytes)
{
    if (!in_smem(smem, n) || ((uintptr_t)smem % n) != 0) { fprintf(stderr, "cp.async bad smem dst\n"); abort(); }
    if (bytes < 0 || bytes > n) { fprintf(stderr, "cp.async bad size %d\n", bytes); abort(); }
    if (bytes > 0 && ((uintptr_t)gmem % n) != 0) { fprintf(stderr, "cp.async misaligned src %p (%d)\n", gmem, n); abort(); }
    memset(smem, 0, n);
    if (bytes) memcpy(smem, gmem, bytes);
}
inline void cp_async16(void *smem, const void *gmem, int b) { cp_async_copy(smem, gmem, 16, b); }
inline void cp_async16_hint(void *smem, const void *gmem, int b, uint64_t) { cp_async_copy(smem, gmem, 16, b); }
inline void cp_async4(void *smem, const void *gmem, int b) { cp_async_copy(smem, gmem, 4, b); }
inline void cp_async_commit() {}
template <int P> inline void cp_async_wait() {}
inline void red_add_hint(float *p, float v, uint64_t) { atomicAdd(p, v); }
inline void red_add_v4_hint(float *p, float4 v, uint64_t)
{
    if (((uintptr_t)p & 15) != 0) { fprintf(stderr, "red.v4 misaligned %p\n", (void *)p); abort(); }
    atomicAdd(p, v.x); atomicAdd(p + 1, v.y); atomicAdd(p + 2, v.z); atomicAdd(p + 3, v.w);
}
struct SmallDiv { int d; float inv; };
inline void divmod(int l, SmallDiv s, int &q, int &r)
{
    int qq = static_cast<int>(static_cast<float>(l) * s.inv);
    int rr = l - qq * s.d;
    if (rr < 0) { --qq; rr += s.d; } else if (rr >= s.d) { ++qq; rr -= s.d; }
    q = qq; r = rr;
}
inline int scan_pixel(int k, int l, int L, int W, SmallDiv divH)
{
    if (k >= 2) l = L - 1 - l;
    if ((k & 1) == 0) return l;
    int w, h; divmod(l, divH, w, h); return h * W + w;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
}  // namespace ss2d
