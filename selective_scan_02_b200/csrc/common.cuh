// common.cuh -- small device helpers shared by the libss2d kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ss2d {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Element access for the two supported storage types.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ float ldg_f32(const T *p) { return to_f32(__ldg(p)); }

// Hardware base-2 exponential and logarithm (MUFU), flush-to-zero.
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2_approx(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log1p(e) for e = exp(-|z|) in [0, 1], as e * r(e) with r(e) = log1p(e) / e a
// degree-7 polynomial fitted on [0, 1] for least maximum relative error (an iterated
// weighted least-squares fit, the Remez method's fixed point).  Relative error
// below 4e-7 over [0, 1] in fp32 Horner evaluation; no MUFU operation.
__device__ __forceinline__ float log1p_unit_f32(float e)
{
    float r = fmaf(-0.008561575785279274f, e, 0.04416891559958458f);
    r = fmaf(r, e, -0.10779239237308502f);
    r = fmaf(r, e, 0.17752929031848907f);
    r = fmaf(r, e, -0.24498216807842255f);
    r = fmaf(r, e, 0.3327595293521881f);
    r = fmaf(r, e, -0.4999743700027466f);
    r = fmaf(r, e, 0.9999998211860657f);
    return e * r;
}

// softplus(z) = log(1 + e^z) = max(z, 0) + log1p(e^-|z|).
__device__ __forceinline__ float softplus_f32(float z)
{
    const float e = ex2_approx(-fabsf(z) * kLog2e);
    return fmaxf(z, 0.0f) + log1p_unit_f32(e);
}


// softplus(z) and its derivative sigmoid(z) = e^z / (1 + e^z), sharing e = exp(-|z|).
__device__ __forceinline__ void softplus_sigmoid_f32(float z, float &sp, float &sig)
{
    const float e = ex2_approx(-fabsf(z) * kLog2e);
    sp = fmaxf(z, 0.0f) + log1p_unit_f32(e);
    sig = __fdividef(z >= 0.0f ? 1.0f : e, 1.0f + e);
}

// Asynchronous global->shared copies (cp.async, L2-cached, bypassing L1).
// `src_bytes` < size zero-fills the remainder of the destination.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem, int src_bytes)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}

// L2 eviction-priority policies for the cache hints below (whole access range).
__device__ __forceinline__ uint64_t l2_policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// cp_async16 with an L2 eviction-priority hint for the source lines.
__device__ __forceinline__ void cp_async16_hint(void *smem, const void *gmem, int src_bytes, uint64_t policy)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(s), "l"(gmem),
                 "r"(src_bytes), "l"(policy));
}

// Relaxed fp32 atomic add without return, with an L2 eviction-priority hint for the line.
__device__ __forceinline__ void red_add_hint(float *gmem, float v, uint64_t policy)
{
    asm volatile("red.global.add.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(gmem), "f"(v), "l"(policy) : "memory");
}

// Relaxed 16-byte vector fp32 atomic add without return (4 consecutive elements), with an
// L2 eviction-priority hint; the address must be 16-byte aligned.
__device__ __forceinline__ void red_add_v4_hint(float *gmem, float4 v, uint64_t policy)
{
    asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(gmem), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

template <int Pending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(Pending)); }

// Quotient and remainder of l by a small positive divisor whose reciprocal
// is precomputed; exact for l < 2^24 (the float product is corrected by one).
struct SmallDiv {
    int d;
    float inv;
};

__device__ __forceinline__ void divmod(int l, SmallDiv s, int &q, int &r)
{
    int qq = static_cast<int>(static_cast<float>(l) * s.inv);
    int rr = l - qq * s.d;
    if (rr < 0) { --qq; rr += s.d; }
    else if (rr >= s.d) { ++qq; rr -= s.d; }
    q = qq;
    r = rr;
}

// Pixel p = h*W + w visited at step l by scan direction k (SS2D article,
// section 4): 0 row-major, 1 column-major, 2 and 3 their reverses.
__device__ __forceinline__ int scan_pixel(int k, int l, int L, int W, SmallDiv divH)
{
    if (k >= 2)
        l = L - 1 - l;
    if ((k & 1) == 0)
        return l;
    int w, h;
    divmod(l, divH, w, h);
    return h * W + w;
}

}  // namespace ss2d
