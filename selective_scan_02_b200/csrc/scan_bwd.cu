// scan_bwd.cu -- instantiations and launcher of the backward scan kernel.
#include "kernels.h"
#include "launch_util.h"
#include "scan_bwd.cuh"

namespace ss2d {

namespace {

// What enters each segment of the segmented backward, from the last segment down:
// in(S-1) = 0, in(s-1) = e(s) + p(s) * in(s).
__global__ void adjoint_carry_in_kernel(const float *__restrict__ e_out, const float *__restrict__ p_out,
                                        float *__restrict__ g_in, long long total, int nseg, int N)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const long long bc = idx / N;
    const int n = (int)(idx % N);
    float c = 0.0f;
    for (int sg = nseg - 1; sg >= 0; --sg) {
        const size_t o = ((size_t)bc * nseg + sg) * N + n;
        g_in[o] = c;
        if (sg > 0)
            c = fmaf(p_out[o], c, e_out[o]);
    }
}

template <int DT>
cudaError_t launch_bwd_t(const BwdArgs &a0, cudaStream_t s)
{
    using S = BwdShape<DT>;
    const BwdLayout lay = S::layout();
    static int configured[kMaxDevices] = {};
    cudaError_t e = configure_smem(scan_bwd_kernel<S>, lay.smem_bytes, configured);
    if (e != cudaSuccess)
        return e;
    BwdArgs a = a0;
    if (a.nseg < 1) {
        a.nseg = 1;
        a.seg_len = a.L;
    }
    a.tiles = (a.D + S::CW - 1) / S::CW;
    const long long items = (long long)a.tiles * 4 * a.B * a.nseg;
    if (items > 0x7fffffffLL || items < 1)
        return cudaErrorInvalidConfiguration;
    if (a.nseg > 1) {
        // first pass over segments 1..nseg-1, then what enters every segment
        // the first pass walks whole 4-step blocks and 16-byte rows: L % 4 == 0
        if (!a.e_out || !a.p_out || !a.g_in || a.seg_len % 32 != 0 || a.L % 4 != 0)
            return cudaErrorInvalidValue;
        static int configured_c[kMaxDevices] = {};
        e = configure_smem(adjoint_carry_kernel<S>, lay.smem_bytes, configured_c);
        if (e != cudaSuccess)
            return e;
        adjoint_carry_kernel<S><<<(unsigned)items, 32, lay.smem_bytes, s>>>(a, lay);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
        const long long total = (long long)a.B * a.C * S::N;
        adjoint_carry_in_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
            a.e_out, a.p_out, a.g_in, total, a.nseg, S::N);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    } else {
        a.g_in = nullptr;
    }
    scan_bwd_kernel<S><<<(unsigned)items, 32, lay.smem_bytes, s>>>(a, lay);
    return cudaGetLastError();
}

}  // namespace

bool scan_bwd_supported(int N, int u_bf16, int delta_bf16, int softplus, int L)
{
    (void)L;  // rows whose length is not a multiple of 4 are staged with 4-byte copies
    return N == 16 && softplus && (u_bf16 != 0) == (delta_bf16 != 0);
}

// One-warp scan_bwd_kernel CTAs resident per B200 SM: its launch bounds allow 8, and each CTA
// takes its shared-memory layout plus the 1 KB the SM reserves per CTA, out of 228 KB.
int scan_bwd_ctas_per_sm()
{
    const int by_smem = (228 * 1024) / (BwdShape<4>::layout().smem_bytes + 1024);
    return by_smem < 8 ? (by_smem > 0 ? by_smem : 1) : 8;
}

void plan_bwd_segments(int B, int D, int L, int *nseg, int *seg_len)
{
    *nseg = 1;
    *seg_len = L;
    const long long items = (long long)B * 4 * ((D + BwdShape<4>::CW - 1) / BwdShape<4>::CW);
    const long long slots = 148LL * scan_bwd_ctas_per_sm();
    if (items >= slots || L < 8 * 32 || L % 4 != 0)
        return;
    // Every segment costs about the same, so the walk takes ceil(items * nseg / slots) waves of
    // seg_len steps: take the fewest segments whose waves are at least 98 % full, else the
    // fullest.  Segments are whole 32-step chunks, at least four of them.
    const int max_ns = L / 128 < 128 ? L / 128 : 128;
    double best = 0.0;
    for (int ns = 2; ns <= max_ns; ++ns) {
        int len = (L + ns - 1) / ns;
        len = (len + 31) / 32 * 32;
        const int n = (L + len - 1) / len;
        const long long work = items * n;
        const double full = (double)work / (double)(((work + slots - 1) / slots) * slots);
        if (full > best + 1e-9) {
            best = full;
            *nseg = n;
            *seg_len = len;
        }
        if (full >= 0.98)
            break;
    }
}

// Only the fp32 instantiation is built: the caller widens bf16 x and dts to fp32 first.
// With a.nseg > 1 the sequences are walked in segments: a first pass and a carry give what
// enters each segment (a.e_out, a.p_out, a.g_in: (B, 4D, nseg, 16) each, from the caller).
cudaError_t launch_scan_bwd(const BwdArgs &a, cudaStream_t s)
{
    return launch_bwd_t<4>(a, s);
}

}  // namespace ss2d
