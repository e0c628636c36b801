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

// Only the fp32 instantiation is built: the caller widens bf16 x and dts to fp32 first.
// With a.nseg > 1 the sequences are walked in segments: a first pass and a carry give what
// enters each segment (a.e_out, a.p_out, a.g_in: (B, 4D, nseg, 16) each, from the caller).
cudaError_t launch_scan_bwd(const BwdArgs &a, cudaStream_t s)
{
    return launch_bwd_t<4>(a, s);
}

}  // namespace ss2d
