// scan.cu -- instantiations and launchers of the selective-scan kernels.
#include "kernels.h"
#include "launch_util.h"
#include "scan.cuh"
#include "scan2.cuh"

namespace ss2d {

namespace {

template <class S>
cudaError_t launch_one(const ScanArgs &a, cudaStream_t s)
{
    ScanArgs args = a;
    S::layout(args);
    static int configured[kMaxDevices] = {};
    cudaError_t e = configure_smem(scan_kernel<S>, args.smem_bytes, configured);
    if (e != cudaSuccess)
        return e;
    args.tiles = (a.per_group + S::CW - 1) / S::CW;
    const long long items = (long long)args.tiles * a.G * a.B * args.nseg;
    if (items > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    scan_kernel<S><<<(unsigned)items, 32, args.smem_bytes, s>>>(args);
    return cudaGetLastError();
}

// The N = 16 kernel with delta computed inside the scan loop (SEGP: first pass of a
// segmented scan).
template <int MODE, int DT, int SEGP = 0, int CL = 0>
cudaError_t launch_two(const ScanArgs &a, cudaStream_t s)
{
    using S = Scan2Shape<MODE, DT, SEGP, CL>;
    const Scan2Layout lay = S::layout();
    static int configured[kMaxDevices] = {};
    cudaError_t e = configure_smem(scan2_kernel<S>, lay.smem_bytes, configured);
    if (e != cudaSuccess)
        return e;
    ScanArgs args = a;
    args.tiles = (a.per_group + S::CW - 1) / S::CW;
    const int gn = a.gn > 0 ? a.gn : a.G;
    if (a.g0 < 0 || a.g0 + gn > a.G)
        return cudaErrorInvalidValue;
    const long long items = (long long)args.tiles * gn * a.B * args.nseg;
    if (items > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    scan2_kernel<S><<<(unsigned)items, 32, lay.smem_bytes, s>>>(args, lay);
    return cudaGetLastError();
}

// Shapes: <N, lanes per channel, channels per lane, CTAs per SM for the register budget, mode,
// element-type variant>.  Every CTA is one warp working on 32/TN * CH channels of one
// (batch, group).  The common N = 16 cases are compiled for their element types (bf16 or
// fp32 u/delta with softplus); everything else reads the types at run time.
template <int MODE, int N, int TN, int CH, int MINB>
cudaError_t by_types(const ScanArgs &a, cudaStream_t s)
{
    const int dt = (a.delta_bf16 ? 1 : 0) | (a.u_bf16 ? 2 : 0) | (a.softplus ? 4 : 0);
    if (N == 16 && a.nseg == 1) {
        if constexpr (MODE == kFusedProj) {
            if (dt == 6 && a.R <= kMaxR)
                return a.ch_last ? launch_two<MODE, 6, 0, 1>(a, s) : launch_two<MODE, 6>(a, s);
        } else if constexpr (MODE == kFused) {
            // a.ckpt: the forward also stores its backward's checkpoints
            if (a.ch_last) {
                if (dt == 7)
                    return a.ckpt ? launch_two<MODE, 7, 3, 1>(a, s) : launch_two<MODE, 7, 0, 1>(a, s);
                if (dt == 4)
                    return a.ckpt ? launch_two<MODE, 4, 3, 1>(a, s) : launch_two<MODE, 4, 0, 1>(a, s);
                return cudaErrorInvalidValue;
            }
            if (dt == 7)
                return a.ckpt ? launch_two<MODE, 7, 3>(a, s) : launch_two<MODE, 7>(a, s);
            if (dt == 4)
                return a.ckpt ? launch_two<MODE, 4, 3>(a, s) : launch_two<MODE, 4>(a, s);
        } else {
            if (dt == 7)
                return launch_two<MODE, 7>(a, s);
            if (dt == 4)
                return launch_two<MODE, 4>(a, s);
        }
    }
    if (a.ch_last)
        return cudaErrorInvalidValue;  // channels-last runs on the N = 16 kernel only
    if constexpr (MODE == kFusedProj) {
        if (dt == 6)  // bf16 x, softplus (no delta input)
            return launch_one<ScanShape<N, TN, CH, MINB, MODE, 6>>(a, s);
    } else {
        if (dt == 7)
            return launch_one<ScanShape<N, TN, CH, MINB, MODE, 7>>(a, s);
        if (dt == 4)
            return launch_one<ScanShape<N, TN, CH, MINB, MODE, 4>>(a, s);
    }
    return launch_one<ScanShape<N, TN, CH, MINB, MODE, kDtRuntime>>(a, s);
}

template <int MODE>
cudaError_t dispatch(const ScanArgs &a, int N, cudaStream_t s)
{
    switch (N) {
    case 16:
        if constexpr (MODE == kStandalone)
            return by_types<MODE, 16, 2, 1, 12>(a, s);
        else
            return by_types<MODE, 16, 4, 1, 12>(a, s);
    case 8: return launch_one<ScanShape<8, 2, 1, 12, MODE, kDtRuntime>>(a, s);
    case 4: return launch_one<ScanShape<4, 1, 1, 8, MODE, kDtRuntime>>(a, s);
    case 2: return launch_one<ScanShape<2, 1, 1, 8, MODE, kDtRuntime>>(a, s);
    case 1: return launch_one<ScanShape<1, 1, 1, 8, MODE, kDtRuntime>>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

// Carries the segment states of a segmented scan: h_in(0) = 0 and
// h_in(s+1) = P(s) h_in(s) + h_end(s), where h_end(s) is the state the first pass
// reached in segment s from a zero start and P(s) the product of its decays (the
// first pass records neither for the last segment).
__global__ void segment_carry_kernel(const float *__restrict__ hend, const float *__restrict__ pend,
                                     float *__restrict__ hin, long long total, int nseg, int N)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const long long bc = idx / N;
    const int n = (int)(idx % N);
    float h = 0.0f;
    for (int sg = 0; sg < nseg; ++sg) {
        const size_t o = ((size_t)bc * nseg + sg) * N + n;
        hin[o] = h;
        if (sg + 1 < nseg)
            h = fmaf(pend[o], h, hend[o]);
    }
}

template <int MODE, int DT, int CL>
cudaError_t launch_segmented(const ScanArgs &a, float *seg_ws, cudaStream_t s)
{
    const size_t n = (size_t)a.B * a.C * a.nseg * 16;
    ScanArgs p1 = a;
    p1.h0 = nullptr;
    p1.ckpt = nullptr;
    p1.hend = seg_ws;
    p1.pend = seg_ws + n;
    cudaError_t e = launch_two<MODE, DT, 1, CL>(p1, s);
    if (e != cudaSuccess)
        return e;
    const long long total = (long long)a.B * a.C * 16;
    segment_carry_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(p1.hend, p1.pend, seg_ws + 2 * n, total,
                                                                          a.nseg, 16);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    ScanArgs p3 = a;
    p3.h0 = seg_ws + 2 * n;
    if constexpr (MODE == kFused) {
        if (a.ckpt)  // the second pass also stores the backward's checkpoints
            return launch_two<MODE, DT, 3, CL>(p3, s);
    }
    return launch_two<MODE, DT, 0, CL>(p3, s);
}

}  // namespace

// One-warp scan2_kernel CTAs resident per B200 SM: its launch bounds allow 12, and each
// CTA takes its shared-memory layout plus the 1 KB the SM reserves per CTA, out of 228 KB.
int scan2_ctas_per_sm(int mode, int dt, int ch_last)
{
    Scan2Layout l{};
    if (mode == kFusedProj)
        l = ch_last ? Scan2Shape<kFusedProj, 6, 0, 1>::layout() : Scan2Shape<kFusedProj, 6>::layout();
    else if (dt & 3)  // bf16 u and delta (the compiled bf16 variant)
        l = ch_last ? Scan2Shape<kFused, 7, 0, 1>::layout() : Scan2Shape<kFused, 7>::layout();
    else
        l = ch_last ? Scan2Shape<kFused, 4, 0, 1>::layout() : Scan2Shape<kFused, 4>::layout();
    const int by_smem = (228 * 1024) / (l.smem_bytes + 1024);
    return by_smem < 12 ? (by_smem > 0 ? by_smem : 1) : 12;
}

void plan_segments(int B, int G, int per_group, int L, int N, int mode, int u_bf16, int delta_bf16, int softplus,
                   int *nseg, int *seg_len)
{
    *nseg = 1;
    *seg_len = L;
    const int dt = (delta_bf16 ? 1 : 0) | (u_bf16 ? 2 : 0) | (softplus ? 4 : 0);
    const bool fused = mode == kFused && (dt == 7 || dt == 4);
    const bool proj = mode == kFusedProj && dt == 6;  // bf16 x, delta from dt_low, softplus
    if (N != 16 || !(fused || proj))
        return;
    const int cw = Scan2Shape<kFused, 7>::CW;  // channels per warp of the N = 16 kernel
    const long long items = (long long)B * G * ((per_group + cw - 1) / cw);
    const long long target = 148LL * scan2_ctas_per_sm(mode, dt, 0);  // one wave
    if (items >= target || L < 8 * kTC)
        return;
    // as many segments as still fit in one wave, each at least four chunks long
    int ns = (int)(target / items);
    ns = ns < L / (4 * kTC) ? ns : L / (4 * kTC);
    if (ns < 2)
        return;
    int len = (L + ns - 1) / ns;
    len = (len + kTC - 1) / kTC * kTC;  // whole chunks: the first pass never sees a partial one
    *seg_len = len;
    *nseg = (L + len - 1) / len;
}

bool scan_reads_transposed_u(int N, int mode, int u_bf16, int delta_bf16, int softplus, int L)
{
    if (N != 16 || ((size_t)L * (u_bf16 ? 2 : 4)) % 16 != 0)
        return false;
    const int dt = (delta_bf16 ? 1 : 0) | (u_bf16 ? 2 : 0) | (softplus ? 4 : 0);
    if (mode == kFused)
        return dt == 7 || dt == 4;
    if (mode == kFusedProj)
        return dt == 6;
    return false;
}

size_t segment_workspace_bytes(int B, int C, int nseg, int N)
{
    return nseg > 1 ? 3 * (size_t)B * C * nseg * N * sizeof(float) : 0;
}

cudaError_t launch_scan_segmented(const ScanArgs &a, int N, int mode, float *seg_ws, cudaStream_t s)
{
    if (N != 16 || a.nseg < 2 || !seg_ws)
        return cudaErrorInvalidValue;
    if (a.seg_len % kTC != 0)
        return cudaErrorInvalidValue;
    const int dt = (a.delta_bf16 ? 1 : 0) | (a.u_bf16 ? 2 : 0) | (a.softplus ? 4 : 0);
    if (mode == kFusedProj) {
        if (dt != 6 || a.R > kMaxR)
            return cudaErrorInvalidValue;
        return a.ch_last ? launch_segmented<kFusedProj, 6, 1>(a, seg_ws, s)
                         : launch_segmented<kFusedProj, 6, 0>(a, seg_ws, s);
    }
    if (mode != kFused)
        return cudaErrorInvalidValue;
    if (dt == 7)
        return a.ch_last ? launch_segmented<kFused, 7, 1>(a, seg_ws, s) : launch_segmented<kFused, 7, 0>(a, seg_ws, s);
    if (dt == 4)
        return a.ch_last ? launch_segmented<kFused, 4, 1>(a, seg_ws, s) : launch_segmented<kFused, 4, 0>(a, seg_ws, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_scan_checkpoints(const ScanArgs &a0, float *ckpt, cudaStream_t s)
{
    ScanArgs a = a0;
    a.nseg = 1;
    a.seg_len = a.L;
    a.h0 = nullptr;
    a.ckpt = ckpt;
    const int dt = (a.delta_bf16 ? 1 : 0) | (a.u_bf16 ? 2 : 0) | (a.softplus ? 4 : 0);
    if (dt == 7)
        return launch_two<kFused, 7, 2>(a, s);
    if (dt == 6)  // bf16 u, fp32 delta (the projection form's backward)
        return launch_two<kFused, 6, 2>(a, s);
    if (dt == 4)
        return launch_two<kFused, 4, 2>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_scan_checkpoints_segmented(const ScanArgs &a0, float *ckpt, float *seg_ws, cudaStream_t s)
{
    if (a0.nseg < 2 || !seg_ws || a0.seg_len % kTC != 0)
        return cudaErrorInvalidValue;
    const int dt = (a0.delta_bf16 ? 1 : 0) | (a0.u_bf16 ? 2 : 0) | (a0.softplus ? 4 : 0);
    if (dt != 7 && dt != 4)
        return cudaErrorInvalidValue;
    const size_t n = (size_t)a0.B * a0.C * a0.nseg * 16;
    ScanArgs p1 = a0;
    p1.h0 = nullptr;
    p1.ckpt = nullptr;
    p1.hend = seg_ws;
    p1.pend = seg_ws + n;
    cudaError_t e = dt == 7 ? launch_two<kFused, 7, 1>(p1, s) : launch_two<kFused, 4, 1>(p1, s);
    if (e != cudaSuccess)
        return e;
    const long long total = (long long)a0.B * a0.C * 16;
    segment_carry_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(p1.hend, p1.pend, seg_ws + 2 * n, total,
                                                                          a0.nseg, 16);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    ScanArgs p2 = a0;
    p2.h0 = seg_ws + 2 * n;
    p2.ckpt = ckpt;
    return dt == 7 ? launch_two<kFused, 7, 2>(p2, s) : launch_two<kFused, 4, 2>(p2, s);
}

cudaError_t launch_scan(const ScanArgs &a0, int N, int mode, cudaStream_t s)
{
    ScanArgs a = a0;
    if (a.nseg <= 0) {
        a.nseg = 1;
        a.seg_len = a.L;
    }
    switch (mode) {
    case kStandalone: return dispatch<kStandalone>(a, N, s);
    case kFused: return dispatch<kFused>(a, N, s);
    case kFusedProj: return dispatch<kFusedProj>(a, N, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ss2d
