// scan.cu -- instantiations and launcher of the selective-scan kernel.
#include "kernels.h"
#include "scan.cuh"

namespace ss2d {

namespace {

template <class S>
cudaError_t launch_one(const ScanArgs &a, cudaStream_t s)
{
    ScanArgs args = a;
    S::layout(args);
    static int configured_bytes = 0;
    if (args.smem_bytes > configured_bytes) {
        cudaError_t e = cudaFuncSetAttribute(scan_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             args.smem_bytes);
        if (e != cudaSuccess)
            return e;
        e = cudaFuncSetAttribute(scan_kernel<S>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess)
            return e;
        configured_bytes = args.smem_bytes;
    }
    args.tiles = (a.per_group + S::CW - 1) / S::CW;
    const long long items = (long long)args.tiles * a.G * a.B;
    if (items > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    scan_kernel<S><<<(unsigned)items, 32, args.smem_bytes, s>>>(args);
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

}  // namespace

cudaError_t launch_scan(const ScanArgs &a, int N, int mode, cudaStream_t s)
{
    switch (mode) {
    case kStandalone: return dispatch<kStandalone>(a, N, s);
    case kFused: return dispatch<kFused>(a, N, s);
    case kFusedProj: return dispatch<kFusedProj>(a, N, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ss2d
