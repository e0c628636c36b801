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

// Shapes: <N, lanes per channel, channels per lane, CTAs per SM for the register budget, mode>.
// Every CTA is one warp working on 32/TN * CH channels of one (batch, group).
template <int MODE>
cudaError_t dispatch(const ScanArgs &a, int N, cudaStream_t s)
{
    switch (N) {
    case 16: return launch_one<ScanShape<16, 4, 2, 12, MODE>>(a, s);
    case 8: return launch_one<ScanShape<8, 2, 2, 8, MODE>>(a, s);
    case 4: return launch_one<ScanShape<4, 1, 1, 8, MODE>>(a, s);
    case 2: return launch_one<ScanShape<2, 1, 1, 8, MODE>>(a, s);
    case 1: return launch_one<ScanShape<1, 1, 1, 8, MODE>>(a, s);
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
