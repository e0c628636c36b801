// scan.cu -- instantiations and launcher of the selective-scan kernel.
#include "kernels.h"
#include "scan.cuh"

namespace ss2d {

namespace {

template <class S, int MODE>
cudaError_t launch_one(const ScanArgs &a, cudaStream_t s)
{
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(scan_kernel<S, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)S::SMEM_BYTES);
        if (e != cudaSuccess)
            return e;
        configured = true;
    }
    ScanArgs args = a;
    args.tiles = (a.per_group + S::CT - 1) / S::CT;
    const long long blocks = (long long)args.tiles * a.G * a.B;
    if (blocks > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    scan_kernel<S, MODE><<<(unsigned)blocks, S::THREADS, S::SMEM_BYTES, s>>>(args);
    return cudaGetLastError();
}

// Channel tile per CTA: 32 channels for the usual widths, 8 for narrow groups;
// up to 4 threads per channel, each holding N/4 states (at least one).
template <int MODE>
cudaError_t dispatch(const ScanArgs &a, int N, cudaStream_t s)
{
    const bool narrow = a.per_group <= 16;
    switch (N) {
    case 16: return narrow ? launch_one<ScanShape<16, 4, 8, 32>, MODE>(a, s) : launch_one<ScanShape<16, 4, 32, 32>, MODE>(a, s);
    case 8: return narrow ? launch_one<ScanShape<8, 2, 8, 32>, MODE>(a, s) : launch_one<ScanShape<8, 2, 32, 32>, MODE>(a, s);
    case 4: return narrow ? launch_one<ScanShape<4, 1, 8, 32>, MODE>(a, s) : launch_one<ScanShape<4, 1, 32, 32>, MODE>(a, s);
    case 2: return narrow ? launch_one<ScanShape<2, 1, 8, 32>, MODE>(a, s) : launch_one<ScanShape<2, 1, 32, 32>, MODE>(a, s);
    case 1: return narrow ? launch_one<ScanShape<1, 1, 8, 32>, MODE>(a, s) : launch_one<ScanShape<1, 1, 32, 32>, MODE>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_scan(const ScanArgs &a, int N, int mode, cudaStream_t s)
{
    return mode == kFused ? dispatch<kFused>(a, N, s) : dispatch<kStandalone>(a, N, s);
}

}  // namespace ss2d
