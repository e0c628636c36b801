// scan_bwd.cu -- instantiations and launcher of the backward scan kernel.
#include "kernels.h"
#include "launch_util.h"
#include "scan_bwd.cuh"

namespace ss2d {

namespace {

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
    a.tiles = (a.D + S::CW - 1) / S::CW;
    const long long items = (long long)a.tiles * 4 * a.B;
    if (items > 0x7fffffffLL || items < 1)
        return cudaErrorInvalidConfiguration;
    scan_bwd_kernel<S><<<(unsigned)items, 32, lay.smem_bytes, s>>>(a, lay);
    return cudaGetLastError();
}

}  // namespace

bool scan_bwd_supported(int N, int u_bf16, int delta_bf16, int softplus, int L)
{
    return N == 16 && softplus && (u_bf16 != 0) == (delta_bf16 != 0) && L % 4 == 0;
}

// Only the fp32 instantiation is built: the caller widens bf16 x and dts to fp32 first.
cudaError_t launch_scan_bwd(const BwdArgs &a, cudaStream_t s)
{
    return launch_bwd_t<4>(a, s);
}

}  // namespace ss2d
