// xproj.cu -- projection path of the fused core (placeholder until built).
#include "xproj.h"

namespace ss2d {

int xproj_supported(int, int, int, int, int, int) { return 1; }

size_t xproj_workspace_bytes(int, int, int, int, int, int) { return 0; }

cudaError_t launch_core_with_projections(const void *, const void *, const float *, const float *, const float *,
                                         const float *, bool, float *, void *, int, int, int, int, int, int,
                                         cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace ss2d
