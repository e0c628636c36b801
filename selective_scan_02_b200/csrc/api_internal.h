// api_internal.h -- argument checks and error text shared by the C ABI files (internal).
#pragma once

#include <cuda_runtime.h>

#include "ss2d.h"

namespace ss2d {

// Checks of ss2d_forward_core's arguments; returns SS2D_OK or the status it would return.
int validate_core_args(const ss2d_core_args *a);

// True when the arguments ask for channels-last x and y.
bool core_channels_last(const ss2d_core_args *a);

// Sets the text ss2d_last_error() returns on the calling thread; returns `status`.
int set_last_error(int status, const char *msg);

// Device address of ss2d_forward_core_static's scratch array on the current device.
cudaError_t static_scratch_address(void **out);

}  // namespace ss2d
