// api_internal.h -- argument checks and error text shared by the C ABI files (internal).
#pragma once

#include <cuda_runtime.h>

#include "ss2d.h"

namespace ss2d {

// Checks of ss2d_forward_core's arguments; returns SS2D_OK or the status it would return.
// With check_y false, y is neither required nor checked against the inputs (a size query).
int validate_core_args(const ss2d_core_args *a, bool check_y = true);

// True when the arguments ask for channels-last x and y.
bool core_channels_last(const ss2d_core_args *a);

// Sets the text ss2d_last_error() returns on the calling thread; returns `status`.
int set_last_error(int status, const char *msg);

// Device address of ss2d_forward_core_static's scratch array on the current device.
cudaError_t static_scratch_address(void **out);

// Slices of ss2d_forward_core_static for these arguments: writes the image count of
// each slice to nb[0 .. max_slices) (nb may be null) and returns the number of
// slices, or -1 if one image needs more scratch than the static array holds.  Every
// slice's workspace (ss2d_forward_core_workspace at that image count) fits the array.
int static_slice_plan(const ss2d_core_args *args, int *nb, int max_slices);

}  // namespace ss2d
