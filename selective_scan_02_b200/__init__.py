"""B200-native (sm_100a) SS2D core: CrossScan -> selective scan -> CrossMerge, its gradient, and the
SS2D block around it (input projection, depthwise convolution, gated normalisation, output projection).

The compute lives in libss2d.so (hand-written CUDA, C ABI in include/ss2d.h);
this package only loads it and marshals torch device tensors into its calls.
"""
from ._binding import (  # noqa: F401
    LIB_PATH,
    SS2D_BF16,
    SS2D_CHANNELS_FIRST,
    SS2D_CHANNELS_LAST,
    SS2D_F32,
    BlockArgs,
    CoreArgs,
    CoreGrads,
    Ss2dError,
    block_device_status,
    block_forward,
    block_forward_workspace_size,
    check_device_status,
    checkpoint_shape,
    cross_merge,
    cross_scan,
    diag_bounded_wait,
    forward_core,
    forward_core_backward,
    forward_core_backward_workspace_size,
    forward_core_static,
    forward_core_workspace_size,
    load_library,
    selective_scan,
)

__all__ = [
    "LIB_PATH", "SS2D_BF16", "SS2D_CHANNELS_FIRST", "SS2D_CHANNELS_LAST", "SS2D_F32", "BlockArgs", "CoreArgs", "CoreGrads",
    "Ss2dError", "block_device_status", "block_forward", "block_forward_workspace_size", "check_device_status", "checkpoint_shape", "cross_merge", "cross_scan", "diag_bounded_wait", "forward_core",
    "forward_core_backward", "forward_core_backward_workspace_size", "forward_core_static",
    "forward_core_workspace_size", "load_library", "selective_scan",
]
