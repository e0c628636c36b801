"""ctypes binding of libss2d.so: argument marshalling only.

Every function here takes torch tensors that already live on a CUDA device,
checks that they are contiguous and of the expected dtype, and passes their
device pointers, sizes and the current CUDA stream to the C ABI declared in
include/ss2d.h.  All computation happens in the library's CUDA kernels; there
is no fallback of any kind.  A missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libss2d.so")

SS2D_MERGE_ATOMIC = 0
SS2D_MERGE_PAGE_ORDER = 1
SS2D_F32 = 0
SS2D_BF16 = 1
SS2D_CHANNELS_FIRST = 0
SS2D_CHANNELS_LAST = 1
_DTYPE_CODE = {torch.float32: SS2D_F32, torch.bfloat16: SS2D_BF16}


class Ss2dError(RuntimeError):
    """A libss2d call returned a non-zero status."""

    def __init__(self, status: int, name: str, message: str):
        super().__init__(f"{name}: {message}")
        self.status = status
        self.name = name


class CoreArgs(ctypes.Structure):
    """Mirror of ss2d_core_args (include/ss2d.h)."""

    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("B", ctypes.c_int), ("D", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("N", ctypes.c_int), ("R", ctypes.c_int),
        ("x", ctypes.c_void_p), ("x_dtype", ctypes.c_int),
        ("dts", ctypes.c_void_p), ("dts_dtype", ctypes.c_int),
        ("Bs", ctypes.c_void_p), ("Cs", ctypes.c_void_p),
        ("A_logs", ctypes.c_void_p), ("Ds", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("delta_softplus", ctypes.c_int),
        ("x_proj_weight", ctypes.c_void_p), ("dt_projs_weight", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("layout", ctypes.c_int),
        ("y_dtype", ctypes.c_int),
        ("ckpt", ctypes.c_void_p),
        ("merge_order", ctypes.c_int),
    ]


class BlockArgs(ctypes.Structure):
    """Mirror of ss2d_block_args (include/ss2d.h)."""

    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("d_model", ctypes.c_int), ("D", ctypes.c_int), ("N", ctypes.c_int), ("R", ctypes.c_int),
        ("d_conv", ctypes.c_int),
        ("x", ctypes.c_void_p),
        ("in_proj_weight", ctypes.c_void_p), ("in_proj_bias", ctypes.c_void_p),
        ("conv_weight", ctypes.c_void_p), ("conv_bias", ctypes.c_void_p),
        ("x_proj_weight", ctypes.c_void_p), ("dt_projs_weight", ctypes.c_void_p), ("dt_projs_bias", ctypes.c_void_p),
        ("A_logs", ctypes.c_void_p), ("Ds", ctypes.c_void_p),
        ("out_norm_weight", ctypes.c_void_p), ("out_norm_bias", ctypes.c_void_p),
        ("out_norm_eps", ctypes.c_float),
        ("out_proj_weight", ctypes.c_void_p), ("out_proj_bias", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("out_dtype", ctypes.c_int),
    ]


class CoreGrads(ctypes.Structure):
    """Mirror of ss2d_core_grads (include/ss2d.h)."""

    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("dy", ctypes.c_void_p), ("dx", ctypes.c_void_p), ("ddts", ctypes.c_void_p),
        ("dA_logs", ctypes.c_void_p), ("dBs", ctypes.c_void_p), ("dCs", ctypes.c_void_p),
        ("dDs", ctypes.c_void_p), ("ddt_bias", ctypes.c_void_p),
        ("dx_proj_weight", ctypes.c_void_p), ("ddt_projs_weight", ctypes.c_void_p),
    ]


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libss2d.so (built in-tree by selective_scan_02_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libss2d.so not found at {LIB_PATH}; build it with selective_scan_02_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ss2d_status_string.argtypes = [I]
    lib.ss2d_status_string.restype = ctypes.c_char_p
    lib.ss2d_last_error.argtypes = []
    lib.ss2d_last_error.restype = ctypes.c_char_p
    lib.ss2d_version.argtypes = []
    lib.ss2d_version.restype = I
    lib.ss2d_cross_scan.argtypes = [P, I, P, I, I, I, I, P]
    lib.ss2d_cross_scan.restype = I
    lib.ss2d_cross_merge.argtypes = [P, P, I, I, I, I, P]
    lib.ss2d_cross_merge.restype = I
    lib.ss2d_selective_scan.argtypes = [P, I, P, I, P, P, P, P, P, I, P, I, I, I, I, I, P]
    lib.ss2d_selective_scan.restype = I
    lib.ss2d_selective_scan_state.argtypes = [P, I, P, I, P, P, P, P, P, I, P, P, P, I, I, I, I, I, P]
    lib.ss2d_selective_scan_state.restype = I
    lib.ss2d_forward_core_workspace.argtypes = [ctypes.POINTER(CoreArgs)]
    lib.ss2d_forward_core_workspace.restype = S
    lib.ss2d_forward_core.argtypes = [ctypes.POINTER(CoreArgs), P, S, P]
    lib.ss2d_forward_core.restype = I
    lib.ss2d_forward_core_static.argtypes = [ctypes.POINTER(CoreArgs), P]
    lib.ss2d_forward_core_static.restype = I
    lib.ss2d_forward_core_backward_workspace.argtypes = [ctypes.POINTER(CoreArgs)]
    lib.ss2d_forward_core_backward_workspace.restype = S
    lib.ss2d_forward_core_backward.argtypes = [ctypes.POINTER(CoreArgs), ctypes.POINTER(CoreGrads), P, S, P]
    lib.ss2d_forward_core_backward.restype = I
    lib.ss2d_device_status.argtypes = [ctypes.POINTER(CoreArgs), P, I, P]
    lib.ss2d_device_status.restype = I
    lib.ss2d_block_forward_workspace.argtypes = [ctypes.POINTER(BlockArgs)]
    lib.ss2d_block_forward_workspace.restype = S
    lib.ss2d_block_forward.argtypes = [ctypes.POINTER(BlockArgs), P, S, P]
    lib.ss2d_block_forward.restype = I
    lib.ss2d_block_device_status.argtypes = [ctypes.POINTER(BlockArgs), P, P]
    lib.ss2d_block_device_status.restype = I
    lib.ss2d_diag_bounded_wait.argtypes = [P, ctypes.c_longlong, P]
    lib.ss2d_diag_bounded_wait.restype = I
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != 0:
        lib = load_library()
        raise Ss2dError(status, lib.ss2d_status_string(status).decode(), lib.ss2d_last_error().decode() or what)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libss2d takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libss2d takes contiguous tensors")
    return t.data_ptr()


def _code(t):
    try:
        return _DTYPE_CODE[t.dtype]
    except KeyError:
        raise ValueError(f"dtype {t.dtype} is not float32 or bfloat16") from None


def _f32(t, name):
    if t is not None and t.dtype != torch.float32:
        raise ValueError(f"{name} must be float32")
    return t


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def cross_scan(x, xs=None, stream=None):
    """x (B,D,H,W) -> xs (B,4,D,H*W), same dtype (ss2d_cross_scan)."""
    B, D, H, W = x.shape
    if xs is None:
        xs = torch.empty((B, 4, D, H * W), dtype=x.dtype, device=x.device)
    _check(load_library().ss2d_cross_scan(_ptr(x), _code(x), _ptr(xs), B, D, H, W, _stream(stream)),
           "ss2d_cross_scan")
    return xs


def cross_merge(ys, H, W, y=None, stream=None):
    """ys (B,4,D,H*W) fp32 -> y (B,D,H,W) fp32 (ss2d_cross_merge)."""
    B, K, D, L = ys.shape
    if K != 4 or L != H * W:
        raise ValueError("ys must be (B, 4, D, H*W)")
    _f32(ys, "ys")
    if y is None:
        y = torch.empty((B, D, H, W), dtype=torch.float32, device=ys.device)
    _check(load_library().ss2d_cross_merge(_ptr(ys), _ptr(y), B, D, H, W, _stream(stream)), "ss2d_cross_merge")
    return y


def selective_scan(u, delta, A_log, Bm, Cm, Dv=None, delta_bias=None, delta_softplus=True, y=None, stream=None,
                   h0=None, return_last_state=False):
    """Selective scan: u, delta (B,C,L); A_log (C,N); Bm, Cm (B,G,N,L) -> y (B,C,L) fp32.

    With h0 (B,C,N) fp32 the scan starts from that state, and with return_last_state it also
    returns the state after the last step, (y, h_last) (ss2d_selective_scan_state); otherwise
    ss2d_selective_scan.
    """
    B, C, L = u.shape
    G, N = Bm.shape[1], Bm.shape[2]
    for t, name in ((A_log, "A_log"), (Bm, "Bm"), (Cm, "Cm"), (Dv, "Dv"), (delta_bias, "delta_bias"), (h0, "h0")):
        _f32(t, name)
    if y is None:
        y = torch.empty((B, C, L), dtype=torch.float32, device=u.device)
    lib = load_library()
    if h0 is None and not return_last_state:
        st = lib.ss2d_selective_scan(
            _ptr(u), _code(u), _ptr(delta), _code(delta), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(Dv),
            _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y), B, C, G, N, L, _stream(stream))
        _check(st, "ss2d_selective_scan")
        return y
    h_last = torch.empty((B, C, N), dtype=torch.float32, device=u.device) if return_last_state else None
    st = lib.ss2d_selective_scan_state(
        _ptr(u), _code(u), _ptr(delta), _code(delta), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(Dv),
        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(h_last), _ptr(y), B, C, G, N, L,
        _stream(stream))
    _check(st, "ss2d_selective_scan_state")
    return (y, h_last) if return_last_state else y


def _core_args(x, A_logs, Ds, dt_bias, y, dts=None, Bs=None, Cs=None, x_proj_weight=None,
               dt_projs_weight=None, delta_softplus=True, channels_last=False, ckpt=None, y_dtype=None,
               page_order=False):
    B, H, W, D = x.shape if channels_last else (x.shape[0], x.shape[2], x.shape[3], x.shape[1])
    N = A_logs.shape[1]
    R = dt_projs_weight.shape[2] if dt_projs_weight is not None else 0
    a = CoreArgs()
    a.struct_size = ctypes.sizeof(CoreArgs)
    a.B, a.D, a.H, a.W, a.N, a.R = B, D, H, W, N, R
    a.x, a.x_dtype = _ptr(x), _code(x)
    a.dts = _ptr(dts)
    a.dts_dtype = _code(dts) if dts is not None else 0
    a.Bs, a.Cs = _ptr(_f32(Bs, "Bs")), _ptr(_f32(Cs, "Cs"))
    a.A_logs, a.Ds, a.dt_bias = _ptr(_f32(A_logs, "A_logs")), _ptr(_f32(Ds, "Ds")), _ptr(_f32(dt_bias, "dt_bias"))
    a.delta_softplus = int(bool(delta_softplus))
    if x_proj_weight is not None and x_proj_weight.dtype != torch.bfloat16:
        raise ValueError("x_proj_weight must be bfloat16")
    a.x_proj_weight = _ptr(x_proj_weight)
    a.dt_projs_weight = _ptr(_f32(dt_projs_weight, "dt_projs_weight"))
    a.y = _ptr(y)
    a.y_dtype = _code(y) if y is not None else (_DTYPE_CODE[y_dtype] if y_dtype is not None else SS2D_F32)
    a.layout = SS2D_CHANNELS_LAST if channels_last else SS2D_CHANNELS_FIRST
    a.ckpt = _ptr(_f32(ckpt, "ckpt"))
    a.merge_order = SS2D_MERGE_PAGE_ORDER if page_order else SS2D_MERGE_ATOMIC
    return a


def checkpoint_shape(x, channels_last=False):
    """Shape of the fp32 checkpoint buffer forward_core can keep for forward_core_backward:
    (B, 4D, ceil(L/16), 16)."""
    B, H, W, D = x.shape if channels_last else (x.shape[0], x.shape[2], x.shape[3], x.shape[1])
    return (B, 4 * D, (H * W + 15) // 16, 16)


def forward_core_workspace_size(x, A_logs, Ds, dt_bias, dts=None, Bs=None, Cs=None, x_proj_weight=None,
                                dt_projs_weight=None, delta_softplus=True, channels_last=False,
                                out_dtype=torch.float32, page_order=False) -> int:
    """Workspace bytes ss2d_forward_core needs for these arguments (out_dtype: y's type)."""
    a = _core_args(x, A_logs, Ds, dt_bias, None, dts, Bs, Cs, x_proj_weight, dt_projs_weight, delta_softplus,
                   channels_last, y_dtype=out_dtype, page_order=page_order)
    lib = load_library()
    n = lib.ss2d_forward_core_workspace(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise Ss2dError(1, "SS2D_ERR_INVALID_ARG", lib.ss2d_last_error().decode())
    return int(n)


def forward_core(x, A_logs, Ds, dt_bias, dts=None, Bs=None, Cs=None, x_proj_weight=None, dt_projs_weight=None,
                 delta_softplus=True, y=None, workspace=None, stream=None, channels_last=False,
                 out_dtype=torch.float32, ckpt=None, page_order=False):
    """Fused SS2D forward core (ss2d_forward_core): x (B,D,H,W) -> y (B,D,H,W) fp32.

    Give either dts (B,4,D,L), Bs, Cs (B,4,N,L), or x_proj_weight (4,R+2N,D) bf16 and
    dt_projs_weight (4,D,R).  A workspace tensor is allocated when needed and none is given.
    With channels_last, x and y are (B,H,W,D) (the page's channel_first=False layout).
    out_dtype (float32 or bfloat16) is the type of a y allocated here; a given y keeps its own.
    ckpt: an fp32 tensor of checkpoint_shape(x) that receives the scan's checkpoints, for a
    later forward_core_backward with the same arguments (dts/Bs/Cs form).
    page_order: merge the four directions in the article's order, deterministically
    (SS2D_MERGE_PAGE_ORDER) instead of with atomics.
    """
    if y is None:
        y = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    a = _core_args(x, A_logs, Ds, dt_bias, y, dts, Bs, Cs, x_proj_weight, dt_projs_weight, delta_softplus,
                   channels_last, ckpt, page_order=page_order)
    lib = load_library()
    need = lib.ss2d_forward_core_workspace(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise Ss2dError(1, "SS2D_ERR_INVALID_ARG", lib.ss2d_last_error().decode())
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_ptr = _ptr(workspace) if need > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if need > 0 else 0
    _check(lib.ss2d_forward_core(ctypes.byref(a), ws_ptr, ws_bytes, _stream(stream)), "ss2d_forward_core")
    return y


def forward_core_static(x, A_logs, Ds, dt_bias, x_proj_weight, dt_projs_weight, delta_softplus=True, y=None,
                        stream=None, channels_last=False):
    """Projection form of the fused core with the library's static scratch (ss2d_forward_core_static).

    For callers that cannot allocate device memory at call time: no workspace is
    taken or allocated.  Calls that overlap on the GPU share the scratch and race.
    """
    if y is None:
        y = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    a = _core_args(x, A_logs, Ds, dt_bias, y, x_proj_weight=x_proj_weight, dt_projs_weight=dt_projs_weight,
                   delta_softplus=delta_softplus, channels_last=channels_last)
    _check(load_library().ss2d_forward_core_static(ctypes.byref(a), _stream(stream)), "ss2d_forward_core_static")
    return y


def forward_core_backward_workspace_size(x, A_logs, Ds, dt_bias, dts=None, Bs=None, Cs=None, delta_softplus=True,
                                         x_proj_weight=None, dt_projs_weight=None, channels_last=False) -> int:
    """Workspace bytes ss2d_forward_core_backward needs for these forward arguments."""
    a = _core_args(x, A_logs, Ds, dt_bias, None, dts, Bs, Cs, x_proj_weight, dt_projs_weight, delta_softplus,
                   channels_last)
    lib = load_library()
    n = lib.ss2d_forward_core_backward_workspace(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise Ss2dError(2, "SS2D_ERR_UNSUPPORTED", lib.ss2d_last_error().decode())
    return int(n)


def forward_core_backward(x, A_logs, Ds, dt_bias, dts=None, Bs=None, Cs=None, dy=None, delta_softplus=True,
                          grads=None, workspace=None, stream=None, x_proj_weight=None, dt_projs_weight=None,
                          channels_last=False, ckpt=None):
    """Gradients of the fused core (ss2d_forward_core_backward).

    dy (B,D,H,W) fp32 is the gradient of the loss with respect to y.  Returns a dict of
    fp32 tensors dx (B,D,H,W), ddts (B,4,D,L), dA_logs (4D,N), dBs, dCs (B,4,N,L), dDs
    and ddt_bias (4D), plus dx_proj_weight (4,R+2N,D) and ddt_projs_weight (4,D,R) in the
    projection form (x_proj_weight and dt_projs_weight given instead of dts, Bs, Cs), where
    ddts, dBs and dCs are the gradients of the projected intermediates.  Pass `grads` (a
    dict of such tensors) to write into existing ones.  A workspace is allocated when none
    (or one too small) is given.  channels_last: x, dy and dx are (B,H,W,D).  ckpt: the
    checkpoints a forward_core call with the same arguments kept (skips their recomputation).
    """
    if dy is None:
        raise ValueError("dy is required")
    B, H, W, D = x.shape if channels_last else (x.shape[0], x.shape[2], x.shape[3], x.shape[1])
    L, N = H * W, A_logs.shape[1]
    dev = x.device
    proj = x_proj_weight is not None
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = dict(dx=torch.empty(tuple(x.shape), **f32), ddts=torch.empty((B, 4, D, L), **f32),
                     dA_logs=torch.empty((4 * D, N), **f32), dBs=torch.empty((B, 4, N, L), **f32),
                     dCs=torch.empty((B, 4, N, L), **f32),
                     dDs=torch.empty((4 * D,), **f32) if Ds is not None else None,
                     ddt_bias=torch.empty((4 * D,), **f32) if dt_bias is not None else None)
        if proj:
            R = dt_projs_weight.shape[2]
            grads["dx_proj_weight"] = torch.empty((4, R + 2 * N, D), **f32)
            grads["ddt_projs_weight"] = torch.empty((4, D, R), **f32)
    _f32(dy, "dy")
    for k, t in grads.items():
        if t is not None:
            _f32(t, k)
    a = _core_args(x, A_logs, Ds, dt_bias, None, dts, Bs, Cs, x_proj_weight, dt_projs_weight, delta_softplus,
                   channels_last, ckpt)
    gr = CoreGrads(ctypes.sizeof(CoreGrads), _ptr(dy), _ptr(grads["dx"]), _ptr(grads.get("ddts")),
                   _ptr(grads["dA_logs"]), _ptr(grads.get("dBs")), _ptr(grads.get("dCs")), _ptr(grads.get("dDs")),
                   _ptr(grads.get("ddt_bias")), _ptr(grads.get("dx_proj_weight")),
                   _ptr(grads.get("ddt_projs_weight")))
    lib = load_library()
    need = lib.ss2d_forward_core_backward_workspace(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise Ss2dError(2, "SS2D_ERR_UNSUPPORTED", lib.ss2d_last_error().decode())
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(lib.ss2d_forward_core_backward(ctypes.byref(a), ctypes.byref(gr), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)),
           "ss2d_forward_core_backward")
    return grads


def check_device_status(x, A_logs, Ds, dt_bias, workspace=None, backward=False, dts=None, Bs=None, Cs=None,
                        x_proj_weight=None, dt_projs_weight=None, delta_softplus=True, channels_last=False,
                        stream=None):
    """Raises Ss2dError (SS2D_ERR_DEVICE) if a tensor-core kernel's bounded wait ran out in the
    last projection-form call on `workspace` (ss2d_device_status).

    Pass that call's arguments and workspace (None after forward_core_static); backward=True
    after forward_core_backward.  Synchronises the stream.  The dts/Bs/Cs form waits on
    nothing and always passes.
    """
    a = _core_args(x, A_logs, Ds, dt_bias, None, dts, Bs, Cs, x_proj_weight, dt_projs_weight, delta_softplus,
                   channels_last)
    _check(load_library().ss2d_device_status(ctypes.byref(a), _ptr(workspace), int(bool(backward)),
                                             _stream(stream)), "ss2d_device_status")


def _bf16(t, name):
    if t is not None and t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16")
    return t


def _block_args(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias, A_logs,
                Ds, out_norm_weight, out_norm_bias, out_proj_weight, in_proj_bias, out_proj_bias, eps, out,
                out_dtype):
    B, H, W, d_model = x.shape
    D = conv_weight.shape[0]
    a = BlockArgs()
    a.struct_size = ctypes.sizeof(BlockArgs)
    a.B, a.H, a.W, a.d_model, a.D = B, H, W, d_model, D
    a.N, a.R, a.d_conv = A_logs.shape[1], dt_projs_weight.shape[2], conv_weight.shape[1]
    a.x = _ptr(_bf16(x, "x"))
    a.in_proj_weight = _ptr(_bf16(in_proj_weight, "in_proj_weight"))
    a.in_proj_bias = _ptr(_f32(in_proj_bias, "in_proj_bias"))
    a.conv_weight = _ptr(_f32(conv_weight, "conv_weight"))
    a.conv_bias = _ptr(_f32(conv_bias, "conv_bias"))
    a.x_proj_weight = _ptr(_bf16(x_proj_weight, "x_proj_weight"))
    a.dt_projs_weight = _ptr(_f32(dt_projs_weight, "dt_projs_weight"))
    a.dt_projs_bias = _ptr(_f32(dt_projs_bias, "dt_projs_bias"))
    a.A_logs, a.Ds = _ptr(_f32(A_logs, "A_logs")), _ptr(_f32(Ds, "Ds"))
    a.out_norm_weight = _ptr(_f32(out_norm_weight, "out_norm_weight"))
    a.out_norm_bias = _ptr(_f32(out_norm_bias, "out_norm_bias"))
    a.out_norm_eps = float(eps)
    a.out_proj_weight = _ptr(_bf16(out_proj_weight, "out_proj_weight"))
    a.out_proj_bias = _ptr(_f32(out_proj_bias, "out_proj_bias"))
    a.out = _ptr(out)
    a.out_dtype = _code(out) if out is not None else _DTYPE_CODE[out_dtype]
    return a


def block_forward_workspace_size(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight,
                                 dt_projs_bias, A_logs, Ds, out_norm_weight, out_norm_bias, out_proj_weight,
                                 in_proj_bias=None, out_proj_bias=None, eps=1e-5, out_dtype=torch.float32) -> int:
    """Workspace bytes ss2d_block_forward needs for these arguments."""
    a = _block_args(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias, A_logs,
                    Ds, out_norm_weight, out_norm_bias, out_proj_weight, in_proj_bias, out_proj_bias, eps, None,
                    out_dtype)
    lib = load_library()
    n = lib.ss2d_block_forward_workspace(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise Ss2dError(1, "SS2D_ERR_INVALID_ARG", lib.ss2d_last_error().decode())
    return int(n)


def block_forward(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias, A_logs,
                  Ds, out_norm_weight, out_norm_bias, out_proj_weight, in_proj_bias=None, out_proj_bias=None,
                  eps=1e-5, out=None, workspace=None, stream=None, out_dtype=torch.float32):
    """The SS2D block (ss2d_block_forward): x (B,H,W,d_model) bf16 -> out (B,H,W,d_model).

    in_proj_weight (2D,d_model) bf16, conv_weight (D,k,k) fp32 (k odd), conv_bias (D) or None,
    x_proj_weight (4,R+2N,D) bf16, dt_projs_weight (4,D,R), dt_projs_bias (4D), A_logs (4D,N),
    Ds (4D), out_norm_weight / out_norm_bias (D), out_proj_weight (d_model,D) bf16; optional
    fp32 projection biases.  A workspace tensor is allocated when none (or too small) is given.
    """
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    a = _block_args(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias, A_logs,
                    Ds, out_norm_weight, out_norm_bias, out_proj_weight, in_proj_bias, out_proj_bias, eps, out,
                    out_dtype)
    lib = load_library()
    need = lib.ss2d_block_forward_workspace(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise Ss2dError(1, "SS2D_ERR_INVALID_ARG", lib.ss2d_last_error().decode())
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(lib.ss2d_block_forward(ctypes.byref(a), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream)), "ss2d_block_forward")
    return out


def block_device_status(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias,
                        A_logs, Ds, out_norm_weight, out_norm_bias, out_proj_weight, workspace, in_proj_bias=None,
                        out_proj_bias=None, eps=1e-5, stream=None, out_dtype=torch.float32):
    """ss2d_block_device_status for the workspace of an earlier block_forward (synchronises)."""
    a = _block_args(x, in_proj_weight, conv_weight, conv_bias, x_proj_weight, dt_projs_weight, dt_projs_bias, A_logs,
                    Ds, out_norm_weight, out_norm_bias, out_proj_weight, in_proj_bias, out_proj_bias, eps, None,
                    out_dtype)
    _check(load_library().ss2d_block_device_status(ctypes.byref(a), _ptr(workspace), _stream(stream)),
           "ss2d_block_device_status")


def diag_bounded_wait(error_word, spin_limit, stream=None):
    """ss2d_diag_bounded_wait: a tensor-core wait that runs out on purpose after spin_limit
    polls and sets error_word (a device int32 tensor, e.g. the first word of a projection-form
    workspace viewed as int32) to 1."""
    if error_word.dtype != torch.int32:
        raise ValueError("error_word must be int32")
    _check(load_library().ss2d_diag_bounded_wait(_ptr(error_word), int(spin_limit), _stream(stream)),
           "ss2d_diag_bounded_wait")
