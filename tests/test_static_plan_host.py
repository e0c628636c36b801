"""Host-side check of ss2d_forward_core_static's slice plan (no GPU).

The static entry point runs the batch in slices that each fit the library's
SS2D_STATIC_SCRATCH_BYTES array.  The projection form's workspace is not linear
in the batch: the segmented scan picks its segment count from the image count,
and its segment states grow with it.  So a plan that extrapolates the size of
one image can overrun the array.  This test sweeps shapes the projection form
accepts and asks the library's own planner (ss2d::static_slice_plan, a C++ symbol
of libss2d.so, host code only) for its slices.  It checks that they cover the
batch and that every slice's workspace (ss2d_forward_core_workspace at that
image count) fits the array.  The pointers are never dereferenced."""
import ctypes
import itertools

import pytest

import selective_scan_02_b200 as ss
from selective_scan_02_b200 import CoreArgs

SCRATCH = 16 << 20  # SS2D_STATIC_SCRATCH_BYTES
PLAN_SYMBOL = "_ZN4ss2d17static_slice_planEPK14ss2d_core_argsPii"
SPAN = 1 << 36      # distinct fake buffers, far enough apart that none overlaps another


@pytest.fixture(scope="module")
def lib():
    lib = ss.load_library()
    plan = lib[PLAN_SYMBOL]
    plan.restype = ctypes.c_int
    plan.argtypes = [ctypes.POINTER(CoreArgs), ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    lib.ss2d_forward_core_workspace.restype = ctypes.c_size_t
    lib.ss2d_forward_core_workspace.argtypes = [ctypes.POINTER(CoreArgs)]
    return lib


def _args(B, D, H, W, R, N=16, channels_last=False):
    a = CoreArgs()
    a.struct_size = ctypes.sizeof(CoreArgs)
    a.B, a.D, a.H, a.W, a.N, a.R = B, D, H, W, N, R
    base = 0x100000000000
    a.x, a.x_dtype = base, 1
    a.A_logs, a.Ds, a.dt_bias = base + SPAN, base + 2 * SPAN, base + 3 * SPAN
    a.x_proj_weight, a.dt_projs_weight = base + 4 * SPAN, base + 5 * SPAN
    a.y = base + 6 * SPAN
    a.delta_softplus = 1
    a.layout = 1 if channels_last else 0
    a.y_dtype = 0
    return a


def _workspace(lib, a, nb):
    q = CoreArgs.from_buffer_copy(a)
    q.B = nb
    return lib.ss2d_forward_core_workspace(ctypes.byref(q))


def _plan(lib, a):
    n = lib[PLAN_SYMBOL](ctypes.byref(a), None, 0)
    if n < 0:
        return None
    buf = (ctypes.c_int * n)()
    assert lib[PLAN_SYMBOL](ctypes.byref(a), buf, n) == n
    return list(buf)


def _check_plan(lib, a):
    plan = _plan(lib, a)
    if plan is None:
        # rejected: then not even one image fits
        assert _workspace(lib, a, 1) > SCRATCH
        return None
    assert sum(plan) == a.B and all(nb > 0 for nb in plan)
    for nb in set(plan):
        w = _workspace(lib, a, nb)
        assert w != ctypes.c_size_t(-1).value
        assert w <= SCRATCH, (a.B, a.D, a.H, a.W, a.R, nb, w)
    return plan


def _old_slice_bytes(lib, a):
    """Workspace of the first slice under the earlier plan, which assumed the workspace is a
    header plus a fixed number of bytes per image (sizes at one and two images)."""
    w1, w2 = _workspace(lib, a, 1), _workspace(lib, a, 2)
    per = (SCRATCH - (w1 - (w2 - w1))) // (w2 - w1)
    return _workspace(lib, a, min(a.B, per))


# Shapes named when the overrun was found (D = 208, 64x64, R = 1, B = 3 and others): each
# must be planned inside the array.
NAMED = [
    (5, 336, 48, 48, 1),
    (3, 208, 64, 64, 1),
    (3, 192, 22, 192, 1),
    (4, 208, 60, 64, 6),
    (3, 224, 31, 128, 2),
]


@pytest.mark.parametrize("B,D,H,W,R", NAMED)
def test_plan_fits_named_shapes(lib, B, D, H, W, R):
    assert _check_plan(lib, _args(B, D, H, W, R)) is not None


def test_plan_sweep(lib):
    """Every accepted shape of the sweep is planned inside the array, including the shapes on
    which extrapolating one image's size (the earlier plan) would overrun it; the sweep must
    contain such shapes, so the non-linear part of the workspace is exercised."""
    shapes = [(9, 16), (22, 192), (28, 32), (31, 128), (48, 48), (56, 56), (60, 64), (64, 64), (100, 104)]
    planned = rejected = overran = 0
    for (H, W), D, R, B in itertools.product(shapes, (16, 64, 192, 208, 224, 336, 352), (1, 2, 6, 16),
                                             (1, 2, 3, 4, 5, 7, 11, 33)):
        a = _args(B, D, H, W, R)
        if lib.ss2d_forward_core_workspace(ctypes.byref(a)) == ctypes.c_size_t(-1).value:
            continue  # shape the projection form does not take
        if _check_plan(lib, a) is None:
            rejected += 1
            continue
        planned += 1
        if B >= 2 and _old_slice_bytes(lib, a) > SCRATCH:
            overran += 1
    assert planned > 500 and rejected > 0 and overran > 0


def test_plan_channels_last(lib):
    for B, D, H, W, R in [(4, 208, 60, 64, 6), (11, 64, 56, 56, 6), (3, 192, 22, 192, 1)]:
        assert _check_plan(lib, _args(B, D, H, W, R, channels_last=True)) is not None
