"""Host-side checks of the C ABI: the library loads without a GPU, exports every
entry point declared in include/ss2d.h, and rejects bad arguments on the host
(before anything is enqueued) with the documented status codes.  The pointers
passed here are never dereferenced: every call fails its argument checks."""
import ctypes
import os
import re

import pytest

import selective_scan_02_b200 as ss
from selective_scan_02_b200 import CoreArgs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA, DEVICE = range(7)
FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names.update(re.findall(r"^[A-Za-z_][\w \*]*?\b(ss2d_\w+)\s*\(", text, flags=re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    return ss.load_library()


def test_library_exports_every_declared_function(lib):
    names = _declared_functions()
    assert {"ss2d_cross_scan", "ss2d_cross_merge", "ss2d_selective_scan", "ss2d_forward_core",
            "ss2d_forward_core_workspace"} <= names
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.ss2d_status_string(OK) == b"SS2D_OK"
    assert lib.ss2d_status_string(MISALIGNED) == b"SS2D_ERR_MISALIGNED"
    assert lib.ss2d_status_string(DEVICE) == b"SS2D_ERR_DEVICE"
    assert lib.ss2d_status_string(99) == b"SS2D_ERR_UNKNOWN"
    assert lib.ss2d_version() == 107


def test_cross_scan_argument_checks(lib):
    assert lib.ss2d_cross_scan(None, 0, FAKE, 1, 1, 2, 2, None) == INVALID
    assert b"non-null" in lib.ss2d_last_error()
    assert lib.ss2d_cross_scan(FAKE, 0, FAKE + 4096, 0, 1, 2, 2, None) == INVALID
    assert lib.ss2d_cross_scan(FAKE, 7, FAKE + 4096, 1, 1, 2, 2, None) == UNSUPPORTED
    assert lib.ss2d_cross_scan(FAKE + 2, 0, FAKE + 4096, 1, 1, 2, 2, None) == MISALIGNED
    assert lib.ss2d_cross_scan(FAKE, 0, FAKE, 1, 1, 2, 2, None) == INVALID  # output overlaps input
    assert lib.ss2d_cross_merge(FAKE, FAKE + 8, 1, 1, 2, 2, None) == MISALIGNED
    assert lib.ss2d_cross_merge(FAKE, FAKE + 16, 1, 1, 2, 2, None) == INVALID  # overlap


def _scan(lib, **kw):
    a = dict(u=FAKE, ud=0, delta=FAKE + (1 << 20), dd=0, A=FAKE + (2 << 20), Bm=FAKE + (3 << 20),
             Cm=FAKE + (4 << 20), Dv=None, bias=None, sp=1, y=FAKE + (8 << 20), B=1, C=4, G=2, N=16, L=8)
    a.update(kw)
    return lib.ss2d_selective_scan(a["u"], a["ud"], a["delta"], a["dd"], a["A"], a["Bm"], a["Cm"], a["Dv"],
                                   a["bias"], a["sp"], a["y"], a["B"], a["C"], a["G"], a["N"], a["L"], None)


def test_selective_scan_argument_checks(lib):
    assert _scan(lib, u=None) == INVALID
    assert _scan(lib, C=5, G=2) == INVALID
    assert _scan(lib, N=3) == UNSUPPORTED
    assert b"N=3" in lib.ss2d_last_error()
    assert _scan(lib, N=32) == UNSUPPORTED
    assert _scan(lib, ud=5) == UNSUPPORTED
    assert _scan(lib, Bm=FAKE + (3 << 20) + 4) == MISALIGNED
    assert _scan(lib, Dv=FAKE + 12) == MISALIGNED
    assert _scan(lib, y=FAKE) == INVALID  # y aliases u
    assert _scan(lib, L=0) == INVALID
    assert _scan(lib, L=(1 << 24) + 1) == INVALID


def test_selective_scan_state_argument_checks(lib):
    def call(h0=FAKE + (20 << 20), h_last=FAKE + (21 << 20), y=FAKE + (8 << 20)):
        return lib.ss2d_selective_scan_state(FAKE, 1, FAKE + (1 << 20), 1, FAKE + (2 << 20), FAKE + (3 << 20),
                                             FAKE + (4 << 20), None, None, 1, h0, h_last, y, 2, 8, 2, 16, 64, None)
    assert call(h0=FAKE + (20 << 20) + 4) == MISALIGNED
    assert call(h_last=FAKE + (21 << 20) + 8) == MISALIGNED
    assert call(h_last=FAKE + (8 << 20)) == INVALID     # h_last overlaps y
    assert call(h_last=FAKE + (1 << 20)) == INVALID     # h_last overlaps delta
    assert call(h0=FAKE + (8 << 20)) == INVALID         # h0 overlaps y
    assert call(h0=FAKE + (21 << 20)) == INVALID        # h0 overlaps h_last


def _core(**kw):
    a = CoreArgs()
    a.struct_size = ctypes.sizeof(CoreArgs)
    a.B, a.D, a.H, a.W, a.N, a.R = 1, 4, 3, 5, 16, 0
    a.x, a.x_dtype = FAKE, 1
    a.dts, a.dts_dtype = FAKE + (1 << 20), 1
    a.Bs, a.Cs = FAKE + (2 << 20), FAKE + (3 << 20)
    a.A_logs, a.Ds, a.dt_bias = FAKE + (4 << 20), FAKE + (5 << 20), FAKE + (6 << 20)
    a.delta_softplus = 1
    a.y = FAKE + (8 << 20)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_forward_core_argument_checks(lib):
    call = lambda a: lib.ss2d_forward_core(ctypes.byref(a), None, 0, None)
    assert call(_core(struct_size=8)) == INVALID
    assert call(_core(dts=None)) == INVALID
    assert call(_core(x_proj_weight=FAKE + (9 << 20), dt_projs_weight=FAKE + (10 << 20))) == INVALID  # both sources
    assert call(_core(dts=None, Bs=None, Cs=None)) == INVALID  # neither source
    assert call(_core(N=5)) == UNSUPPORTED
    assert call(_core(dts_dtype=3)) == UNSUPPORTED
    assert call(_core(x=FAKE + 8)) == MISALIGNED
    assert call(_core(y=FAKE)) == INVALID  # y aliases x
    assert lib.ss2d_forward_core_workspace(ctypes.byref(_core(N=5))) == ctypes.c_size_t(-1).value
    assert lib.ss2d_forward_core_workspace(ctypes.byref(_core())) == 0
    # the query does not need y's address; a bf16 y adds its fp32 accumulation buffer (B*D*L floats)
    assert lib.ss2d_forward_core_workspace(ctypes.byref(_core(y=None))) == 0
    assert lib.ss2d_forward_core_workspace(ctypes.byref(_core(y=None, y_dtype=1))) == 1 * 4 * 3 * 5 * 4
    assert call(_core(y=None)) == INVALID  # the call itself needs y
    assert lib.ss2d_forward_core(None, None, 0, None) == INVALID


def _grads(**kw):
    g = ss.CoreGrads()
    g.struct_size = ctypes.sizeof(ss.CoreGrads)
    g.dy = FAKE + (20 << 20)
    g.dx, g.ddts, g.dA_logs = FAKE + (21 << 20), FAKE + (22 << 20), FAKE + (23 << 20)
    g.dBs, g.dCs, g.dDs, g.ddt_bias = FAKE + (24 << 20), FAKE + (25 << 20), FAKE + (26 << 20), FAKE + (27 << 20)
    for k, v in kw.items():
        setattr(g, k, v)
    return g


def test_forward_core_backward_argument_checks(lib):
    good = dict(H=4, W=4)  # H*W = 16: bf16 rows of 16-byte multiples
    call = lambda a, g, ws=FAKE + (40 << 20), n=1 << 30: lib.ss2d_forward_core_backward(
        ctypes.byref(a), ctypes.byref(g) if g is not None else None, ws, n, None)
    query = lambda a: lib.ss2d_forward_core_backward_workspace(ctypes.byref(a))
    assert call(_core(**good), None) == INVALID
    assert call(_core(**good), _grads(struct_size=8)) == INVALID
    assert call(_core(**good), _grads(dBs=None)) == INVALID
    assert call(_core(**good, N=4), _grads(), n=16) == WORKSPACE        # N < 16 runs padded to 16 states
    assert call(_core(**good, dts_dtype=0), _grads()) == UNSUPPORTED    # mixed bf16 x / fp32 dts
    assert call(_core(**good, delta_softplus=0), _grads()) == UNSUPPORTED
    assert call(_core(H=3, W=5), _grads(), n=16) == WORKSPACE           # rows of 15 elements: 4-byte staging
    assert call(_core(**good, dts=None, Bs=None, Cs=None, R=2, x_proj_weight=FAKE + (9 << 20),
                      dt_projs_weight=FAKE + (10 << 20)), _grads()) == UNSUPPORTED  # D = 4: no x_proj GEMM
    assert call(_core(**good), _grads(dx=FAKE + (21 << 20) + 8)) == MISALIGNED
    assert call(_core(**good), _grads(dx=FAKE)) == INVALID               # dx overlaps x
    assert call(_core(**good), _grads(dCs=FAKE + (24 << 20))) == INVALID  # dCs overlaps dBs
    assert call(_core(**good), _grads(), n=16) == WORKSPACE
    assert call(_core(**good), _grads(), ws=None) == WORKSPACE
    # workspace: checkpoints (B, 4D, ceil(L/16), 16), x and dy with transposed planes, and for bf16
    # inputs fp32 copies of x and dts; all fp32, each rounded up to 256 bytes
    r256 = lambda n: (n + 255) // 256 * 256
    B, D, L = 1, 4, 16
    base = r256(B * 4 * D * 1 * 16 * 4) + r256(B * D * L * 4) + r256(B * D * L * 4)
    assert query(_core(**good, y=None)) == base + r256(B * D * L * 4) + r256(B * 4 * D * L * 4)
    assert query(_core(**good, y=None, x_dtype=0, dts_dtype=0)) == base
    # N < 16: A_log (4D, 16) twice and B, C, dB, dC (B, 4, 16, L) padded to 16 states follow
    pad = 2 * r256(4 * D * 16 * 4) + 4 * r256(B * 4 * 16 * L * 4)
    assert query(_core(**good, N=4, y=None)) == base + r256(B * D * L * 4) + r256(B * 4 * D * L * 4) + pad
    assert query(_core(**good, N=5)) == ctypes.c_size_t(-1).value
    assert lib.ss2d_forward_core_backward_workspace(None) == ctypes.c_size_t(-1).value
    # one image of 32x32: the checkpoint pass and the backward walk 8 segments of 128 steps;
    # their first-pass and carry states, (3, B, 4D, 8, 16) fp32, follow the fp32 copies
    D1, L1 = 16, 1024
    base1 = r256(4 * D1 * 64 * 16 * 4) + 2 * r256(D1 * L1 * 4) + r256(D1 * L1 * 4) + r256(4 * D1 * L1 * 4)
    assert query(_core(B=1, D=D1, H=32, W=32, y=None)) == base1 + r256(3 * 4 * D1 * 8 * 16 * 4)


def test_forward_core_backward_projection_checks(lib):
    # projection form: N = 16, D % 16 == 0 and R <= 64; weight gradients required
    proj = dict(D=16, H=2, W=8, R=2, dts=None, Bs=None, Cs=None, x_proj_weight=FAKE + (9 << 20),
                dt_projs_weight=FAKE + (10 << 20))
    wgrads = dict(ddts=None, dBs=None, dCs=None, dx_proj_weight=FAKE + (28 << 20), ddt_projs_weight=FAKE + (29 << 20))
    call = lambda a, g, ws=FAKE + (40 << 20), n=1 << 30: lib.ss2d_forward_core_backward(
        ctypes.byref(a), ctypes.byref(g), ws, n, None)
    query = lambda a: lib.ss2d_forward_core_backward_workspace(ctypes.byref(a))
    assert call(_core(**proj), _grads(**dict(wgrads, dx_proj_weight=None))) == INVALID   # weight gradient missing
    assert call(_core(**dict(proj, R=65)), _grads(**wgrads)) == UNSUPPORTED             # R > 64
    assert call(_core(**dict(proj, D=24)), _grads(**wgrads)) == UNSUPPORTED             # D % 16 != 0
    assert call(_core(**dict(proj, N=8)), _grads(**wgrads)) == UNSUPPORTED              # N != 16
    assert b"N = 16" in lib.ss2d_last_error()
    assert call(_core(**dict(proj, delta_softplus=0)), _grads(**wgrads)) == UNSUPPORTED
    assert call(_core(**dict(proj, B=16384)), _grads(**wgrads)) == UNSUPPORTED          # grid y of dt_proj's adjoints
    assert b"16383" in lib.ss2d_last_error()
    assert call(_core(**proj), _grads(**dict(wgrads, dx_proj_weight=FAKE + (9 << 20)))) == INVALID  # overlaps Wx
    assert call(_core(**proj), _grads(**dict(wgrads, ddt_projs_weight=FAKE + (28 << 20)))) == INVALID  # two overlap
    assert call(_core(**proj), _grads(**wgrads), n=16) == WORKSPACE
    # the dts/Bs/Cs form takes no weight gradients, and an ABI-102 grads struct (without them) still works there
    good = dict(H=4, W=4)
    assert call(_core(**good), _grads(dx_proj_weight=FAKE + (28 << 20))) == INVALID
    assert call(_core(**good), _grads(struct_size=ss.CoreGrads.dx_proj_weight.offset), n=16) == WORKSPACE
    assert call(_core(**good), _grads(struct_size=ss.CoreGrads.dx_proj_weight.offset + 8)) == INVALID
    # workspace: the direct form's (fp32 copies of x and dts included), then the x_proj error word,
    # x_dbl (B, 4, R+2N, L), B and C copies, their gradients, ddts, the gradient of dt_low and
    # 148 partial sums of the x_proj weight gradient
    r256 = lambda n: (n + 255) // 256 * 256
    B, D, L, N, R = 1, 16, 16, 16, 2
    direct = r256(B * 4 * D * 1 * 16 * 4) + 2 * r256(B * D * L * 4) + r256(B * D * L * 4) + r256(B * 4 * D * L * 4)
    extra = 256 + r256(B * 4 * (R + 2 * N) * L * 4) + 4 * r256(B * 4 * N * L * 4) + r256(B * 4 * D * L * 4) \
        + r256(B * 4 * R * L * 4) + r256(148 * 4 * (R + 2 * N) * D * 4)
    assert query(_core(**proj, y=None)) == direct + extra
    # channels-last: channels-first copies of x (bf16), dy and dx (fp32) follow
    assert query(_core(**proj, y=None, layout=1)) == direct + extra + r256(B * D * L * 2) + 2 * r256(B * D * L * 4)


def test_device_status_argument_checks(lib):
    """ss2d_device_status: these calls all return before touching the device."""
    call = lambda a, ws=FAKE + (40 << 20), backward=0: lib.ss2d_device_status(
        ctypes.byref(a) if a is not None else None, ws, backward, None)
    proj = dict(D=16, H=2, W=8, R=2, dts=None, Bs=None, Cs=None, x_proj_weight=FAKE + (9 << 20),
                dt_projs_weight=FAKE + (10 << 20))
    assert call(None) == INVALID
    assert call(_core(), backward=2) == INVALID
    assert call(_core(N=5)) == UNSUPPORTED                      # arguments the forward rejects
    assert call(_core(**dict(proj, N=8)), backward=1) == UNSUPPORTED  # ... or the backward rejects
    assert call(_core(**proj), ws=None, backward=1) == WORKSPACE
    assert call(_core(**proj), ws=FAKE + (40 << 20) + 8) == MISALIGNED
    # the dts/Bs/Cs form waits on nothing: OK without a workspace, forward or backward, y not needed
    assert call(_core(y=None), ws=None) == OK
    assert call(_core(H=4, W=4, y=None), ws=None, backward=1) == OK


def test_forward_core_checkpoint_checks(lib):
    # ckpt: (B, 4D, ceil(L/16), 16) fp32 kept by the forward for its backward (dts/Bs/Cs form only)
    call = lambda a: lib.ss2d_forward_core(ctypes.byref(a), None, 0, None)
    query = lambda a: lib.ss2d_forward_core_workspace(ctypes.byref(a))
    ck = FAKE + (30 << 20)
    good = dict(H=4, W=4)
    assert query(_core(**good, ckpt=ck)) == query(_core(**good))                    # no extra workspace
    assert call(_core(**good, ckpt=ck + 8)) == MISALIGNED
    assert call(_core(**good, ckpt=FAKE + (1 << 20))) == INVALID                     # overlaps dts
    assert call(_core(**good, ckpt=FAKE + (8 << 20))) == INVALID                     # overlaps y
    assert call(_core(**good, ckpt=ck, N=8)) == UNSUPPORTED
    assert call(_core(**good, ckpt=ck, dts_dtype=0)) == UNSUPPORTED                 # x and dts of one type
    assert call(_core(**good, ckpt=ck, delta_softplus=0)) == UNSUPPORTED
    assert call(_core(D=16, H=2, W=8, R=2, dts=None, Bs=None, Cs=None, x_proj_weight=FAKE + (9 << 20),
                      dt_projs_weight=FAKE + (10 << 20), ckpt=ck)) == UNSUPPORTED   # projection form
    # a struct without the member (ABI 103) is accepted and keeps no checkpoints
    assert query(_core(**good, struct_size=CoreArgs.ckpt.offset)) == query(_core(**good))
    # the backward: a gradient may not overlap the checkpoints it reads
    bcall = lambda a, g: lib.ss2d_forward_core_backward(ctypes.byref(a), ctypes.byref(g), FAKE + (40 << 20),
                                                        1 << 30, None)
    assert bcall(_core(**good, ckpt=ck), _grads(dDs=ck)) == INVALID


def test_forward_core_layout_checks(lib):
    call = lambda a: lib.ss2d_forward_core(ctypes.byref(a), None, 0, None)
    query = lambda a: lib.ss2d_forward_core_workspace(ctypes.byref(a))
    assert query(_core(struct_size=CoreArgs.layout.offset)) == 0          # struct without `layout`: channels-first
    assert query(_core(struct_size=CoreArgs.layout.offset + 2)) == ctypes.c_size_t(-1).value
    assert call(_core(layout=5)) == INVALID
    assert call(_core(layout=1, N=8)) == UNSUPPORTED                        # channels-last runs with N = 16
    assert call(_core(layout=1, dts_dtype=0)) == UNSUPPORTED                # x and dts of one type
    assert call(_core(layout=1, D=4)) == UNSUPPORTED                        # 4 bf16 channels: 8-byte runs
    assert query(_core(layout=1, D=8, H=4, W=4)) == 0                       # no transposed copy of x
    # y_dtype: struct without it keeps fp32; bf16 y adds y's fp32 sum to the workspace
    assert query(_core(struct_size=CoreArgs.y_dtype.offset, layout=1, D=8, H=4, W=4)) == 0
    assert call(_core(y_dtype=7)) == UNSUPPORTED
    assert query(_core(layout=1, D=8, H=4, W=4, y_dtype=1)) == 1 * 8 * 16 * 4
    # where channels-last x needs a channels-first copy (the projection form's GEMM, the backward),
    # one launch transposes each image's (H*W, D) matrix in at most 65535 tiles of 32x32
    big = dict(layout=1, D=96, H=1024, W=1024, y=None)            # 32768 * 3 tiles
    proj = dict(R=6, dts=None, Bs=None, Cs=None, x_proj_weight=FAKE + (9 << 20), dt_projs_weight=FAKE + (10 << 20))
    assert query(_core(**big, **proj)) == ctypes.c_size_t(-1).value
    assert b"65535" in lib.ss2d_last_error()
    assert query(_core(**big)) != ctypes.c_size_t(-1).value        # the direct form reads channel runs in place
    bwd_query = lambda a: lib.ss2d_forward_core_backward_workspace(ctypes.byref(a))
    assert bwd_query(_core(**big)) == ctypes.c_size_t(-1).value
    assert b"65535" in lib.ss2d_last_error()
    assert bwd_query(_core(**dict(big, H=512))) != ctypes.c_size_t(-1).value  # 16384 * 3 tiles
    # channels-first: the plane transpose of x (the column orders' rows; the backward's x and dy)
    # is one launch of at most 65535 tiles of 32x32
    long_rows = dict(H=2, W=1 << 21, y=None)                                 # 1 * 65536 tiles, rows aligned
    assert query(_core(**long_rows)) == ctypes.c_size_t(-1).value
    assert b"65535" in lib.ss2d_last_error()
    assert query(_core(H=1, W=(1 << 21) + 1, y=None)) != ctypes.c_size_t(-1).value  # unaligned rows: no copy
    assert bwd_query(_core(**dict(long_rows, W=(1 << 21) + 4))) == ctypes.c_size_t(-1).value
    assert b"65535" in lib.ss2d_last_error()


def test_binding_rejects_host_tensors():
    import torch

    x = torch.zeros(1, 2, 3, 3)
    with pytest.raises(ValueError):
        ss.cross_scan(x)


def test_bench_segment_mirror_matches_library(lib):
    # bench.py counts the kernels of a segmented scan from its own copy of the segment plan;
    # the library's workspace size (segment states + the transposed copy of x) reveals its plan
    import dataclasses
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from selective_scan_02_b200.inputs import WORKLOADS
    cases = [("vmamba_t_stage1", {}), ("vmamba_t_stage1", {"B": 1}), ("vmamba_t_stage1", {"B": 8}),
             ("hires_long", {}), ("stage3_short", {}), ("tiny", {})]
    for name, over in cases:
        wl = dataclasses.replace(WORKLOADS[name], **over)
        esize = 2 if wl.x_dtype == "bf16" else 4
        G = 1 << 36  # tensors of these sizes need fake addresses far apart
        a = _core(B=wl.B, D=wl.D, H=wl.H, W=wl.W, N=wl.N, x_dtype=1 if wl.x_dtype == "bf16" else 0,
                  dts_dtype=1 if wl.dt_dtype == "bf16" else 0, x=FAKE, dts=FAKE + G, Bs=FAKE + 2 * G,
                  Cs=FAKE + 3 * G, A_logs=FAKE + 4 * G, Ds=FAKE + 5 * G, dt_bias=FAKE + 6 * G, y=FAKE + 7 * G)
        ws = lib.ss2d_forward_core_workspace(ctypes.byref(a))
        transposed = wl.B * wl.D * wl.L * esize if (wl.N == 16 and (wl.L * esize) % 16 == 0) else 0
        per_seg = 3 * wl.B * 4 * wl.D * wl.N * 4
        seg_bytes = ws - transposed
        nseg = seg_bytes // per_seg if seg_bytes > 0 else 1
        assert seg_bytes in (0, nseg * per_seg), (name, over, ws)
        assert bench.planned_segments(wl) == nseg, (name, over, nseg)


def test_projection_large_dt_rank_checks(lib):
    # dt_ranks above 16 are supported channels-first (dts materialised in the workspace) and
    # rejected channels-last; above 64 they are rejected
    G = 1 << 36
    base = dict(B=1, D=64, H=8, W=12, N=16, x_dtype=1, x=FAKE, dts=None, Bs=None, Cs=None, A_logs=FAKE + G, Ds=FAKE + 2 * G,
                dt_bias=FAKE + 3 * G, x_proj_weight=FAKE + 4 * G, dt_projs_weight=FAKE + 5 * G, y=FAKE + 6 * G)
    small = _core(R=16, **base)
    large = _core(R=24, **base)
    ws_small = lib.ss2d_forward_core_workspace(ctypes.byref(small))
    ws_large = lib.ss2d_forward_core_workspace(ctypes.byref(large))
    L, D = 8 * 12, 64
    # x_dbl grows by 4*(24-16) rows; dts (1, 4, D, L) fp32 is added; the fused path's transposed
    # copy of x (1, D, W, H) bf16 is not needed
    assert ws_large - ws_small == 4 * 8 * L * 4 + 4 * D * L * 4 - D * L * 2
    cl = _core(R=24, layout=1, **base)
    assert lib.ss2d_forward_core_workspace(ctypes.byref(cl)) == ctypes.c_size_t(-1).value
    assert b"R <= 16" in lib.ss2d_last_error()
    assert lib.ss2d_forward_core_workspace(ctypes.byref(_core(R=65, **base))) == ctypes.c_size_t(-1).value


def test_page_order_merge_checks(lib):
    # SS2D_MERGE_PAGE_ORDER: dts/Bs/Cs form, N = 16, softplus on, x and dts of one type
    assert lib.ss2d_forward_core(ctypes.byref(_core(merge_order=1)), None, 0, None) in (OK, WORKSPACE, CUDA)
    assert lib.ss2d_forward_core(ctypes.byref(_core(merge_order=2)), None, 0, None) == INVALID
    assert lib.ss2d_forward_core(ctypes.byref(_core(merge_order=1, N=8)), None, 0, None) == UNSUPPORTED
    assert lib.ss2d_forward_core(ctypes.byref(_core(merge_order=1, dts_dtype=0)), None, 0, None) == UNSUPPORTED
    # every direction stores its output once: the workspace grows by the four outputs in scan order
    G = 1 << 36
    base = dict(B=2, D=192, H=256, W=256, N=16, x=FAKE, dts=FAKE + G, Bs=FAKE + 2 * G, Cs=FAKE + 3 * G,
                A_logs=FAKE + 4 * G, Ds=FAKE + 5 * G, dt_bias=FAKE + 6 * G, y=FAKE + 7 * G)
    ws_atomic = lib.ss2d_forward_core_workspace(ctypes.byref(_core(**base)))
    ws_page = lib.ss2d_forward_core_workspace(ctypes.byref(_core(merge_order=1, **base)))
    assert ws_atomic % 256 == 0 and ws_page == ws_atomic + 4 * 2 * 192 * 256 * 256 * 4
    # channel-first y is merged in one launch of 32x32 tiles per plane: rejected on the host when
    # there are more than 65535 (fp32 x of odd length: no transposed copy, whose check would say so)
    big = dict(base, B=1, D=16, H=1, W=(1 << 24) - 1, x_dtype=0, dts_dtype=0)
    assert lib.ss2d_forward_core(ctypes.byref(_core(merge_order=1, **big)), None, 0, None) == UNSUPPORTED
    assert b"65535 tiles" in lib.ss2d_last_error()
    assert lib.ss2d_forward_core_workspace(ctypes.byref(_core(merge_order=0, **big))) != ctypes.c_size_t(-1).value
    # callers built against the struct without merge_order still get the atomic merge
    old = _core(**base)
    old.struct_size = CoreArgs.merge_order.offset
    assert lib.ss2d_forward_core_workspace(ctypes.byref(old)) == ws_atomic


def _block(**kw):
    from selective_scan_02_b200 import BlockArgs

    a = BlockArgs()
    a.struct_size = ctypes.sizeof(BlockArgs)
    a.B, a.H, a.W, a.d_model, a.D, a.N, a.R, a.d_conv = 2, 8, 8, 32, 64, 16, 4, 3
    span = 1 << 30  # distinct fake buffers, far enough apart not to overlap
    names = ["x", "in_proj_weight", "conv_weight", "conv_bias", "x_proj_weight", "dt_projs_weight", "dt_projs_bias",
             "A_logs", "Ds", "out_norm_weight", "out_norm_bias", "out_proj_weight", "out"]
    for i, n in enumerate(names):
        setattr(a, n, FAKE + i * span)
    a.out_norm_eps = 1e-5
    a.out_dtype = 0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_block_argument_checks(lib):
    """ss2d_block_forward checks everything on the host and enqueues nothing on failure; the
    workspace size follows its layout (error word, the core's workspace, xz, x_c, y)."""
    from selective_scan_02_b200 import BlockArgs

    lib.ss2d_block_forward_workspace.restype = ctypes.c_size_t
    lib.ss2d_block_forward_workspace.argtypes = [ctypes.POINTER(BlockArgs)]
    lib.ss2d_block_forward.argtypes = [ctypes.POINTER(BlockArgs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    none = ctypes.c_size_t(-1).value

    def ws(a):
        return lib.ss2d_block_forward_workspace(ctypes.byref(a))

    def run(a, wsp=FAKE + (40 << 30), nbytes=1 << 40):
        return lib.ss2d_block_forward(ctypes.byref(a), wsp, nbytes, None)

    good = _block()
    n = ws(good)
    assert n != none
    # the core's workspace for the same shape in its projection form, then the block's buffers;
    # the block runs the core channels-last where N = 16, dt_rank <= 16 and D <= 768, else
    # channel-first
    def core_ws(R, layout):
        core = CoreArgs()
        core.struct_size = ctypes.sizeof(CoreArgs)
        core.B, core.D, core.H, core.W, core.N, core.R = 2, 64, 8, 8, 16, R
        core.x, core.x_dtype, core.A_logs = FAKE, 1, FAKE + (7 << 30)
        core.x_proj_weight, core.dt_projs_weight, core.delta_softplus = FAKE + (4 << 30), FAKE + (5 << 30), 1
        core.layout = layout
        lib.ss2d_forward_core_workspace.restype = ctypes.c_size_t
        return lib.ss2d_forward_core_workspace(ctypes.byref(core))

    M, D = 2 * 64, 64

    def r256(v):
        return (v + 255) // 256 * 256

    def block_ws(cw):
        return 256 + r256(cw) + r256(M * 2 * D * 2) + r256(M * D * 2) + r256(M * D * 4)

    assert n == block_ws(core_ws(4, 1))
    assert ws(_block(R=24)) == block_ws(core_ws(24, 0))
    assert run(good, nbytes=n - 1) == WORKSPACE
    assert run(good, wsp=None) == WORKSPACE
    assert run(good, wsp=FAKE + (40 << 30) + 8) == MISALIGNED
    assert run(good, wsp=good.out) == INVALID  # workspace overlaps out
    assert run(_block(struct_size=8)) == INVALID
    assert run(_block(d_conv=2)) == INVALID and b"odd" in lib.ss2d_last_error()
    assert run(_block(d_conv=9)) == UNSUPPORTED
    assert run(_block(d_model=40)) == UNSUPPORTED
    assert run(_block(D=72)) == UNSUPPORTED
    assert run(_block(D=1664)) == UNSUPPORTED and b"1648" in lib.ss2d_last_error()
    assert run(_block(N=8)) == UNSUPPORTED
    assert run(_block(R=65)) == UNSUPPORTED  # the core's projection form takes R <= 64
    assert run(_block(out_dtype=5)) == UNSUPPORTED
    assert run(_block(out_norm_eps=0.0)) == INVALID
    assert run(_block(x=None)) == INVALID
    assert run(_block(out=None)) == INVALID
    assert ws(_block(out=None)) == n  # the size query does not need out
    assert run(_block(conv_weight=FAKE + (2 << 30) + 4)) == MISALIGNED
    assert run(_block(out=FAKE)) == INVALID and b"overlaps" in lib.ss2d_last_error()
    assert run(_block(B=0)) == INVALID
    assert ws(_block(B=0)) == none
