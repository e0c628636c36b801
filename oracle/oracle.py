"""ctypes front end of the CPU oracle (ss2d_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path.  It converts numpy
arrays to contiguous fp64 and calls the plain sequential C restatement of the
SS2D forward core and of its gradient (liboracle.so).  Every function but one
is marshalling around a C call; forward_core_proj_bwd composes C calls with
library einsums (the adjoints of the two linear projections), as its docstring
states.  forward_core_f32 calls the same C source compiled with an fp32 element
type (liboracle_f32.so); it exists only to time an fp32 CPU baseline and is not
a parity reference.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss2d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_LIB32 = os.path.join(_HERE, "liboracle_f32.so")
_lib = None
_lib32 = None


def build(force: bool = False) -> str:
    """Compile ss2d_oracle.c into liboracle.so (fp64) and liboracle_f32.so (the fp32
    instantiation, for timing only) with gcc (plain -O2, no fast-math)."""
    for lib, extra in ((_LIB, []), (_LIB32, ["-DORACLE_REAL=float"])):
        if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(_SRC):
            cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", *extra, "-o", lib, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_cross_scan.argtypes = [P, P, I, I, I, I]
        _lib.oracle_cross_merge.argtypes = [P, P, I, I, I, I]
        _lib.oracle_x_proj.argtypes = [P, P, P, I, I, I, I]
        _lib.oracle_dt_proj.argtypes = [P, P, P, I, I, I, I, I]
        _lib.oracle_selective_scan.argtypes = [P, P, P, P, P, P, P, I, P, I, I, I, I, I, P, P]
        _lib.oracle_selective_scan_ckpt.argtypes = [P, P, P, P, P, P, P, I, P, I, I, I, I, I, I, P]
        _lib.oracle_forward_core.argtypes = [P, P, P, P, P, P, P, I, P, P, P, I, I, I, I, I, I]
        _lib.oracle_selective_scan_bwd.argtypes = [P, P, P, P, P, P, P, I, P, P, P, P, P, P, P, P, I, I, I, I, I]
        _lib.oracle_forward_core_bwd.argtypes = [P, P, P, P, P, P, P, I, P, P, P, P, P, P, P, P, I, I, I, I, I]
        for f in (_lib.oracle_cross_scan, _lib.oracle_cross_merge, _lib.oracle_x_proj,
                  _lib.oracle_dt_proj, _lib.oracle_selective_scan, _lib.oracle_selective_scan_ckpt,
                  _lib.oracle_forward_core,
                  _lib.oracle_selective_scan_bwd, _lib.oracle_forward_core_bwd):
            f.restype = None
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def cross_scan(x):
    """x (B,D,H,W) -> xs (B,4,D,H*W)."""
    x = _f64(x)
    B, D, H, W = x.shape
    xs = np.empty((B, 4, D, H * W), dtype=np.float64)
    _load().oracle_cross_scan(_ptr(x), _ptr(xs), B, D, H, W)
    return xs


def cross_merge(out_y, H, W):
    """out_y (B,4,D,L) -> y (B,D,H,W)."""
    out_y = _f64(out_y)
    B, K, D, L = out_y.shape
    assert K == 4 and L == H * W
    y = np.empty((B, D, H, W), dtype=np.float64)
    _load().oracle_cross_merge(_ptr(out_y), _ptr(y), B, D, H, W)
    return y


def x_proj(xs, weight):
    """xs (B,4,D,L), weight (4,Cp,D) -> x_dbl (B,4,Cp,L)."""
    xs, weight = _f64(xs), _f64(weight)
    B, K, D, L = xs.shape
    Cp = weight.shape[1]
    out = np.empty((B, 4, Cp, L), dtype=np.float64)
    _load().oracle_x_proj(_ptr(xs), _ptr(weight), _ptr(out), B, D, L, Cp)
    return out


def dt_proj(x_dbl, weight, N):
    """x_dbl (B,4,R+2N,L) (first R rows used), weight (4,D,R) -> dts (B,4,D,L)."""
    x_dbl, weight = _f64(x_dbl), _f64(weight)
    B, K, Cp, L = x_dbl.shape
    _, D, R = weight.shape
    assert Cp == R + 2 * N
    out = np.empty((B, 4, D, L), dtype=np.float64)
    _load().oracle_dt_proj(_ptr(x_dbl), _ptr(weight), _ptr(out), B, D, L, R, N)
    return out


def selective_scan(u, delta, A_log, Bm, Cm, Dv=None, delta_bias=None, delta_softplus=True,
                   h0=None, return_last_state=False):
    """u, delta (B,C,L); A_log (C,N); Bm, Cm (B,G,N,L) -> y (B,C,L) [, h_last (B,C,N)]."""
    u, delta, A_log, Bm, Cm = _f64(u), _f64(delta), _f64(A_log), _f64(Bm), _f64(Cm)
    Dv, delta_bias, h0 = _f64(Dv), _f64(delta_bias), _f64(h0)
    B, C, L = u.shape
    G, N = Bm.shape[1], Bm.shape[2]
    assert delta.shape == u.shape and A_log.shape == (C, N) and Cm.shape == Bm.shape
    assert C % G == 0
    y = np.empty((B, C, L), dtype=np.float64)
    h_last = np.empty((B, C, N), dtype=np.float64) if return_last_state else None
    _load().oracle_selective_scan(_ptr(u), _ptr(delta), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(Dv),
                                  _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y),
                                  B, C, G, N, L, _ptr(h0), _ptr(h_last))
    return (y, h_last) if return_last_state else y


def selective_scan_ckpt(u, delta, A_log, Bm, Cm, every, Dv=None, delta_bias=None, delta_softplus=True):
    """selective_scan from a zero state that also returns the state before every `every`-th
    step: y (B,C,L) and ckpt (B,C,ceil(L/every),N), ckpt[b,c,j] = h_{j*every-1} (zero for j=0)."""
    u, delta, A_log, Bm, Cm = _f64(u), _f64(delta), _f64(A_log), _f64(Bm), _f64(Cm)
    Dv, delta_bias = _f64(Dv), _f64(delta_bias)
    B, C, L = u.shape
    G, N = Bm.shape[1], Bm.shape[2]
    assert delta.shape == u.shape and A_log.shape == (C, N) and Cm.shape == Bm.shape and every > 0
    y = np.empty((B, C, L), dtype=np.float64)
    ck = np.empty((B, C, (L + every - 1) // every, N), dtype=np.float64)
    _load().oracle_selective_scan_ckpt(_ptr(u), _ptr(delta), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(Dv),
                                       _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y),
                                       B, C, G, N, L, int(every), _ptr(ck))
    return y, ck


def forward_core(x, A_logs, Ds, dt_bias, dts=None, Bs=None, Cs=None, x_proj_weight=None,
                 dt_projs_weight=None, delta_softplus=True):
    """SS2D forward core, channel-first: x (B,D,H,W) -> y (B,D,H,W)."""
    x, A_logs, Ds, dt_bias = _f64(x), _f64(A_logs), _f64(Ds), _f64(dt_bias)
    dts, Bs, Cs = _f64(dts), _f64(Bs), _f64(Cs)
    x_proj_weight, dt_projs_weight = _f64(x_proj_weight), _f64(dt_projs_weight)
    B, D, H, W = x.shape
    N = A_logs.shape[1]
    R = 0
    if x_proj_weight is not None:
        R = dt_projs_weight.shape[2]
        assert x_proj_weight.shape == (4, R + 2 * N, D)
    else:
        assert dts is not None and Bs is not None and Cs is not None
    y = np.empty((B, D, H, W), dtype=np.float64)
    _load().oracle_forward_core(_ptr(x), _ptr(dts), _ptr(A_logs), _ptr(Bs), _ptr(Cs), _ptr(Ds),
                                _ptr(dt_bias), int(bool(delta_softplus)), _ptr(x_proj_weight),
                                _ptr(dt_projs_weight), _ptr(y), B, D, H, W, N, R)
    return y


def forward_core_f32(x, A_logs, Ds, dt_bias, dts, Bs, Cs, delta_softplus=True):
    """forward_core (dts/Bs/Cs form) in the oracle's fp32 instantiation, for timing an fp32
    CPU baseline only (parity is always taken against the fp64 forward_core).  Inputs are
    converted to contiguous fp32; the C call releases the GIL, so threads can split a batch."""
    global _lib32
    if _lib32 is None:
        build()
        _lib32 = ctypes.CDLL(_LIB32)
        P, I = ctypes.c_void_p, ctypes.c_int
        _lib32.oracle_forward_core.argtypes = [P, P, P, P, P, P, P, I, P, P, P, I, I, I, I, I, I]
        _lib32.oracle_forward_core.restype = None
    f = [np.ascontiguousarray(a, dtype=np.float32) for a in (x, dts, A_logs, Bs, Cs, Ds, dt_bias)]
    B, D, H, W = f[0].shape
    N = f[2].shape[1]
    y = np.empty((B, D, H, W), dtype=np.float32)
    _lib32.oracle_forward_core(_ptr(f[0]), _ptr(f[1]), _ptr(f[2]), _ptr(f[3]), _ptr(f[4]), _ptr(f[5]),
                               _ptr(f[6]), int(bool(delta_softplus)), None, None, _ptr(y), B, D, H, W, N, 0)
    return y


def selective_scan_bwd(u, delta, A_log, Bm, Cm, Dv, delta_bias, delta_softplus, dy):
    """Gradient of selective_scan (zero initial state) given dy (B,C,L).  Returns a dict with
    du, ddelta (B,C,L), dA_log (C,N), dBm, dCm (B,G,N,L), dDv, ddelta_bias (C)."""
    u, delta, A_log, Bm, Cm, dy = _f64(u), _f64(delta), _f64(A_log), _f64(Bm), _f64(Cm), _f64(dy)
    Dv, delta_bias = _f64(Dv), _f64(delta_bias)
    B, C, L = u.shape
    G, N = Bm.shape[1], Bm.shape[2]
    assert delta.shape == u.shape == dy.shape and A_log.shape == (C, N) and Cm.shape == Bm.shape
    out = dict(du=np.empty((B, C, L)), ddelta=np.empty((B, C, L)), dA_log=np.empty((C, N)),
               dBm=np.empty((B, G, N, L)), dCm=np.empty((B, G, N, L)), dDv=np.empty(C), ddelta_bias=np.empty(C))
    _load().oracle_selective_scan_bwd(_ptr(u), _ptr(delta), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(Dv),
                                      _ptr(delta_bias), int(bool(delta_softplus)), _ptr(dy),
                                      _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dA_log"]), _ptr(out["dBm"]),
                                      _ptr(out["dCm"]), _ptr(out["dDv"]), _ptr(out["ddelta_bias"]), B, C, G, N, L)
    return out


def forward_core_bwd(x, A_logs, Ds, dt_bias, dts, Bs, Cs, dy, delta_softplus=True):
    """Gradient of forward_core (dts/Bs/Cs form) given dy (B,D,H,W).  Returns a dict with
    dx (B,D,H,W), ddts (B,4,D,L), dA_logs (4D,N), dBs, dCs (B,4,N,L), dDs, ddt_bias (4D)."""
    x, A_logs, Ds, dt_bias = _f64(x), _f64(A_logs), _f64(Ds), _f64(dt_bias)
    dts, Bs, Cs, dy = _f64(dts), _f64(Bs), _f64(Cs), _f64(dy)
    B, D, H, W = x.shape
    N = A_logs.shape[1]
    L = H * W
    assert dy.shape == x.shape and dts.shape == (B, 4, D, L) and Bs.shape == (B, 4, N, L)
    out = dict(dx=np.empty((B, D, H, W)), ddts=np.empty((B, 4, D, L)), dA_logs=np.empty((4 * D, N)),
               dBs=np.empty((B, 4, N, L)), dCs=np.empty((B, 4, N, L)), dDs=np.empty(4 * D),
               ddt_bias=np.empty(4 * D))
    _load().oracle_forward_core_bwd(_ptr(x), _ptr(dts), _ptr(A_logs), _ptr(Bs), _ptr(Cs), _ptr(Ds),
                                    _ptr(dt_bias), int(bool(delta_softplus)), _ptr(dy),
                                    _ptr(out["dx"]), _ptr(out["ddts"]), _ptr(out["dA_logs"]), _ptr(out["dBs"]),
                                    _ptr(out["dCs"]), _ptr(out["dDs"]), _ptr(out["ddt_bias"]), B, D, H, W, N)
    return out


def forward_core_proj_bwd(x, x_proj_weight, dt_projs_weight, A_logs, Ds, dt_bias, dy, delta_softplus=True):
    """Gradient of forward_core in its projection form (x_proj and dt_proj of section 3.2
    of the SS2D article) given dy (B,D,H,W).

    The chain rule through the steps of the forward, in the forward's order:
      xs = CrossScan(x); x_dbl = x_proj(xs); dts = dt_proj(x_dbl[:, :, :R]);
      Bs, Cs = x_dbl[:, :, R:R+N], x_dbl[:, :, R+N:]; y = core(x, dts, Bs, Cs).
    The core's gradient is forward_core_bwd; the two projections are linear maps whose
    adjoints are the transposed contractions (library einsums), and CrossScan's adjoint is
    CrossMerge.  Returns a dict with dx (B,D,H,W), dx_proj_weight (4,R+2N,D),
    ddt_projs_weight (4,D,R), dA_logs (4D,N), dDs, ddt_bias (4D), and the gradients of
    the intermediates: ddts (B,4,D,L), dBs, dCs (B,4,N,L), in scan order."""
    x, Wx, Wdt, dy = _f64(x), _f64(x_proj_weight), _f64(dt_projs_weight), _f64(dy)
    B, D, H, W = x.shape
    N = np.asarray(A_logs).shape[1]
    R = Wdt.shape[2]
    assert Wx.shape == (4, R + 2 * N, D) and Wdt.shape == (4, D, R) and dy.shape == x.shape
    xs = cross_scan(x)
    x_dbl = x_proj(xs, Wx)
    dts = dt_proj(x_dbl, Wdt, N)
    Bs = np.ascontiguousarray(x_dbl[:, :, R:R + N])
    Cs = np.ascontiguousarray(x_dbl[:, :, R + N:])
    g = forward_core_bwd(x, A_logs, Ds, dt_bias, dts, Bs, Cs, dy, delta_softplus)
    # dts[b,k,d,l] = sum_r Wdt[k,d,r] x_dbl[b,k,r,l]
    d_dtlow = np.einsum("kdr,bkdl->bkrl", Wdt, g["ddts"])
    dWdt = np.einsum("bkdl,bkrl->kdr", g["ddts"], x_dbl[:, :, :R])
    # x_dbl[b,k,c,l] = sum_d Wx[k,c,d] xs[b,k,d,l]
    d_xdbl = np.concatenate([d_dtlow, g["dBs"], g["dCs"]], axis=2)
    dWx = np.einsum("bkcl,bkdl->kcd", d_xdbl, xs)
    dxs = np.einsum("kcd,bkcl->bkdl", Wx, d_xdbl)
    dx = g["dx"] + cross_merge(dxs, H, W)
    return dict(dx=dx, dx_proj_weight=dWx, ddt_projs_weight=dWdt, dA_logs=g["dA_logs"], dDs=g["dDs"],
                ddt_bias=g["ddt_bias"], ddts=g["ddts"], dBs=g["dBs"], dCs=g["dCs"])
