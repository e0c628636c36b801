"""The general selective-scan kernel runs on the host, against the oracle, without a GPU.

selective_scan_02_b200/csrc/scan.cuh (scan_kernel: every N in {1, 2, 4, 8, 16}, element types
read at run time; the path for N < 16 and for type mixes the N = 16 kernel is not compiled
for) is compiled for the CPU with tests/emu/: one std::thread per lane, shuffles and
__syncwarp on a barrier, cp.async as copies that check their shared-memory destination and
global-source alignment, merge atomics as atomic adds, and exp2/log2 from the C library in
place of the hardware units, under AddressSanitizer and UBSan.  The warp shapes are the
library's for each N.  Standalone scans (with and without D, bias, softplus, an initial state
and the final state; rows that are not 16-byte aligned; ragged channel tiles), the fused core
and its projection mode are compared with the oracle.
"""
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as orc
from tests.emu_build import build_emulator
from selective_scan_02_b200.inputs import Workload, bf16_bits, make_inputs, random_scan_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_scan_02_b200", "csrc")


def _rel_err(got, ref):
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-30)))


@pytest.fixture(scope="module")
def emulator(tmp_path_factory):
    d = tmp_path_factory.mktemp("scan_emu")
    src = open(os.path.join(CSRC, "scan.cuh")).read()
    body = src[src.index("enum ScanMode"):]
    body = body.replace("extern __shared__ __align__(16) unsigned char smem_raw[];",
                        "unsigned char *smem_raw = g_warp->smem;")
    return build_emulator(d, '#pragma once\n#include "common_emu.h"\nnamespace ss2d {\n' + body, "scan_emu_main.cpp")


def _store(a, dt):
    if dt == "bf16":
        return bf16_bits(np.ascontiguousarray(a, np.float32)).astype(np.uint16)
    return np.ascontiguousarray(a, np.float32)


def _f32(a, path):
    np.ascontiguousarray(a, np.float32).tofile(path)


def _run(emulator, d, mode, B, C, H, W, N, G, ub, db, sp, hasD, hasb, h0, last, R=0):
    args = [emulator] + [str(v) for v in (mode, B, C, H, W, N, G, int(ub), int(db), int(sp), int(hasD), int(hasb),
                                           int(h0), int(last), R)] + [d]
    r = subprocess.run(args, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]


SCAN_CASES = [
    # B, C, G, N, L, u dtype, delta dtype, softplus, D and bias, h0, h_last
    (2, 24, 2, 16, 100, "bf16", "f32", True, True, False, True),   # N = 16, a type mix scan2 does not cover
    (1, 16, 1, 8, 37, "f32", "f32", True, True, True, True),       # rows not 16-byte aligned, state passing
    (2, 20, 2, 4, 33, "bf16", "bf16", False, False, False, False),  # softplus off, no D / bias, ragged tile
    (1, 8, 1, 2, 64, "f32", "bf16", True, True, True, False),
    (1, 40, 4, 1, 129, "bf16", "f32", True, True, False, True),    # ragged tile of 10 channels per group
]


@pytest.mark.parametrize("case", SCAN_CASES)
def test_general_scan_kernel_standalone_matches_oracle(emulator, tmp_path, case):
    B, C, G, N, L, udt, ddt, sp, hasDb, hash0, last = case
    inp = random_scan_inputs(90 + B + C + N + L, B, C, G, N, L, udt, ddt)
    delta, bias = inp["delta"], inp["delta_bias"]
    if not sp:  # without softplus the step size is taken as given: keep it positive
        delta, bias = np.abs(delta), None
    Dv = inp["Dv"] if hasDb else None
    bias = bias if hasDb else None
    h0 = np.random.default_rng(L).standard_normal((B, C, N)).astype(np.float32) if hash0 else None
    d = str(tmp_path)
    _store(inp["u"], udt).tofile(f"{d}/u")
    _store(delta, ddt).tofile(f"{d}/delta")
    for a, n in [(inp["Bm"], "Bm"), (inp["Cm"], "Cm"), (inp["A_log"], "A"), (Dv, "Dv"), (bias, "bias"), (h0, "h0")]:
        if a is not None:
            _f32(a, f"{d}/{n}")
    _run(emulator, d, 0, B, C, 1, L, N, G, udt == "bf16", ddt == "bf16", sp, Dv is not None, bias is not None,
         h0 is not None, last)
    ref_y, ref_h = orc.selective_scan(inp["u"], delta, inp["A_log"], inp["Bm"], inp["Cm"], Dv, bias, sp,
                                      h0=h0, return_last_state=True)
    tol = 5e-3 if "bf16" in (udt, ddt) else 2e-3
    y = np.fromfile(f"{d}/y", np.float32).astype(np.float64)
    assert _rel_err(y, ref_y.reshape(-1)) <= tol
    if last:
        h = np.fromfile(f"{d}/hlast", np.float32).astype(np.float64)
        assert _rel_err(h, ref_h.reshape(-1)) <= tol


CORE_CASES = [
    # B, D, H, W, N, dtype (x and dts), R (0: dts/Bs/Cs form)
    (1, 8, 8, 8, 4, "f32", 0),      # the tiny workload's shape
    (2, 20, 6, 10, 8, "bf16", 0),   # H != W, a ragged channel tile
    (1, 16, 5, 7, 2, "f32", 0),     # rows not 16-byte aligned
    (1, 16, 8, 8, 8, "bf16", 3),    # projection mode
    (2, 24, 6, 8, 4, "bf16", 2),    # projection mode, ragged tile
]


@pytest.mark.parametrize("case", CORE_CASES)
def test_general_scan_kernel_fused_core_matches_oracle(emulator, tmp_path, case):
    B, D, H, W, N, dt, R = case
    inp = make_inputs(Workload("emu_g", B, D, H, W, N, R, dt, dt, 110 + B + D + H + W + N + R))
    d = str(tmp_path)
    _store(inp["x"], dt).tofile(f"{d}/u")
    for k, n in [("A_logs", "A"), ("Ds", "Dv"), ("dt_bias", "bias")]:
        _f32(inp[k], f"{d}/{n}")
    if R:
        _f32(orc.x_proj(orc.cross_scan(inp["x"]), inp["x_proj_weight"]), f"{d}/xdbl")
        _f32(inp["dt_projs_weight"], f"{d}/Wdt")
        ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"],
                               x_proj_weight=inp["x_proj_weight"], dt_projs_weight=inp["dt_projs_weight"])
    else:
        _store(inp["dts"], dt).tofile(f"{d}/delta")
        _f32(inp["Bs"], f"{d}/Bm")
        _f32(inp["Cs"], f"{d}/Cm")
        ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"],
                               Cs=inp["Cs"])
    _run(emulator, d, 2 if R else 1, B, D, H, W, N, 4, dt == "bf16", dt == "bf16" and not R, True, True, True,
         False, False, R)
    y = np.fromfile(f"{d}/y", np.float32).astype(np.float64)
    assert _rel_err(y, ref.reshape(-1)) <= (5e-3 if dt == "bf16" else 2e-3)
