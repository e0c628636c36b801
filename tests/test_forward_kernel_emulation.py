"""The forward scan kernel runs on the host, against the oracle, without a GPU.

selective_scan_02_b200/csrc/scan2.cuh (the fused N = 16 core: staging, the in-loop delta,
the scan and the merge) is compiled for the CPU with tests/emu/: one std::thread per lane,
shuffles and __syncwarp on a barrier, cp.async as copies that check their shared-memory
destination and global-source alignment, merge atomics as atomic adds, and exp2/log2 from
the C library in place of the hardware units.  AddressSanitizer and UBSan watch every
access.  y is compared with oracle.forward_core for bf16 and fp32 inputs, channels-first
and channels-last, whole and segmented sequences, a ragged channel tile and a partial chunk;
where the pass keeps the backward's checkpoints, they are compared with the fp64 recurrence.
The page-order merge's plain stores (per-direction outputs, each element once) and the kernel's
projection mode (dt_proj fused into the loop, rows of x_dbl) are run the same way.
"""
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import oracle as orc
from tests.emu_build import build_emulator
from selective_scan_02_b200.inputs import Workload, bf16_bits, make_inputs
from tests.ckpt_reference import checkpoints

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_scan_02_b200", "csrc")


def _rel_err(got, ref):
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-30)))


@pytest.fixture(scope="module")
def emulator(tmp_path_factory):
    d = tmp_path_factory.mktemp("fwd_emu")
    scan = open(os.path.join(CSRC, "scan.cuh")).read()
    # the modes, constants and argument struct of scan.cuh (not its older kernel)
    decls = scan[scan.index("enum ScanMode"):scan.index("template <int N_, int TN_, int CH_, int MINB_")]
    src = open(os.path.join(CSRC, "scan2.cuh")).read()
    body = src[src.index("namespace ss2d {") + len("namespace ss2d {"):]
    body = body.replace("extern __shared__ __align__(16) unsigned char smem_raw[];",
                        "unsigned char *smem_raw = g_warp->smem;")
    body = re.sub(r"__device__ __forceinline__ float bf16_(lo|hi)\(uint32_t w\) \{[^}]*\}\n", "", body)
    # the carry kernel of the segmented scan, from the launchers' file
    cu = open(os.path.join(CSRC, "scan.cu")).read()
    carry = cu[cu.index("__global__ void segment_carry_kernel"):
               cu.index("template <int MODE, int DT, int CL>\ncudaError_t launch_segmented")]
    header = '#pragma once\n#include "common_emu.h"\nnamespace ss2d {\n' + decls + body
    return build_emulator(d, header + "\nnamespace ss2d {\n" + carry + "}\n", "fwd_emu_main.cpp")


CASES = [
    # B, D, H, W, dtype, channels_last, nseg, seg_len, keep checkpoints
    (1, 16, 8, 12, "bf16", False, 1, 96, False),     # three whole chunks
    (2, 24, 10, 12, "bf16", False, 1, 120, True),    # a ragged channel tile, a partial last chunk
    (1, 16, 8, 8, "f32", False, 1, 64, False),
    (1, 16, 16, 16, "bf16", False, 4, 64, True),     # segmented: first pass, carry, second pass
    (1, 16, 8, 12, "bf16", True, 1, 96, True),       # channels-last x and y
    (1, 8, 8, 8, "f32", True, 1, 64, False),         # channels-last, fewer channels than a tile
]


@pytest.mark.parametrize("case", CASES)
def test_forward_kernel_host_emulation_matches_oracle(emulator, tmp_path, case):
    B, D, H, W, dt, cl, nseg, seg_len, keep = case
    wl = Workload("emu_f", B, D, H, W, 16, 0, dt, dt, 60 + B + D + H + W)
    inp = make_inputs(wl)
    d = str(tmp_path)
    store = (lambda a: bf16_bits(np.ascontiguousarray(a, np.float32)).astype(np.uint16)) if dt == "bf16" else \
        (lambda a: np.ascontiguousarray(a, np.float32))
    x = inp["x"]
    store(x.transpose(0, 2, 3, 1) if cl else x).tofile(f"{d}/x")
    if not cl:
        store(np.swapaxes(x, 2, 3)).tofile(f"{d}/xT")
    store(inp["dts"]).tofile(f"{d}/dts")
    for k, n in [("A_logs", "A"), ("Bs", "Bm"), ("Cs", "Cm"), ("Ds", "Dv"), ("dt_bias", "bias")]:
        np.ascontiguousarray(inp[k], np.float32).tofile(f"{d}/{n}")
    r = subprocess.run([emulator, str(B), str(D), str(H), str(W), "1" if dt == "bf16" else "0", "1" if cl else "0",
                        d, str(nseg), str(seg_len), "1" if keep else "0"], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    y = np.fromfile(f"{d}/y", np.float32).astype(np.float64)
    ref = orc.forward_core(x, inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"], Cs=inp["Cs"])
    if cl:
        ref = ref.transpose(0, 2, 3, 1)
    assert _rel_err(y, ref.reshape(-1)) <= 2e-3
    if keep:  # the checkpoints the pass that produces y stores for the backward
        ck = np.fromfile(f"{d}/ckpt", np.float32).astype(np.float64)
        assert _rel_err(ck, checkpoints(inp, B, D, H * W, 16).reshape(-1)) <= 2e-3


CKPT_ONLY_CASES = [
    # B, D, H, W, dtype, nseg, seg_len: the backward's checkpoint pass (checkpoints alone)
    (2, 24, 10, 12, "bf16", 1, 120),   # bf16 rows read as they are, a ragged channel tile
    (1, 16, 16, 16, "bf16", 4, 64),    # segmented: first pass, carry, checkpoints from the carried states
    (1, 16, 8, 8, "f32", 1, 64),
]


@pytest.mark.parametrize("case", CKPT_ONLY_CASES)
def test_checkpoint_pass_host_emulation_matches_recurrence(emulator, tmp_path, case):
    B, D, H, W, dt, nseg, seg_len = case
    wl = Workload("emu_ck", B, D, H, W, 16, 0, dt, dt, 70 + B + D + H + W)
    inp = make_inputs(wl)
    d = str(tmp_path)
    store = (lambda a: bf16_bits(np.ascontiguousarray(a, np.float32)).astype(np.uint16)) if dt == "bf16" else \
        (lambda a: np.ascontiguousarray(a, np.float32))
    x = inp["x"]
    store(x).tofile(f"{d}/x")
    store(np.swapaxes(x, 2, 3)).tofile(f"{d}/xT")
    store(inp["dts"]).tofile(f"{d}/dts")
    for k, n in [("A_logs", "A"), ("Bs", "Bm"), ("Cs", "Cm"), ("Ds", "Dv"), ("dt_bias", "bias")]:
        np.ascontiguousarray(inp[k], np.float32).tofile(f"{d}/{n}")
    r = subprocess.run([emulator, str(B), str(D), str(H), str(W), "1" if dt == "bf16" else "0", "0", d, str(nseg),
                        str(seg_len), "2"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    ck = np.fromfile(f"{d}/ckpt", np.float32).astype(np.float64)
    assert _rel_err(ck, checkpoints(inp, B, D, H * W, 16).reshape(-1)) <= 2e-3


@pytest.mark.parametrize("case", [(2, 24, 10, 12), (1, 16, 8, 16)])
def test_mixed_checkpoint_pass_matches_recurrence(emulator, tmp_path, case):
    """bf16 u with fp32 dts: the projection form's backward runs its checkpoint pass on bf16 x
    as it is and the expanded fp32 dts."""
    B, D, H, W = case
    wl = Workload("emu_mx", B, D, H, W, 16, 0, "bf16", "f32", 75 + B + D + H + W)
    inp = make_inputs(wl)
    d = str(tmp_path)
    b16 = lambda a: bf16_bits(np.ascontiguousarray(a, np.float32)).astype(np.uint16)
    x = inp["x"]
    b16(x).tofile(f"{d}/x")
    b16(np.swapaxes(x, 2, 3)).tofile(f"{d}/xT")
    np.ascontiguousarray(inp["dts"], np.float32).tofile(f"{d}/dts")
    for k, n in [("A_logs", "A"), ("Bs", "Bm"), ("Cs", "Cm"), ("Ds", "Dv"), ("dt_bias", "bias")]:
        np.ascontiguousarray(inp[k], np.float32).tofile(f"{d}/{n}")
    r = subprocess.run([emulator, str(B), str(D), str(H), str(W), "2", "0", d, "1", str(H * W), "2"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    ck = np.fromfile(f"{d}/ckpt", np.float32).astype(np.float64)
    assert _rel_err(ck, checkpoints(inp, B, D, H * W, 16).reshape(-1)) <= 2e-3


PAGE_CASES = [
    # B, D, H, W, dtype, channels_last, nseg, seg_len: the page-order merge's plain stores
    (1, 16, 8, 12, "bf16", False, 1, 96),      # channel-first: the four outputs in scan order
    (2, 24, 10, 12, "bf16", False, 1, 120),    # a ragged channel tile, a partial last chunk
    (1, 16, 16, 16, "bf16", False, 4, 64),     # segmented
    (1, 16, 7, 7, "f32", False, 1, 49),        # rows not 16-byte aligned
    (1, 16, 8, 12, "bf16", True, 1, 96),       # channels-last: per-direction copies of y
    (1, 8, 8, 8, "f32", True, 1, 64),
]


@pytest.mark.parametrize("case", PAGE_CASES)
def test_forward_kernel_page_order_outputs_match_oracle(emulator, tmp_path, case):
    """With per-direction output buffers every element is stored once.  Channel-first: the four
    outputs in scan order equal the oracle's selective scan of CrossScan(x), and the page's
    CrossMerge of them its forward core.  Channels-last: ((y0 + y2) + y1) + y3 of the four
    copies equals the forward core."""
    B, D, H, W, dt, cl, nseg, seg_len = case
    wl = Workload("emu_pg", B, D, H, W, 16, 0, dt, dt, 90 + B + D + H + W)
    inp = make_inputs(wl)
    d = str(tmp_path)
    store = (lambda a: bf16_bits(np.ascontiguousarray(a, np.float32)).astype(np.uint16)) if dt == "bf16" else \
        (lambda a: np.ascontiguousarray(a, np.float32))
    x = inp["x"]
    store(x.transpose(0, 2, 3, 1) if cl else x).tofile(f"{d}/x")
    if not cl:
        store(np.swapaxes(x, 2, 3)).tofile(f"{d}/xT")
    store(inp["dts"]).tofile(f"{d}/dts")
    for k, n in [("A_logs", "A"), ("Bs", "Bm"), ("Cs", "Cm"), ("Ds", "Dv"), ("dt_bias", "bias")]:
        np.ascontiguousarray(inp[k], np.float32).tofile(f"{d}/{n}")
    r = subprocess.run([emulator, str(B), str(D), str(H), str(W), "1" if dt == "bf16" else "0", "1" if cl else "0",
                        d, str(nseg), str(seg_len), "0", "0", "1"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    L = H * W
    ref = orc.forward_core(x, inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"], Cs=inp["Cs"])
    if cl:
        parts = [np.fromfile(f"{d}/{n}", np.float32).astype(np.float64) for n in ("y", "yb1", "yb2", "yb3")]
        assert all(np.all(p != -12345.0) for p in parts)  # every element stored
        y = ((parts[0] + parts[2]) + parts[1]) + parts[3]
        assert _rel_err(y, ref.transpose(0, 2, 3, 1).reshape(-1)) <= 2e-3
    else:
        ys = np.fromfile(f"{d}/ys", np.float32).astype(np.float64).reshape(B, 4, D, L)
        assert np.all(ys != -12345.0)
        ys_ref = orc.selective_scan(orc.cross_scan(x).reshape(B, 4 * D, L), inp["dts"].reshape(B, 4 * D, L),
                                    inp["A_logs"], inp["Bs"], inp["Cs"], Dv=inp["Ds"], delta_bias=inp["dt_bias"],
                                    delta_softplus=True)
        assert _rel_err(ys.reshape(-1), ys_ref.reshape(-1)) <= 2e-3
        assert _rel_err(orc.cross_merge(ys, H, W).reshape(-1), ref.reshape(-1)) <= 2e-3


PROJ_CASES = [
    # B, D, H, W, R, channels_last, nseg, seg_len: the projection mode (dt_proj fused in the loop)
    (1, 16, 8, 16, 6, False, 1, 128),
    (2, 24, 10, 12, 4, False, 1, 120),    # a ragged channel tile, a partial last chunk
    (1, 16, 16, 16, 6, False, 4, 64),     # segmented
    (1, 16, 8, 12, 2, True, 1, 96),       # channels-last x and y
]


@pytest.mark.parametrize("case", PROJ_CASES)
def test_forward_kernel_projection_mode_matches_oracle(emulator, tmp_path, case):
    """The kernel's projection mode reads dt_low, B and C rows of x_dbl and computes
    dt = W_dt . dt_low in the loop; x_dbl is the oracle's x_proj of the cross-scanned x."""
    B, D, H, W, R, cl, nseg, seg_len = case
    wl = Workload("emu_p", B, D, H, W, 16, R, "bf16", "bf16", 80 + B + D + H + W + R)
    inp = make_inputs(wl)
    d = str(tmp_path)
    store = lambda a: bf16_bits(np.ascontiguousarray(a, np.float32)).astype(np.uint16)
    x = inp["x"]
    store(x.transpose(0, 2, 3, 1) if cl else x).tofile(f"{d}/x")
    if not cl:
        store(np.swapaxes(x, 2, 3)).tofile(f"{d}/xT")
    xdbl = orc.x_proj(orc.cross_scan(x), inp["x_proj_weight"])
    np.ascontiguousarray(xdbl, np.float32).tofile(f"{d}/xdbl")
    np.ascontiguousarray(inp["dt_projs_weight"], np.float32).tofile(f"{d}/Wdt")
    for k, n in [("A_logs", "A"), ("Ds", "Dv"), ("dt_bias", "bias")]:
        np.ascontiguousarray(inp[k], np.float32).tofile(f"{d}/{n}")
    r = subprocess.run([emulator, str(B), str(D), str(H), str(W), "1", "1" if cl else "0", d, str(nseg),
                        str(seg_len), "0", str(R)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    y = np.fromfile(f"{d}/y", np.float32).astype(np.float64)
    ref = orc.forward_core(x, inp["A_logs"], inp["Ds"], inp["dt_bias"], x_proj_weight=inp["x_proj_weight"],
                           dt_projs_weight=inp["dt_projs_weight"])
    if cl:
        ref = ref.transpose(0, 2, 3, 1)
    assert _rel_err(y, ref.reshape(-1)) <= 5e-3


FULL = os.environ.get("SS2D_EMU_FULL") == "1"


@pytest.mark.skipif(not FULL, reason="one stage-1 image takes about 20 s per case; set SS2D_EMU_FULL=1")
@pytest.mark.parametrize("case", [(1, 192, 56, 56, "bf16", False, 1, 3136, True),
                                  (1, 192, 56, 56, "bf16", True, 1, 3136, False)])
def test_forward_kernel_host_emulation_stage1_image(emulator, tmp_path, case):
    """One image of the stage-1 workload (D = 192, 56x56, bf16) at its full size."""
    test_forward_kernel_host_emulation_matches_oracle(emulator, tmp_path, case)


@pytest.mark.skipif(not FULL, reason="one image of the projection workload takes about 30 s; set SS2D_EMU_FULL=1")
def test_forward_kernel_projection_mode_full_image(emulator, tmp_path):
    """One image of the projection workload (D = 192, 56x56, R = 6) at its full size."""
    test_forward_kernel_projection_mode_matches_oracle(emulator, tmp_path, (1, 192, 56, 56, 6, False, 1, 3136))
