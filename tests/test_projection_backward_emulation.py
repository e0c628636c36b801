"""dt_proj's kernels of the projection form's backward run on the host, without a GPU.

dtproj_expand_kernel, dtproj_dgrad_kernel and dtproj_wgrad_kernel (selective_scan_02_b200/
csrc/proj_bwd.cu) are compiled for the CPU with tests/emu/: one std::thread per thread of
each CTA, warp shuffles on a per-warp barrier, __syncthreads on a per-CTA barrier, under
AddressSanitizer and UBSan.  On x_dbl from the oracle's x_proj and a seeded gradient of dts
they must give dt_proj's output (the oracle's dt_proj) and its two adjoints, the transposed
contractions d dt_low[b,k,r,l] = sum_d W_dt[k,d,r] ddts[b,k,d,l] and
dW_dt[k,d,r] = sum_{b,l} ddts[b,k,d,l] dt_low[b,k,r,l].  Cases cover a ragged last block of
steps, a ragged channel tile, both register widths of the weight-gradient kernel (R <= 8 and
R <= 16) and several images per CTA with a ragged last slice.
"""
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as orc
from tests.emu_build import build_emulator
from selective_scan_02_b200.inputs import Workload, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_scan_02_b200", "csrc")


def _rel_err(got, ref):
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-30)))


@pytest.fixture(scope="module")
def emulator(tmp_path_factory):
    d = tmp_path_factory.mktemp("projbwd_emu")
    scan = open(os.path.join(CSRC, "scan.cuh")).read()
    decls = scan[scan.index("enum ScanMode"):scan.index("struct ScanArgs")]
    src = open(os.path.join(CSRC, "proj_bwd.cu")).read()
    body = src[src.index("__device__ __forceinline__ float warp_sum"):src.index("int sm_count()")]
    body = body.replace("extern __shared__ float sw[];", "float *sw = reinterpret_cast<float *>(g_warp->smem);")
    body = body.replace("__shared__ float sw[kDtChunk * kMaxRLarge];",
                        "float *sw = reinterpret_cast<float *>(g_warp->smem);")
    body = body.replace("extern __shared__ __align__(16) float adj_smem[];",
                        "float *adj_smem = reinterpret_cast<float *>(g_warp->smem);")
    body = body.replace("__shared__ float red[kWgTile * RM][kWgThreads / 32];",
                        "auto &red = *reinterpret_cast<float (*)[kWgTile * RM][kWgThreads / 32]>(g_warp->smem);")
    header = '#pragma once\n#include "common_emu.h"\nnamespace ss2d {\n' + decls + body + "}  // namespace ss2d\n"
    return build_emulator(d, header, "projbwd_emu_main.cpp")


@pytest.mark.parametrize("B,D,H,W,R,bpb", [
    (1, 16, 8, 16, 6, 1),     # one block of 128 steps, R <= 8
    (2, 24, 10, 15, 4, 1),    # L = 150: a ragged second block of steps; a ragged channel tile of the weight gradient
    (3, 16, 6, 8, 12, 2),     # R <= 16; two images per CTA, the last slice one image
    (1, 32, 4, 8, 16, 1),     # the largest R the scan fuses
    (2, 16, 6, 8, 24, 1),     # R = 24: the chunked expansion and dt_low gradient, two channels per weight-gradient CTA
    # R = 48: one channel per weight-gradient CTA; two 64-channel weight chunks (64 + 16).  About two
    # minutes under the emulator, so opt-in (SS2D_EMU_FULL=1); the GPU suite runs R = 48 at D = 64
    # and D = 1536
    pytest.param(1, 80, 2, 4, 48, 1, marks=pytest.mark.skipif(os.environ.get("SS2D_EMU_FULL") != "1",
                                                              reason="set SS2D_EMU_FULL=1")),
])
def test_dt_proj_backward_kernels_match_definitions(emulator, tmp_path, B, D, H, W, R, bpb):
    N, L = 16, H * W
    inp = make_inputs(Workload("emu_pb", B, D, H, W, N, R, "bf16", "bf16", 150 + B + D + H + W + R))
    xdbl = orc.x_proj(orc.cross_scan(inp["x"]), inp["x_proj_weight"]).astype(np.float32)
    Wdt = np.ascontiguousarray(inp["dt_projs_weight"], np.float32)
    ddts = np.random.default_rng(R + L).standard_normal((B, 4, D, L)).astype(np.float32)
    d = str(tmp_path)
    xdbl.tofile(f"{d}/xdbl")
    Wdt.tofile(f"{d}/Wdt")
    ddts.tofile(f"{d}/ddts")
    r = subprocess.run([emulator] + [str(v) for v in (B, D, H, W, N, R, bpb)] + [d], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    x64, w64, g64 = xdbl.astype(np.float64), Wdt.astype(np.float64), ddts.astype(np.float64)
    dts = np.fromfile(f"{d}/dts", np.float32).astype(np.float64)
    assert _rel_err(dts, orc.dt_proj(x64, w64, N).reshape(-1)) <= 1e-4  # fp32 sums against fp64
    dtlow = np.fromfile(f"{d}/dtlow", np.float32).astype(np.float64)
    assert _rel_err(dtlow, np.einsum("kdr,bkdl->bkrl", w64, g64).reshape(-1)) <= 1e-4
    dW = np.fromfile(f"{d}/dWdt", np.float32).astype(np.float64)
    assert _rel_err(dW, np.einsum("bkdl,bkrl->kdr", g64, x64[:, :, :R]).reshape(-1)) <= 1e-4


@pytest.mark.parametrize("B,D,H,W,R,ctas", [
    (1, 16, 8, 16, 6, 1),     # two 64-step tiles walked by one CTA per direction
    (2, 24, 10, 14, 4, 3),    # L = 140: a ragged third tile (12 steps); three CTAs, two tiles each
    (3, 16, 6, 8, 12, 2),     # R <= 16 (16 registers per sum); one tile per image, the CTAs uneven
    (1, 32, 4, 8, 16, 1),     # the largest R of the fused kernel
    (2, 256, 4, 8, 6, 5),     # D = 256, every thread a channel; more CTAs than tiles (idle CTAs add zeros)
])
def test_fused_dt_proj_adjoints_match_definitions(emulator, tmp_path, B, D, H, W, R, ctas):
    # dtproj_adj_kernel: d dt_low and dW_dt from one shared-memory copy of each ddts tile
    N, L = 16, H * W
    inp = make_inputs(Workload("emu_pa", B, D, H, W, N, R, "bf16", "bf16", 170 + B + D + H + W + R))
    xdbl = orc.x_proj(orc.cross_scan(inp["x"]), inp["x_proj_weight"]).astype(np.float32)
    Wdt = np.ascontiguousarray(inp["dt_projs_weight"], np.float32)
    ddts = np.random.default_rng(R + L + 1).standard_normal((B, 4, D, L)).astype(np.float32)
    d = str(tmp_path)
    xdbl.tofile(f"{d}/xdbl")
    Wdt.tofile(f"{d}/Wdt")
    ddts.tofile(f"{d}/ddts")
    r = subprocess.run([emulator] + [str(v) for v in (B, D, H, W, N, R, 1)] + [d, str(ctas)], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    x64, w64, g64 = xdbl.astype(np.float64), Wdt.astype(np.float64), ddts.astype(np.float64)
    dtlow = np.fromfile(f"{d}/dtlow", np.float32).astype(np.float64)
    assert _rel_err(dtlow, np.einsum("kdr,bkdl->bkrl", w64, g64).reshape(-1)) <= 1e-4
    dW = np.fromfile(f"{d}/dWdt", np.float32).astype(np.float64)
    assert _rel_err(dW, np.einsum("bkdl,bkrl->kdr", g64, x64[:, :, :R]).reshape(-1)) <= 1e-4
