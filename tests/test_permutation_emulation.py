"""The permutation kernels run on the host, against the oracle, without a GPU.

CrossScan, CrossMerge, the plane transposes (fp32 and bf16 on 32x32 tiles), the bf16-pair
transpose on 64x64 tiles and the register-only bf16 transpose of 8x8 blocks, both of which also
zero y (selective_scan_02_b200/csrc/perm.cu)
are compiled for the CPU with tests/emu/: one std::thread per CUDA thread, __syncthreads on a
per-CTA barrier, each CTA's shared tiles in its own buffer, under AddressSanitizer and UBSan,
in the launchers' grids.  Shapes span several tiles with ragged edges.  Results must equal
the oracle's CrossScan and CrossMerge and numpy's transpose bit for bit (integer-valued data
for the merge's sums), and every element of y must be zeroed.
"""
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import oracle as orc
from tests.emu_build import build_emulator
from selective_scan_02_b200.inputs import bf16_bits

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_scan_02_b200", "csrc")


@pytest.fixture(scope="module")
def emulator(tmp_path_factory):
    d = tmp_path_factory.mktemp("perm_emu")
    src = open(os.path.join(CSRC, "perm.cu")).read()
    body = src[src.index("constexpr int kTile"):src.index("// bf16 -> fp32, eight elements per 16-byte load")]
    # the kernels' shared tiles live in the emulated CTA's shared memory
    smem = "g_warp->smem"
    body = re.sub(r"__shared__ (\w+) (\w+)\[(\w+)\]\[([^\]]+)\];",
                  lambda m: f"auto &{m.group(2)} = *reinterpret_cast<{m.group(1)} (*)[{m.group(3)}][{m.group(4)}]>"
                            f"({smem}{' + sizeof(float) * kTile * (kTile + 1)' if m.group(2) == 't3' else ''});",
                  body)
    extra = ("struct alignas(16) uint4 { unsigned x, y, z, w; };\n"
             "inline uint4 make_uint4(unsigned a, unsigned b, unsigned c, unsigned d) { return {a, b, c, d}; }\n")
    header = '#pragma once\n#include "common_emu.h"\n' + extra + 'namespace ss2d {\n' + body + "}  // namespace ss2d\n"
    return build_emulator(d, header, "perm_emu_main.cpp")


def _run(emulator, d, which, B, D, H, W):
    r = subprocess.run([emulator, str(which), str(B), str(D), str(H), str(W), d], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]


SHAPES = [(1, 2, 40, 70), (2, 1, 33, 5), (1, 1, 1, 37)]


@pytest.mark.parametrize("B,D,H,W", SHAPES)
@pytest.mark.parametrize("bf16", [False, True])
def test_cross_scan_and_transpose_kernels_are_exact(emulator, tmp_path, B, D, H, W, bf16):
    x = np.random.default_rng(H * W + D).standard_normal((B, D, H, W)).astype(np.float32)
    d = str(tmp_path)
    if bf16:
        bits = bf16_bits(x).astype(np.uint16)
        x = (bits.astype(np.uint32) << 16).view(np.float32)
        bits.tofile(f"{d}/x")
        read = lambda shape: (np.fromfile(f"{d}/out", np.uint16).astype(np.uint32) << 16).view(np.float32) \
            .reshape(shape)
    else:
        x.tofile(f"{d}/x")
        read = lambda shape: np.fromfile(f"{d}/out", np.float32).reshape(shape)
    _run(emulator, d, 1 if bf16 else 0, B, D, H, W)
    assert np.array_equal(read((B, 4, D, H * W)), orc.cross_scan(x).astype(np.float32))
    _run(emulator, d, 4 if bf16 else 3, B, D, H, W)
    assert np.array_equal(read((B, D, W, H)), np.swapaxes(x, 2, 3))


def test_cross_merge_kernel_is_exact(emulator, tmp_path):
    B, D, H, W = 2, 3, 37, 45
    ys = np.random.default_rng(5).integers(-1000, 1000, size=(B, 4, D, H * W)).astype(np.float32)
    d = str(tmp_path)
    ys.tofile(f"{d}/x")
    _run(emulator, d, 2, B, D, H, W)
    assert np.array_equal(np.fromfile(f"{d}/out", np.float32).reshape(B, D, H, W), orc.cross_merge(ys, H, W))


@pytest.mark.parametrize("B,D,H,W", [(1, 2, 70, 130), (2, 1, 6, 10), (1, 1, 2, 64), (1, 2, 66, 72)])
def test_pair_transpose_kernel_is_exact_and_zeroes_y(emulator, tmp_path, B, D, H, W):
    x = np.random.default_rng(H + W).standard_normal((B, D, H, W)).astype(np.float32)
    bits = bf16_bits(x).astype(np.uint16)
    d = str(tmp_path)
    bits.tofile(f"{d}/x")
    np.full((B, D, H, W), np.nan, np.float32).tofile(f"{d}/y")
    _run(emulator, d, 5, B, D, H, W)
    assert np.array_equal(np.fromfile(f"{d}/out", np.uint16).reshape(B, D, W, H), np.swapaxes(bits, 2, 3))
    assert np.all(np.fromfile(f"{d}/y", np.float32) == 0.0)


@pytest.mark.parametrize("B,D,H,W", [(2, 3, 16, 24), (1, 2, 56, 56), (1, 1, 8, 8), (3, 1, 40, 8)])
def test_block_transpose_kernel_is_exact_and_zeroes_y(emulator, tmp_path, B, D, H, W):
    # bf16 planes with H and W multiples of 8: one 8x8 block per thread, regrouped in registers
    x = np.random.default_rng(7 * H + W).standard_normal((B, D, H, W)).astype(np.float32)
    bits = bf16_bits(x).astype(np.uint16)
    d = str(tmp_path)
    bits.tofile(f"{d}/x")
    np.full((B, D, H, W), np.nan, np.float32).tofile(f"{d}/y")
    _run(emulator, d, 6, B, D, H, W)
    assert np.array_equal(np.fromfile(f"{d}/out", np.uint16).reshape(B, D, W, H), np.swapaxes(bits, 2, 3))
    assert np.all(np.fromfile(f"{d}/y", np.float32) == 0.0)
