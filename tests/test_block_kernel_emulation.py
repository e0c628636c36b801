"""The SS2D block's CUDA-core kernels run on the host, against the block oracle, without a GPU.

dwconv_silu_kernel (the depthwise convolution with its bias and SiLU, written channel-first or
channels-last), norm_gate_kernel (LayerNorm over D gated by SiLU(z), channel-first y) and
norm_gate_cl_kernel (the same on channels-last y) of selective_scan_02_b200/csrc/block.cu
are compiled for the CPU with tests/emu/: one std::thread per CUDA thread, __syncthreads on a
per-CTA barrier, each CTA's shared memory in its own buffer, the launchers' grids, under
AddressSanitizer and UBSan.  The results are compared with oracle/block.py's depthwise_conv,
silu and layer_norm (fp64, rounded to bf16 where the block stores): equal except for rare
one-unit bf16 rounding flips at ties (the kernel computes in fp32).  Shapes span ragged
column, row, channel and pixel tiles, kernel sizes 1/3/5/7, rows whose length is not a
multiple of 4 (the normalisation's scalar loads), both z paths of the channel-first
normalisation (shared-memory tile and global reads) and 1 to 12 channel pairs per lane for the
channels-last one."""
import os
import subprocess

import numpy as np
import pytest

from oracle import block as ob
from tests.emu_build import build_emulator
from selective_scan_02_b200.inputs import bf16_bits, round_bf16

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "selective_scan_02_b200", "csrc", "block.cu")

EXTRA = """
struct alignas(16) uint4 { unsigned x, y, z, w; };
inline uint4 make_uint4(unsigned a, unsigned b, unsigned c, unsigned d) { return {a, b, c, d}; }
inline __nv_bfloat16 __float2bfloat16_rn(float f)
{
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    __nv_bfloat16 b;
    b.v = (uint16_t)(u >> 16);
    return b;
}
inline float __expf(float x) { return expf(x); }
inline uint32_t pack_bf16x2(float lo, float hi)
{
    return (uint32_t)__float2bfloat16_rn(lo).v | ((uint32_t)__float2bfloat16_rn(hi).v << 16);
}
"""


@pytest.fixture(scope="module")
def emulator(tmp_path_factory):
    d = tmp_path_factory.mktemp("block_emu")
    src = open(KERNEL).read()
    body = src[src.index("constexpr int kCvThreads"):src.index("// Host side.")]
    body = body[:body.rindex("// ----")]
    body = body.replace("extern __shared__ __align__(16) unsigned char cv_smem[];",
                        "unsigned char *cv_smem = g_warp->smem;")
    body = body.replace("extern __shared__ float sy[];", "float *sy = reinterpret_cast<float *>(g_warp->smem);")
    assert "__shared__" not in body
    header = '#pragma once\n#include "common_emu.h"\n' + EXTRA + "namespace ss2d {\n" + body + "}  // namespace ss2d\n"
    return build_emulator(d, header, "block_emu_main.cpp")


def _bf16_file(path, a):
    bf16_bits(np.ascontiguousarray(a, np.float32)).tofile(path)


def _read_bf16(path, shape):
    return (np.fromfile(path, np.uint16).astype(np.uint32) << 16).view(np.float32).reshape(shape).astype(np.float64)


def _close_with_flips(got, ref):
    """Equal except for rare one-unit flips of the bf16 rounding (the two sides round from
    values that differ in their last fp32 bits)."""
    diff = got != ref
    assert np.mean(diff) <= 2e-3, np.mean(diff)
    if diff.any():
        ulp = 2.0 ** (np.floor(np.log2(np.abs(ref[diff]) + 1e-30)) - 7)
        assert np.all(np.abs(got[diff] - ref[diff]) <= ulp * 1.0001)


CONV_CASES = [
    (1, 5, 37, 80, 3),    # odd width (scalar stores): two column tiles (32 + 5), a ragged row tile (4 + 1), channel tiles 64 + 16
    (2, 9, 7, 32, 5),     # 5x5 kernel wider than the image is high/wide in places
    (1, 6, 11, 48, 1),    # 1x1 kernel
    (1, 8, 33, 64, 7),    # 7x7 kernel (the shared-memory tap path)
    (2, 7, 40, 80, 3),    # even width: bf16 pairs out; column tiles 32 + 8, channel tiles 64 + 16, rows 4 + 3
    (1, 4, 34, 16, 1),    # even width, 1x1 kernel, a 2-column last tile
]


@pytest.mark.parametrize("channels_last", [False, True])
@pytest.mark.parametrize("B,H,W,D,k", CONV_CASES)
def test_conv_kernel_matches_oracle(emulator, tmp_path, B, H, W, D, k, channels_last):
    rng = np.random.default_rng(B * 1000 + H * 100 + W + D + k)
    xz = round_bf16(rng.standard_normal((B, H, W, 2 * D)).astype(np.float32))
    w = rng.uniform(-1.0 / k, 1.0 / k, (D, k, k)).astype(np.float32)
    bias = rng.uniform(-0.5, 0.5, D).astype(np.float32)
    d = str(tmp_path)
    _bf16_file(f"{d}/xz", xz)
    w.tofile(f"{d}/w")
    bias.tofile(f"{d}/bias")
    which = "3" if channels_last else "0"
    r = subprocess.run([emulator, which, str(B), str(H), str(W), str(D), d, str(k)], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    ref = ob.round_bf16(ob.silu(ob.depthwise_conv(xz[..., :D].astype(np.float64), w, bias)))  # (B, H, W, D)
    if channels_last:
        got = _read_bf16(f"{d}/out", (B, H, W, D))
    else:
        got = _read_bf16(f"{d}/out", (B, D, H, W))
        ref = ref.transpose(0, 3, 1, 2)
    _close_with_flips(got, ref)


@pytest.mark.parametrize("which,B,H,W,D", [
    (1, 2, 5, 9, 48),     # L = 45: a ragged 32-pixel tile, rows not a multiple of 4 (scalar loads)
    (1, 1, 8, 8, 64),     # L = 64: 16-byte loads, two full tiles
    (2, 1, 6, 7, 32),     # z read from global memory (the wide-D path)
])
def test_norm_gate_kernel_matches_oracle(emulator, tmp_path, which, B, H, W, D):
    rng = np.random.default_rng(which * 100 + B + H + W + D)
    L = H * W
    y = (rng.standard_normal((B, D, L)) * 2.0 + 0.3).astype(np.float32)
    xz = round_bf16(rng.standard_normal((B * L, 2 * D)).astype(np.float32))
    gamma = rng.uniform(0.5, 1.5, D).astype(np.float32)
    beta = (rng.standard_normal(D) * 0.1).astype(np.float32)
    d = str(tmp_path)
    y.tofile(f"{d}/y")
    _bf16_file(f"{d}/xz", xz)
    gamma.tofile(f"{d}/gamma")
    beta.tofile(f"{d}/beta")
    r = subprocess.run([emulator, str(which), str(B), str(H), str(W), str(D), d], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    got = _read_bf16(f"{d}/out", (B * L, D))
    yt = y.astype(np.float64).transpose(0, 2, 1).reshape(B * L, D)
    ref = ob.round_bf16(ob.layer_norm(yt, gamma, beta, 1e-5) * ob.silu(xz[:, D:].astype(np.float64)))
    _close_with_flips(got, ref)


@pytest.mark.parametrize("B,H,W,D", [
    (2, 5, 9, 48),     # 24 channel pairs: one register per lane, lanes 24..31 idle; 90 pixels, a ragged CTA
    (1, 8, 8, 192),    # stage-1 channels: 3 pairs per lane
    (1, 3, 7, 208),    # 104 pairs: 4 per lane, the last partly idle
    (1, 2, 3, 768),    # the largest D of the kernel: 12 pairs per lane
])
def test_channels_last_norm_gate_kernel_matches_oracle(emulator, tmp_path, B, H, W, D):
    # norm_gate_cl_kernel: y as (B*H*W, D) rows, warp = pixel
    rng = np.random.default_rng(B * 7 + H + W + D)
    L = H * W
    y = (rng.standard_normal((B * L, D)) * 2.0 - 0.4).astype(np.float32)
    xz = round_bf16(rng.standard_normal((B * L, 2 * D)).astype(np.float32))
    gamma = rng.uniform(0.5, 1.5, D).astype(np.float32)
    beta = (rng.standard_normal(D) * 0.1).astype(np.float32)
    d = str(tmp_path)
    y.tofile(f"{d}/y")
    _bf16_file(f"{d}/xz", xz)
    gamma.tofile(f"{d}/gamma")
    beta.tofile(f"{d}/beta")
    r = subprocess.run([emulator, "4", str(B), str(H), str(W), str(D), d], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    got = _read_bf16(f"{d}/out", (B * L, D))
    ref = ob.round_bf16(ob.layer_norm(y.astype(np.float64), gamma, beta, 1e-5) * ob.silu(xz[:, D:].astype(np.float64)))
    _close_with_flips(got, ref)
