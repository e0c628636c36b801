"""Seeded synthetic inputs for the SS2D forward core.

This module only draws numbers.  It holds none of the arithmetic of the
forward core itself, so that both the CUDA path and the CPU oracle can take
their inputs from it without sharing any of the computation.

Shapes follow the SS2D module of the VMamba article ("Deep dive into the SS2D
module of VMamba", sections 1 and 3): x is (B, D, H, W) channel-first,
dts is (B, 4, D, L), Bs / Cs are (B, 4, N, L), A_logs / Ds / dt_bias are per
channel over the four directions (4*D), with L = H*W.  Parameter draws follow
the same article's initialisation recipes (section 2.1 for the dt bias and the
dt_proj weight, section 2.2 for A_log).

Every workload is seeded with ``numpy.random.default_rng(seed)`` and draws in
a fixed order: x, dt, dt-bias uniform, B, C, x_proj weight, dt_proj weight.
bf16 values are produced by round-to-nearest-even from fp32 and are kept as
fp32 arrays holding exactly representable bf16 values (``bf16_bits`` gives the
raw 16-bit patterns).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

DT_MIN = 1e-3
DT_MAX = 1e-1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic SS2D-core problem.

    name      short identifier
    B, D      batch and inner channels (d_inner = ssm_ratio * d_model)
    H, W      spatial size; L = H * W
    N         state size (d_state)
    R         dt_rank; 0 means dts / Bs / Cs are given directly (no projections)
    x_dtype   'bf16' or 'f32' storage of x (the scan input u)
    dt_dtype  'bf16' or 'f32' storage of dts
    seed      numpy default_rng seed
    """

    name: str
    B: int
    D: int
    H: int
    W: int
    N: int
    R: int
    x_dtype: str
    dt_dtype: str
    seed: int
    description: str = ""

    @property
    def L(self) -> int:
        return self.H * self.W

    @property
    def elements(self) -> int:
        """Scan elements B * 4 * D * L (the throughput unit)."""
        return self.B * 4 * self.D * self.L


# The five synthetic problems: a tiny fp32 case, the VMamba-T stage-1 shape,
# the stage-3 shape (many short sequences), a 256x256 high-resolution scan
# (long sequences) and the full core with the per-direction projections.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 8, 8, 8, 4, 0, "f32", "f32", 0,
                     "tiny SS2D core, fp32, B1 D8 8x8 N4"),
    "vmamba_t_stage1": Workload("vmamba_t_stage1", 32, 192, 56, 56, 16, 0, "bf16", "bf16", 1,
                                "VMamba-T stage-1 scan, B32 D192 56x56 N16, bf16 u/dt, fp32 B/C"),
    "stage3_short": Workload("stage3_short", 32, 768, 14, 14, 16, 0, "bf16", "bf16", 2,
                             "stage-3 shape, B32 D768 14x14 N16, bf16 u/dt, fp32 B/C"),
    "hires_long": Workload("hires_long", 2, 192, 256, 256, 16, 0, "f32", "f32", 3,
                           "high-resolution long scan, B2 D192 256x256 N16, fp32"),
    "proj": Workload("proj", 64, 192, 56, 56, 16, 6, "bf16", "bf16", 4,
                     "full forward core with x_proj/dt_proj, B64 D192 56x56 N16 R6, bf16 x/W_x"),
}
WORKLOAD_ORDER = ["tiny", "vmamba_t_stage1", "stage3_short", "hires_long", "proj"]


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    rounded = (bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return rounded.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of an array of bf16-representable fp32 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def dt_bias_init(rng: np.random.Generator, n: int) -> np.ndarray:
    """dt_proj bias per the article's dt_init: dt ~ logU[dt_min, dt_max], bias = softplus^-1(dt)."""
    dt = np.exp(rng.random(n) * (math.log(DT_MAX) - math.log(DT_MIN)) + math.log(DT_MIN))
    inv_dt = dt + np.log(-np.expm1(-dt))
    return inv_dt.astype(np.float32)


def make_inputs(wl: Workload, with_dts: bool | None = None) -> dict:
    """Draw every input of one workload.

    Returns a dict of contiguous numpy arrays:
      x (B,D,H,W), A_logs (4D,N), Ds (4D), dt_bias (4D) and either
      dts (B,4,D,L), Bs (B,4,N,L), Cs (B,4,N,L)         when wl.R == 0, or
      x_proj_weight (4,R+2N,D), dt_projs_weight (4,D,R) when wl.R > 0.
    All arrays are fp32; bf16-stored tensors hold bf16-representable values.
    """
    rng = np.random.default_rng(wl.seed)
    B, D, H, W, N, R, L = wl.B, wl.D, wl.H, wl.W, wl.N, wl.R, wl.L
    out = {}
    out["x"] = _store(rng.standard_normal((B, D, H, W), dtype=np.float32), wl.x_dtype)
    if with_dts is None:
        with_dts = R == 0
    if with_dts:
        out["dts"] = _store(rng.standard_normal((B, 4, D, L), dtype=np.float32) * np.float32(0.5), wl.dt_dtype)
    out["dt_bias"] = dt_bias_init(rng, 4 * D)
    if R == 0:
        out["Bs"] = rng.standard_normal((B, 4, N, L), dtype=np.float32)
        out["Cs"] = rng.standard_normal((B, 4, N, L), dtype=np.float32)
    else:
        bound = D ** -0.5
        out["x_proj_weight"] = round_bf16(rng.uniform(-bound, bound, (4, R + 2 * N, D)).astype(np.float32))
        dt_std = R ** -0.5
        out["dt_projs_weight"] = rng.uniform(-dt_std, dt_std, (4, D, R)).astype(np.float32)
    # A_log = log(1..N) for every channel of every direction; D = 1.
    out["A_logs"] = np.ascontiguousarray(np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (4 * D, 1)).astype(np.float32))
    out["Ds"] = np.ones(4 * D, dtype=np.float32)
    return out


def random_scan_inputs(seed: int, B: int, C: int, G: int, N: int, L: int,
                       u_dtype: str = "f32", dt_dtype: str = "f32",
                       dt_scale: float = 0.5) -> dict:
    """Inputs for the standalone selective scan on (B, C, L) with G groups of B/C."""
    rng = np.random.default_rng(seed)
    out = {
        "u": _store(rng.standard_normal((B, C, L), dtype=np.float32), u_dtype),
        "delta": _store(rng.standard_normal((B, C, L), dtype=np.float32) * np.float32(dt_scale), dt_dtype),
        "delta_bias": dt_bias_init(rng, C),
        "Bm": rng.standard_normal((B, G, N, L), dtype=np.float32),
        "Cm": rng.standard_normal((B, G, N, L), dtype=np.float32),
        "A_log": np.ascontiguousarray(np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (C, 1)).astype(np.float32)),
        "Dv": rng.standard_normal(C, dtype=np.float32),
    }
    return out


def random_core_inputs(seed: int, B: int, D: int, H: int, W: int, N: int, R: int = 0,
                       x_dtype: str = "f32", dt_dtype: str = "f32") -> dict:
    """Inputs of an ad-hoc forward-core problem (same recipe as the named workloads)."""
    wl = Workload("adhoc", B, D, H, W, N, R, x_dtype, dt_dtype, seed)
    return make_inputs(wl)


@dataclasses.dataclass(frozen=True)
class BlockWorkload:
    """One synthetic problem for the whole SS2D block (input projection, depthwise
    convolution, core, gated output normalisation, output projection).

    d_model   the block's input and output channels; D = d_inner is the core's width
    d_conv    kernel size of the depthwise convolution (odd)
    The rest as in Workload; x is channels last, (B, H, W, d_model), bf16."""

    name: str
    B: int
    H: int
    W: int
    d_model: int
    D: int
    N: int
    R: int
    d_conv: int
    seed: int
    description: str = ""

    @property
    def L(self) -> int:
        return self.H * self.W

    @property
    def elements(self) -> int:
        """Scan elements of the block's core, B * 4 * D * L."""
        return self.B * 4 * self.D * self.L


# The block at the shape of the projection workload: VMamba-T stage 1 (d_model 96,
# ssm_ratio 2, dt_rank ceil(96 / 16) = 6), batch 64.
BLOCK_WORKLOADS = {
    "block_stage1": BlockWorkload("block_stage1", 64, 56, 56, 96, 192, 16, 6, 3, 5,
                                  "SS2D block, B64 56x56 d_model 96 D192 N16 R6 d_conv 3, bf16 x"),
}


def make_block_inputs(wl: BlockWorkload, in_proj_bias: bool = False, out_proj_bias: bool = False) -> dict:
    """Draw every input of one block workload, in this order: x, in_proj weight, conv weight
    and bias, x_proj weight, dt_proj weight, dt bias, out_norm weight and bias, out_proj
    weight, then the optional projection biases.

    Linear and convolution weights are uniform in +-fan_in^-0.5 (fan_in d_model for the
    input projection, D for x_proj and the output projection, d_conv^2 for the depthwise
    kernel, dt_rank for dt_proj); the dt bias and A_log follow make_inputs.  The output
    normalisation's weight is uniform in [0.5, 1.5) and its bias N(0, 0.1^2), so that both
    affine terms matter.  bf16-stored tensors (x and the three projection weights) hold
    bf16-representable fp32 values."""
    rng = np.random.default_rng(wl.seed)
    B, H, W, dm, D, N, R, k = wl.B, wl.H, wl.W, wl.d_model, wl.D, wl.N, wl.R, wl.d_conv
    out = {}
    out["x"] = round_bf16(rng.standard_normal((B, H, W, dm), dtype=np.float32))
    b = dm ** -0.5
    out["in_proj_weight"] = round_bf16(rng.uniform(-b, b, (2 * D, dm)).astype(np.float32))
    b = 1.0 / k
    out["conv_weight"] = rng.uniform(-b, b, (D, k, k)).astype(np.float32)
    out["conv_bias"] = rng.uniform(-b, b, D).astype(np.float32)
    b = D ** -0.5
    out["x_proj_weight"] = round_bf16(rng.uniform(-b, b, (4, R + 2 * N, D)).astype(np.float32))
    b = R ** -0.5
    out["dt_projs_weight"] = rng.uniform(-b, b, (4, D, R)).astype(np.float32)
    out["dt_projs_bias"] = dt_bias_init(rng, 4 * D)
    out["out_norm_weight"] = rng.uniform(0.5, 1.5, D).astype(np.float32)
    out["out_norm_bias"] = (rng.standard_normal(D) * 0.1).astype(np.float32)
    b = D ** -0.5
    out["out_proj_weight"] = round_bf16(rng.uniform(-b, b, (dm, D)).astype(np.float32))
    out["A_logs"] = np.ascontiguousarray(np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (4 * D, 1)).astype(np.float32))
    out["Ds"] = np.ones(4 * D, dtype=np.float32)
    if in_proj_bias:
        out["in_proj_bias"] = rng.uniform(-dm ** -0.5, dm ** -0.5, 2 * D).astype(np.float32)
    if out_proj_bias:
        out["out_proj_bias"] = rng.uniform(-D ** -0.5, D ** -0.5, dm).astype(np.float32)
    return out
