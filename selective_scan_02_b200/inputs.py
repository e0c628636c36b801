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
