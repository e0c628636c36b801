"""Poisoned buffers: every output element is written, and no workspace byte is read before it
is written.

Each entry point runs with its outputs and its workspace filled with NaN first (all-ones bytes,
a NaN in fp32 and in bf16).  An output element the kernels never write, or a workspace value
read before the call wrote it, then shows as a NaN, or as a value off the oracle; the results
must be finite and match the fp64 oracle within the usual limits.  Small shapes that still
span several tiles, a ragged tail, the segmented walks and the padded small-N backward.
"""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from oracle import oracle as orc
from selective_scan_02_b200.inputs import Workload, bf16_bits, make_inputs, random_scan_inputs

pytestmark = pytest.mark.gpu

TOL_FWD_F32, TOL_FWD_BF16 = 2e-3, 5e-3
TOL_BWD_F32, TOL_BWD_BF16 = 5e-3, 1e-2


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "an output element was not written, or a NaN was read"
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-30)))


def dev(a, dtype="f32"):
    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.float().cpu().numpy()


def nan_like(shape, dtype=torch.float32):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


def poisoned_workspace(nbytes):
    return torch.full((max(nbytes, 16),), 0xFF, dtype=torch.uint8, device="cuda")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ss.load_library()


def test_permutations_write_every_element():
    rng = np.random.default_rng(3)
    x = rng.integers(-1000, 1000, size=(2, 5, 7, 9)).astype(np.float32)
    xs = ss.cross_scan(dev(x), xs=nan_like((2, 4, 5, 63)))
    assert np.array_equal(host(xs), orc.cross_scan(x))
    ys = rng.integers(-1000, 1000, size=(2, 4, 5, 63)).astype(np.float32)
    y = ss.cross_merge(dev(ys), 7, 9, y=nan_like((2, 5, 7, 9)))
    assert np.array_equal(host(y), orc.cross_merge(ys, 7, 9))


@pytest.mark.parametrize("N,L,dt", [(16, 100, "bf16"), (16, 37, "f32"), (4, 129, "f32"), (8, 33, "bf16")])
def test_standalone_scan_writes_every_element(N, L, dt):
    B, C, G = 2, 24, 2
    inp = random_scan_inputs(11 + N + L, B, C, G, N, L, dt, dt)
    t = dict(u=dev(inp["u"], dt), delta=dev(inp["delta"], dt), A_log=dev(inp["A_log"]), Bm=dev(inp["Bm"]),
             Cm=dev(inp["Cm"]), Dv=dev(inp["Dv"]), delta_bias=dev(inp["delta_bias"]))
    ref, h_ref = orc.selective_scan(inp["u"], inp["delta"], inp["A_log"], inp["Bm"], inp["Cm"], inp["Dv"],
                                    inp["delta_bias"], return_last_state=True)
    tol = TOL_FWD_BF16 if dt == "bf16" else TOL_FWD_F32
    y = ss.selective_scan(**t, y=nan_like((B, C, L)))
    assert rel_err(host(y), ref) <= tol
    y, h = ss.selective_scan(**t, y=nan_like((B, C, L)), return_last_state=True)
    assert rel_err(host(y), ref) <= tol
    assert rel_err(host(h), h_ref) <= tol


CORE_CASES = [
    # B, D, H, W, dtype, channels_last, bf16 y
    (2, 24, 10, 12, "bf16", False, False),   # a ragged channel tile, a partial last chunk
    (1, 16, 32, 32, "f32", False, False),    # segmented (few channels, a long sequence)
    (1, 16, 30, 24, "bf16", False, True),    # segmented with a partial last segment, bf16 y
    (2, 32, 8, 12, "bf16", True, False),     # channels-last x and y
    (1, 32, 32, 32, "f32", True, True),      # channels-last, segmented, bf16 y
]


@pytest.mark.parametrize("case", CORE_CASES)
def test_forward_core_with_poisoned_workspace(case):
    B, D, H, W, dt, cl, ybf = case
    inp = make_inputs(Workload("poison", B, D, H, W, 16, 0, dt, dt, 500 + B + D + H + W))
    ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"],
                           Cs=inp["Cs"])
    x = inp["x"].transpose(0, 2, 3, 1) if cl else inp["x"]
    if cl:
        ref = ref.transpose(0, 2, 3, 1)
    t = dict(x=dev(np.ascontiguousarray(x), dt), dts=dev(inp["dts"], dt), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    ydt = torch.bfloat16 if ybf else torch.float32
    ws = poisoned_workspace(ss.forward_core_workspace_size(**t, channels_last=cl, out_dtype=ydt))
    ck = nan_like(ss.checkpoint_shape(t["x"], channels_last=cl))
    y = ss.forward_core(**t, channels_last=cl, y=nan_like(x.shape, ydt), workspace=ws, ckpt=ck)
    tol = 1e-2 if ybf else (TOL_FWD_BF16 if dt == "bf16" else TOL_FWD_F32)
    assert rel_err(host(y), ref) <= tol
    assert torch.isfinite(ck).all()


@pytest.mark.parametrize("case", [(2, 32, 9, 16, 6, False), (1, 32, 32, 32, 6, False), (2, 32, 8, 16, 4, True)])
def test_forward_core_projections_with_poisoned_workspace(case):
    B, D, H, W, R, cl = case
    inp = make_inputs(Workload("poison_p", B, D, H, W, 16, R, "bf16", "bf16", 520 + B + D + H + W + R))
    ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], x_proj_weight=inp["x_proj_weight"],
                           dt_projs_weight=inp["dt_projs_weight"])
    x = inp["x"].transpose(0, 2, 3, 1) if cl else inp["x"]
    if cl:
        ref = ref.transpose(0, 2, 3, 1)
    t = dict(x=dev(np.ascontiguousarray(x), "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]),
             dt_bias=dev(inp["dt_bias"]), x_proj_weight=dev(inp["x_proj_weight"], "bf16"),
             dt_projs_weight=dev(inp["dt_projs_weight"]))
    ws = poisoned_workspace(ss.forward_core_workspace_size(**t, channels_last=cl))
    y = ss.forward_core(**t, channels_last=cl, y=nan_like(x.shape), workspace=ws)
    assert rel_err(host(y), ref) <= TOL_FWD_BF16
    ss.check_device_status(**t, channels_last=cl, workspace=ws)


def _nan_grads(B, D, H, W, N, R, cl):
    L = H * W
    g = dict(dx=nan_like((B, H, W, D) if cl else (B, D, H, W)), ddts=nan_like((B, 4, D, L)),
             dA_logs=nan_like((4 * D, N)), dBs=nan_like((B, 4, N, L)), dCs=nan_like((B, 4, N, L)),
             dDs=nan_like((4 * D,)), ddt_bias=nan_like((4 * D,)))
    if R:
        g["dx_proj_weight"] = nan_like((4, R + 2 * N, D))
        g["ddt_projs_weight"] = nan_like((4, D, R))
    return g


BWD_CASES = [
    # B, D, H, W, N, dtype, channels_last
    (2, 24, 8, 12, 16, "bf16", False),   # a ragged channel tile
    (1, 16, 32, 32, 16, "f32", False),   # segmented walk
    (1, 16, 30, 24, 16, "bf16", False),  # segmented, a partial last segment
    (2, 16, 8, 8, 4, "f32", False),      # N = 4, padded to 16 states
    (2, 32, 8, 12, 16, "bf16", True),    # channels-last x, dy and dx
]


@pytest.mark.parametrize("case", BWD_CASES)
def test_backward_with_poisoned_outputs_and_workspace(case):
    B, D, H, W, N, dt, cl = case
    inp = make_inputs(Workload("poison_b", B, D, H, W, N, 0, dt, dt, 540 + B + D + H + W + N))
    dy = np.random.default_rng(7).standard_normal((B, D, H, W)).astype(np.float32)
    ref = orc.forward_core_bwd(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], inp["dts"], inp["Bs"],
                               inp["Cs"], dy)
    x, dyl = (inp["x"].transpose(0, 2, 3, 1), dy.transpose(0, 2, 3, 1)) if cl else (inp["x"], dy)
    t = dict(x=dev(np.ascontiguousarray(x), dt), dts=dev(inp["dts"], dt), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    ws = poisoned_workspace(ss.forward_core_backward_workspace_size(**t, channels_last=cl))
    g = ss.forward_core_backward(**t, dy=dev(np.ascontiguousarray(dyl)), grads=_nan_grads(B, D, H, W, N, 0, cl),
                                 workspace=ws, channels_last=cl)
    tol = TOL_BWD_BF16 if dt == "bf16" else TOL_BWD_F32
    for k in ("dx", "ddts", "dA_logs", "dBs", "dCs", "dDs", "ddt_bias"):
        r = ref[k].transpose(0, 2, 3, 1) if (cl and k == "dx") else ref[k]
        assert rel_err(host(g[k]), r) <= tol, k


@pytest.mark.parametrize("case", [(2, 32, 8, 16, 6, False), (1, 32, 32, 32, 6, False), (2, 32, 8, 16, 4, True)])
def test_projection_backward_with_poisoned_outputs_and_workspace(case):
    B, D, H, W, R, cl = case
    N = 16
    inp = make_inputs(Workload("poison_pb", B, D, H, W, N, R, "bf16", "bf16", 560 + B + D + H + W + R))
    dy = np.random.default_rng(8).standard_normal((B, D, H, W)).astype(np.float32)
    ref = orc.forward_core_proj_bwd(inp["x"], inp["x_proj_weight"], inp["dt_projs_weight"], inp["A_logs"],
                                    inp["Ds"], inp["dt_bias"], dy)
    x, dyl = (inp["x"].transpose(0, 2, 3, 1), dy.transpose(0, 2, 3, 1)) if cl else (inp["x"], dy)
    t = dict(x=dev(np.ascontiguousarray(x), "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]),
             dt_bias=dev(inp["dt_bias"]), x_proj_weight=dev(inp["x_proj_weight"], "bf16"),
             dt_projs_weight=dev(inp["dt_projs_weight"]))
    ws = poisoned_workspace(ss.forward_core_backward_workspace_size(**t, channels_last=cl))
    g = ss.forward_core_backward(**t, dy=dev(np.ascontiguousarray(dyl)), grads=_nan_grads(B, D, H, W, N, R, cl),
                                 workspace=ws, channels_last=cl)
    ss.check_device_status(**t, channels_last=cl, workspace=ws, backward=True)
    for k in ("dx", "dx_proj_weight", "ddt_projs_weight", "dA_logs", "dDs", "ddt_bias", "ddts", "dBs", "dCs"):
        r = ref[k].transpose(0, 2, 3, 1) if (cl and k == "dx") else ref[k]
        assert rel_err(host(g[k]), r) <= TOL_BWD_BF16, k
