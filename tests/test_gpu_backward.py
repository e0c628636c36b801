"""GPU parity of the backward of the fused core against the fp64 oracle gradient.

ss2d_forward_core_backward (checkpoint pass + reverse-scan kernel) is compared,
gradient by gradient, with oracle.forward_core_bwd on the same seeded inputs
(bf16 tensors hold the values the oracle reads as fp64), using the error measure
of the forward parity tests: max |gpu - oracle| / (|oracle| + 1e-3 * rms(oracle)).
"""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from oracle import oracle as orc
from selective_scan_02_b200.inputs import WORKLOADS, Workload, bf16_bits, make_inputs

pytestmark = pytest.mark.gpu

# The gradients sum many more fp32 terms than the forward (dA_log over every step and
# batch element, dB/dC over a direction's channels), hence the looser limits.
TOL_F32 = 5e-3
TOL_BF16 = 1e-2

GRAD_KEYS = [("dx", "dx"), ("ddts", "ddts"), ("dA_logs", "dA_logs"), ("dBs", "dBs"), ("dCs", "dCs"),
             ("dDs", "dDs"), ("ddt_bias", "ddt_bias")]


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite values in the GPU output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-30)))


def dev(a, dtype="f32"):
    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.float().cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ss.load_library()


def _run(inp, wl, dy):
    t = dict(x=dev(inp["x"], wl.x_dtype), dts=dev(inp["dts"], wl.dt_dtype), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    return {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(dy)).items()}


def _ref(inp, dy):
    return orc.forward_core_bwd(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], inp["dts"], inp["Bs"],
                                inp["Cs"], dy)


BWD_CASES = [
    # B, D, H, W, dtype (x and dts)
    (1, 16, 8, 8, "f32"),      # 4 chunks of 16 steps, one full channel tile
    (2, 24, 8, 12, "bf16"),    # a ragged second tile of 8 channels, H != W
    (1, 16, 4, 4, "bf16"),     # a single chunk
    (1, 8, 5, 4, "f32"),       # a partial last chunk (4 steps), fewer channels than a tile
    (1, 32, 16, 20, "bf16"),   # 20 chunks
    (2, 16, 12, 8, "f32"),
    (1, 16, 1, 16, "bf16"),    # H = 1: the column orders visit the same pixels as the row orders
    (2, 16, 7, 7, "bf16"),     # L = 49 (VMamba-T stage 4): rows staged with 4-byte copies
    (1, 24, 3, 5, "f32"),      # L = 15, a ragged channel tile
]


@pytest.mark.parametrize("case", BWD_CASES)
def test_forward_core_backward_matches_oracle(case):
    B, D, H, W, dt = case
    wl = Workload("bwd", B, D, H, W, 16, 0, dt, dt, 300 + B + D + H + W)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((B, D, H, W)).astype(np.float32)
    got = _run(inp, wl, dy)
    ref = _ref(inp, dy)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    errs = {k: rel_err(got[k], ref[r]) for k, r in GRAD_KEYS}
    assert all(e <= tol for e in errs.values()), errs


def test_forward_core_backward_rejects_unsupported():
    wl = Workload("bwd", 1, 16, 3, 5, 16, 0, "bf16", "f32", 5)  # bf16 x with fp32 dts
    inp = make_inputs(wl)
    t = dict(x=dev(inp["x"], "bf16"), dts=dev(inp["dts"], "f32"), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    with pytest.raises(ss.Ss2dError) as e:
        ss.forward_core_backward(**t, dy=torch.zeros((1, 16, 3, 5), device="cuda"))
    assert e.value.name == "SS2D_ERR_UNSUPPORTED"


def test_forward_core_backward_is_linear_in_dy():
    # the gradient is linear in dy: grad(2 dy1 - dy2) = 2 grad(dy1) - grad(dy2)
    wl = Workload("bwd", 1, 16, 8, 8, 16, 0, "f32", "f32", 11)
    inp = make_inputs(wl)
    rng = np.random.default_rng(12)
    dy1 = rng.standard_normal((1, 16, 8, 8)).astype(np.float32)
    dy2 = rng.standard_normal((1, 16, 8, 8)).astype(np.float32)
    g1, g2 = _run(inp, wl, dy1), _run(inp, wl, dy2)
    g3 = _run(inp, wl, (2 * dy1 - dy2).astype(np.float32))
    for k, _ in GRAD_KEYS:
        comb = 2 * g1[k].astype(np.float64) - g2[k]
        assert rel_err(g3[k], comb) <= 1e-3, k


def test_stage1_backward_sampled():
    # Full stage-1 shapes on two batch elements (the per-image gradients do not mix across
    # the batch; the parameter gradients are the sums over these two images).
    base = WORKLOADS["vmamba_t_stage1"]
    wl = Workload("stage1_b2", 2, base.D, base.H, base.W, base.N, 0, base.x_dtype, base.dt_dtype, base.seed)
    inp = make_inputs(wl)
    dy = np.random.default_rng(99).standard_normal((2, base.D, base.H, base.W)).astype(np.float32)
    got = _run(inp, wl, dy)
    ref = _ref(inp, dy)
    errs = {k: rel_err(got[k], ref[r]) for k, r in GRAD_KEYS}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


# ---- projection form: x_proj (tensor cores) and dt_proj recomputed, their adjoints after the scan's

PROJ_KEYS = [("dx", "dx"), ("dx_proj_weight", "dx_proj_weight"), ("ddt_projs_weight", "ddt_projs_weight"),
             ("dA_logs", "dA_logs"), ("dDs", "dDs"), ("ddt_bias", "ddt_bias"), ("ddts", "ddts"), ("dBs", "dBs"),
             ("dCs", "dCs")]


def _proj_run(inp, dy):
    t = dict(x=dev(inp["x"], "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]),
             x_proj_weight=dev(inp["x_proj_weight"], "bf16"), dt_projs_weight=dev(inp["dt_projs_weight"]))
    return {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(dy)).items()}


def _proj_ref(inp, dy):
    return orc.forward_core_proj_bwd(inp["x"], inp["x_proj_weight"], inp["dt_projs_weight"], inp["A_logs"],
                                     inp["Ds"], inp["dt_bias"], dy)


PROJ_BWD_CASES = [
    # B, D, H, W, R
    (1, 16, 4, 8, 2),      # one x_proj tile, one 8x8 tile of the dx kernel
    (2, 32, 5, 8, 6),      # ragged pixel tiles (H = 5), two images
    (1, 64, 8, 16, 6),     # two 8x8 tiles per x_proj tile, 64 channels
    (1, 80, 12, 8, 16),    # a ragged channel block of the weight-gradient kernels, R = 16 (R + 2N = 48)
]


@pytest.mark.parametrize("case", PROJ_BWD_CASES)
def test_projection_backward_matches_oracle(case):
    B, D, H, W, R = case
    wl = Workload("projbwd", B, D, H, W, 16, R, "bf16", "bf16", 500 + B + D + H + W + R)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 2).standard_normal((B, D, H, W)).astype(np.float32)
    got = _proj_run(inp, dy)
    ref = _proj_ref(inp, dy)
    errs = {k: rel_err(got[k], ref[r]) for k, r in PROJ_KEYS}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


# The other VMamba-T stages and the shapes the tensor-core adjoints of x_proj do not tile:
# x_proj's adjoints then run on the CUDA cores in fp32, and dt_ranks above 16 take the chunked
# dt_proj kernels; at 7x7 the scan's backward stages its rows with 4-byte copies.
PROJ_BWD_STAGE_CASES = [
    (2, 1536, 7, 7, 48),   # stage 4: d_model 768, dt_rank 48, L = 49
    (1, 64, 7, 7, 4),      # 7x7 with a small channel count
    # B, D, H, W, R
    (1, 384, 28, 28, 12),  # stage 2: d_model 192, dt_rank 12 (D > 256, W % 8 != 0)
    (1, 768, 14, 14, 24),  # stage 3: d_model 384, dt_rank 24
    (2, 48, 6, 10, 6),     # W = 10
    (1, 272, 8, 16, 6),    # 272 channels: more than one MMA's N
    (1, 64, 8, 16, 48),    # dt_rank 48: 4 (R + 2N) = 320 rows of x_dbl
]


@pytest.mark.parametrize("case", PROJ_BWD_STAGE_CASES)
def test_projection_backward_other_stages(case):
    B, D, H, W, R = case
    wl = Workload("projbwd_st", B, D, H, W, 16, R, "bf16", "bf16", 800 + B + D + H + W + R)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 2).standard_normal((B, D, H, W)).astype(np.float32)
    got = _proj_run(inp, dy)
    ref = _proj_ref(inp, dy)
    errs = {k: rel_err(got[k], ref[r]) for k, r in PROJ_KEYS}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


def test_projection_backward_without_intermediates():
    # ddts / dBs / dCs are optional in the projection form; the other gradients do not change
    wl = Workload("projbwd", 1, 16, 4, 8, 16, 2, "bf16", "bf16", 77)
    inp = make_inputs(wl)
    dy = np.random.default_rng(78).standard_normal((1, 16, 4, 8)).astype(np.float32)
    t = dict(x=dev(inp["x"], "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]),
             x_proj_weight=dev(inp["x_proj_weight"], "bf16"), dt_projs_weight=dev(inp["dt_projs_weight"]))
    full = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(dy)).items()}
    f32 = dict(dtype=torch.float32, device="cuda")
    grads = dict(dx=torch.empty((1, 16, 4, 8), **f32), dA_logs=torch.empty((64, 16), **f32),
                 dDs=torch.empty(64, **f32), ddt_bias=torch.empty(64, **f32),
                 dx_proj_weight=torch.empty((4, 34, 16), **f32), ddt_projs_weight=torch.empty((4, 16, 2), **f32))
    part = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(dy), grads=grads).items()}
    for k in grads:
        assert rel_err(part[k], full[k]) <= 1e-4, k


def test_projection_backward_full_shapes_two_images():
    # the projection workload's shapes (D = 192, 56x56, R = 6) on two images
    base = WORKLOADS["proj"]
    wl = Workload("proj_b2", 2, base.D, base.H, base.W, base.N, base.R, base.x_dtype, base.dt_dtype, base.seed)
    inp = make_inputs(wl)
    dy = np.random.default_rng(98).standard_normal((2, base.D, base.H, base.W)).astype(np.float32)
    got = _proj_run(inp, dy)
    ref = _proj_ref(inp, dy)
    errs = {k: rel_err(got[k], ref[r]) for k, r in PROJ_KEYS}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


# The additivity holds exactly in real arithmetic.  Both sides are fp32 sums of about 10^5
# products in different orders (per-CTA partial sums, atomics), so entries that cancel to near
# zero differ by fp32 rounding measured against the error floor of 1e-3 * rms.
TOL_ADDITIVE = 5e-3


def _halves_sum_check(run, inp_full, B, keys):
    """Batch additivity at full size: the parameter gradients of the whole batch equal the sums
    of those of its two halves (the per-image terms do not interact)."""
    full = run(inp_full, slice(0, B))
    a = run(inp_full, slice(0, B // 2))
    b = run(inp_full, slice(B // 2, B))
    for k in keys:
        assert rel_err(full[k], a[k].astype(np.float64) + b[k]) <= TOL_ADDITIVE, k
    return full


def test_stage1_backward_full_batch_sampled():
    # the bench's call: the whole stage-1 batch (B = 32); dx of two images against the oracle,
    # which computes them image by image, and the parameter gradients by batch additivity
    wl = WORKLOADS["vmamba_t_stage1"]
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((wl.B, wl.D, wl.H, wl.W)).astype(np.float32)

    def run(inp, sl):
        t = dict(x=dev(inp["x"][sl], wl.x_dtype), dts=dev(inp["dts"][sl], wl.dt_dtype), Bs=dev(inp["Bs"][sl]),
                 Cs=dev(inp["Cs"][sl]), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
        return {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(dy[sl])).items()}

    full = _halves_sum_check(run, inp, wl.B, ["dA_logs", "dDs", "ddt_bias"])
    for b in (0, wl.B - 1):
        one = slice(b, b + 1)
        ref = orc.forward_core_bwd(inp["x"][one], inp["A_logs"], inp["Ds"], inp["dt_bias"], inp["dts"][one],
                                   inp["Bs"][one], inp["Cs"][one], dy[one])
        for k in ("dx", "ddts", "dBs", "dCs"):
            assert rel_err(full[k][one], ref[k]) <= TOL_BF16, (b, k)


def test_projection_backward_full_batch_sampled():
    # the bench's call on the projection workload (B = 64): dx and the intermediates' gradients
    # of two images against the oracle, the weight gradients by batch additivity
    wl = WORKLOADS["proj"]
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((wl.B, wl.D, wl.H, wl.W)).astype(np.float32)

    def run(inp, sl):
        t = dict(x=dev(inp["x"][sl], "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]),
                 dt_bias=dev(inp["dt_bias"]), x_proj_weight=dev(inp["x_proj_weight"], "bf16"),
                 dt_projs_weight=dev(inp["dt_projs_weight"]))
        return {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(dy[sl])).items()}

    full = _halves_sum_check(run, inp, wl.B, ["dx_proj_weight", "ddt_projs_weight", "dA_logs", "dDs", "ddt_bias"])
    for b in (0, wl.B - 1):
        one = slice(b, b + 1)
        ref = orc.forward_core_proj_bwd(inp["x"][one], inp["x_proj_weight"], inp["dt_projs_weight"], inp["A_logs"],
                                        inp["Ds"], inp["dt_bias"], dy[one])
        for k in ("dx", "ddts", "dBs", "dCs"):
            assert rel_err(full[k][one], ref[k]) <= TOL_BF16, (b, k)


@pytest.mark.parametrize("case", [(1, 16, 8, 8, "f32"), (2, 32, 6, 8, "bf16"), (1, 16, 7, 7, "bf16")])
def test_backward_channels_last(case):
    # channels-last x, dy and dx (the page's default layout): the same gradients, transposed
    B, D, H, W, dt = case
    wl = Workload("bwd_cl", B, D, H, W, 16, 0, dt, dt, 600 + B + D + H + W)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((B, D, H, W)).astype(np.float32)
    cl = lambda a: np.ascontiguousarray(a.transpose(0, 2, 3, 1))
    t = dict(x=dev(cl(inp["x"]), dt), dts=dev(inp["dts"], dt), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    got = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(cl(dy)), channels_last=True).items()}
    ref = _ref(inp, dy)
    ref["dx"] = cl(ref["dx"])
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    errs = {k: rel_err(got[k], ref[r]) for k, r in GRAD_KEYS}
    assert all(e <= tol for e in errs.values()), errs


def test_projection_backward_channels_last():
    B, D, H, W, R = 2, 32, 5, 8, 6
    wl = Workload("projbwd_cl", B, D, H, W, 16, R, "bf16", "bf16", 611)
    inp = make_inputs(wl)
    dy = np.random.default_rng(612).standard_normal((B, D, H, W)).astype(np.float32)
    cl = lambda a: np.ascontiguousarray(a.transpose(0, 2, 3, 1))
    t = dict(x=dev(cl(inp["x"]), "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]),
             x_proj_weight=dev(inp["x_proj_weight"], "bf16"), dt_projs_weight=dev(inp["dt_projs_weight"]))
    got = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(cl(dy)), channels_last=True).items()}
    ref = _proj_ref(inp, dy)
    ref["dx"] = cl(ref["dx"])
    errs = {k: rel_err(got[k], ref[r]) for k, r in PROJ_KEYS}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


# ---- checkpoints kept by the forward ---------------------------------------------------------

CKPT_CASES = [
    # B, D, H, W, dtype, channels_last, segmented forward
    (2, 24, 8, 12, "bf16", False, False),
    (1, 16, 8, 8, "f32", False, False),
    (2, 32, 6, 8, "bf16", True, False),
    (1, 16, 32, 32, "bf16", False, True),   # one image, L = 1024: the forward runs in 8 segments
]

# Kept against recomputed checkpoints.  Unsegmented, both are the same fp32 sequence of
# operations, so the gradients differ only by atomic ordering.  A segmented forward starts
# each segment from a carried state, P*h + h_end, with P = exp2(a * (sum of delta)); that
# rounds differently from 128 single-step decays, and dC (read straight off the states)
# shows up to about 5e-4 against the 1e-3*rms floor.
TOL_KEPT = 1e-4
TOL_KEPT_SEGMENTED = 2e-3


@pytest.mark.parametrize("case", CKPT_CASES)
def test_forward_checkpoints_feed_the_backward(case):
    B, D, H, W, dt, cl, seg = case
    wl = Workload("ckpt", B, D, H, W, 16, 0, dt, dt, 700 + B + D + H + W)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((B, D, H, W)).astype(np.float32)
    tr = (lambda a: np.ascontiguousarray(a.transpose(0, 2, 3, 1))) if cl else (lambda a: a)
    t = dict(x=dev(tr(inp["x"]), dt), dts=dev(inp["dts"], dt), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    ck = torch.full(ss.checkpoint_shape(t["x"], channels_last=cl), float("nan"), device="cuda")
    y_plain = host(ss.forward_core(**t, channels_last=cl))
    y_kept = host(ss.forward_core(**t, channels_last=cl, ckpt=ck))
    # keeping the checkpoints leaves y as it was, up to the order in which the merge's four fp32
    # atomic additions land (it varies between runs)
    assert rel_err(y_kept, y_plain) <= 1e-5
    assert np.all(np.isfinite(host(ck)))           # every checkpoint written
    g_kept = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(tr(dy)), channels_last=cl,
                                                              ckpt=ck).items()}
    g_own = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(tr(dy)), channels_last=cl).items()}
    ref = _ref(inp, dy)
    ref["dx"] = tr(ref["dx"])
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    for k, r in GRAD_KEYS:
        assert rel_err(g_kept[k], g_own[k]) <= (TOL_KEPT_SEGMENTED if seg else TOL_KEPT), k
        assert rel_err(g_kept[k], ref[r]) <= tol, k



# ---- segmented walk: few images with long sequences ---------------------------------------------

SEG_BWD_CASES = [
    # B, D, H, W, dtype, channels_last -- segments as the library plans them
    (1, 16, 32, 32, "f32", False),    # L = 1024: 8 segments of 128 steps
    (1, 32, 24, 40, "bf16", False),   # L = 960: 6 segments of 160
    (2, 16, 20, 36, "f32", False),    # L = 720: 5 segments, the last one 80 steps
    (1, 16, 32, 32, "bf16", True),    # channels-last
    (4, 192, 32, 32, "f32", False),   # checkpoint pass in 7 segments of 160 steps, the walk in 5 of 224
    (4, 192, 32, 32, "bf16", False),  # bf16 checkpoint pass (read as is) in 8 segments of 128, the walk in 5 of 224
    (2, 64, 20, 30, "bf16", False),   # L = 600 (rows of whole 16-byte pieces): both segmented, bf16 copies widened
]


@pytest.mark.parametrize("case", SEG_BWD_CASES)
def test_segmented_backward_matches_oracle(case):
    B, D, H, W, dt, cl = case
    wl = Workload("bwd_seg", B, D, H, W, 16, 0, dt, dt, 800 + B + D + H + W)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((B, D, H, W)).astype(np.float32)
    tr = (lambda a: np.ascontiguousarray(a.transpose(0, 2, 3, 1))) if cl else (lambda a: a)
    t = dict(x=dev(tr(inp["x"]), dt), dts=dev(inp["dts"], dt), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    got = {k: host(v) for k, v in ss.forward_core_backward(**t, dy=dev(tr(dy)), channels_last=cl).items()}
    ref = _ref(inp, dy)
    ref["dx"] = tr(ref["dx"])
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    errs = {k: rel_err(got[k], ref[r]) for k, r in GRAD_KEYS}
    assert all(e <= tol for e in errs.values()), errs


def test_segmented_projection_backward_matches_oracle():
    B, D, H, W, R = 1, 16, 32, 32, 4
    wl = Workload("projbwd_seg", B, D, H, W, 16, R, "bf16", "bf16", 812)
    inp = make_inputs(wl)
    dy = np.random.default_rng(813).standard_normal((B, D, H, W)).astype(np.float32)
    got = _proj_run(inp, dy)
    ref = _proj_ref(inp, dy)
    errs = {k: rel_err(got[k], ref[r]) for k, r in PROJ_KEYS}
    assert all(e <= TOL_BF16 for e in errs.values()), errs


def test_long_scan_backward_full_size_sampled():
    # the 256x256 workload (B = 2, fp32) in the bench's call, walked in segments; dx and ddts of
    # two channels against the oracle, which computes them from those channels' four sequences
    wl = WORKLOADS["hires_long"]
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((wl.B, wl.D, wl.H, wl.W)).astype(np.float32)
    t = dict(x=dev(inp["x"], wl.x_dtype), dts=dev(inp["dts"], wl.dt_dtype), Bs=dev(inp["Bs"]), Cs=dev(inp["Cs"]),
             A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))
    g = ss.forward_core_backward(**t, dy=dev(dy))
    dx, ddts = host(g["dx"]), host(g["ddts"])
    D = wl.D
    for d in (0, D - 1):
        chans = [k * D + d for k in range(4)]
        ref = orc.forward_core_bwd(inp["x"][:, d:d + 1], inp["A_logs"][chans], inp["Ds"][chans],
                                   inp["dt_bias"][chans], inp["dts"][:, :, d:d + 1], inp["Bs"], inp["Cs"],
                                   dy[:, d:d + 1])
        assert rel_err(dx[:, d:d + 1], ref["dx"]) <= TOL_F32, d
        assert rel_err(ddts[:, :, d:d + 1], ref["ddts"]) <= TOL_F32, d


# ---- state sizes below 16: the kernels run 16 states with inert padded ones -----------------

SMALL_N_CASES = [
    # B, D, H, W, N, dtype
    (1, 16, 8, 8, 4, "f32"),
    (2, 24, 8, 12, 8, "bf16"),
    (1, 8, 4, 8, 1, "f32"),
    (1, 16, 6, 8, 2, "bf16"),
]


@pytest.mark.parametrize("case", SMALL_N_CASES)
def test_backward_small_state_matches_oracle(case):
    B, D, H, W, N, dt = case
    wl = Workload("bwd_n", B, D, H, W, N, 0, dt, dt, 900 + B + D + H + W + N)
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((B, D, H, W)).astype(np.float32)
    got = _run(inp, wl, dy)
    ref = _ref(inp, dy)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    errs = {k: rel_err(got[k], ref[r]) for k, r in GRAD_KEYS}
    assert all(e <= tol for e in errs.values()), errs


def test_tiny_workload_backward():
    # the tiny configuration (N = 4, fp32) in full
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((wl.B, wl.D, wl.H, wl.W)).astype(np.float32)
    got = _run(inp, wl, dy)
    ref = _ref(inp, dy)
    errs = {k: rel_err(got[k], ref[r]) for k, r in GRAD_KEYS}
    assert all(e <= TOL_F32 for e in errs.values()), errs
