"""GPU parity: the CUDA path of libss2d against the fp64 CPU oracle.

Every comparison feeds both sides the same seeded inputs (bf16 tensors hold
the same values the oracle reads as fp64).  Error measure: max over elements
of |gpu - oracle| / (|oracle| + 1e-3 * rms(oracle)); limits 2e-3 for fp32
u/delta and 5e-3 with bf16 u/delta.  Permutations are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from oracle import oracle as orc
from selective_scan_02_b200.inputs import WORKLOADS, bf16_bits, make_inputs, random_scan_inputs

pytestmark = pytest.mark.gpu

TOL_F32 = 2e-3
TOL_BF16 = 5e-3


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite values in the GPU output"
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    den = np.abs(ref) + 1e-3 * rms + 1e-30
    return float(np.max(np.abs(got - ref) / den)) if ref.size else 0.0


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


# ----------------------------------------------------------------------------
# CrossScan / CrossMerge
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(2, 3, 5, 7), (1, 8, 8, 8), (2, 5, 33, 65), (1, 2, 1, 9), (1, 2, 70, 1)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_cross_scan_bit_exact(shape, dtype):
    rng = np.random.default_rng(sum(shape))
    x = rng.standard_normal(shape, dtype=np.float32)
    if dtype == "bf16":
        from selective_scan_02_b200.inputs import round_bf16
        x = round_bf16(x)
    xs = host(ss.cross_scan(dev(x, dtype)))
    np.testing.assert_array_equal(xs.astype(np.float64), orc.cross_scan(x))


@pytest.mark.parametrize("shape", [(2, 3, 5, 7), (2, 4, 33, 40), (1, 1, 1, 1)])
def test_cross_merge_integer_exact_and_float(shape):
    B, D, H, W = shape
    rng = np.random.default_rng(B * D + H * W)
    ys_int = rng.integers(-1000, 1000, (B, 4, D, H * W)).astype(np.float32)
    y = host(ss.cross_merge(dev(ys_int), H, W))
    np.testing.assert_array_equal(y.astype(np.float64), orc.cross_merge(ys_int, H, W))
    ys = rng.standard_normal((B, 4, D, H * W), dtype=np.float32)
    y = host(ss.cross_merge(dev(ys), H, W))
    np.testing.assert_allclose(y, orc.cross_merge(ys, H, W), rtol=1e-6, atol=1e-6)


# ----------------------------------------------------------------------------
# Standalone selective scan
# ----------------------------------------------------------------------------

SCAN_CASES = [
    # B, C, G, N, L, u_dtype, dt_dtype, softplus, with_D, with_bias
    (1, 8, 1, 4, 64, "f32", "f32", True, True, True),
    (2, 8, 2, 16, 37, "f32", "f32", True, True, True),
    (2, 40, 2, 16, 100, "bf16", "bf16", True, True, True),
    (1, 64, 4, 16, 196, "bf16", "f32", True, False, True),
    (2, 24, 3, 8, 70, "f32", "bf16", False, True, False),
    (1, 96, 1, 4, 33, "f32", "f32", True, True, True),
    (2, 12, 2, 2, 45, "f32", "f32", True, True, True),
    (1, 70, 1, 1, 129, "f32", "f32", True, True, True),
    (3, 4, 4, 16, 1, "f32", "f32", True, True, True),
    (1, 130, 2, 16, 300, "f32", "f32", True, True, True),
]


@pytest.mark.parametrize("case", SCAN_CASES)
def test_selective_scan_matches_oracle(case):
    B, C, G, N, L, ud, dd, sp, with_D, with_bias = case
    inp = random_scan_inputs(1000 + B * 7 + C + N + L, B, C, G, N, L, ud, dd)
    Dv = inp["Dv"] if with_D else None
    bias = inp["delta_bias"] if with_bias else None
    delta = inp["delta"] if sp else np.abs(inp["delta"]) + np.float32(0.05)
    if not sp and dd == "bf16":
        from selective_scan_02_b200.inputs import round_bf16
        delta = round_bf16(delta)
    y = ss.selective_scan(dev(inp["u"], ud), dev(delta, dd), dev(inp["A_log"]), dev(inp["Bm"]), dev(inp["Cm"]),
                          dev(Dv) if Dv is not None else None, dev(bias) if bias is not None else None, sp)
    ref = orc.selective_scan(inp["u"], delta, inp["A_log"], inp["Bm"], inp["Cm"], Dv, bias, sp)
    tol = TOL_BF16 if "bf16" in (ud, dd) else TOL_F32
    assert rel_err(host(y), ref) <= tol


def test_selective_scan_is_deterministic():
    inp = random_scan_inputs(5, 2, 64, 2, 16, 300, "bf16", "bf16")
    args = [dev(inp["u"], "bf16"), dev(inp["delta"], "bf16"), dev(inp["A_log"]), dev(inp["Bm"]), dev(inp["Cm"]),
            dev(inp["Dv"]), dev(inp["delta_bias"]), True]
    a = host(ss.selective_scan(*args))
    b = host(ss.selective_scan(*args))
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("N", [1, 16])
def test_softplus_accuracy_over_its_domain(N):
    # A_log = -30 (A ~ -1e-13, so every decay is 1 in fp32), u = 1, B = 1, C = 1/N, D = 0, L = 1:
    # the scan's only output is delta = softplus(z), here for z spread over [-15, 15], once per
    # channel.  Both branches of the kernels' log1p (series below e^-|z| = 1/8, hardware log2
    # above) and the hardware exp2 are compared with the fp64 oracle, element by element.
    C = 4096
    z = np.linspace(-15.0, 15.0, C).astype(np.float32).reshape(1, C, 1)
    u = np.ones((1, C, 1), dtype=np.float32)
    A_log = np.full((C, N), -30.0, dtype=np.float32)
    Bm = np.ones((1, 1, N, 1), dtype=np.float32)
    Cm = np.full((1, 1, N, 1), 1.0 / N, dtype=np.float32)
    y = host(ss.selective_scan(dev(u), dev(z), dev(A_log), dev(Bm), dev(Cm), None, None, True))
    ref = orc.selective_scan(u, z, A_log, Bm, Cm, None, None, True)
    rel = np.abs(y.astype(np.float64) - ref) / np.abs(ref)
    assert float(rel.max()) <= 3e-6, (float(rel.max()), float(z.reshape(-1)[int(rel.argmax())]))


STATE_CASES = [
    # B, C, G, N, L, dtype: both kernels (N = 16 and N < 16), ragged L (padding steps past the end)
    (2, 40, 2, 16, 100, "bf16"),
    (1, 16, 1, 16, 37, "f32"),
    (2, 24, 3, 8, 70, "f32"),
    (1, 32, 2, 4, 33, "bf16"),
    (1, 16, 1, 16, 3, "f32"),
    (2, 130, 2, 16, 321, "f32"),
]


@pytest.mark.parametrize("case", STATE_CASES)
def test_selective_scan_state_passing_matches_oracle(case):
    B, C, G, N, L, dt = case
    inp = random_scan_inputs(2000 + B + C + N + L, B, C, G, N, L, dt, dt)
    h0 = np.random.default_rng(L).standard_normal((B, C, N)).astype(np.float32)
    args = [dev(inp["u"], dt), dev(inp["delta"], dt), dev(inp["A_log"]), dev(inp["Bm"]), dev(inp["Cm"]),
            dev(inp["Dv"]), dev(inp["delta_bias"]), True]
    y, h_last = ss.selective_scan(*args, h0=dev(h0), return_last_state=True)
    ref_y, ref_h = orc.selective_scan(inp["u"], inp["delta"], inp["A_log"], inp["Bm"], inp["Cm"], inp["Dv"],
                                      inp["delta_bias"], True, h0=h0, return_last_state=True)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    assert rel_err(host(y), ref_y) <= tol
    assert rel_err(host(h_last), ref_h) <= tol
    # zero initial state with the final state returned
    y0, h0_last = ss.selective_scan(*args, return_last_state=True)
    r0_y, r0_h = orc.selective_scan(inp["u"], inp["delta"], inp["A_log"], inp["Bm"], inp["Cm"], inp["Dv"],
                                    inp["delta_bias"], True, return_last_state=True)
    assert rel_err(host(y0), r0_y) <= tol and rel_err(host(h0_last), r0_h) <= tol


@pytest.mark.parametrize("N,split", [(16, 61), (16, 96), (8, 50)])
def test_selective_scan_in_two_pieces_equals_whole(N, split):
    # scanning [0, m) and then [m, L) from the first piece's final state gives the scan of [0, L)
    B, C, G, L = 2, 32, 2, 160
    inp = random_scan_inputs(77 + N + split, B, C, G, N, L, "f32", "f32")
    whole_y, whole_h = ss.selective_scan(dev(inp["u"]), dev(inp["delta"]), dev(inp["A_log"]), dev(inp["Bm"]),
                                         dev(inp["Cm"]), dev(inp["Dv"]), dev(inp["delta_bias"]), True,
                                         return_last_state=True)
    parts, h = [], None
    for lo, hi in ((0, split), (split, L)):
        cut = lambda a: np.ascontiguousarray(a[..., lo:hi])
        y, h = ss.selective_scan(dev(cut(inp["u"])), dev(cut(inp["delta"])), dev(inp["A_log"]), dev(cut(inp["Bm"])),
                                 dev(cut(inp["Cm"])), dev(inp["Dv"]), dev(inp["delta_bias"]), True, h0=h,
                                 return_last_state=True)
        parts.append(host(y))
    assert rel_err(np.concatenate(parts, axis=-1), host(whole_y)) <= 1e-4
    assert rel_err(host(h), host(whole_h)) <= 1e-4


# ----------------------------------------------------------------------------
# Fused forward core
# ----------------------------------------------------------------------------

def _core_dev(inp, wl):
    return dict(x=dev(inp["x"], wl.x_dtype), dts=dev(inp["dts"], wl.dt_dtype), Bs=dev(inp["Bs"]),
                Cs=dev(inp["Cs"]), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]))


def _core_ref(inp):
    return orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"],
                            Cs=inp["Cs"])


CORE_CASES = [
    # B, D, H, W, N, x_dtype, dt_dtype
    (1, 8, 8, 8, 4, "f32", "f32"),
    (2, 8, 5, 7, 16, "f32", "f32"),
    (2, 40, 9, 6, 16, "bf16", "bf16"),
    (1, 33, 14, 14, 16, "bf16", "bf16"),
    (1, 16, 1, 13, 8, "f32", "f32"),
    (2, 5, 11, 1, 16, "f32", "f32"),
    (1, 64, 12, 20, 16, "bf16", "bf16"),
    # few channels and long sequences: run as a segmented scan (first pass, carry, second pass)
    (1, 16, 64, 64, 16, "f32", "f32"),
    (1, 24, 48, 40, 16, "bf16", "bf16"),
    (2, 8, 33, 31, 16, "f32", "f32"),
]


@pytest.mark.parametrize("case", CORE_CASES)
def test_forward_core_matches_oracle(case):
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N, xd, dd = case
    wl = Workload("case", B, D, H, W, N, 0, xd, dd, 77 + B + D + H + W + N)
    inp = make_inputs(wl)
    y = ss.forward_core(**_core_dev(inp, wl))
    tol = TOL_BF16 if "bf16" in (xd, dd) else TOL_F32
    assert rel_err(host(y), _core_ref(inp)) <= tol


CL_CASES = [
    # B, D, H, W, dtype (x and dts): channels-last x and y, (B, H, W, D)
    (2, 24, 9, 6, "bf16"),
    (1, 16, 8, 8, "f32"),
    (2, 40, 14, 14, "bf16"),
    (1, 8, 33, 31, "f32"),
    (1, 16, 64, 64, "f32"),     # long sequences, few channels: segmented scan
    (1, 24, 48, 40, "bf16"),    # segmented, ragged channel tile
]


@pytest.mark.parametrize("case", CL_CASES)
def test_forward_core_channels_last_matches_oracle(case):
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, dt = case
    wl = Workload("cl", B, D, H, W, 16, 0, dt, dt, 500 + B + D + H + W)
    inp = make_inputs(wl)
    t = _core_dev(inp, wl)
    t["x"] = dev(np.ascontiguousarray(inp["x"].transpose(0, 2, 3, 1)), dt)   # (B, H, W, D)
    y = ss.forward_core(**t, channels_last=True)
    assert tuple(y.shape) == (B, H, W, D)
    ref = _core_ref(inp).transpose(0, 2, 3, 1)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    assert rel_err(host(y), ref) <= tol


@pytest.mark.parametrize("channels_last", [False, True])
def test_forward_core_bf16_output(channels_last):
    # y in bf16: the fp32 core rounded to nearest even, so within the bf16 tolerance plus one
    # bf16 rounding (2^-8 relative) of the oracle
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W = 2, 24, 12, 10
    wl = Workload("ybf16", B, D, H, W, 16, 0, "bf16", "bf16", 9)
    inp = make_inputs(wl)
    t = _core_dev(inp, wl)
    ref = _core_ref(inp)
    if channels_last:
        t["x"] = dev(np.ascontiguousarray(inp["x"].transpose(0, 2, 3, 1)), "bf16")
        ref = ref.transpose(0, 2, 3, 1)
    y = ss.forward_core(**t, channels_last=channels_last, out_dtype=torch.bfloat16)
    assert y.dtype == torch.bfloat16
    y32 = ss.forward_core(**t, channels_last=channels_last)
    # the same fp32 sum rounded once (atomic order may move the sum's last bit: at most one bf16 step)
    np.testing.assert_allclose(host(y), host(y32.to(torch.bfloat16)), rtol=2.0 ** -7, atol=0)
    assert rel_err(host(y), ref) <= TOL_BF16 + 2.0 ** -8


def test_forward_core_tiny_workload():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl)
    y = ss.forward_core(**_core_dev(inp, wl))
    assert rel_err(host(y), _core_ref(inp)) <= TOL_F32


def test_forward_core_identity_scan_is_four_x():
    """C = 0 and D = 1 make the scan the identity: the fused core and the unfused
    chain CrossScan -> scan -> CrossMerge both return exactly 4x (integer x)."""
    rng = np.random.default_rng(21)
    B, D, H, W, N = 2, 36, 10, 13, 16
    from selective_scan_02_b200.inputs import Workload
    wl = Workload("id", B, D, H, W, N, 0, "f32", "f32", 21)
    inp = make_inputs(wl)
    inp["x"] = rng.integers(-300, 300, (B, D, H, W)).astype(np.float32)
    inp["Cs"][:] = 0.0
    inp["Ds"][:] = 1.0
    y = host(ss.forward_core(**_core_dev(inp, wl)))
    np.testing.assert_array_equal(y, 4 * inp["x"])
    t = _core_dev(inp, wl)
    xs = ss.cross_scan(t["x"])
    ys = ss.selective_scan(xs.view(B, 4 * D, H * W), t["dts"].view(B, 4 * D, H * W), t["A_logs"], t["Bs"], t["Cs"],
                           t["Ds"], t["dt_bias"], True)
    y2 = host(ss.cross_merge(ys.view(B, 4, D, H * W), H, W))
    np.testing.assert_array_equal(y2, 4 * inp["x"])


def test_unfused_chain_matches_fused_core():
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N = 2, 48, 12, 9, 16
    wl = Workload("chain", B, D, H, W, N, 0, "bf16", "bf16", 31)
    inp = make_inputs(wl)
    t = _core_dev(inp, wl)
    fused = host(ss.forward_core(**t))
    xs = ss.cross_scan(t["x"])
    ys = ss.selective_scan(xs.view(B, 4 * D, H * W), t["dts"].view(B, 4 * D, H * W), t["A_logs"], t["Bs"], t["Cs"],
                           t["Ds"], t["dt_bias"], True)
    chain = host(ss.cross_merge(ys.view(B, 4, D, H * W), H, W))
    ref = _core_ref(inp)
    assert rel_err(chain, ref) <= TOL_BF16
    assert rel_err(fused, ref) <= TOL_BF16
    np.testing.assert_allclose(fused, chain, rtol=1e-5, atol=1e-5 * float(np.sqrt(np.mean(ref * ref))))


# ----------------------------------------------------------------------------
# Full-size workloads: the GPU runs the whole problem; the oracle checks
# sampled (b, d) planes, each of which depends on four channel sequences.
# ----------------------------------------------------------------------------

def _sample_planes(wl, seed, count):
    rng = np.random.default_rng(seed)
    bs = rng.integers(0, wl.B, count)
    ds = rng.integers(0, wl.D, count)
    ds[0], bs[0] = wl.D - 1, wl.B - 1  # always include the last channel tile
    return list(zip(bs.tolist(), ds.tolist()))


def _oracle_plane(inp, b, d, D):
    sl = lambda a: a[b:b + 1]
    chans = [k * D + d for k in range(4)]
    return orc.forward_core(inp["x"][b:b + 1, d:d + 1], inp["A_logs"][chans], inp["Ds"][chans],
                            inp["dt_bias"][chans], dts=sl(inp["dts"])[:, :, d:d + 1], Bs=sl(inp["Bs"]),
                            Cs=sl(inp["Cs"]))[0, 0]


@pytest.mark.parametrize("name,count", [("vmamba_t_stage1", 12), ("stage3_short", 24), ("hires_long", 3)])
def test_full_workload_sampled(name, count):
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    t = _core_dev(inp, wl)
    y = ss.forward_core(**t)
    torch.cuda.synchronize()
    tol = TOL_BF16 if "bf16" in (wl.x_dtype, wl.dt_dtype) else TOL_F32
    worst = 0.0
    for b, d in _sample_planes(wl, 5, count):
        got = y[b, d].float().cpu().numpy()
        worst = max(worst, rel_err(got, _oracle_plane(inp, b, d, wl.D)))
    assert worst <= tol, worst
    assert torch.isfinite(y).all().item()


def test_full_stage1_standalone_scan_sampled():
    """The standalone scan on the materialised cross-scanned stage-1 input (B=32, C=768, L=3136)."""
    wl = WORKLOADS["vmamba_t_stage1"]
    inp = make_inputs(wl)
    t = _core_dev(inp, wl)
    B, D, L = wl.B, wl.D, wl.L
    xs = ss.cross_scan(t["x"]).view(B, 4 * D, L)
    y = ss.selective_scan(xs, t["dts"].view(B, 4 * D, L), t["A_logs"], t["Bs"], t["Cs"], t["Ds"], t["dt_bias"], True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(8)
    xs_np = orc.cross_scan(inp["x"][:1])  # only used for batch 0 channels below
    worst = 0.0
    for c in list(rng.integers(0, 4 * D, 6)) + [4 * D - 1]:
        k = c // D
        ref = orc.selective_scan(xs_np[0:1, k, c % D][:, None], inp["dts"][0:1, k, c % D][:, None],
                                 inp["A_logs"][c:c + 1], inp["Bs"][0:1, k:k + 1], inp["Cs"][0:1, k:k + 1],
                                 inp["Ds"][c:c + 1], inp["dt_bias"][c:c + 1], True)
        worst = max(worst, rel_err(y[0, c].cpu().numpy()[None, None], ref))
    assert worst <= TOL_BF16, worst


# ----------------------------------------------------------------------------
# Projection path: x_proj on tensor cores, dt_proj fused into the scan
# ----------------------------------------------------------------------------

def _proj_dev(inp):
    return dict(x=dev(inp["x"], "bf16"), A_logs=dev(inp["A_logs"]), Ds=dev(inp["Ds"]), dt_bias=dev(inp["dt_bias"]),
                x_proj_weight=dev(inp["x_proj_weight"], "bf16"), dt_projs_weight=dev(inp["dt_projs_weight"]))


def _proj_ref(inp):
    return orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], x_proj_weight=inp["x_proj_weight"],
                            dt_projs_weight=inp["dt_projs_weight"])


PROJ_CASES = [
    # B, D, H, W, N, R
    (1, 16, 8, 8, 4, 2),
    (2, 32, 9, 16, 16, 6),
    (1, 64, 14, 24, 16, 4),
    (2, 16, 5, 8, 8, 3),
]


@pytest.mark.parametrize("case", PROJ_CASES)
def test_forward_core_with_projections_matches_oracle(case):
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N, R = case
    wl = Workload("projcase", B, D, H, W, N, R, "bf16", "bf16", 300 + B + D + H + W + N + R)
    inp = make_inputs(wl)
    t = _proj_dev(inp)
    ws_bytes = ss.forward_core_workspace_size(**t)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    y = ss.forward_core(**t, workspace=ws)
    assert rel_err(host(y), _proj_ref(inp)) <= TOL_BF16
    assert int(ws[:4].view(torch.int32).item()) == 0  # no bounded wait ran out


# The other VMamba-T stages (SS2D article section 1: d_inner = 2 d_model; the overview page's
# four stages at 56, 28, 14 and 7 pixels), and widths that are not multiples of 8 or channel
# counts whose weights do not fit next to an x tile: these run the chunked x_proj kernel
# (128-pixel row-major tiles, 64-channel reduction chunks).
STAGE_PROJ_CASES = [
    # B, D, H, W, N, R
    (2, 384, 28, 28, 16, 12),   # stage 2: d_model 192, dt_rank 12
    (1, 768, 14, 14, 16, 16),   # stage 3 shape with the largest dt_rank the scan fuses
    (1, 1536, 7, 7, 16, 8),     # stage 4 shape, 49 pixels (rows not 16-byte aligned)
    (2, 48, 6, 10, 16, 6),      # W = 10, L = 60: element-wise x staging
    (1, 80, 9, 9, 8, 5),        # 80 channels = one 64-channel chunk and one of 16
    # dt_ranks above 16: dts is made by a separate dt_proj kernel and the direct-form scan
    # reads B and C from x_dbl's rows
    (1, 768, 14, 14, 16, 24),   # stage 3: d_model 384, dt_rank 24
    (1, 1536, 7, 7, 16, 48),    # stage 4: d_model 768, dt_rank 48 (4 (R + 2N) = 320 columns: two GEMM launches)
    (2, 64, 8, 12, 16, 20),
]


def test_static_entry_with_large_dt_rank():
    from selective_scan_02_b200.inputs import Workload
    inp = make_inputs(Workload("projstage_s", 3, 128, 10, 10, 16, 40, "bf16", "bf16", 611))
    t = _proj_dev(inp)
    ref = _proj_ref(inp)
    for _ in range(2):
        assert rel_err(host(ss.forward_core_static(**t)), ref) <= TOL_BF16


@pytest.mark.parametrize("case", STAGE_PROJ_CASES)
def test_forward_core_with_projections_other_stages(case):
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N, R = case
    wl = Workload("projstage", B, D, H, W, N, R, "bf16", "bf16", 500 + B + D + H + W + N + R)
    inp = make_inputs(wl)
    t = _proj_dev(inp)
    ws = torch.zeros(ss.forward_core_workspace_size(**t), dtype=torch.uint8, device="cuda")
    y = ss.forward_core(**t, workspace=ws)
    assert rel_err(host(y), _proj_ref(inp)) <= TOL_BF16
    assert int(ws[:4].view(torch.int32).item()) == 0  # no bounded wait ran out


@pytest.mark.parametrize("case", [(2, 192, 7, 12, 16, 6), (1, 400, 5, 5, 16, 4)])
def test_chunked_projection_gemm_matches_einsum_oracle(case):
    """x_dbl of the chunked x_proj kernel (any width, any multiple-of-16 channel count) against
    the oracle's x_proj of the cross-scanned x, in each direction's scan order."""
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N, R = case
    inp = make_inputs(Workload("gemm2", B, D, H, W, N, R, "bf16", "bf16", 78 + D))
    t = _proj_dev(inp)
    ws = torch.zeros(ss.forward_core_workspace_size(**t), dtype=torch.uint8, device="cuda")
    ss.forward_core(**t, workspace=ws)
    torch.cuda.synchronize()
    Cp, L = R + 2 * N, H * W
    got = ws[256:256 + B * 4 * Cp * L * 4].view(torch.float32).view(B, 4, Cp, L).cpu().numpy()
    ref = orc.x_proj(orc.cross_scan(inp["x"]), inp["x_proj_weight"])
    rms = float(np.sqrt(np.mean(ref * ref)))
    assert float(np.max(np.abs(got - ref))) <= 1e-4 * rms


@pytest.mark.parametrize("case", [(2, 32, 8, 8, 6), (1, 48, 9, 16, 4)])
def test_forward_core_with_projections_channels_last(case):
    # channels-last x and y with the projections: the GEMM runs on a channels-first copy of x
    # made in the workspace, the scan reads x's channel runs directly
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, R = case
    wl = Workload("proj_cl", B, D, H, W, 16, R, "bf16", "bf16", 40 + B + D + H + W + R)
    inp = make_inputs(wl)
    t = _proj_dev(inp)
    t["x"] = dev(np.ascontiguousarray(inp["x"].transpose(0, 2, 3, 1)), "bf16")
    y = ss.forward_core(**t, channels_last=True)
    assert rel_err(host(y), _proj_ref(inp).transpose(0, 2, 3, 1)) <= TOL_BF16
    ys = ss.forward_core_static(**t, channels_last=True)
    assert rel_err(host(ys), _proj_ref(inp).transpose(0, 2, 3, 1)) <= TOL_BF16


PROJ_SEG_CASES = [
    # B, D, H, W, R, channels_last: few images with long sequences run as a segmented scan
    (1, 32, 32, 32, 6, False),    # 8 segments of 128 steps
    (1, 16, 30, 24, 2, False),    # L = 720: 5 segments, the last one 80 steps (a partial chunk)
    (2, 32, 24, 16, 6, True),     # channels-last x and y, segmented
]


@pytest.mark.parametrize("case", PROJ_SEG_CASES)
def test_forward_core_with_projections_segmented(case):
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, R, cl = case
    wl = Workload("proj_seg", B, D, H, W, 16, R, "bf16", "bf16", 70 + B + D + H + W + R)
    inp = make_inputs(wl)
    t = _proj_dev(inp)
    ref = _proj_ref(inp)
    if cl:
        t["x"] = dev(np.ascontiguousarray(inp["x"].transpose(0, 2, 3, 1)), "bf16")
        ref = ref.transpose(0, 2, 3, 1)
    plain = ss.forward_core_workspace_size(**t, channels_last=cl)
    # the workspace holds the segment states on top of x_dbl and the copy of x
    L, Cp = H * W, R + 32
    assert plain > 256 + B * 4 * Cp * L * 4 + B * D * L * 2
    ws = torch.zeros(plain, dtype=torch.uint8, device="cuda")
    y = ss.forward_core(**t, channels_last=cl, workspace=ws)
    assert rel_err(host(y), ref) <= TOL_BF16
    assert int(ws[:4].view(torch.int32).item()) == 0


def test_device_status_after_projection_calls():
    """ss2d_device_status after real projection-form calls (forward, static forward, backward):
    every bounded wait ended, so each reports SS2D_OK.  The workspaces start filled with nonzero
    bytes, so a status word read from the wrong place would not be zero.  A nonzero word
    planted from the host (the whole workspace set to ones) is reported as SS2D_ERR_DEVICE,
    and the next call clears it."""
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N, R = 2, 32, 8, 16, 16, 6
    inp = make_inputs(Workload("status", B, D, H, W, N, R, "bf16", "bf16", 91))
    t = _proj_dev(inp)
    ws = torch.full((ss.forward_core_workspace_size(**t),), 0x5A, dtype=torch.uint8, device="cuda")
    y = ss.forward_core(**t, workspace=ws)
    ss.check_device_status(**t, workspace=ws)
    ws.fill_(1)
    with pytest.raises(ss.Ss2dError) as e:
        ss.check_device_status(**t, workspace=ws)
    assert e.value.status == 6 and e.value.name == "SS2D_ERR_DEVICE"
    ss.forward_core(**t, workspace=ws, y=y)
    ss.check_device_status(**t, workspace=ws)
    ss.forward_core_static(**t)
    ss.check_device_status(**t)
    dy = torch.randn(y.shape, generator=torch.Generator(device="cuda").manual_seed(5), device="cuda")
    bws = torch.full((ss.forward_core_backward_workspace_size(**t),), 0x5A, dtype=torch.uint8, device="cuda")
    ss.forward_core_backward(**t, dy=dy, workspace=bws)
    ss.check_device_status(**t, workspace=bws, backward=True)
    bws.fill_(1)
    with pytest.raises(ss.Ss2dError):
        ss.check_device_status(**t, workspace=bws, backward=True)


def test_projection_gemm_matches_einsum_oracle():
    """The tensor-core x_proj writes x_dbl (B, 4, R+2N, L) in each direction's scan order into the
    workspace after a 256-byte header; compare it with the oracle's x_proj of the cross-scanned x."""
    from selective_scan_02_b200.inputs import Workload
    B, D, H, W, N, R = 2, 64, 10, 24, 16, 6
    wl = Workload("gemm", B, D, H, W, N, R, "bf16", "bf16", 77)
    inp = make_inputs(wl)
    t = _proj_dev(inp)
    ws = torch.zeros(ss.forward_core_workspace_size(**t), dtype=torch.uint8, device="cuda")
    ss.forward_core(**t, workspace=ws)
    torch.cuda.synchronize()
    Cp, L = R + 2 * N, H * W
    got = ws[256:256 + B * 4 * Cp * L * 4].view(torch.float32).view(B, 4, Cp, L).cpu().numpy()
    ref = orc.x_proj(orc.cross_scan(inp["x"]), inp["x_proj_weight"])
    rms = float(np.sqrt(np.mean(ref * ref)))
    assert float(np.max(np.abs(got - ref))) <= 1e-4 * rms


def test_full_projection_workload_sampled():
    """The full projection workload (B=64, D=192, 56x56, N=16, R=6) on the GPU; the oracle checks
    sampled (b, d) planes: x_proj of image b over all channels, then dt_proj, scan and merge for d."""
    wl = WORKLOADS["proj"]
    inp = make_inputs(wl)
    t = _proj_dev(inp)
    y = ss.forward_core(**t)
    torch.cuda.synchronize()
    D, N, R = wl.D, wl.N, wl.R
    rng = np.random.default_rng(44)
    worst = 0.0
    for b in [0, wl.B - 1] + list(rng.integers(0, wl.B, 1)):
        xs = orc.cross_scan(inp["x"][b:b + 1])
        x_dbl = orc.x_proj(xs, inp["x_proj_weight"])
        for d in [0, D - 1] + list(rng.integers(0, D, 2)):
            chans = [k * D + d for k in range(4)]
            dts = orc.dt_proj(x_dbl, inp["dt_projs_weight"][:, d:d + 1], N)
            out = orc.selective_scan(xs[:, :, d].reshape(1, 4, wl.L), dts.reshape(1, 4, wl.L), inp["A_logs"][chans],
                                     x_dbl[:, :, R:R + N], x_dbl[:, :, R + N:], inp["Ds"][chans],
                                     inp["dt_bias"][chans], True)
            ref = orc.cross_merge(out.reshape(1, 4, 1, wl.L), wl.H, wl.W)[0, 0]
            worst = max(worst, rel_err(y[b, d].cpu().numpy(), ref))
    assert worst <= TOL_BF16, worst
