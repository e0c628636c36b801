"""The page-order merge (SS2D_MERGE_PAGE_ORDER) of the fused core on the GPU.

The SS2D article's section 3.3 sums the four directions' outputs as
y0 + inv_y0 + wh_y + invwh_y.  With the page-order merge every
direction stores its output once, without atomics, and one pass adds the four in that
order, so y is ((y0 + y2) + y1) + y3 bit for bit on every run.  Checked here: two runs give the
same bits; the result matches the oracle; and where the scans are not split into
segments it equals, bit for bit, the unfused chain CrossScan -> selective scan ->
ss2d_cross_merge (which adds in the same order)."""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from oracle import oracle as orc
from selective_scan_02_b200.inputs import Workload, bf16_bits, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"bf16": 5e-3, "f32": 2e-3}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _dev(a, dtype="f32"):
    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms)))


def _inputs(B, D, H, W, dt, seed):
    wl = Workload("merge", B, D, H, W, 16, 0, dt, dt, seed)
    inp = make_inputs(wl)
    t = dict(x=_dev(inp["x"], dt), dts=_dev(inp["dts"], dt), Bs=_dev(inp["Bs"]), Cs=_dev(inp["Cs"]),
             A_logs=_dev(inp["A_logs"]), Ds=_dev(inp["Ds"]), dt_bias=_dev(inp["dt_bias"]))
    return inp, t


CASES = [
    # B, D, H, W, dtype
    (2, 64, 32, 32, "bf16"),   # L = 1024: each direction's launch is scanned in segments
    (1, 40, 24, 40, "f32"),    # a ragged channel tile, H != W, fp32
    (3, 32, 12, 16, "bf16"),   # L = 192: not segmented
    (2, 32, 7, 7, "bf16"),     # L = 49: rows not 16-byte aligned (4-byte staging, one-step stores)
]


@pytest.mark.parametrize("case", CASES)
def test_page_order_merge_is_deterministic_and_matches_oracle(case):
    B, D, H, W, dt = case
    inp, t = _inputs(B, D, H, W, dt, 700 + B + D + H + W)
    y1 = ss.forward_core(**t, page_order=True)
    y2 = ss.forward_core(**t, page_order=True)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))  # the same bits on both runs
    ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"],
                           Cs=inp["Cs"])
    assert _rel_err(y1.cpu().numpy(), ref) <= TOL[dt]
    # and the same values as the atomic merge, up to the order of the four additions
    ya = ss.forward_core(**t)
    assert _rel_err(y1.cpu().numpy(), ya.double().cpu().numpy()) <= 1e-5


def test_page_order_merge_equals_unfused_chain_bit_for_bit():
    # L = 192 < 256: neither path splits the sequences into segments, so the per-step
    # arithmetic is the same and ss2d_cross_merge adds the four outputs in the same order
    B, D, H, W = 2, 32, 12, 16
    inp, t = _inputs(B, D, H, W, "bf16", 731)
    L = H * W
    y = ss.forward_core(**t, page_order=True)
    xs = ss.cross_scan(t["x"]).view(B, 4 * D, L)
    ys = ss.selective_scan(xs, t["dts"].view(B, 4 * D, L), t["A_logs"], t["Bs"], t["Cs"], t["Ds"], t["dt_bias"],
                           True)
    ym = ss.cross_merge(ys.view(B, 4, D, L), H, W)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int32), ym.view(torch.int32))


def test_page_order_merge_bf16_output_and_full_stage1_is_deterministic():
    # the stage-1 shape at two images (bf16 y rounds the fp32 page-order sum once)
    inp, t = _inputs(2, 192, 56, 56, "bf16", 1)
    y1 = ss.forward_core(**t, page_order=True, out_dtype=torch.bfloat16)
    y2 = ss.forward_core(**t, page_order=True, out_dtype=torch.bfloat16)
    yf = ss.forward_core(**t, page_order=True)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y1, yf.to(torch.bfloat16))


@pytest.mark.parametrize("case", [(2, 32, 12, 16, "bf16"), (1, 48, 10, 14, "f32"), (1, 16, 5, 7, "f32")])
def test_page_order_merge_channels_last(case):
    # channels-last x and y: direction 0 stores into y, the others into copies of y, then the
    # four are added element-wise in the page's order
    B, D, H, W, dt = case
    inp, t = _inputs(B, D, H, W, dt, 760 + B + D + H + W)
    t["x"] = t["x"].permute(0, 2, 3, 1).contiguous()
    y1 = ss.forward_core(**t, channels_last=True, page_order=True)
    y2 = ss.forward_core(**t, channels_last=True, page_order=True)
    ya = ss.forward_core(**t, channels_last=True)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"],
                           Cs=inp["Cs"]).transpose(0, 2, 3, 1)
    assert _rel_err(y1.cpu().numpy(), ref) <= TOL[dt]
    # the same four fp32 terms added in another order: three roundings each way, relative to
    # |y| + 1e-3 rms(y) where the terms cancel
    assert _rel_err(y1.cpu().numpy(), ya.double().cpu().numpy()) <= 5e-5


def test_page_order_merge_keeps_checkpoints():
    # the page-order forward can keep its backward's checkpoints too: y is unchanged, bit for bit,
    # and the backward reading them matches the backward that recomputes them
    B, D, H, W = 2, 32, 12, 16
    inp, t = _inputs(B, D, H, W, "bf16", 733)
    ck = torch.full(ss.checkpoint_shape(t["x"]), float("nan"), device="cuda")
    y0 = ss.forward_core(**t, page_order=True)
    y1 = ss.forward_core(**t, page_order=True, ckpt=ck)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))
    assert bool(torch.isfinite(ck).all())
    dy = torch.from_numpy(np.random.default_rng(734).standard_normal((B, D, H, W)).astype(np.float32)).cuda()
    g_kept = ss.forward_core_backward(**t, dy=dy, ckpt=ck)
    g_own = ss.forward_core_backward(**t, dy=dy)
    torch.cuda.synchronize()
    for k in g_own:
        ref = g_own[k].double().cpu().numpy()
        assert _rel_err(g_kept[k].cpu().numpy(), ref) <= 1e-4, k
