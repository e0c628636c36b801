"""GPU parity of the SS2D block (ss2d_block_forward) against the block oracle.

The block (SS2D article, section 1; VMamba overview page, section 2.2) runs the input
projection and the output projection on the tensor cores, the depthwise convolution with
SiLU and the gated LayerNorm in their own kernels, and the core in between.  Each case
compares the whole block's output with oracle/block.py (fp64, rounding to bf16 where the
block stores), element by element, within the core's bf16 tolerance (5e-3 relative) plus
a term for rounding flips at the bf16 storage points, taken from the oracle's own
sensitivity to that rounding (_assert_block_parity states the bound).  Cases span ragged 128-row tiles, widths
and channel counts that are not multiples of the kernels' tiles, several column passes of
the projections, every built kernel size, the four VMamba-T stage shapes, and the full
stage-1 batch of 64 images (checked on its first and last image)."""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from oracle import block as ob
from selective_scan_02_b200.inputs import BLOCK_WORKLOADS, BlockWorkload, bf16_bits, make_block_inputs

pytestmark = pytest.mark.gpu

TOL = 5e-3
BF16_KEYS = ("x", "in_proj_weight", "x_proj_weight", "out_proj_weight")


def _assert_block_parity(got, ref, ref_unrounded, tol=TOL, rms_tol=1e-3):
    """The block stores xz, x_c and g in bf16.  Both sides round there, from values that
    differ by their fp32 / fp64 arithmetic (about 1e-7 relative), so now and then a value next
    to a rounding tie lands on the other bf16 neighbour: a flip of one unit in the last place.
    A flip in x_c moves the core's output along the whole scan lines through that pixel
    (the decays reach hundreds of steps), and the LayerNorm and the output projection spread
    a change of y over every output channel of the pixel.  The oracle evaluated without the
    storage rounding (ref_unrounded) gives, per output, the size of the effect that rounding
    errors of that magnitude at the storage points have; flips are a few such errors, so the
    per-element bound adds twice the per-pixel rms of |ref - ref_unrounded| to the core's
    metric:
      (i)   every element: |got - ref| <= tol (|ref| + 1e-3 rms(ref)) + 2 env(pixel),
            env(pixel) = rms over the pixel's output channels of |ref - ref_unrounded|;
      (ii)  over the whole output: rms(got - ref) <= rms_tol rms(ref)."""
    got = np.asarray(got, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    diff = np.abs(got - ref)
    env = np.sqrt(np.mean((ref - ref_unrounded) ** 2, axis=-1, keepdims=True))
    bound = tol * (np.abs(ref) + 1e-3 * rms) + 2.0 * env
    assert np.all(diff <= bound), (float(np.max(diff / bound)), float(np.max(diff) / rms))
    assert float(np.sqrt(np.mean(diff * diff))) <= rms_tol * rms, float(np.sqrt(np.mean(diff * diff))) / rms


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _dev(inp):
    out = {}
    for k, v in inp.items():
        if k in BF16_KEYS:
            out[k] = torch.from_numpy(bf16_bits(v).view(np.int16)).view(torch.bfloat16).cuda()
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()
    return out


def _rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms)))


def _gpu(t, **kw):
    return ss.block_forward(t["x"], t["in_proj_weight"], t["conv_weight"], t.get("conv_bias"), t["x_proj_weight"],
                            t["dt_projs_weight"], t["dt_projs_bias"], t["A_logs"], t["Ds"], t["out_norm_weight"],
                            t["out_norm_bias"], t["out_proj_weight"], in_proj_bias=t.get("in_proj_bias"),
                            out_proj_bias=t.get("out_proj_bias"), **kw)


def _oracle(inp, b0=0, b1=None, store_bf16=True):
    sl = slice(b0, b1)
    return ob.block_forward(inp["x"][sl], inp["in_proj_weight"], inp["conv_weight"], inp.get("conv_bias"),
                            inp["x_proj_weight"], inp["dt_projs_weight"], inp["dt_projs_bias"], inp["A_logs"],
                            inp["Ds"], inp["out_norm_weight"], inp["out_norm_bias"], inp["out_proj_weight"],
                            in_proj_bias=inp.get("in_proj_bias"), out_proj_bias=inp.get("out_proj_bias"),
                            store_bf16=store_bf16)


def _refs(inp, b0=0, b1=None):
    return _oracle(inp, b0, b1), _oracle(inp, b0, b1, store_bf16=False)


CASES = [
    # B, H, W, d_model, D, R, d_conv, biases
    (2, 12, 12, 32, 64, 4, 3, True),      # small, both projection biases
    (1, 10, 13, 48, 80, 3, 3, False),     # 130 pixels (ragged 128-row tile), D not a multiple of 64
    (3, 9, 7, 16, 32, 2, 5, True),        # 5x5 kernel wider than the image's short side
    (2, 6, 11, 32, 48, 4, 1, False),      # 1x1 kernel
    (1, 8, 40, 64, 128, 4, 7, True),      # 7x7 kernel, two 32-column conv tiles
    (2, 16, 16, 96, 192, 6, 3, False),    # stage-1 channels: 2D = 384, two column passes
]


@pytest.mark.parametrize("case", CASES)
def test_block_matches_oracle(case):
    B, H, W, dm, D, R, k, biases = case
    wl = BlockWorkload("t", B, H, W, dm, D, 16, R, k, 100 + B + H + W + dm + k)
    inp = make_block_inputs(wl, in_proj_bias=biases, out_proj_bias=biases)
    out = _gpu(_dev(inp))
    torch.cuda.synchronize()
    assert out.shape == (B, H, W, dm)
    _assert_block_parity(out.cpu().numpy(), *_refs(inp))


STAGES = [
    # VMamba-T stages 2, 3 and 4: d_model 192 / 384 / 768, D = 2 d_model, dt_rank ceil(d_model / 16)
    (1, 28, 28, 192, 384, 12),
    (1, 14, 14, 384, 768, 24),
    (2, 7, 7, 768, 1536, 48),
]


@pytest.mark.parametrize("case", STAGES)
def test_block_other_stages(case):
    B, H, W, dm, D, R = case
    wl = BlockWorkload("stage", B, H, W, dm, D, 16, R, 3, 200 + dm)
    inp = make_block_inputs(wl)
    out = _gpu(_dev(inp))
    torch.cuda.synchronize()
    _assert_block_parity(out.cpu().numpy(), *_refs(inp))


def test_block_bf16_output():
    wl = BlockWorkload("bf", 2, 12, 20, 32, 64, 16, 4, 3, 300)
    inp = make_block_inputs(wl, out_proj_bias=True)
    t = _dev(inp)
    o32 = _gpu(t)
    o16 = _gpu(t, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16
    # a bf16 output adds one rounding of at most 2^-9 relative (about 2^-9 / sqrt(3) rms)
    _assert_block_parity(o16.float().cpu().numpy(), *_refs(inp), tol=TOL + 2.0 ** -9, rms_tol=1e-3 + 2.0 ** -9)
    # and is the fp32 output rounded, up to the core's atomic merge order
    assert _rel_err(o16.float().cpu().numpy(), o32.double().cpu().numpy()) <= 2.0 ** -8


def test_block_full_stage1_batch():
    """The block at VMamba-T stage 1 with the batch of 64 images the bench times; the oracle
    checks the first and the last image (images are independent)."""
    wl = BLOCK_WORKLOADS["block_stage1"]
    inp = make_block_inputs(wl)
    t = _dev(inp)
    ws = torch.empty(ss.block_forward_workspace_size(t["x"], t["in_proj_weight"], t["conv_weight"], t["conv_bias"],
                                                     t["x_proj_weight"], t["dt_projs_weight"], t["dt_projs_bias"],
                                                     t["A_logs"], t["Ds"], t["out_norm_weight"], t["out_norm_bias"],
                                                     t["out_proj_weight"]), dtype=torch.uint8, device="cuda")
    out = _gpu(t, workspace=ws)
    ss.block_device_status(t["x"], t["in_proj_weight"], t["conv_weight"], t["conv_bias"], t["x_proj_weight"],
                           t["dt_projs_weight"], t["dt_projs_bias"], t["A_logs"], t["Ds"], t["out_norm_weight"],
                           t["out_norm_bias"], t["out_proj_weight"], ws)
    got = out.cpu().numpy()
    for b in (0, wl.B - 1):
        _assert_block_parity(got[b:b + 1], *_refs(inp, b, b + 1))


def test_block_rejects_before_enqueueing():
    wl = BlockWorkload("rej", 1, 8, 8, 32, 64, 16, 4, 3, 400)
    inp = make_block_inputs(wl)
    t = _dev(inp)
    out = torch.full((1, 8, 8, 32), 7.0, device="cuda")
    bad = dict(t)
    bad["conv_weight"] = torch.zeros((64, 2, 2), device="cuda")  # even kernel size
    with pytest.raises(ss.Ss2dError) as e:
        _gpu(bad, out=out)
    assert e.value.name == "SS2D_ERR_INVALID_ARG"
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
