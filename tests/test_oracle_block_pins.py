"""Pins of the block oracle (oracle/block.py) against facts that do not come from it.

Each step of the SS2D block (SS2D article, section 1; VMamba overview page, section 2.2)
is pinned by closed forms, special cases and library routines:
  - bf16 rounding: hand-worked ties and torch's float32 -> bfloat16 conversion;
  - SiLU: exact values and the identity SiLU(z) - SiLU(-z) = z; torch's silu;
  - the depthwise convolution: a centred delta kernel is the identity, an off-centre one a
    shift with zero fill; scipy's correlate2d and torch's grouped conv2d on random data;
  - LayerNorm: the output variance var / (var + eps) in closed form, invariance under
    y -> a*y + c (with eps scaled by a^2), torch's layer_norm;
  - the linear maps: a brute-force double loop and identity weights;
  - the whole block: a configuration whose core reduces to a per-channel scale (C = 0, so the
    output is the skip term), with a delta convolution, against a first-principles
    composition; and the block's non-core steps recomposed from torch's library routines.
A mistake such as swapping the x and z halves of the input projection, a wrong padding, a
missing SiLU, an unbiased variance or a dropped gate fails at least one of these."""
import numpy as np
import pytest
import scipy.signal
import torch
import torch.nn.functional as F

from oracle import block as ob
from selective_scan_02_b200.inputs import BlockWorkload, make_block_inputs


def test_round_bf16_ties_and_library():
    one = 1.0
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even pattern (1.0)
    assert ob.round_bf16(np.array([one + 2.0 ** -8]))[0] == one
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert ob.round_bf16(np.array([one + 3 * 2.0 ** -8]))[0] == one + 2.0 ** -6
    # just above a tie rounds up, negative values mirror
    assert ob.round_bf16(np.array([one + 2.0 ** -8 + 2.0 ** -20]))[0] == one + 2.0 ** -7
    assert ob.round_bf16(np.array([-(one + 3 * 2.0 ** -8)]))[0] == -(one + 2.0 ** -6)
    rng = np.random.default_rng(0)
    a = rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ob.round_bf16(a), ref)


def test_silu_values_and_identity():
    assert ob.silu(np.array([0.0]))[0] == 0.0
    assert ob.silu(np.array([1.0]))[0] == pytest.approx(1.0 / (1.0 + np.exp(-1.0)), rel=1e-15)
    z = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(ob.silu(z) - ob.silu(-z), z, rtol=0, atol=1e-13)
    assert ob.silu(np.array([-800.0]))[0] == 0.0  # exp overflow gives -0, not nan
    ref = F.silu(torch.from_numpy(z)).numpy()
    np.testing.assert_allclose(ob.silu(z), ref, rtol=1e-14, atol=1e-300)


@pytest.mark.parametrize("k", [1, 3, 5, 7])
def test_depthwise_conv_delta_kernels(k):
    rng = np.random.default_rng(k)
    x = rng.standard_normal((2, 6, 9, 5))
    r = (k - 1) // 2
    w = np.zeros((5, k, k))
    w[:, r, r] = 1.0
    bias = rng.standard_normal(5)
    np.testing.assert_array_equal(ob.depthwise_conv(x, w, bias), x + bias)
    if k > 1:
        # a one at (i, j) reads x[h + i - r, w + j - r]: a shift with zeros from outside
        i, j = 0, k - 1
        w = np.zeros((5, k, k))
        w[:, i, j] = 1.0
        got = ob.depthwise_conv(x, w)
        di, dj = i - r, j - r
        ref = np.zeros_like(x)
        H, W = x.shape[1:3]
        for h in range(H):
            for ww in range(W):
                hs, ws = h + di, ww + dj
                if 0 <= hs < H and 0 <= ws < W:
                    ref[:, h, ww, :] = x[:, hs, ws, :]
        np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("k", [3, 5])
def test_depthwise_conv_matches_libraries(k):
    rng = np.random.default_rng(10 + k)
    B, H, W, D = 2, 7, 11, 4
    x = rng.standard_normal((B, H, W, D))
    w = rng.standard_normal((D, k, k))
    bias = rng.standard_normal(D)
    got = ob.depthwise_conv(x, w, bias)
    for b in range(B):
        for d in range(D):
            ref = scipy.signal.correlate2d(x[b, :, :, d], w[d], mode="same", boundary="fill") + bias[d]
            np.testing.assert_allclose(got[b, :, :, d], ref, rtol=1e-12, atol=1e-12)
    ref = F.conv2d(torch.from_numpy(x).permute(0, 3, 1, 2), torch.from_numpy(w)[:, None], torch.from_numpy(bias),
                   padding=k // 2, groups=D).permute(0, 2, 3, 1).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_layer_norm_closed_form_and_library():
    rng = np.random.default_rng(3)
    y = rng.standard_normal((5, 64)) * 3 + 2
    eps = 1e-5
    out = ob.layer_norm(y, np.ones(64), np.zeros(64), eps)
    var = y.var(axis=-1)
    np.testing.assert_allclose(out.mean(axis=-1), 0, atol=1e-13)
    np.testing.assert_allclose((out ** 2).mean(axis=-1), var / (var + eps), rtol=1e-12)
    # invariance under an affine change of y when eps is scaled with the variance
    a, c = 7.5, -3.0
    np.testing.assert_allclose(ob.layer_norm(a * y + c, np.ones(64), np.zeros(64), eps * a * a), out, rtol=1e-11,
                               atol=1e-12)
    g, bta = rng.uniform(0.5, 1.5, 64), rng.standard_normal(64)
    ref = F.layer_norm(torch.from_numpy(y), (64,), torch.from_numpy(g), torch.from_numpy(bta), eps).numpy()
    np.testing.assert_allclose(ob.layer_norm(y, g, bta, eps), ref, rtol=1e-12, atol=1e-12)


def test_linear_brute_force_and_identity():
    rng = np.random.default_rng(4)
    a = rng.standard_normal((3, 4, 6))
    w = rng.standard_normal((5, 6))
    bias = rng.standard_normal(5)
    got = ob.linear(a, w, bias)
    for i in range(3):
        for j in range(4):
            for m in range(5):
                assert got[i, j, m] == pytest.approx(sum(a[i, j, kk] * w[m, kk] for kk in range(6)) + bias[m],
                                                     rel=1e-13, abs=1e-13)
    eye = np.vstack([np.eye(6), np.zeros((2, 6))])
    np.testing.assert_array_equal(ob.linear(a, eye)[..., :6], a)
    np.testing.assert_array_equal(ob.linear(a, eye)[..., 6:], 0)


def _small_block(seed=7, B=2, H=6, W=5, dm=32, D=48, N=16, R=4, k=3, **kw):
    wl = BlockWorkload("pin", B, H, W, dm, D, N, R, k, seed)
    return make_block_inputs(wl, **kw)


def _call(inp, eps=1e-5):
    return ob.block_forward(inp["x"], inp["in_proj_weight"], inp["conv_weight"], inp["conv_bias"],
                            inp["x_proj_weight"], inp["dt_projs_weight"], inp["dt_projs_bias"], inp["A_logs"],
                            inp["Ds"], inp["out_norm_weight"], inp["out_norm_bias"], inp["out_proj_weight"],
                            in_proj_bias=inp.get("in_proj_bias"), out_proj_bias=inp.get("out_proj_bias"), eps=eps,
                            intermediates=True)


def test_block_with_skip_only_core_matches_first_principles():
    """C = 0 (the x_proj rows that produce C are zero) leaves each direction's output at
    Ds * u, so the merged core output is (sum of the four directions' Ds) * x_c.  A centred
    delta kernel without bias makes x_c = bf16(SiLU(x_in)).  The block output then follows
    from the definitions alone, with no scan and no convolution."""
    inp = _small_block(in_proj_bias=True, out_proj_bias=True)
    N, R, D = 16, 4, 48
    inp["x_proj_weight"][:, R + N:, :] = 0.0
    inp["conv_weight"][:] = 0.0
    inp["conv_weight"][:, 1, 1] = 1.0
    inp["conv_bias"][:] = 0.0
    rng = np.random.default_rng(9)
    inp["Ds"] = rng.uniform(0.5, 1.5, 4 * D).astype(np.float32)
    out, mid = _call(inp)

    def bf(a):
        return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()

    x = inp["x"].astype(np.float64)
    xz = bf(np.einsum("bhwc,oc->bhwo", x, inp["in_proj_weight"].astype(np.float64)) + inp["in_proj_bias"])
    x_in, z = xz[..., :D], xz[..., D:]
    x_c = bf(x_in / (1 + np.exp(-x_in)))
    ds = inp["Ds"].astype(np.float64).reshape(4, D).sum(axis=0)
    y = ds * x_c
    mu = y.mean(-1, keepdims=True)
    sd = np.sqrt(((y - mu) ** 2).mean(-1, keepdims=True) + 1e-5)
    g = bf(((y - mu) / sd * inp["out_norm_weight"] + inp["out_norm_bias"]) * (z / (1 + np.exp(-z))))
    ref = np.einsum("bhwc,oc->bhwo", g, inp["out_proj_weight"].astype(np.float64)) + inp["out_proj_bias"]
    np.testing.assert_allclose(mid["y"], y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_block_steps_match_torch_library_routines():
    """The block's steps around the core recomposed from torch's linear, conv2d (groups = D),
    silu and layer_norm in fp64, with the oracle's own core output as the middle step."""
    inp = _small_block(seed=11, H=7, W=9, k=5, in_proj_bias=True)
    out, mid = _call(inp)
    t = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in inp.items()}
    D = 48

    def bf(a):
        return a.float().to(torch.bfloat16).double()

    xz = bf(F.linear(t["x"], t["in_proj_weight"], t["in_proj_bias"]))
    np.testing.assert_array_equal(mid["xz"], xz.numpy())
    x_in, z = xz[..., :D], xz[..., D:]
    conv = F.conv2d(x_in.permute(0, 3, 1, 2), t["conv_weight"][:, None], t["conv_bias"], padding=2, groups=D)
    x_c = bf(F.silu(conv)).permute(0, 2, 3, 1)
    # equal up to the rare bf16 tie that fp64 rounding order can move
    assert np.mean(mid["x_c"] != x_c.numpy()) < 1e-3
    np.testing.assert_allclose(mid["x_c"], x_c.numpy(), rtol=1e-2, atol=0)
    y = torch.from_numpy(mid["y"])
    g = bf(F.layer_norm(y, (D,), t["out_norm_weight"], t["out_norm_bias"], 1e-5) * F.silu(z))
    assert np.mean(mid["g"] != g.numpy()) < 1e-3
    ref = F.linear(torch.from_numpy(mid["g"]), t["out_proj_weight"])
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_block_gate_and_split_order_matter():
    """Swapping the x and z halves of the input projection changes the output (so the pins
    above see the split order), and a zero gate branch zeroes the output."""
    inp = _small_block(seed=13)
    out, _ = _call(inp)
    sw = dict(inp)
    D = 48
    sw["in_proj_weight"] = np.concatenate([inp["in_proj_weight"][D:], inp["in_proj_weight"][:D]])
    out_sw, _ = _call(sw)
    assert np.max(np.abs(out_sw - out)) > 0.1 * np.max(np.abs(out))
    zg = dict(inp)
    zg["in_proj_weight"] = inp["in_proj_weight"].copy()
    zg["in_proj_weight"][D:] = 0.0
    out_z, _ = _call(zg)
    assert np.all(out_z == 0.0)


def test_block_storage_rounding_switch():
    """store_bf16=True leaves xz, x_c and g on the bf16 grid; store_bf16=False keeps them in
    fp64, and the two outputs differ by the effect of rounding errors of at most 2^-9 relative
    at those points (small against the output, but not zero)."""
    inp = _small_block(seed=17)
    out, mid = _call(inp)
    for k in ("xz", "x_c", "g"):
        np.testing.assert_array_equal(ob.round_bf16(mid[k]), mid[k])
    raw = ob.block_forward(inp["x"], inp["in_proj_weight"], inp["conv_weight"], inp["conv_bias"],
                           inp["x_proj_weight"], inp["dt_projs_weight"], inp["dt_projs_bias"], inp["A_logs"],
                           inp["Ds"], inp["out_norm_weight"], inp["out_norm_bias"], inp["out_proj_weight"],
                           store_bf16=False)
    rms = np.sqrt(np.mean(out ** 2))
    gap = np.sqrt(np.mean((out - raw) ** 2)) / rms
    assert 1e-5 < gap < 2.0 ** -6
