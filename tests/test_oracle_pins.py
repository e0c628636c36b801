"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a
hand-derived fixture, a closed form, a library routine applied to a special
case, an invariant, or a brute-force evaluation written from a different
formula.  None of them needs a GPU.
"""
import math
import os

import numpy as np
import pytest

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_fixture(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows[key] = vals
    return rows


# ----------------------------------------------------------------------------
# cross scan / cross merge
# ----------------------------------------------------------------------------

def test_cross_scan_direction_table_golden():
    """Hand-derived 2x3 example of the four scan orders (VMamba SS2D article, section 4)."""
    fx = _read_fixture("cross_scan_direction_table.txt")
    H, W = int(fx["H"][0]), int(fx["H"][2])
    plane = np.array([float(v) for v in fx["plane"]]).reshape(1, 1, H, W)
    xs = orc.cross_scan(plane)
    for k in range(4):
        expect = np.array([float(v) for v in fx[f"dir{k}"]])
        np.testing.assert_array_equal(xs[0, k, 0], expect)


def test_page_test_cross_scan_assertions():
    """The article's test_cross_scan (section 5): x (2,64,32,32) -> xs (2,4,64,1024),
    direction 0 is x.flatten() and direction 1 is x.T.flatten(), read per batch element."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((2, 64, 32, 32))
    xs = orc.cross_scan(x)
    assert xs.shape == (2, 4, 64, 1024)
    for b in range(2):
        for d in (0, 17, 63):
            np.testing.assert_array_equal(xs[b, 0, d], x[b, d].flatten())
            np.testing.assert_array_equal(xs[b, 1, d], x[b, d].T.flatten())


@pytest.mark.parametrize("H,W", [(3, 5), (7, 4), (1, 6), (6, 1), (8, 8)])
def test_cross_scan_matches_numpy_transpose_flip(H, W):
    """Index formulas of the four orders against numpy's transpose and flip."""
    rng = np.random.default_rng(H * 31 + W)
    B, D = 2, 3
    x = rng.standard_normal((B, D, H, W))
    xs = orc.cross_scan(x)
    L = H * W
    hw = x.reshape(B, D, L)
    wh = np.swapaxes(x, 2, 3).reshape(B, D, L)
    np.testing.assert_array_equal(xs[:, 0], hw)
    np.testing.assert_array_equal(xs[:, 1], wh)
    np.testing.assert_array_equal(xs[:, 2], hw[:, :, ::-1])
    np.testing.assert_array_equal(xs[:, 3], wh[:, :, ::-1])


@pytest.mark.parametrize("H,W", [(3, 5), (4, 4), (5, 2)])
def test_cross_merge_is_adjoint_of_cross_scan(H, W):
    """Merging sums each direction back onto the pixel it was read from, so it is the
    transpose of the scan gather: <scan(x), ys> == <x, merge(ys)>."""
    rng = np.random.default_rng(7 + H + W)
    B, D = 2, 3
    x = rng.standard_normal((B, D, H, W))
    ys = rng.standard_normal((B, 4, D, H * W))
    lhs = float(np.sum(orc.cross_scan(x) * ys))
    rhs = float(np.sum(x * orc.cross_merge(ys, H, W)))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_merge_of_scan_is_four_x_exact():
    """With the scan as the identity, CrossMerge(CrossScan(x)) == 4x exactly (integer data)."""
    rng = np.random.default_rng(5)
    x = rng.integers(-1000, 1000, size=(2, 3, 6, 9)).astype(np.float64)
    y = orc.cross_merge(orc.cross_scan(x), 6, 9)
    np.testing.assert_array_equal(y, 4 * x)


def test_cross_merge_single_direction_placement():
    """A one-hot in one direction's scan position lands on the pixel that order visits."""
    H, W = 3, 4
    L = H * W
    order = {
        0: [h * W + w for h in range(H) for w in range(W)],
        1: [h * W + w for w in range(W) for h in range(H)],
    }
    order[2] = order[0][::-1]
    order[3] = order[1][::-1]
    for k in range(4):
        for l in (0, 1, 5, L - 1):
            ys = np.zeros((1, 4, 1, L))
            ys[0, k, 0, l] = 1.0
            y = orc.cross_merge(ys, H, W).reshape(L)
            expect = np.zeros(L)
            expect[order[k][l]] = 1.0
            np.testing.assert_array_equal(y, expect)


# ----------------------------------------------------------------------------
# selective scan
# ----------------------------------------------------------------------------

def _softplus_lib(z):
    return np.logaddexp(0.0, z)


def _brute_force_scan(u, delta, A_log, Bm, Cm, Dv, bias, softplus_on):
    """O(L^2 N) unrolled form: y_l = sum_{j<=l} sum_n C_l[n] exp(A_n (S_l - S_j)) dt_j B_j[n] u_j + D u_l,
    with S the running sum of dt -- the product of the per-step decays written as one exponential."""
    B, C, L = u.shape
    G, N = Bm.shape[1], Bm.shape[2]
    y = np.zeros((B, C, L))
    for b in range(B):
        for c in range(C):
            g = c * G // C
            z = delta[b, c] + (bias[c] if bias is not None else 0.0)
            dt = _softplus_lib(z) if softplus_on else z
            S = np.concatenate([[0.0], np.cumsum(dt)])  # S[l+1] = dt_0 + ... + dt_l
            A = -np.exp(A_log[c])
            for l in range(L):
                tot = 0.0
                for j in range(l + 1):
                    decay = np.exp(A * (S[l + 1] - S[j + 1]))
                    tot += np.sum(Cm[b, g, :, l] * decay * dt[j] * Bm[b, g, :, j]) * u[b, c, j]
                y[b, c, l] = tot + (Dv[c] if Dv is not None else 0.0) * u[b, c, l]
    return y


@pytest.mark.parametrize("N,G,softplus_on,L", [(1, 1, True, 7), (3, 2, True, 9), (4, 4, False, 6), (2, 1, True, 1)])
def test_scan_matches_brute_force(N, G, softplus_on, L):
    rng = np.random.default_rng(100 + N * 10 + G + L)
    B, C = 2, 4
    u = rng.standard_normal((B, C, L))
    delta = rng.standard_normal((B, C, L)) * 0.5 + (0.0 if softplus_on else 1.0)
    A_log = np.log(rng.uniform(0.5, 3.0, (C, N)))
    Bm = rng.standard_normal((B, G, N, L))
    Cm = rng.standard_normal((B, G, N, L))
    Dv = rng.standard_normal(C)
    bias = rng.uniform(-2, -0.5, C) if softplus_on else rng.uniform(0.0, 0.3, C)
    got = orc.selective_scan(u, delta, A_log, Bm, Cm, Dv, bias, softplus_on)
    ref = _brute_force_scan(u, delta, A_log, Bm, Cm, Dv, bias, softplus_on)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_scan_lti_equals_causal_convolution():
    """Constant dt, B, C: y = K * u + D u with K_m = sum_n C_n exp(dt A_n)^m dt B_n
    (VSSD article, section 3.1), evaluated with numpy.convolve."""
    rng = np.random.default_rng(3)
    L, N = 40, 4
    u = rng.standard_normal((1, 1, L))
    dt_raw = 0.3
    delta = np.full((1, 1, L), dt_raw)
    A_log = np.log(np.array([[0.5, 1.0, 2.0, 4.0]]))
    Bn = rng.standard_normal(N)
    Cn = rng.standard_normal(N)
    Bm = np.tile(Bn[None, None, :, None], (1, 1, 1, L))
    Cm = np.tile(Cn[None, None, :, None], (1, 1, 1, L))
    Dv = np.array([0.7])
    got = orc.selective_scan(u, delta, A_log, Bm, Cm, Dv, None, False)[0, 0]
    A = -np.exp(A_log[0])
    m = np.arange(L)
    K = np.sum(Cn[:, None] * np.exp(dt_raw * A)[:, None] ** m[None, :] * dt_raw * Bn[:, None], axis=0)
    ref = np.convolve(u[0, 0], K)[:L] + Dv[0] * u[0, 0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_scan_golden_halving_kernel():
    """Hand-derived LTI case with A_bar = 1/2 (fixture lti_halving_kernel.txt)."""
    fx = _read_fixture("lti_halving_kernel.txt")
    L = int(fx["L"][0])
    ln2 = float(fx["ln2"][0])
    assert abs(ln2 - math.log(2.0)) < 1e-15
    ones = np.ones((1, 1, 1, L))
    for name in ("impulse", "step"):
        u = np.array([float(v) for v in fx[f"{name}_u"]]).reshape(1, 1, L)
        expect = np.array([float(v) for v in fx[f"{name}_y_over_ln2"]]) * ln2
        y = orc.selective_scan(u, np.full((1, 1, L), ln2), np.zeros((1, 1)), ones, ones, None, None, False)
        np.testing.assert_allclose(y[0, 0], expect, rtol=1e-14, atol=1e-15)


def test_scan_cumsum_special_case():
    """A_log = -30 makes A ~ -1e-13, so every decay is 1 to within 1e-12 over these lengths;
    with B = C = 1 and N = 1 the scan is the running sum of dt * u (numpy.cumsum)."""
    rng = np.random.default_rng(9)
    B, C, L = 2, 3, 200
    u = rng.standard_normal((B, C, L))
    delta = rng.standard_normal((B, C, L))
    bias = rng.uniform(-3, 0, C)
    A_log = np.full((C, 1), -30.0)
    ones = np.ones((B, 1, 1, L))
    Dv = rng.standard_normal(C)
    y = orc.selective_scan(u, delta, A_log, ones, ones, Dv, bias, True)
    dt = _softplus_lib(delta + bias[None, :, None])
    ref = np.cumsum(dt * u, axis=-1) + Dv[None, :, None] * u
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-9)


def test_scan_memoryless_special_case():
    """A_log = +5 (A ~ -148) and dt >= 0.5 without softplus give decays below e^-74: every
    step forgets the past, so y_l = sum_n C_l dt_l B_l u_l + D u_l element by element."""
    rng = np.random.default_rng(10)
    B, C, G, N, L = 2, 4, 2, 3, 30
    u = rng.standard_normal((B, C, L))
    delta = rng.uniform(0.5, 2.0, (B, C, L))
    bias = rng.uniform(0.0, 0.5, C)
    A_log = np.full((C, N), 5.0)
    Bm = rng.standard_normal((B, G, N, L))
    Cm = rng.standard_normal((B, G, N, L))
    Dv = rng.standard_normal(C)
    y = orc.selective_scan(u, delta, A_log, Bm, Cm, Dv, bias, False)
    dt = delta + bias[None, :, None]
    grp = np.repeat(np.arange(G), C // G)
    ref = np.einsum("bcnl,bcnl->bcl", Cm[:, grp], Bm[:, grp]) * dt * u + Dv[None, :, None] * u
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def _brute_force_states(u, delta, A_log, Bm, bias, softplus_on):
    """h_l[n] = sum_{j<=l} exp(A_n (S_l - S_j)) dt_j B_j[n] u_j for every l, from the same
    cumulative-sum form as _brute_force_scan (not the step-by-step recurrence)."""
    B, C, L = u.shape
    G, N = Bm.shape[1], Bm.shape[2]
    h = np.zeros((B, C, L, N))
    for b in range(B):
        for c in range(C):
            g = c * G // C
            z = delta[b, c] + (bias[c] if bias is not None else 0.0)
            dt = _softplus_lib(z) if softplus_on else z
            S = np.concatenate([[0.0], np.cumsum(dt)])
            A = -np.exp(A_log[c])
            for l in range(L):
                for j in range(l + 1):
                    h[b, c, l] += np.exp(A * (S[l + 1] - S[j + 1])) * dt[j] * Bm[b, g, :, j] * u[b, c, j]
    return h


@pytest.mark.parametrize("every,L", [(4, 13), (16, 16), (5, 1), (3, 9)])
def test_scan_checkpoints_match_brute_force_states(every, L):
    """selective_scan_ckpt records h_{j*every - 1} (zero for j = 0): against the unrolled states."""
    rng = np.random.default_rng(40 + every + L)
    B, C, G, N = 2, 4, 2, 3
    u = rng.standard_normal((B, C, L))
    delta = rng.standard_normal((B, C, L)) * 0.5
    A_log = np.log(rng.uniform(0.5, 3.0, (C, N)))
    Bm = rng.standard_normal((B, G, N, L))
    Cm = rng.standard_normal((B, G, N, L))
    bias = rng.uniform(-2, -0.5, C)
    y, ck = orc.selective_scan_ckpt(u, delta, A_log, Bm, Cm, every, delta_bias=bias, delta_softplus=True)
    h = _brute_force_states(u, delta, A_log, Bm, bias, True)
    nck = (L + every - 1) // every
    assert ck.shape == (B, C, nck, N)
    np.testing.assert_array_equal(ck[:, :, 0], 0.0)
    for j in range(1, nck):
        np.testing.assert_allclose(ck[:, :, j], h[:, :, j * every - 1], rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(y, orc.selective_scan(u, delta, A_log, Bm, Cm, None, bias, True))


def test_scan_checkpoints_cumsum_and_memoryless():
    """Closed forms of the recorded states: the running sum of dt * u when every decay is 1
    (A_log = -30, B = 1), and the last step's dt B u when every decay is ~0 (A_log = +5)."""
    rng = np.random.default_rng(41)
    B, C, L, every = 2, 3, 64, 16
    u = rng.standard_normal((B, C, L))
    delta = rng.standard_normal((B, C, L))
    bias = rng.uniform(-3, 0, C)
    ones = np.ones((B, 1, 1, L))
    _, ck = orc.selective_scan_ckpt(u, delta, np.full((C, 1), -30.0), ones, ones, every, delta_bias=bias)
    run = np.cumsum(_softplus_lib(delta + bias[None, :, None]) * u, axis=-1)
    for j in range(1, L // every):
        np.testing.assert_allclose(ck[:, :, j, 0], run[:, :, j * every - 1], rtol=1e-9, atol=1e-9)
    dpos = rng.uniform(0.5, 2.0, (B, C, L))
    Bm = rng.standard_normal((B, 1, 2, L))
    _, ck = orc.selective_scan_ckpt(u, dpos, np.full((C, 2), 5.0), Bm, Bm, every, delta_softplus=False)
    for j in range(1, L // every):
        l = j * every - 1
        ref = dpos[:, :, l, None] * Bm[:, 0, None, :, l] * u[:, :, l, None]
        np.testing.assert_allclose(ck[:, :, j], ref, rtol=1e-12, atol=1e-14)


def test_scan_single_step_any_delta_with_softplus():
    """L = 1 has no history, so y = sum_n C dt B u + D u for any dt; dt from numpy.logaddexp."""
    rng = np.random.default_rng(12)
    B, C, N = 3, 5, 4
    u = rng.standard_normal((B, C, 1))
    delta = rng.standard_normal((B, C, 1)) * 4
    bias = rng.standard_normal(C)
    A_log = rng.standard_normal((C, N))
    Bm = rng.standard_normal((B, 1, N, 1))
    Cm = rng.standard_normal((B, 1, N, 1))
    Dv = rng.standard_normal(C)
    y = orc.selective_scan(u, delta, A_log, Bm, Cm, Dv, bias, True)
    dt = _softplus_lib(delta + bias[None, :, None])
    ref = np.sum(Cm[:, 0] * Bm[:, 0], axis=1)[:, None, :] * dt * u + Dv[None, :, None] * u
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-14)


def test_scan_state_passing_and_linearity():
    """Scanning [0, m) then [m, L) from the carried state equals one scan of [0, L); the scan
    is linear in u at fixed dt, B, C."""
    rng = np.random.default_rng(13)
    B, C, G, N, L, m = 2, 4, 2, 5, 50, 17
    u = rng.standard_normal((B, C, L))
    delta = rng.standard_normal((B, C, L)) * 0.5
    bias = rng.uniform(-4, -1, C)
    A_log = np.log(rng.uniform(0.5, 8, (C, N)))
    Bm = rng.standard_normal((B, G, N, L))
    Cm = rng.standard_normal((B, G, N, L))
    Dv = rng.standard_normal(C)
    full, h_full = orc.selective_scan(u, delta, A_log, Bm, Cm, Dv, bias, True, return_last_state=True)
    y1, h1 = orc.selective_scan(u[..., :m], delta[..., :m], A_log, Bm[..., :m], Cm[..., :m], Dv, bias, True,
                                return_last_state=True)
    y2, h2 = orc.selective_scan(u[..., m:], delta[..., m:], A_log, Bm[..., m:], Cm[..., m:], Dv, bias, True,
                                h0=h1, return_last_state=True)
    np.testing.assert_allclose(np.concatenate([y1, y2], -1), full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h2, h_full, rtol=1e-12, atol=1e-13)
    u2 = rng.standard_normal((B, C, L))
    a, b = 0.75, -2.5
    lhs = orc.selective_scan(a * u + b * u2, delta, A_log, Bm, Cm, Dv, bias, True)
    rhs = a * full + b * orc.selective_scan(u2, delta, A_log, Bm, Cm, Dv, bias, True)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------
# projections and the full core
# ----------------------------------------------------------------------------

def test_x_proj_and_dt_proj_match_einsum():
    rng = np.random.default_rng(14)
    B, D, L, R, N = 2, 5, 7, 3, 2
    xs = rng.standard_normal((B, 4, D, L))
    wx = rng.standard_normal((4, R + 2 * N, D))
    wdt = rng.standard_normal((4, D, R))
    x_dbl = orc.x_proj(xs, wx)
    np.testing.assert_allclose(x_dbl, np.einsum("bkdl,kcd->bkcl", xs, wx), rtol=1e-13, atol=1e-13)
    dts = orc.dt_proj(x_dbl, wdt, N)
    np.testing.assert_allclose(dts, np.einsum("bkrl,kdr->bkdl", x_dbl[:, :, :R], wdt), rtol=1e-13, atol=1e-13)


def _core_inputs(rng, B, D, H, W, N):
    L = H * W
    return dict(
        x=rng.standard_normal((B, D, H, W)),
        dts=rng.standard_normal((B, 4, D, L)) * 0.5,
        Bs=rng.standard_normal((B, 4, N, L)),
        Cs=rng.standard_normal((B, 4, N, L)),
        A_logs=np.log(rng.uniform(0.5, 6.0, (4 * D, N))),
        Ds=rng.standard_normal(4 * D),
        dt_bias=rng.uniform(-5, -1, 4 * D),
    )


def _only_direction(inp, k, D):
    """Zero C and D of every direction but k, so the merge sees only direction k."""
    out = {key: v.copy() for key, v in inp.items()}
    for j in range(4):
        if j != k:
            out["Cs"][:, j] = 0.0
            out["Ds"][j * D:(j + 1) * D] = 0.0
    return out


def _core(inp):
    return orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"],
                            Bs=inp["Bs"], Cs=inp["Cs"])


def test_core_is_sum_of_single_directions():
    rng = np.random.default_rng(15)
    B, D, H, W, N = 2, 3, 4, 5, 3
    inp = _core_inputs(rng, B, D, H, W, N)
    full = _core(inp)
    parts = sum(_core(_only_direction(inp, k, D)) for k in range(4))
    np.testing.assert_allclose(full, parts, rtol=1e-12, atol=1e-12)


def test_core_reverse_direction_is_flip_of_forward():
    """Direction 2 on the spatially flipped input, given direction 0's parameters, equals the
    flip of direction 0's output (and likewise 3 against 1): the reverse scans change the
    recursion direction only (VSSD article, section 2.2)."""
    rng = np.random.default_rng(16)
    B, D, H, W, N = 1, 2, 3, 5, 4
    inp = _core_inputs(rng, B, D, H, W, N)
    for fwd, rev in ((0, 2), (1, 3)):
        a = _only_direction(inp, fwd, D)
        b = {key: v.copy() for key, v in a.items()}
        b["x"] = inp["x"][:, :, ::-1, ::-1].copy()
        for key in ("dts", "Bs", "Cs"):
            b[key][:, rev] = a[key][:, fwd]
            b[key][:, fwd] = 0.0
        for key in ("A_logs", "Ds", "dt_bias"):
            b[key][rev * D:(rev + 1) * D] = a[key][fwd * D:(fwd + 1) * D]
        b["Ds"][fwd * D:(fwd + 1) * D] = 0.0
        ya = _core(a)
        yb = _core(b)
        np.testing.assert_allclose(yb, ya[:, :, ::-1, ::-1], rtol=1e-12, atol=1e-13)


def test_core_vertical_direction_is_horizontal_on_transpose():
    """Direction 1 on x equals direction 0 on x^T (H and W swapped), transposed back."""
    rng = np.random.default_rng(17)
    B, D, H, W, N = 2, 2, 3, 4, 3
    inp = _core_inputs(rng, B, D, H, W, N)
    a = _only_direction(inp, 1, D)
    b = {key: v.copy() for key, v in a.items()}
    b["x"] = np.swapaxes(inp["x"], 2, 3).copy()
    for key in ("dts", "Bs", "Cs"):
        b[key][:, 0] = a[key][:, 1]
        b[key][:, 1] = 0.0
    for key in ("A_logs", "Ds", "dt_bias"):
        b[key][0:D] = a[key][D:2 * D]
    b["Ds"][D:2 * D] = 0.0
    np.testing.assert_allclose(np.swapaxes(_core(b), 2, 3), _core(a), rtol=1e-12, atol=1e-13)


def test_core_identity_scan_gives_four_x():
    """C = 0 and D = 1 make the scan the identity: the core returns 4x exactly."""
    rng = np.random.default_rng(18)
    B, D, H, W, N = 2, 3, 5, 4, 2
    inp = _core_inputs(rng, B, D, H, W, N)
    inp["x"] = rng.integers(-500, 500, (B, D, H, W)).astype(np.float64)
    inp["Cs"][:] = 0.0
    inp["Ds"][:] = 1.0
    np.testing.assert_array_equal(_core(inp), 4 * inp["x"])


def test_core_with_projections_matches_einsum_composition():
    """The projection path equals the given-dts path fed with einsum-computed projections."""
    rng = np.random.default_rng(19)
    B, D, H, W, N, R = 2, 4, 3, 5, 2, 3
    L = H * W
    x = rng.standard_normal((B, D, H, W))
    wx = rng.standard_normal((4, R + 2 * N, D)) * 0.4
    wdt = rng.standard_normal((4, D, R)) * 0.5
    A_logs = np.log(rng.uniform(0.5, 4.0, (4 * D, N)))
    Ds = rng.standard_normal(4 * D)
    bias = rng.uniform(-4, -1, 4 * D)
    got = orc.forward_core(x, A_logs, Ds, bias, x_proj_weight=wx, dt_projs_weight=wdt)
    hw = x.reshape(B, D, L)
    wh = np.swapaxes(x, 2, 3).reshape(B, D, L)
    xs = np.stack([hw, wh, hw[:, :, ::-1], wh[:, :, ::-1]], axis=1)
    x_dbl = np.einsum("bkdl,kcd->bkcl", xs, wx)
    dts = np.einsum("bkrl,kdr->bkdl", x_dbl[:, :, :R], wdt)
    ref = orc.forward_core(x, A_logs, Ds, bias, dts=dts, Bs=x_dbl[:, :, R:R + N], Cs=x_dbl[:, :, R + N:])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
