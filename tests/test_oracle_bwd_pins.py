"""Pins of the oracle's gradient (oracle_selective_scan_bwd, oracle_forward_core_bwd).

The gradient oracle is checked against things other than itself:
  - central finite differences of the (separately pinned) forward oracle, for
    every input of the scan and of the core, with softplus on and off;
  - closed forms of two special cases where the recurrence collapses: the
    cumulative sum (A ~ 0, N = 1, B = C = 1) and the memoryless scan (decay ~ 0).
A dropped term, a wrong sign, a transposed index or a missed sum over a group's
channels changes at least one of these.
"""
import numpy as np
import pytest

from oracle import oracle as orc


def _scan_inputs(rng, B, C, G, N, L, softplus_on):
    # Without softplus the step size is dt + bias itself, which must stay positive for the
    # decays exp(dt A) to stay below one; draw both positive there.
    if softplus_on:
        delta, bias = rng.normal(scale=0.7, size=(B, C, L)), rng.normal(scale=0.5, size=C)
    else:
        delta, bias = rng.uniform(0.05, 1.0, size=(B, C, L)), rng.uniform(0.0, 0.3, size=C)
    return dict(u=rng.normal(size=(B, C, L)), delta=delta,
                A_log=np.log(rng.uniform(0.3, 3.0, size=(C, N))), Bm=rng.normal(size=(B, G, N, L)),
                Cm=rng.normal(size=(B, G, N, L)), Dv=rng.normal(size=C), delta_bias=bias)


def _fd_check(loss, params, grads, names, rng, eps=1e-5, max_entries=40, rtol=1e-6):
    """Central differences of loss() w.r.t. sampled entries of each named parameter array."""
    for name in names:
        p = params[name]
        flat = p.reshape(-1)
        idx = np.arange(flat.size) if flat.size <= max_entries else rng.choice(flat.size, max_entries, replace=False)
        g = grads[name].reshape(-1)
        scale = max(1.0, float(np.abs(g).max()))
        for i in idx:
            old = flat[i]
            flat[i] = old + eps
            lp = loss()
            flat[i] = old - eps
            lm = loss()
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[i]) <= rtol * scale + 1e-8 * abs(fd), (name, int(i), fd, g[i])


@pytest.mark.parametrize("softplus_on", [True, False])
@pytest.mark.parametrize("B,C,G,N,L", [(2, 4, 2, 3, 9), (1, 3, 1, 4, 6), (1, 2, 2, 1, 1)])
def test_scan_gradient_matches_finite_differences(softplus_on, B, C, G, N, L):
    rng = np.random.default_rng(100 + B * 7 + C + N + L)
    p = _scan_inputs(rng, B, C, G, N, L, softplus_on)
    w = rng.normal(size=(B, C, L))

    def loss():
        y = orc.selective_scan(p["u"], p["delta"], p["A_log"], p["Bm"], p["Cm"], p["Dv"], p["delta_bias"],
                               softplus_on)
        return float(np.sum(w * y))

    gr = orc.selective_scan_bwd(p["u"], p["delta"], p["A_log"], p["Bm"], p["Cm"], p["Dv"], p["delta_bias"],
                                softplus_on, w)
    grads = dict(u=gr["du"], delta=gr["ddelta"], A_log=gr["dA_log"], Bm=gr["dBm"], Cm=gr["dCm"], Dv=gr["dDv"],
                 delta_bias=gr["ddelta_bias"])
    _fd_check(loss, p, grads, list(grads), rng)


def test_scan_gradient_cumsum_closed_form():
    # A_log = -30 makes A ~ -1e-13, so dA = 1 to double precision; with N = 1, B = C = 1 and
    # no softplus, y_l = sum_{j<=l} delta_j u_j + D u_l.  For loss = sum(dy * y):
    #   du_l = delta_l * S_l + D dy_l,  ddelta_l = u_l * S_l,  dD = sum dy u,  with S_l = sum_{m>=l} dy_m.
    rng = np.random.default_rng(7)
    B, C, L = 2, 3, 11
    u = rng.normal(size=(B, C, L))
    delta = rng.uniform(0.1, 1.0, size=(B, C, L))
    A_log = np.full((C, 1), -30.0)
    ones = np.ones((B, 1, 1, L))
    Dv = rng.normal(size=C)
    dy = rng.normal(size=(B, C, L))
    gr = orc.selective_scan_bwd(u, delta, A_log, ones, ones, Dv, None, False, dy)
    S = np.flip(np.cumsum(np.flip(dy, -1), -1), -1)
    np.testing.assert_allclose(gr["du"], delta * S + Dv[None, :, None] * dy, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(gr["ddelta"], u * S, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(gr["dDv"], np.sum(dy * u, axis=(0, 2)), rtol=1e-12)
    np.testing.assert_allclose(gr["ddelta_bias"], np.sum(u * S, axis=(0, 2)), rtol=1e-11)
    # dB_l = sum_c S_l delta_l u_l-style terms: g_l = S_l here, so dB_l = sum_c S_l delta_l u_l
    np.testing.assert_allclose(gr["dBm"][:, 0, 0], np.sum(S * delta * u, axis=1), rtol=1e-10, atol=1e-11)
    # dC_l = sum_c dy_l h_l with h_l = cumsum(delta u)
    h = np.cumsum(delta * u, axis=-1)
    np.testing.assert_allclose(gr["dCm"][:, 0, 0], np.sum(dy * h, axis=1), rtol=1e-10, atol=1e-11)


def test_scan_gradient_memoryless_closed_form():
    # A_log = +5 (A ~ -148) with delta >= 0.5 and no softplus: dA <= e^-74, so every state is
    # only its own step's input: h_l = delta_l B_l u_l, y_l = sum_n C_l delta_l B_l u_l + D u_l.
    rng = np.random.default_rng(8)
    B, C, G, N, L = 1, 4, 2, 3, 7
    u = rng.normal(size=(B, C, L))
    delta = rng.uniform(0.5, 1.5, size=(B, C, L))
    A_log = np.full((C, N), 5.0)
    Bm = rng.normal(size=(B, G, N, L))
    Cm = rng.normal(size=(B, G, N, L))
    Dv = rng.normal(size=C)
    dy = rng.normal(size=(B, C, L))
    gr = orc.selective_scan_bwd(u, delta, A_log, Bm, Cm, Dv, None, False, dy)
    grp = np.arange(C) // (C // G)
    Bc, Cc = Bm[:, grp], Cm[:, grp]                  # (B, C, N, L)
    CB = np.sum(Cc * Bc, axis=2)                     # (B, C, L)
    np.testing.assert_allclose(gr["du"], CB * delta * dy + Dv[None, :, None] * dy, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr["ddelta"], CB * u * dy, rtol=1e-12, atol=1e-12)
    dBc = Cc * (delta * u * dy)[:, :, None, :]
    dCc = Bc * (delta * u * dy)[:, :, None, :]
    for g in range(G):
        np.testing.assert_allclose(gr["dBm"][:, g], dBc[:, grp == g].sum(1), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(gr["dCm"][:, g], dCc[:, grp == g].sum(1), rtol=1e-12, atol=1e-12)
    assert np.all(np.abs(gr["dA_log"]) < 1e-20)


@pytest.mark.parametrize("softplus_on", [True, False])
@pytest.mark.parametrize("B,D,H,W,N", [(1, 3, 3, 4, 2), (2, 2, 2, 3, 3)])
def test_core_gradient_matches_finite_differences(softplus_on, B, D, H, W, N):
    rng = np.random.default_rng(200 + D * H * W + N)
    L = H * W
    s = _scan_inputs(rng, B, 4 * D, 4, N, L, softplus_on)
    p = dict(x=rng.normal(size=(B, D, H, W)), dts=s["delta"].reshape(B, 4, D, L), A_logs=s["A_log"],
             Bs=s["Bm"], Cs=s["Cm"], Ds=s["Dv"], dt_bias=s["delta_bias"])
    w = rng.normal(size=(B, D, H, W))

    def loss():
        y = orc.forward_core(p["x"], p["A_logs"], p["Ds"], p["dt_bias"], dts=p["dts"], Bs=p["Bs"], Cs=p["Cs"],
                             delta_softplus=softplus_on)
        return float(np.sum(w * y))

    gr = orc.forward_core_bwd(p["x"], p["A_logs"], p["Ds"], p["dt_bias"], p["dts"], p["Bs"], p["Cs"], w,
                              delta_softplus=softplus_on)
    grads = dict(x=gr["dx"], dts=gr["ddts"], A_logs=gr["dA_logs"], Bs=gr["dBs"], Cs=gr["dCs"], Ds=gr["dDs"],
                 dt_bias=gr["ddt_bias"])
    _fd_check(loss, p, grads, list(grads), rng, max_entries=30)


@pytest.mark.parametrize("softplus_on", [True, False])
@pytest.mark.parametrize("B,D,H,W,N,R", [(1, 3, 3, 4, 2, 1), (2, 2, 2, 3, 3, 2)])
def test_core_projection_gradient_matches_finite_differences(softplus_on, B, D, H, W, N, R):
    # The projection form: the gradient reaches x through both u and x_proj, and the
    # weights of x_proj and dt_proj through dts, B and C.
    rng = np.random.default_rng(300 + D * H * W + N + R)
    Cp = R + 2 * N
    p = dict(x=rng.normal(size=(B, D, H, W)), x_proj_weight=rng.normal(scale=0.5, size=(4, Cp, D)),
             dt_projs_weight=rng.normal(scale=0.5, size=(4, D, R)), A_logs=np.log(rng.uniform(0.3, 3.0, size=(4 * D, N))),
             Ds=rng.normal(size=4 * D), dt_bias=rng.normal(scale=0.5, size=4 * D))
    if not softplus_on:
        # without softplus the step is dt_proj(x_dbl) + bias itself; a large bias keeps it positive
        p["dt_bias"] = rng.uniform(4.0, 5.0, size=4 * D)
        p["dt_projs_weight"] = rng.uniform(-0.05, 0.05, size=(4, D, R))
        p["x_proj_weight"][:, :R] *= 0.1
    w = rng.normal(size=(B, D, H, W))

    def loss():
        y = orc.forward_core(p["x"], p["A_logs"], p["Ds"], p["dt_bias"], x_proj_weight=p["x_proj_weight"],
                             dt_projs_weight=p["dt_projs_weight"], delta_softplus=softplus_on)
        return float(np.sum(w * y))

    gr = orc.forward_core_proj_bwd(p["x"], p["x_proj_weight"], p["dt_projs_weight"], p["A_logs"], p["Ds"],
                                   p["dt_bias"], w, delta_softplus=softplus_on)
    grads = dict(x=gr["dx"], x_proj_weight=gr["dx_proj_weight"], dt_projs_weight=gr["ddt_projs_weight"],
                 A_logs=gr["dA_logs"], Ds=gr["dDs"], dt_bias=gr["ddt_bias"])
    _fd_check(loss, p, grads, list(grads), rng, max_entries=40)


def test_core_projection_gradient_intermediates():
    # The intermediate gradients are those of the dts/Bs/Cs form at the projected inputs, and
    # the weight gradients are their contractions: with every x_proj row but one zero, the
    # gradient of that row is the intermediate gradient of its slot summed against xs.
    rng = np.random.default_rng(41)
    B, D, H, W, N, R = 1, 2, 2, 3, 2, 1
    L = H * W
    x = rng.normal(size=(B, D, H, W))
    Wx = rng.normal(scale=0.5, size=(4, R + 2 * N, D))
    Wdt = rng.normal(scale=0.5, size=(4, D, R))
    A_logs, Ds, bias = np.log(rng.uniform(0.3, 3.0, size=(4 * D, N))), rng.normal(size=4 * D), rng.normal(size=4 * D)
    dy = rng.normal(size=(B, D, H, W))
    gr = orc.forward_core_proj_bwd(x, Wx, Wdt, A_logs, Ds, bias, dy)
    xs = orc.cross_scan(x)
    # dBs[b,k,n,l] pairs with x_dbl row R + n; its weight gradient is sum_l dBs * xs
    for k in range(4):
        for n in range(N):
            want = np.einsum("l,dl->d", gr["dBs"][0, k, n], xs[0, k])
            np.testing.assert_allclose(gr["dx_proj_weight"][k, R + n], want, rtol=1e-12, atol=1e-12)
    assert gr["ddts"].shape == (B, 4, D, L)


def test_scan_gradient_hand_derived_two_step_case():
    """The two-step scan of the fixture two_step_scan_gradient.txt, its output and every
    gradient derived by hand (values a + b*exp(-1))."""
    import math
    import os

    fx = {}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "two_step_scan_gradient.txt")
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            fx[k] = [float(t) for t in v]
    e = math.exp(-1.0)
    val = lambda k: np.array([a + b * e for a, b in zip(fx[k][0::2], fx[k][1::2])])
    u = np.array([1.0, 2.0]).reshape(1, 1, 2)
    delta = np.array([0.5, 1.0]).reshape(1, 1, 2)
    Bm = np.array([2.0, 1.0]).reshape(1, 1, 1, 2)
    Cm = np.array([1.0, 3.0]).reshape(1, 1, 1, 2)
    A_log, Dv, bias = np.zeros((1, 1)), np.array([0.5]), np.zeros(1)
    dy = np.ones((1, 1, 2))
    y = orc.selective_scan(u, delta, A_log, Bm, Cm, Dv, bias, False)
    np.testing.assert_allclose(y.reshape(-1), val("y"), rtol=1e-14)
    g = orc.selective_scan_bwd(u, delta, A_log, Bm, Cm, Dv, bias, False, dy)
    for key, fkey in [("du", "du"), ("dBm", "dB"), ("dCm", "dC"), ("ddelta", "ddelta"), ("ddelta_bias", "dbias"),
                      ("dA_log", "dA_log"), ("dDv", "dD")]:
        np.testing.assert_allclose(g[key].reshape(-1), val(fkey), rtol=1e-13, atol=1e-15, err_msg=key)
