"""Pins of the oracle's VJP-of-VJP (FlashCart App. C Eq. C2 and the
direction-tensor derivatives that force training needs, paragraph after
Eq. C2) against things other than itself:

* the Hessian-vector product of <ybar, T_l(r/|r|)> against central
  differences of the analytic Jacobian (pinned in test_oracle_tensors),
  against the homogeneity identity H r = -grad (T_l depends on r/|r| only)
  and against symmetry;
* the whole VJP-of-VJP as the gradient of
  L = <vx, x_bar> + <vw, w_bar> + <vr, r_bar> built from the oracle's
  (pinned) VJP: L is linear in g, x and w, so central differences along
  random directions are exact up to rounding; along the edge vectors a
  central difference with a small step;
* special cases that reduce to the forward convolution: with only vx the
  g-gradient is the forward of vx, with only vw it is the forward with
  weights vw."""
import numpy as np
import pytest

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O


def rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("l", [1, 2, 3, 4])
def test_hvp_matches_differences_of_the_jacobian(l):
    g = rng(10 + l)
    for _ in range(3):
        r = g.normal(size=3) * 1.7
        yb = g.normal(size=2 * l + 1)
        v = g.normal(size=3)
        h = 1e-5
        jp = O.direction_jac(l, r + h * v).T @ yb
        jm = O.direction_jac(l, r - h * v).T @ yb
        fd = (jp - jm) / (2 * h)
        hv = O.direction_hvp(l, r, yb, v)
        assert np.max(np.abs(hv - fd)) <= 1e-7 * max(1.0, np.max(np.abs(fd)))


@pytest.mark.parametrize("l", [1, 2, 3, 4])
def test_hvp_homogeneity_and_symmetry(l):
    g = rng(20 + l)
    r = g.normal(size=3) * 0.9
    yb = g.normal(size=2 * l + 1)
    grad = O.direction_jac(l, r).T @ yb
    # F(lambda r) = F(r)  =>  H r = -grad F
    np.testing.assert_allclose(O.direction_hvp(l, r, yb, r), -grad, atol=1e-12 * (1 + np.abs(grad).max()))
    a, b = g.normal(size=3), g.normal(size=3)
    np.testing.assert_allclose(a @ O.direction_hvp(l, r, yb, b), b @ O.direction_hvp(l, r, yb, a),
                               rtol=1e-12, atol=1e-12)


def vjp_functional(wl, L, C, g, x, w, vec, cot, sum_paths):
    """L = <vx, x_bar> + <vw, w_bar> + <vr, r_bar> from the oracle VJP."""
    xb, wb, rb = O.edge_conv_vjp(L, L, L, C, wl["edge_index"], vec, x, w, g, wl["n_nodes"],
                                 sum_paths=sum_paths)
    tot = 0.0
    if cot.get("vx") is not None:
        tot += np.sum(np.asarray(cot["vx"], np.float64) * xb)
    if cot.get("vw") is not None:
        tot += np.sum(np.asarray(cot["vw"], np.float64).reshape(wb.shape) * wb)
    if cot.get("vr") is not None:
        tot += np.sum(np.asarray(cot["vr"], np.float64) * rb)
    return tot


def small_case(L, C, sum_paths, seed):
    wl = W.tiny(seed)
    E = wl["edge_index"].shape[1]
    d = W.conv_inputs(wl["n_nodes"], wl["edge_index"], L, C, seed + 7, with_grad=True,
                      sum_paths=sum_paths)
    cot = W.cotangents(wl["n_nodes"], E, L, C, seed + 8, wl["edge_vec"])
    return wl, d, cot


@pytest.mark.parametrize("L,C,sum_paths", [(2, 3, False), (3, 2, False), (3, 2, True)])
def test_vvjp_is_the_gradient_of_the_vjp_functional(L, C, sum_paths):
    wl, d, cot = small_case(L, C, sum_paths, 31 + L)
    x = d["x"].astype(np.float64)
    w = d["w"].astype(np.float64)
    g0 = d["g"].astype(np.float64)
    vec = wl["edge_vec"].astype(np.float64)
    gh, xh, wh, rh = O.edge_conv_vjp_vjp(L, L, L, C, wl["edge_index"], vec, x, w, g0,
                                         cot["vx"], cot["vw"], cot["vr"], wl["n_nodes"],
                                         sum_paths=sum_paths)
    F = lambda g=g0, x=x, w=w, vec=vec: vjp_functional(wl, L, C, g, x, w, vec, cot, sum_paths)
    r = rng(L + 100)
    for _ in range(2):
        # linear in g, x and w: a central difference with step 1 is exact
        dg = r.normal(size=g0.shape)
        lhs = (F(g=g0 + dg) - F(g=g0 - dg)) / 2
        assert abs(lhs - np.sum(gh * dg)) <= 1e-9 * max(1.0, abs(lhs))
        dx = r.normal(size=x.shape)
        lhs = (F(x=x + dx) - F(x=x - dx)) / 2
        assert abs(lhs - np.sum(xh * dx)) <= 1e-9 * max(1.0, abs(lhs))
        dw = r.normal(size=w.shape)
        lhs = (F(w=w + dw) - F(w=w - dw)) / 2
        assert abs(lhs - np.sum(wh * dw)) <= 1e-9 * max(1.0, abs(lhs))
        # nonlinear in the edge vectors
        dr = r.normal(size=vec.shape)
        h = 1e-6
        lhs = (F(vec=vec + h * dr) - F(vec=vec - h * dr)) / (2 * h)
        assert abs(lhs - np.sum(rh * dr)) <= 1e-6 * max(1.0, abs(lhs))


def test_vvjp_special_cases_reduce_to_the_forward():
    L, C = 2, 4
    wl, d, cot = small_case(L, C, False, 5)
    ei, ev, N = wl["edge_index"], wl["edge_vec"], wl["n_nodes"]
    # only vx: g_hat = sum_e w f(vx, y) = the forward of vx; x_hat = 0
    gh, xh, wh, rh = O.edge_conv_vjp_vjp(L, L, L, C, ei, ev, d["x"], d["w"], d["g"],
                                         cot["vx"], None, None, N)
    z = O.edge_conv(L, L, L, C, ei, ev, cot["vx"], d["w"], N)
    np.testing.assert_allclose(gh, z, rtol=1e-12, atol=1e-12)
    assert np.all(xh == 0)
    # its w_hat is the first VJP's w_bar taken at x := vx
    _, wb, _ = O.edge_conv_vjp(L, L, L, C, ei, ev, cot["vx"], d["w"], d["g"], N)
    np.testing.assert_allclose(wh, wb, rtol=1e-12, atol=1e-12)
    # only vw: g_hat = the forward with weights vw; w_hat = 0
    gh, xh, wh, rh = O.edge_conv_vjp_vjp(L, L, L, C, ei, ev, d["x"], d["w"], d["g"],
                                         None, cot["vw"], None, N)
    z = O.edge_conv(L, L, L, C, ei, ev, d["x"], cot["vw"], N)
    np.testing.assert_allclose(gh, z, rtol=1e-12, atol=1e-12)
    assert np.all(wh == 0)
    # and its x_hat is the first VJP's x_bar with weights vw
    xb, _, _ = O.edge_conv_vjp(L, L, L, C, ei, ev, d["x"], cot["vw"], d["g"], N)
    np.testing.assert_allclose(xh, xb, rtol=1e-12, atol=1e-12)


def test_vvjp_edge_mask_selects_edges():
    L, C = 2, 2
    wl, d, cot = small_case(L, C, False, 9)
    E = wl["edge_index"].shape[1]
    m = np.zeros(E, np.uint8)
    m[::3] = 1
    full = O.edge_conv_vjp_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], d["x"], d["w"],
                               d["g"], cot["vx"], cot["vw"], cot["vr"], wl["n_nodes"])
    part = O.edge_conv_vjp_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], d["x"], d["w"],
                               d["g"], cot["vx"], cot["vw"], cot["vr"], wl["n_nodes"],
                               edge_mask=m)
    sel = m.astype(bool)
    np.testing.assert_allclose(part[2][sel], full[2][sel], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(part[3][sel], full[3][sel], rtol=1e-12, atol=1e-12)
    assert np.all(part[2][~sel] == 0) and np.all(part[3][~sel] == 0)
