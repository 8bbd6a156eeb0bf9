"""Pins of the oracle's receiver-sorted edge convolution (Sec. 4 Eq. 1, App. D
layout) and its VJP (App. C Eq. C1) to closed forms, symmetry properties and
finite differences.  FlashCart, arXiv 2610.06409."""
import numpy as np
import pytest

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from test_oracle_tensors import rand_rot, rotate_dense

RNG = np.random.default_rng(7)


def small_graph(n=6, k=3, seed=0):
    pos, ei, ev = W.random_graph(n, k, 3.0, seed)
    return ei, ev.astype(np.float64)


def layout(lmax, sum_paths=False):
    ps = O.paths(lmax, lmax, lmax)
    Pl = [sum(1 for p in ps if p[2] == l) for l in range(lmax + 1)]
    eta = []
    seen = [0] * (lmax + 1)
    for p in ps:
        eta.append(seen[p[2]])
        seen[p[2]] += 1
    off, o = [], 0
    for l in range(lmax + 1):
        off.append(o)
        o += (2 * l + 1) * (1 if sum_paths else Pl[l])
    return ps, Pl, eta, off, o


def test_closed_form_paths_and_layout():
    """(0,l)->l gives x_0 T_l(r), (l,0)->l gives x_l and (1,1)->0 gives the
    dot product x_1 . r-hat (normalisation T (x) T -> T); check them at the
    App. D offsets off(l) + (c P_l + eta) C + k."""
    L, C, N = 3, 3, 5
    ei, ev = small_graph(N, 2, 1)
    E = ei.shape[1]
    x = RNG.normal(size=(N, (L + 1) ** 2 * C))
    w = RNG.normal(size=(E, 23, C))
    z = O.edge_conv(L, L, L, C, ei, ev, x, w, N)
    ps, Pl, eta, off, zr = layout(L)
    xr = x.reshape(N, (L + 1) ** 2, C)
    zz = z.reshape(N, zr, C)
    for p, (l1, l2, l3) in enumerate(ps):
        if not ((l1 == 0 and l2 == l3) or (l2 == 0 and l1 == l3)
                or (l1, l2, l3) == (1, 1, 0)):
            continue
        ref = np.zeros((N, 2 * l3 + 1, C))
        for e in range(E):
            u, v = ei[0, e], ei[1, e]
            r = ev[e]
            rh = r / np.linalg.norm(r)
            if l1 == 0:
                f = xr[v, 0][None, :] * O.direction(l2, r)[:, None]
            elif l2 == 0:
                f = xr[v, l1 * l1:l1 * l1 + 2 * l1 + 1]
            else:
                f = (rh[:, None] * xr[v, 1:4]).sum(0)[None, :]
            ref[u] += w[e, p][None, :] * f
        got = np.stack([zz[:, off[l3] + c * Pl[l3] + eta[p]]
                        for c in range(2 * l3 + 1)], axis=1)
        np.testing.assert_allclose(got, ref, atol=1e-12)


def test_direction_l1_closed_form_is_rhat():
    r = RNG.normal(size=3)
    np.testing.assert_allclose(O.direction(1, r), r / np.linalg.norm(r),
                               atol=1e-15)


def rotate_features(R, feat, lmax, C, blocks=None):
    """feat [N][rows*C] in node layout (P_l = 1) -> rotated copy."""
    N = feat.shape[0]
    f = feat.reshape(N, -1, C).copy()
    out = np.empty_like(f)
    rows = blocks if blocks is not None else [(l, l * l, 1) for l in range(lmax + 1)]
    for (l, start, P) in rows:
        for n in range(N):
            for eta in range(P):
                for k in range(C):
                    comps = f[n, start + np.arange(2 * l + 1) * P + eta, k]
                    d = rotate_dense(R, O.stf_dense(l, comps))
                    out[n, start + np.arange(2 * l + 1) * P + eta, k] = \
                        O.stf_extract(l, d)
    return out.reshape(N, -1)


@pytest.mark.parametrize("reflect", [False, True])
def test_layer_equivariance(reflect):
    L, C, N = 2, 2, 5
    ei, ev = small_graph(N, 3, 2)
    E = ei.shape[1]
    x = RNG.normal(size=(N, (L + 1) ** 2 * C))
    w = RNG.normal(size=(E, 11, C))
    R = rand_rot(RNG, reflect)
    z = O.edge_conv(L, L, L, C, ei, ev, x, w, N)
    zr = O.edge_conv(L, L, L, C, ei, ev @ R.T, rotate_features(R, x, L, C), w, N)
    ps, Pl, eta, off, _ = layout(L)
    blocks = [(l, off[l], Pl[l]) for l in range(L + 1)]
    np.testing.assert_allclose(zr, rotate_features(R, z, L, C, blocks),
                               atol=1e-10 * np.abs(z).max())


def test_edge_order_invariance_sum_paths_and_parity():
    L, C, N = 2, 3, 6
    ei, ev = small_graph(N, 3, 3)
    E = ei.shape[1]
    x = RNG.normal(size=(N, 9 * C))
    w = RNG.normal(size=(E, 11, C))
    z = O.edge_conv(L, L, L, C, ei, ev, x, w, N)
    perm = RNG.permutation(E)
    z2 = O.edge_conv(L, L, L, C, ei[:, perm], ev[perm], x, w[perm], N)
    np.testing.assert_allclose(z2, z, atol=1e-12)
    # summed paths = sum over eta of the separate outputs
    zs = O.edge_conv(L, L, L, C, ei, ev, x, w, N, sum_paths=True)
    ps, Pl, eta, off, zr = layout(L)
    zz = z.reshape(N, zr, C)
    ref = np.zeros((N, 9, C))
    for l in range(L + 1):
        for c in range(2 * l + 1):
            ref[:, l * l + c] = zz[:, off[l] + c * Pl[l]:off[l] + (c + 1) * Pl[l]].sum(1)
    np.testing.assert_allclose(zs.reshape(N, 9, C), ref, atol=1e-12)
    # inverting every edge vector scales path (l1,l2)->l3 by (-1)^l2
    zn = O.edge_conv(L, L, L, C, ei, -ev, x, w, N).reshape(N, zr, C)
    for p, (l1, l2, l3) in enumerate(ps):
        for c in range(2 * l3 + 1):
            s = off[l3] + c * Pl[l3] + eta[p]
            np.testing.assert_allclose(zn[:, s], (-1) ** l2 * zz[:, s], atol=1e-12)


def test_empty_and_isolated_receivers():
    L, C, N = 2, 2, 4
    ei = np.array([[1, 1], [0, 2]], dtype=np.int32)
    ev = RNG.normal(size=(2, 3))
    x = RNG.normal(size=(N, 9 * C))
    w = RNG.normal(size=(2, 11, C))
    z = O.edge_conv(L, L, L, C, ei, ev, x, w, N)
    assert np.all(z[[0, 2, 3]] == 0) and np.abs(z[1]).max() > 0
    z0 = O.edge_conv(L, L, L, C, np.zeros((2, 0), np.int32), np.zeros((0, 3)),
                     x, np.zeros((0, 11, C)), N)
    assert z0.shape == (N, 35 * C) and np.all(z0 == 0)


def test_receiver_mask_selects_rows():
    L, C, N = 2, 2, 6
    ei, ev = small_graph(N, 3, 4)
    x = RNG.normal(size=(N, 9 * C))
    w = RNG.normal(size=(ei.shape[1], 11, C))
    z = O.edge_conv(L, L, L, C, ei, ev, x, w, N)
    m = np.zeros(N, np.uint8)
    m[[1, 4]] = 1
    zm = O.edge_conv(L, L, L, C, ei, ev, x, w, N, recv_mask=m)
    np.testing.assert_allclose(zm[[1, 4]], z[[1, 4]], atol=0)
    assert np.all(zm[[0, 2, 3, 5]] == 0)


# ---------------------------------------------------------------------------
# VJP (App. C Eq. C1) against finite differences
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L,sum_paths", [(2, False), (3, False), (2, True)])
def test_vjp_finite_differences(L, sum_paths):
    C, N = 2, 5
    ei, ev = small_graph(N, 2, 5)
    E = ei.shape[1]
    P = len(O.paths(L, L, L))
    x = RNG.normal(size=(N, (L + 1) ** 2 * C))
    w = RNG.normal(size=(E, P, C))
    zr = O.zrow(L, L, L, sum_paths)
    g = RNG.normal(size=(N, zr * C))

    def loss(x_, w_, ev_):
        return float((O.edge_conv(L, L, L, C, ei, ev_, x_, w_, N,
                                  sum_paths=sum_paths) * g).sum())
    xb, wb, rb = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, g, N,
                                 sum_paths=sum_paths)
    # x and w enter bilinearly: central differences are exact up to rounding
    h = 1e-3
    for _ in range(6):
        i = RNG.integers(x.size)
        d = np.zeros(x.size); d[i] = h
        fd = (loss(x + d.reshape(x.shape), w, ev) - loss(x - d.reshape(x.shape), w, ev)) / (2 * h)
        assert abs(fd - xb.ravel()[i]) < 1e-9 * max(1, abs(fd))
        j = RNG.integers(w.size)
        d = np.zeros(w.size); d[j] = h
        fd = (loss(x, w + d.reshape(w.shape), ev) - loss(x, w - d.reshape(w.shape), ev)) / (2 * h)
        assert abs(fd - wb.ravel()[j]) < 1e-9 * max(1, abs(fd))
    h = 1e-5
    for e in range(E):
        for b in range(3):
            d = np.zeros_like(ev); d[e, b] = h
            fd = (loss(x, w, ev + d) - loss(x, w, ev - d)) / (2 * h)
            assert abs(fd - rb[e, b]) < 1e-6 * max(1, abs(fd))
    # the direction tensors depend on r-hat only: r_bar . r = 0
    np.testing.assert_allclose((rb * ev).sum(1), 0.0, atol=1e-9)


def test_vjp_edge_mask_is_partial_sum():
    L, C, N = 2, 2, 5
    ei, ev = small_graph(N, 3, 6)
    E = ei.shape[1]
    x = RNG.normal(size=(N, 9 * C))
    w = RNG.normal(size=(E, 11, C))
    g = RNG.normal(size=(N, 35 * C))
    full = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, g, N)
    m = np.zeros(E, np.uint8); m[::2] = 1
    a = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, g, N, edge_mask=m)
    b = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, g, N, edge_mask=1 - m)
    for fa, fb, ff in zip(a, b, full):
        np.testing.assert_allclose(fa + fb, ff, atol=1e-12)
