"""Pins of the oracle's odd-J (parity-changing) products and convolution.

FlashCart (arXiv 2610.06409) App. B, paragraph after Eq. (B1), and Sec. 7
"Limitations": the symbolic construction extends to products of opposite
parity by one Levi-Civita contraction, with parity tracked explicitly.  The
pages print no formula, so the oracle takes the plain reading: contract
n = (l1 + l2 - l3 - 1)/2 index pairs, one index of each input through
epsilon, then the symmetric trace-free part with no further factor.  These
tests tie that reading to things other than its own code: the cross
product, the axial vector of a commutator, the generator of rotations,
symmetry and tracelessness, O(3) equivariance with the det(R) of a
pseudo-tensor, exchange antisymmetry, and central differences of the
convolution's VJP."""
import itertools

import numpy as np
import pytest

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from test_oracle_tensors import is_symmetric, max_trace, rand_rot, rotate_dense

RNG = np.random.default_rng(11)


def odd_paths(L):
    return [(a, b, c) for (a, b, c) in itertools.product(range(L + 1), repeat=3)
            if O.odd_admissible(a, b, c)]


def test_path_rule_and_counts():
    """l1, l2 >= 1, |l1 - l2| <= l3 <= l1 + l2 - 1, l1 + l2 + l3 odd; no
    pseudoscalar outputs (l3 = 0 would need l1 = l2 and an odd sum)."""
    for (a, b, c) in itertools.product(range(5), repeat=3):
        expect = a >= 1 and b >= 1 and abs(a - b) <= c <= a + b - 1 and (a + b + c) % 2 == 1
        assert O.odd_admissible(a, b, c) == expect
    assert all(c > 0 for (_, _, c) in odd_paths(4))
    assert [len(O.paths(L, L, L, odd=True)) for L in (1, 2, 3, 4)] == [1, 4, 11, 23]
    assert O.paths(3, 3, 3, odd=True)[0] == (1, 1, 1)


def test_vector_vector_is_the_cross_product():
    for _ in range(5):
        x, y = RNG.normal(size=3), RNG.normal(size=3)
        np.testing.assert_allclose(O.product_odd(1, 1, 1, x, y), np.cross(x, y), atol=1e-14)


def test_rank2_rank2_to_vector_is_the_commutator_axial_vector():
    """(2,2)->1: one pair contracted, one through epsilon: the axial vector
    of X Y, i.e. (M12 - M21, M20 - M02, M01 - M10) with M = X Y."""
    for _ in range(5):
        xc, yc = RNG.normal(size=5), RNG.normal(size=5)
        M = O.stf_dense(2, xc) @ O.stf_dense(2, yc)
        ref = np.array([M[1, 2] - M[2, 1], M[2, 0] - M[0, 2], M[0, 1] - M[1, 0]])
        np.testing.assert_allclose(O.product_odd(2, 2, 1, xc, yc), ref, atol=1e-13)


def rodrigues(n, t):
    """Rotation by angle t about the unit axis n (right-hand rule)."""
    n = n / np.linalg.norm(n)
    K = np.array([[0.0, -n[2], n[1]], [n[2], 0.0, -n[0]], [-n[1], n[0], 0.0]])
    return np.eye(3) + np.sin(t) * K + (1.0 - np.cos(t)) * (K @ K)


@pytest.mark.parametrize("l", [1, 2, 3, 4, 5])
def test_rank_l_with_vector_is_the_rotation_generator(l):
    """(l,1)->l with a unit vector n equals -(1/l) d/dt [R_n(t) x] at t = 0
    (central differences of the dense rotation; no Levi-Civita symbol)."""
    xc = RNG.normal(size=2 * l + 1)
    n = RNG.normal(size=3)
    n /= np.linalg.norm(n)
    xd = O.stf_dense(l, xc)
    h = 1e-5
    d = (rotate_dense(rodrigues(n, h), xd) - rotate_dense(rodrigues(n, -h), xd)) / (2 * h)
    ref = -O.stf_extract(l, d) / l
    np.testing.assert_allclose(O.product_odd(l, 1, l, xc, n), ref, atol=1e-8)


@pytest.mark.parametrize("path", odd_paths(4))
def test_outputs_are_stf_and_exchange_antisymmetric(path):
    l1, l2, l3 = path
    x, y = RNG.normal(size=2 * l1 + 1), RNG.normal(size=2 * l2 + 1)
    d = O.product_odd_dense(l1, l2, l3, x, y)
    scale = max(np.abs(d).max(), 1e-300)
    assert is_symmetric(d) <= 1e-13 * scale
    assert max_trace(d) <= 1e-13 * scale
    # swapping the inputs flips the sign of the epsilon contraction
    np.testing.assert_allclose(O.product_odd(l2, l1, l3, y, x), -O.product_odd(l1, l2, l3, x, y),
                               atol=1e-12 * scale)
    # bilinearity
    x2 = RNG.normal(size=2 * l1 + 1)
    np.testing.assert_allclose(O.product_odd(l1, l2, l3, 2.0 * x - 0.5 * x2, y),
                               2.0 * O.product_odd(l1, l2, l3, x, y)
                               - 0.5 * O.product_odd(l1, l2, l3, x2, y), atol=1e-11 * scale)


@pytest.mark.parametrize("reflect", [False, True])
@pytest.mark.parametrize("path", odd_paths(3))
def test_pseudo_tensor_equivariance(path, reflect):
    """f(R x, R y) = det(R) R f(x, y) for every orthogonal R: a rotation
    acts as on a true tensor, a reflection adds a sign."""
    l1, l2, l3 = path
    R = rand_rot(RNG, reflect)
    x, y = RNG.normal(size=2 * l1 + 1), RNG.normal(size=2 * l2 + 1)
    xr = O.stf_extract(l1, rotate_dense(R, O.stf_dense(l1, x)))
    yr = O.stf_extract(l2, rotate_dense(R, O.stf_dense(l2, y)))
    lhs = O.product_odd(l1, l2, l3, xr, yr)
    rhs = np.linalg.det(R) * O.stf_extract(l3, rotate_dense(R, O.product_odd_dense(l1, l2, l3, x, y)))
    np.testing.assert_allclose(lhs, rhs, atol=1e-10 * max(1.0, np.abs(rhs).max()))


def test_odd_convolution_closed_form_and_parity():
    """The (1,1)->1 slot of the odd convolution is sum_e w x_1 x r-hat; and
    inverting every edge vector multiplies path (l1,l2)->l3 by (-1)^l2."""
    L, C, N = 3, 2, 6
    pos, ei, ev = W.random_graph(N, 3, 3.0, 4)
    ev = ev.astype(np.float64)
    E = ei.shape[1]
    ps = O.paths(L, L, L, odd=True)
    P = len(ps)
    x = RNG.normal(size=(N, (L + 1) ** 2 * C))
    w = RNG.normal(size=(E, P, C))
    z = O.edge_conv(L, L, L, C, ei, ev, x, w, N, odd=True)
    zr = O.zrow(L, L, L, odd=True)
    Pl = [sum(1 for p in ps if p[2] == l) for l in range(L + 1)]
    off = np.concatenate([[0], np.cumsum([(2 * l + 1) * Pl[l] for l in range(L + 1)])])
    zz = z.reshape(N, zr, C)
    xr = x.reshape(N, -1, C)
    ref = np.zeros((N, 3, C))
    for e in range(E):
        u, v = ei[:, e]
        rh = ev[e] / np.linalg.norm(ev[e])
        for k in range(C):
            ref[u, :, k] += w[e, 0, k] * np.cross(xr[v, 1:4, k], rh)
    # path 0 is (1,1)->1, eta 0 of rank 1: slots off(1) + c P_1 + 0
    got = zz[:, off[1] + np.arange(3) * Pl[1], :]
    np.testing.assert_allclose(got, ref, atol=1e-12)
    zi = O.edge_conv(L, L, L, C, ei, -ev, x, w, N, odd=True).reshape(N, zr, C)
    for p, (l1, l2, l3) in enumerate(ps):
        eta = sum(1 for q in ps[:p] if q[2] == l3)
        sl = off[l3] + np.arange(2 * l3 + 1) * Pl[l3] + eta
        np.testing.assert_allclose(zi[:, sl, :], (-1) ** l2 * zz[:, sl, :], atol=1e-12)


@pytest.mark.parametrize("L", [2, 3])
def test_odd_convolution_vjp_central_differences(L):
    C, N = 2, 5
    pos, ei, ev = W.random_graph(N, 2, 3.0, 5)
    ev = ev.astype(np.float64)
    E = ei.shape[1]
    P = len(O.paths(L, L, L, odd=True))
    x = RNG.normal(size=(N, (L + 1) ** 2 * C))
    w = RNG.normal(size=(E, P, C))
    g = RNG.normal(size=(N, O.zrow(L, L, L, odd=True) * C))

    def loss(x_, w_, ev_):
        return float((O.edge_conv(L, L, L, C, ei, ev_, x_, w_, N, odd=True) * g).sum())
    xb, wb, rb = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, g, N, odd=True)
    h = 1e-3   # bilinear in x and w: exact up to rounding
    for _ in range(8):
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
    np.testing.assert_allclose((rb * ev).sum(1), 0.0, atol=1e-9)
