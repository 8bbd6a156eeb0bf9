"""Pins of the FP64 oracle's tensor algebra to facts the FlashCart pages and
textbook mathematics fix (not to the oracle's own formulas).

Pages: FlashCart, arXiv 2610.06409 -- Sec. 2 (STF spaces), Sec. 3 (independent
components, trace relation, the (1,1)->2 example), App. B (T_l, Eq. B1),
App. C (Table C1 operation counts).
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
from numpy.polynomial import legendre

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(20261202)


def rand_rot(rng, reflect=False):
    q, r = np.linalg.qr(rng.normal(size=(3, 3)))
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    if reflect:
        q = -q
    return q


def rotate_dense(R, t):
    for ax in range(t.ndim):
        t = np.moveaxis(np.tensordot(R, t, axes=([1], [ax])), 0, ax)
    return t


def is_symmetric(t):
    l = t.ndim
    return max((np.abs(t - np.transpose(t, p)).max()
                for p in itertools.permutations(range(l))), default=0.0)


def max_trace(t):
    if t.ndim < 2:
        return 0.0
    return np.abs(np.trace(t, axis1=0, axis2=1)).max()


# ---------------------------------------------------------------------------
# independent components and the trace relation (Sec. 2, Sec. 3)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("l", range(0, 7))
def test_component_choice(l):
    comps = [O.comp_pxyz(l, c) for c in range(2 * l + 1)]
    # 2l+1 = (l+1)(l+2)/2 symmetric minus l(l-1)/2 trace conditions
    assert len(comps) == (l + 1) * (l + 2) // 2 - l * (l - 1) // 2
    assert len(set(comps)) == len(comps)
    for px, py, pz in comps:
        assert px + py + pz == l and pz <= 1 and min(px, py, pz) >= 0


@pytest.mark.parametrize("l", range(0, 7))
def test_reconstruction_is_stf_and_roundtrips(l):
    c = RNG.normal(size=2 * l + 1)
    d = O.stf_dense(l, c)
    assert is_symmetric(d) < 1e-12
    assert max_trace(d) < 1e-11 * max(1.0, np.abs(d).max())
    np.testing.assert_allclose(O.stf_extract(l, d), c, rtol=0, atol=1e-13)
    # the 2l+1 components span the whole STF space: the dense images of the
    # unit vectors are linearly independent
    M = np.stack([O.stf_dense(l, np.eye(2 * l + 1)[i]).ravel()
                  for i in range(2 * l + 1)])
    assert np.linalg.matrix_rank(M) == 2 * l + 1


@pytest.mark.parametrize("l", range(2, 6))
def test_trace_relation(l):
    """x_{px,py,pz} = -x_{px+2,py,pz-2} - x_{px,py+2,pz-2}, Sec. 3."""
    c = RNG.normal(size=2 * l + 1)
    d = O.stf_dense(l, c)

    def ent(px, py, pz):
        return d[tuple([0] * px + [1] * py + [2] * pz)]
    for pz in range(2, l + 1):
        for px in range(0, l - pz + 1):
            py = l - pz - px
            assert abs(ent(px, py, pz) + ent(px + 2, py, pz - 2)
                       + ent(px, py + 2, pz - 2)) < 1e-12


# ---------------------------------------------------------------------------
# generic trace removal: textbook closed forms and projector properties
# ---------------------------------------------------------------------------

def test_detrace_rank2_closed_form():
    S = RNG.normal(size=(3, 3))
    S = S + S.T
    ref = S - np.eye(3) * np.trace(S) / 3.0
    np.testing.assert_allclose(O.detrace(2, S), ref, atol=1e-14)


def test_detrace_rank3_closed_form():
    A = RNG.normal(size=(3, 3, 3))
    S = sum(np.transpose(A, p) for p in itertools.permutations(range(3))) / 6
    t = np.einsum("iik->k", S)
    I = np.eye(3)
    ref = S - (np.einsum("ij,k->ijk", I, t) + np.einsum("ik,j->ijk", I, t)
               + np.einsum("jk,i->ijk", I, t)) / 5.0
    np.testing.assert_allclose(O.detrace(3, S), ref, atol=1e-14)


@pytest.mark.parametrize("l", range(2, 6))
def test_detrace_is_projector(l):
    A = RNG.normal(size=(3,) * l)
    S = O.permavg(l, A)
    D = O.detrace(l, S)
    assert is_symmetric(D) < 1e-12 and max_trace(D) < 1e-12
    np.testing.assert_allclose(O.detrace(l, D), D, atol=1e-12)


# ---------------------------------------------------------------------------
# direction tensors (App. B)
# ---------------------------------------------------------------------------

def test_direction_low_ranks_closed_form():
    r = RNG.normal(size=3)
    u = r / np.linalg.norm(r)
    assert abs(O.direction_dense(0, r) - 1.0) < 1e-15
    np.testing.assert_allclose(O.direction_dense(1, r), u, atol=1e-15)
    np.testing.assert_allclose(O.direction_dense(2, r),
                               1.5 * (np.outer(u, u) - np.eye(3) / 3), atol=1e-15)


@pytest.mark.parametrize("l", range(0, 7))
def test_direction_normalisation_and_legendre(l):
    r = RNG.normal(size=3)
    u = r / np.linalg.norm(r)
    T = O.direction_dense(l, r)
    assert is_symmetric(T) < 1e-12 and max_trace(T) < 1e-11
    full = T
    for _ in range(l):
        full = np.tensordot(full, u, axes=([0], [0]))
    assert abs(float(full) - 1.0) < 1e-12           # App. B: contraction = 1
    zz = T[(2,) * l] if l else T
    assert abs(float(zz) - legendre.legval(u[2], [0] * l + [1])) < 1e-12
    # natural parity (Sec. 2): T_l(-r) = (-1)^l T_l(r)
    np.testing.assert_allclose(O.direction_dense(l, -r), (-1) ** l * T,
                               atol=1e-13)


@pytest.mark.parametrize("l", range(0, 5))
def test_direction_jacobian_finite_difference(l):
    r = RNG.normal(size=3) * 2.0
    J = O.direction_jac(l, r)
    h = 1e-6
    fd = np.stack([(O.direction(l, r + h * e) - O.direction(l, r - h * e))
                   / (2 * h) for e in np.eye(3)], axis=1)
    np.testing.assert_allclose(J, fd, atol=1e-8)
    # T depends on the direction only
    np.testing.assert_allclose(J @ r, 0.0, atol=1e-12)


# ---------------------------------------------------------------------------
# products (Sec. 2, Sec. 3, App. B, App. C)
# ---------------------------------------------------------------------------

def test_paths_and_counts_golden():
    cases = json.load(open(os.path.join(GOLDEN, "path_counts.json")))["cases"]
    for c in cases:
        ps = O.paths(c["lin"], c["ledge"], c["lout"])
        if "paths" in c:
            assert len(ps) == c["paths"]
        if "output_components" in c:
            assert sum(2 * l3 + 1 for _, _, l3 in ps) == c["output_components"]
    assert len(O.paths(2, 2, 2)) == 11 and len(O.paths(3, 3, 3)) == 23
    assert len(O.paths(4, 4, 4)) == 42


def test_admissibility_rule():
    for l1, l2, l3 in itertools.product(range(6), repeat=3):
        tri = abs(l1 - l2) <= l3 <= l1 + l2
        assert O.admissible(l1, l2, l3) == (tri and (l1 + l2 + l3) % 2 == 0)


def test_worked_example_112_golden():
    g = json.load(open(os.path.join(GOLDEN, "product_112_xx.json")))
    K = O.path_coeffs(1, 1, 2)              # [a][b1][b2]
    idx = {"x": 0, "y": 1, "z": 2}
    expect = np.zeros((3, 3))
    for t in g["terms"]:
        expect[idx[t["x"]], idx[t["y"]]] = float(Fraction(t["coef"]))
    assert O.comp_pxyz(2, 0) == (2, 0, 0)   # component 0 of rank 2 is xx
    np.testing.assert_allclose(K[0], expect, atol=1e-15)


def test_table_c1_operation_counts_golden():
    g = json.load(open(os.path.join(GOLDEN, "table_c1_opcounts.json")))
    for row in g["rows"]:
        L = row["max_rank"]
        ncpl, ops = 0, 0
        for l3 in range(L + 1):
            for l1 in range(L + 1):
                for l2 in range(l1, L + 1):
                    if not O.admissible(l1, l2, l3):
                        continue
                    ncpl += 1
                    K = O.path_coeffs(l1, l2, l3)
                    for a in range(2 * l3 + 1):
                        c = K[a][np.abs(K[a]) > 1e-12]
                        if len(c) == 0:
                            continue
                        ops += 2 * len(c) - 1 + int(
                            np.sum(np.abs(np.abs(c) - 1.0) > 1e-9))
        assert ncpl == row["couplings"]
        assert ops == row["independent_ops"]


@pytest.mark.parametrize("path", O.paths(4, 4, 4))
def test_product_routes_agree_and_output_is_stf(path):
    l1, l2, l3 = path
    x, y = RNG.normal(size=2 * l1 + 1), RNG.normal(size=2 * l2 + 1)
    d0 = O.product_dense(l1, l2, l3, x, y, route=0)
    d1 = O.product_dense(l1, l2, l3, x, y, route=1)
    scale = max(1.0, np.abs(d0).max())
    assert np.abs(d0 - d1).max() < 1e-13 * scale
    assert is_symmetric(d0) < 1e-12 * scale
    assert max_trace(d0) < 1e-12 * scale
    assert np.abs(d0).max() > 0


@pytest.mark.parametrize("path", O.paths(4, 4, 4))
def test_product_equivariance_o3(path):
    l1, l2, l3 = path
    x, y = RNG.normal(size=2 * l1 + 1), RNG.normal(size=2 * l2 + 1)
    for reflect in (False, True):
        R = rand_rot(RNG, reflect)
        xr = O.stf_extract(l1, rotate_dense(R, O.stf_dense(l1, x)))
        yr = O.stf_extract(l2, rotate_dense(R, O.stf_dense(l2, y)))
        lhs = O.product_dense(l1, l2, l3, xr, yr)
        rhs = rotate_dense(R, O.product_dense(l1, l2, l3, x, y))
        assert np.abs(lhs - rhs).max() < 1e-10 * max(1.0, np.abs(rhs).max())


@pytest.mark.parametrize("path", O.paths(4, 4, 4))
def test_product_normalisation_on_direction_tensors(path):
    """Reading of C_{l1 l2 l3}: T_l1 (x) T_l2 -> T_l3 at any direction."""
    l1, l2, l3 = path
    r = RNG.normal(size=3)
    f = O.product(l1, l2, l3, O.direction(l1, r), O.direction(l2, r))
    np.testing.assert_allclose(f, O.direction(l3, r), atol=1e-12)


@pytest.mark.parametrize("l", range(0, 6))
def test_scalar_coupling_is_legendre(l):
    r, s = RNG.normal(size=3), RNG.normal(size=3)
    c = (r @ s) / np.linalg.norm(r) / np.linalg.norm(s)
    f = O.product(l, l, 0, O.direction(l, r), O.direction(l, s))[0]
    assert abs(f - legendre.legval(c, [0] * l + [1])) < 1e-12


def test_product_is_bilinear_and_exchange_symmetric():
    for l1, l2, l3 in O.paths(3, 3, 3):
        x1, x2 = RNG.normal(size=(2, 2 * l1 + 1))
        y1 = RNG.normal(size=2 * l2 + 1)
        a = 0.7
        lhs = O.product(l1, l2, l3, a * x1 + x2, y1)
        rhs = a * O.product(l1, l2, l3, x1, y1) + O.product(l1, l2, l3, x2, y1)
        np.testing.assert_allclose(lhs, rhs, atol=1e-12)
        # Sec. 3: exchanged paths share one expression with swapped operands
        np.testing.assert_allclose(O.product(l1, l2, l3, x1, y1),
                                   O.product(l2, l1, l3, y1, x1), atol=1e-12)
