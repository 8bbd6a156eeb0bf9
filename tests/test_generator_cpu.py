"""The product-side generator (exact rational polynomials) against the FP64
oracle (dense index contractions): two independent derivations of the same
coefficients from the FlashCart pages must agree."""
import numpy as np
import pytest

from cartesian_tensor_products_b200.gen import fc_algebra as G
from cartesian_tensor_products_b200.gen import fc_codegen as CG
from oracle import oracle as O


@pytest.mark.parametrize("path", G.paths(4, 4, 4))
def test_bilinear_coefficients_match_oracle(path):
    K = np.array(G.path_coefficients(*path), dtype=np.float64)
    np.testing.assert_allclose(K, O.path_coeffs(*path), atol=1e-14)


@pytest.mark.parametrize("l", range(0, 5))
def test_direction_polynomials_match_oracle(l):
    rng = np.random.default_rng(l)
    for _ in range(4):
        r = rng.normal(size=3)
        u = r / np.linalg.norm(r)
        ys = [sum(float(c) * u[0] ** m[0] * u[1] ** m[1] * u[2] ** m[2]
                  for m, c in p.items()) for p in G.direction_polys(l)]
        np.testing.assert_allclose(ys, O.direction(l, r), atol=1e-14)


def test_component_order_matches_oracle():
    for l in range(6):
        assert G.components(l) == [O.comp_pxyz(l, c) for c in range(2 * l + 1)]


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5])
def test_forward_groups_cover_every_row_once(L):
    T = CG.Tables(L)
    groups = CG.partition_rows(T, CG.NGROUPS[L])
    rows = [r for g in groups for r in g]
    assert sorted(rows) == sorted((p, a) for p in range(T.P)
                                  for a in range(2 * T.paths[p][2] + 1))
    # the generated M entries of all groups add up to the nonzeros of M
    codes = [CG.GroupCode(T, g, i) for i, g in enumerate(groups)]
    nnz = sum(len(T.mrow(p, a)) for p in range(T.P) if not T.is_identity(p)
              for a in range(2 * T.paths[p][2] + 1))
    assert sum(c.NM for c in codes) == nnz


@pytest.mark.parametrize("path", G.odd_paths(4, 4, 4))
def test_odd_path_coefficients_match_oracle(path):
    """Odd-J paths: r . (grad a x grad b) on polynomials (generator) against
    the dense epsilon contraction (oracle)."""
    K = np.array(G.odd_path_coefficients(*path), dtype=np.float64)
    np.testing.assert_allclose(K, O.path_coeffs_odd(*path), atol=1e-14)
    assert G.odd_paths(4, 4, 4) == O.paths(4, 4, 4, odd=True)
