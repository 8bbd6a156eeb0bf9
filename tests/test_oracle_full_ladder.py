"""Pins of the oracle's full correlation ladder (FlashCart Sec. 5 Eq. 2:
products keep every path, a learned map mixes paths and channels per output
rank) against things other than itself: the order-1 closed form, the
reduction to the (separately pinned) path-reduced ladder when every map is
diagonal in the channels, a brute-force expansion from the pinned pairwise
product, and O(3) equivariance."""
import numpy as np
import pytest

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import node_blocks, rot_matrices, rotate_rows


def rank_paths(L):
    P = O.paths(L, L, L)
    return P, [sum(1 for p in P if p[2] == l) for l in range(L + 1)]


@pytest.mark.parametrize("L", [1, 2, 3])
def test_order_one_is_the_per_rank_map(L):
    C, N = 3, 4
    d = W.full_ladder_inputs(N, L, C, 1, 3)
    _, z = O.full_ladder(L, C, 1, d["A"], d["W1"], d["Wq"])
    A = d["A"].astype(np.float64).reshape(N, -1, C)
    ref = np.zeros_like(A)
    for l in range(L + 1):
        ref[:, l * l:(l + 1) ** 2] = np.einsum("jk,nck->ncj", d["W1"][l].astype(np.float64),
                                               A[:, l * l:(l + 1) ** 2])
    np.testing.assert_allclose(z.reshape(N, -1, C), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L,order", [(2, 3), (3, 4)])
def test_channel_diagonal_maps_give_the_path_reduced_ladder(L, order):
    """W1 = I and W_q[l][j][eta C + k] = delta_jk a_q[eta][k]: each step is the
    path-reduced product with path weights a_q followed by an identity mix."""
    C, N = 4, 5
    P, Pl = rank_paths(L)
    rng = np.random.default_rng(7)
    A = rng.normal(size=(N, (L + 1) ** 2 * C))
    a = rng.normal(size=(order - 1, len(P), C))
    W1 = np.stack([np.eye(C)] * (L + 1))
    Wq = np.zeros((order - 1, C * len(P) * C))
    for q in range(order - 1):
        off = 0
        for l in range(L + 1):
            K = Pl[l] * C
            blk = np.zeros((C, K))
            eta = 0
            for p, (l1, l2, l3) in enumerate(P):
                if l3 != l:
                    continue
                blk[np.arange(C), eta * C + np.arange(C)] = a[q, p]
                eta += 1
            Wq[q, off:off + C * K] = blk.ravel()
            off += C * K
    _, z = O.full_ladder(L, C, order, A, W1, Wq)
    mix = np.stack([np.stack([np.eye(C)] * (L + 1))] * (order - 1))
    _, zr = O.ladder(L, C, order, A, a, mix)
    np.testing.assert_allclose(z, zr, rtol=1e-12, atol=1e-12)


def test_brute_force_two_steps():
    L, C, N, order = 1, 2, 3, 2
    d = W.full_ladder_inputs(N, L, C, order, 11)
    st, z = O.full_ladder(L, C, order, d["A"], d["W1"], d["Wq"])
    P, Pl = rank_paths(L)
    A = d["A"].astype(np.float64).reshape(N, -1, C)
    W1 = d["W1"].astype(np.float64)
    phi1 = np.zeros_like(A)
    for l in range(L + 1):
        phi1[:, l * l:(l + 1) ** 2] = np.einsum("jk,nck->ncj", W1[l], A[:, l * l:(l + 1) ** 2])
    Wq = d["Wq"][0].astype(np.float64)
    phi2 = np.zeros_like(A)
    off = 0
    for l in range(L + 1):
        K = Pl[l] * C
        Wl = Wq[off:off + C * K].reshape(C, K)
        off += C * K
        eta = 0
        for (l1, l2, l3) in P:
            if l3 != l:
                continue
            for n in range(N):
                for k in range(C):
                    f = O.product(l1, l2, l3, phi1[n, l1 * l1:(l1 + 1) ** 2, k],
                                  A[n, l2 * l2:(l2 + 1) ** 2, k])
                    for j in range(C):
                        phi2[n, l * l:(l + 1) ** 2, j] += Wl[j, eta * C + k] * f
            eta += 1
    np.testing.assert_allclose(st[0].reshape(N, -1, C), phi1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st[1].reshape(N, -1, C), phi2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z.reshape(N, -1, C), phi1 + phi2, rtol=1e-12, atol=1e-12)


def test_equivariance():
    L, C, N, order = 3, 3, 4, 3
    d = W.full_ladder_inputs(N, L, C, order, 13)
    rng = np.random.default_rng(3)
    q, r = np.linalg.qr(rng.normal(size=(3, 3)))
    R = q * np.sign(np.diag(r))
    D = rot_matrices(R, L)
    _, z = O.full_ladder(L, C, order, d["A"], d["W1"], d["Wq"])
    Ar = rotate_rows(D, d["A"], node_blocks(L), C)
    _, zr = O.full_ladder(L, C, order, Ar, d["W1"], d["Wq"])
    np.testing.assert_allclose(zr, rotate_rows(D, z, node_blocks(L), C), rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------------------
# reverse pass of the full ladder
# ---------------------------------------------------------------------------

def _loss(L, C, order, A, W1, Wq, gz):
    _, z = O.full_ladder(L, C, order, A, W1, Wq)
    return float((z * gz).sum())


@pytest.mark.parametrize("L,order", [(1, 3), (2, 3), (3, 2)])
def test_full_ladder_vjp_central_differences(L, order):
    """Every entry of A_bar, W1_bar and Wq_bar against central differences of
    <gz, z> (z is a polynomial of degree `order` in A and of degree 1 in each
    map, so the map gradients are exact up to rounding and the A step error
    is O(h^2))."""
    C, N = 2, 2
    d = W.full_ladder_inputs(N, L, C, order, 21 + L)
    A, W1, Wq = (d[k].astype(np.float64) for k in ("A", "W1", "Wq"))
    gz = np.random.default_rng(5).normal(size=A.shape)
    Ab, W1b, Wqb = O.full_ladder_vjp(L, C, order, A, W1, Wq, gz)
    h = 1e-5
    for arr, grad in ((A, Ab), (W1, W1b), (Wq, Wqb)):
        flat, g = arr.reshape(-1), grad.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            fp = _loss(L, C, order, A, W1, Wq, gz)
            flat[i] = keep - h
            fm = _loss(L, C, order, A, W1, Wq, gz)
            flat[i] = keep
            assert abs((fp - fm) / (2 * h) - g[i]) <= 1e-6 * max(1.0, abs(g[i])), (i, g[i])


@pytest.mark.parametrize("L,order", [(2, 3), (3, 4)])
def test_full_ladder_vjp_reduces_to_path_reduced_ladder_vjp(L, order):
    """W1 = I and Wq[l][j][eta C + k] = M_l[j][k] a[eta][k] make every full
    step the path-reduced product (weights a) followed by the per-rank mix M,
    i.e. the separately pinned product ladder.  Then A_bar equals its A1_bar
    and, by the chain rule through that parametrisation,
    path_w_bar[p][k] = sum_j Wq_bar[l][j][eta C + k] M_l[j][k] and
    mix_bar[l][j][k] = sum_{p -> l} Wq_bar[l][j][eta C + k] a[p][k]."""
    C, N = 3, 4
    P, Pl = rank_paths(L)
    rng = np.random.default_rng(17)
    A = rng.normal(size=(N, (L + 1) ** 2 * C))
    a = rng.normal(size=(order - 1, len(P), C))
    M = rng.normal(size=(order - 1, L + 1, C, C)) / np.sqrt(C)
    gz = rng.normal(size=A.shape)
    W1 = np.stack([np.eye(C)] * (L + 1))
    Wq = np.zeros((order - 1, C * len(P) * C))
    offs = np.concatenate([[0], np.cumsum([C * p * C for p in Pl])])
    etas = []
    for q in range(order - 1):
        eta_of = {}
        for l in range(L + 1):
            blk = np.zeros((C, Pl[l] * C))
            eta = 0
            for p, (l1, l2, l3) in enumerate(P):
                if l3 != l:
                    continue
                blk[:, eta * C:(eta + 1) * C] = M[q, l] * a[q, p][None, :]
                eta_of[p] = eta
                eta += 1
            Wq[q, offs[l]:offs[l + 1]] = blk.ravel()
        etas.append(eta_of)
    Ab, _, Wqb = O.full_ladder_vjp(L, C, order, A, W1, Wq, gz)
    A1b, pwb, mxb = O.ladder_vjp(L, C, order, A, a, M, gz)
    np.testing.assert_allclose(Ab, A1b, rtol=1e-11, atol=1e-11)
    for q in range(order - 1):
        for p, (l1, l2, l3) in enumerate(P):
            blk = Wqb[q, offs[l3]:offs[l3 + 1]].reshape(C, Pl[l3] * C)
            e = etas[q][p]
            g = blk[:, e * C:(e + 1) * C]                      # [j][k]
            np.testing.assert_allclose((g * M[q, l3]).sum(0), pwb[q, p], rtol=1e-10, atol=1e-10)
        for l in range(L + 1):
            blk = Wqb[q, offs[l]:offs[l + 1]].reshape(C, Pl[l] * C)
            acc = np.zeros((C, C))
            for p, (l1, l2, l3) in enumerate(P):
                if l3 == l:
                    e = etas[q][p]
                    acc += blk[:, e * C:(e + 1) * C] * a[q, p][None, :]
            np.testing.assert_allclose(acc, mxb[q, l], rtol=1e-10, atol=1e-10)


def test_full_ladder_vjp_node_mask_and_order_one():
    """Masked nodes contribute nothing; order 1 leaves only the first map."""
    L, C, N = 2, 3, 5
    d = W.full_ladder_inputs(N, L, C, 3, 8)
    gz = d["gz"].astype(np.float64)
    m = np.array([1, 0, 1, 0, 0], np.uint8)
    Ab, W1b, Wqb = O.full_ladder_vjp(L, C, 3, d["A"], d["W1"], d["Wq"], gz, node_mask=m)
    Ab2, W1b2, Wqb2 = O.full_ladder_vjp(L, C, 3, d["A"], d["W1"], d["Wq"], gz * m[:, None])
    assert np.all(Ab[m == 0] == 0)
    np.testing.assert_allclose(Ab[m == 1], Ab2[m == 1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(W1b, W1b2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Wqb, Wqb2, rtol=1e-12, atol=1e-12)
    Ab1, W1b1, _ = O.full_ladder_vjp(L, C, 1, d["A"], d["W1"], None, gz)
    A = d["A"].astype(np.float64).reshape(N, -1, C)
    G = gz.reshape(N, -1, C)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) ** 2)
        np.testing.assert_allclose(W1b1[l], np.einsum("ncj,nck->jk", G[:, sl], A[:, sl]),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Ab1.reshape(N, -1, C)[:, sl],
                                   np.einsum("jk,ncj->nck", d["W1"][l].astype(np.float64), G[:, sl]),
                                   rtol=1e-12, atol=1e-12)
