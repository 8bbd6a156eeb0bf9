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
