"""Pins of the oracle's node-local product ladder (FlashCart Sec. 5 Eq. 2 with
path-reduced products, App. E) to closed forms, equivariance and finite
differences."""
import numpy as np
import pytest

from oracle import oracle as O
from test_oracle_conv import rotate_features
from test_oracle_tensors import rand_rot

RNG = np.random.default_rng(11)


def path_index(L, path):
    return O.paths(L, L, L).index(path)


def test_scalar_chain_closed_form():
    """Only the (0,0)->0 path weighted: A_{v+1}[0] = M_v (A_v[0] * A_1[0]),
    higher ranks of A_{v+1} vanish, z = sum_v A_v."""
    L, C, N, order = 2, 4, 3, 4
    P = len(O.paths(L, L, L))
    A1 = RNG.normal(size=(N, 9 * C))
    pw = np.zeros((order - 1, P, C))
    pw[:, path_index(L, (0, 0, 0)), :] = RNG.normal(size=(order - 1, C))
    mix = RNG.normal(size=(order - 1, L + 1, C, C))
    states, z = O.ladder(L, C, order, A1, pw, mix)
    a = A1.reshape(N, 9, C)
    s0 = a[:, 0]
    zref = a.copy()
    cur = s0
    for v in range(order - 1):
        cur = (pw[v, 0][None, :] * cur * s0) @ mix[v, 0].T
        st = states[v].reshape(N, 9, C)
        np.testing.assert_allclose(st[:, 0], cur, atol=1e-12)
        assert np.all(st[:, 1:] == 0)
        zref[:, 0] += cur
    np.testing.assert_allclose(z.reshape(N, 9, C), zref, atol=1e-12)


def test_vector_chain_closed_form():
    """Paths (0,0)->0 and (0,1)->1 with unit weights and identity mixing:
    A_{v+1}[0] = A_1[0]^(v+1), A_{v+1}[1] = A_v[0] A_1[1] = A_1[0]^v A_1[1]."""
    L, C, N, order = 1, 3, 4, 5
    P = len(O.paths(L, L, L))
    A1 = RNG.normal(size=(N, 4 * C))
    pw = np.zeros((order - 1, P, C))
    pw[:, path_index(L, (0, 0, 0))] = 1.0
    pw[:, path_index(L, (0, 1, 1))] = 1.0
    mix = np.broadcast_to(np.eye(C), (order - 1, L + 1, C, C)).copy()
    _, z = O.ladder(L, C, order, A1, pw, mix)
    a = A1.reshape(N, 4, C)
    s = a[:, 0]
    zs = sum(s ** q for q in range(1, order + 1))
    zv = a[:, 1:4] * sum(s ** q for q in range(0, order))[:, None, :]
    zz = z.reshape(N, 4, C)
    np.testing.assert_allclose(zz[:, 0], zs, atol=1e-12)
    np.testing.assert_allclose(zz[:, 1:4], zv, atol=1e-12)


def test_order_one_is_identity():
    L, C, N = 2, 2, 3
    A1 = RNG.normal(size=(N, 9 * C))
    states, z = O.ladder(L, C, 1, A1, np.zeros((0, 11, C)), np.zeros((0, 3, C, C)))
    np.testing.assert_allclose(z, A1, atol=0)


@pytest.mark.parametrize("reflect", [False, True])
def test_ladder_equivariance(reflect):
    L, C, N, order = 2, 2, 2, 3
    P = len(O.paths(L, L, L))
    A1 = RNG.normal(size=(N, 9 * C))
    pw = RNG.normal(size=(order - 1, P, C))
    mix = RNG.normal(size=(order - 1, L + 1, C, C))
    R = rand_rot(RNG, reflect)
    _, z = O.ladder(L, C, order, A1, pw, mix)
    _, zr = O.ladder(L, C, order, rotate_features(R, A1, L, C), pw, mix)
    np.testing.assert_allclose(zr, rotate_features(R, z, L, C),
                               atol=1e-10 * np.abs(z).max())


def test_ladder_vjp_finite_differences():
    L, C, N, order = 2, 2, 3, 4
    P = len(O.paths(L, L, L))
    A1 = RNG.normal(size=(N, 9 * C))
    pw = RNG.normal(size=(order - 1, P, C))
    mix = RNG.normal(size=(order - 1, L + 1, C, C)) / np.sqrt(C)
    gz = RNG.normal(size=(N, 9 * C))

    def loss(a, p, m):
        return float((O.ladder(L, C, order, a, p, m)[1] * gz).sum())
    A1b, pwb, mxb = O.ladder_vjp(L, C, order, A1, pw, mix, gz)
    h = 1e-5
    for arr, grad, which in ((A1, A1b, 0), (pw, pwb, 1), (mix, mxb, 2)):
        for _ in range(8):
            i = RNG.integers(arr.size)
            d = np.zeros(arr.size); d[i] = h
            d = d.reshape(arr.shape)
            args_p = [A1, pw, mix]; args_m = [A1, pw, mix]
            args_p[which] = arr + d; args_m[which] = arr - d
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad.ravel()[i]) < 1e-6 * max(1.0, abs(fd))


def test_ladder_node_mask():
    L, C, N, order = 2, 2, 4, 3
    P = len(O.paths(L, L, L))
    A1 = RNG.normal(size=(N, 9 * C))
    pw = RNG.normal(size=(order - 1, P, C))
    mix = RNG.normal(size=(order - 1, L + 1, C, C))
    gz = RNG.normal(size=(N, 9 * C))
    m = np.array([1, 0, 1, 0], np.uint8)
    _, z = O.ladder(L, C, order, A1, pw, mix)
    _, zm = O.ladder(L, C, order, A1, pw, mix, node_mask=m)
    np.testing.assert_allclose(zm[[0, 2]], z[[0, 2]], atol=0)
    gzm = gz * m[:, None]
    full = O.ladder_vjp(L, C, order, A1, pw, mix, gzm)
    part = O.ladder_vjp(L, C, order, A1, pw, mix, gz, node_mask=m)
    for a, b in zip(full, part):
        np.testing.assert_allclose(b, a, atol=1e-12)
