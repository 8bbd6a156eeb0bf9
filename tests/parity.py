"""Helpers shared by the GPU parity tests (test infrastructure)."""
import numpy as np

from oracle import oracle as O

FWD_TOL = 1e-5      # max relative error, forward (normwise: max|d| / max|ref|)
VJP_TOL = 1e-4      # max relative error, VJPs


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def rot_matrices(R, lmax):
    """D_l(R): rotation of the 2l+1 independent components of rank-l STF
    tensors, built from the oracle's dense reconstruction."""
    out = []
    for l in range(lmax + 1):
        n = 2 * l + 1
        D = np.zeros((n, n))
        for c in range(n):
            d = O.stf_dense(l, np.eye(n)[c])
            for ax in range(l):
                d = np.moveaxis(np.tensordot(R, d, axes=([1], [ax])), 0, ax)
            D[:, c] = O.stf_extract(l, d)
        out.append(D)
    return out


def rotate_rows(D, feat, blocks, C):
    """feat [N][rows*C]; blocks = [(l, start_row, P_l)] -> rotated copy."""
    N = feat.shape[0]
    f = feat.reshape(N, -1, C).astype(np.float64)
    out = f.copy()
    for (l, start, P) in blocks:
        n = 2 * l + 1
        blk = f[:, start:start + n * P].reshape(N, n, P, C)
        out[:, start:start + n * P] = np.einsum("ab,nbpc->napc", D[l], blk).reshape(N, n * P, C)
    return out.reshape(N, -1)


def node_blocks(lmax):
    return [(l, l * l, 1) for l in range(lmax + 1)]


def out_blocks(lmax):
    ps = O.paths(lmax, lmax, lmax)
    Pl = [sum(1 for p in ps if p[2] == l) for l in range(lmax + 1)]
    blocks, o = [], 0
    for l in range(lmax + 1):
        blocks.append((l, o, Pl[l]))
        o += (2 * l + 1) * Pl[l]
    return blocks


def ragged_graph(n_nodes, degrees, box, seed):
    """Receiver-sorted random graph with the given in-degree per receiver
    (senders distinct, no self-edges)."""
    g = np.random.default_rng(seed)
    pos = g.uniform(0, box, size=(n_nodes, 3))
    recv, send = [], []
    for u, k in enumerate(degrees):
        k = min(k, n_nodes - 1)
        s = g.choice(n_nodes - 1, size=k, replace=False)
        s = np.where(s >= u, s + 1, s)
        recv += [u] * k
        send += sorted(s.tolist())
    ei = np.array([recv, send], dtype=np.int32).reshape(2, -1)
    ev = (pos[ei[1]] - pos[ei[0]]).astype(np.float32)
    return ei, ev
