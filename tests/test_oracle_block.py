"""Pins of the oracle's interaction block (envelope-weighted convolution with
summed paths, product ladder, E = sum of rank-0 outputs, forces): energy
finite differences against the forces, zero net force, and invariance of E
under rotations of the whole configuration (FlashCart Sec. 2: E is
invariant, F = -grad E transforms as a vector)."""
import numpy as np

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import node_blocks, rot_matrices, rotate_rows

L, C, ORDER = 2, 4, 3


def small_block():
    d = W.diamond(cells=2, cutoff=3.0, channels=C, lmax=L, order=ORDER, seed=11)
    return d


def energy(d, pos):
    ei = d["edge_index"]
    ev = pos[ei[1]] - pos[ei[0]] + d["shift"]
    e, _, _ = O.block_energy_forces(L, C, ORDER, ei, ev, d["x"], d["omega"], d["path_w"],
                                    d["mix_w"], d["n_nodes"], d["cutoff"], d["edge_scale"])
    return e.sum()


def test_block_forces_match_energy_differences():
    d = small_block()
    pos = d["pos64"]
    ei = d["edge_index"]
    ev = pos[ei[1]] - pos[ei[0]] + d["shift"]
    _, _, F = O.block_energy_forces(L, C, ORDER, ei, ev, d["x"], d["omega"], d["path_w"],
                                    d["mix_w"], d["n_nodes"], d["cutoff"], d["edge_scale"])
    rng = np.random.default_rng(0)
    h = 1e-5
    for i in rng.choice(d["n_nodes"], 3, replace=False):
        for k in range(3):
            dp = np.zeros_like(pos)
            dp[i, k] = h
            fd = (energy(d, pos + dp) - energy(d, pos - dp)) / (2 * h)
            assert abs(-fd - F[i, k]) < 1e-6 * max(1.0, np.abs(F).max())
    # translation invariance: no net force
    assert np.abs(F.sum(0)).max() < 1e-9 * max(1.0, np.abs(F).max())


def test_block_energy_rotation_invariant():
    d = small_block()
    pos = d["pos64"]
    ei = d["edge_index"]
    ev = pos[ei[1]] - pos[ei[0]] + d["shift"]
    rng = np.random.default_rng(1)
    q, r = np.linalg.qr(rng.normal(size=(3, 3)))
    R = q * np.sign(np.diag(r))
    xr = rotate_rows(rot_matrices(R, L), d["x"], node_blocks(L), C)
    e0, _, F0 = O.block_energy_forces(L, C, ORDER, ei, ev, d["x"], d["omega"], d["path_w"],
                                      d["mix_w"], d["n_nodes"], d["cutoff"], d["edge_scale"])
    e1, _, F1 = O.block_energy_forces(L, C, ORDER, ei, ev @ R.T, xr, d["omega"], d["path_w"],
                                      d["mix_w"], d["n_nodes"], d["cutoff"], d["edge_scale"])
    np.testing.assert_allclose(e1, e0, atol=1e-10 * np.abs(e0).max())
    np.testing.assert_allclose(F1, F0 @ R.T, atol=1e-9 * np.abs(F0).max())


def test_envelope_closed_form_and_cutoff():
    ev = np.array([[0.0, 0.0, 1.0], [0.0, 2.5, 0.0], [3.0, 4.0, 0.0]])
    s, sp, r = O.envelope(ev, 5.0, 2.0)
    np.testing.assert_allclose(s[:2], (np.cos(np.pi * r[:2] / 5.0) + 1.0), atol=1e-15)
    assert s[2] == 0.0 and sp[2] == 0.0          # |r| = 5 is at the cutoff
    h = 1e-6
    for j in range(2):
        sp_fd = (O.envelope(ev[j:j + 1] * (1 + h / r[j]), 5.0, 2.0)[0][0]
                 - O.envelope(ev[j:j + 1] * (1 - h / r[j]), 5.0, 2.0)[0][0]) / (2 * h)
        assert abs(sp_fd - sp[j]) < 1e-8
