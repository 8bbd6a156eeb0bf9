"""GPU parity of the interaction block (envelope-weighted edge convolution with
summed paths, order-5 product ladder, E = sum of rank-0 outputs, forces from
the VJPs) against the FP64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import FWD_TOL, VJP_TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_block(fc, d):
    L, order = d["lmax"], d["order"]
    ei, ev = dev(d["edge_index"]), dev(d["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, d["n_nodes"])
    energy, F, z = fc.interaction_block(L, order, rowptr, ei, ev, dev(d["x"]), dev(d["omega"]),
                                        dev(d["path_w"]), dev(d["mix_w"]), d["cutoff"],
                                        d["edge_scale"])
    torch.cuda.synchronize()
    C = d["channels"]
    return float(energy.item()), F.cpu().numpy(), z[:, :C].sum(1).cpu().numpy()


def test_small_diamond_block_full(fc):
    d = W.diamond(cells=2, cutoff=3.0, channels=8, lmax=3, order=5, seed=12)
    E, F, e_node = gpu_block(fc, d)
    re, _, rF = O.block_energy_forces(3, 8, 5, d["edge_index"], d["edge_vec"], d["x"],
                                      d["omega"], d["path_w"], d["mix_w"], d["n_nodes"],
                                      d["cutoff"], d["edge_scale"])
    assert rel_err(e_node, re) <= FWD_TOL
    assert abs(E - re.sum()) <= FWD_TOL * np.abs(re).sum()
    assert rel_err(F, rF) <= VJP_TOL


def test_diamond_1000_sampled(fc):
    """The 1000-atom diamond cell at full size.  Per-atom energies are
    node-local given the atom's incoming edges; an atom's force needs the
    edge gradients of its incoming edges and of the edges it sends on, which
    the oracle forms over exactly those receivers."""
    d = W.diamond()
    E, F, e_node = gpu_block(fc, d)
    recv, send = d["edge_index"]
    atoms = np.array([0, 517])
    need = set(atoms.tolist())
    for i in atoms:
        need |= set(recv[send == i].tolist())
    mask = np.zeros(d["n_nodes"], np.uint8)
    mask[sorted(need)] = 1
    re, dEdr, _ = O.block_energy_forces(d["lmax"], d["channels"], d["order"], d["edge_index"],
                                        d["edge_vec"], d["x"], d["omega"], d["path_w"],
                                        d["mix_w"], d["n_nodes"], d["cutoff"], d["edge_scale"],
                                        recv_mask=mask)
    rows = np.nonzero(mask)[0]
    assert rel_err(e_node[rows], re[rows]) <= FWD_TOL
    # normwise against the whole force tensor: max over the sampled atoms of
    # |F_i - ref_i| <= 1e-4 max|F| (the full reference is not formed)
    fmax = np.abs(F).max()
    for i in atoms:
        ref = -(dEdr[send == i].sum(0) - dEdr[recv == i].sum(0))
        assert np.abs(F[i] - ref).max() <= VJP_TOL * fmax
    # translation invariance at full size
    assert np.abs(F.sum(0)).max() <= 1e-3 * np.abs(F).max()
    assert np.isfinite(E)
