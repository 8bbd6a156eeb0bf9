"""GPU parity of fc_edge_conv (FlashCart Sec. 4 Eq. 1, Algorithm 1) against
the FP64 oracle, through the C ABI.  Tolerance: max relative error 1e-5."""
import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import (FWD_TOL, node_blocks, out_blocks, ragged_graph, rel_err,
                    rot_matrices, rotate_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def gpu_conv(fc, wl, sum_paths=False, lmax=None):
    L = wl["lmax"] if lmax is None else lmax
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    z = fc.edge_conv(L, rowptr, ei, ev, dev(wl["x"]), dev(wl["w"]), sum_paths=sum_paths)
    torch.cuda.synchronize()
    return z.cpu().numpy()


def oracle_conv(wl, sum_paths=False, recv_mask=None):
    L, C = wl["lmax"], wl["channels"]
    return O.edge_conv(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"],
                       wl["w"], wl["n_nodes"], sum_paths=sum_paths, recv_mask=recv_mask)


@pytest.fixture(scope="module")
def micro():
    return W.microbench()


def test_tiny_full(fc):
    wl = W.tiny()
    assert rel_err(gpu_conv(fc, wl), oracle_conv(wl)) <= FWD_TOL


def test_tiny_rank4_forward(fc):
    wl = W.tiny_r4()
    assert rel_err(gpu_conv(fc, wl), oracle_conv(wl)) <= FWD_TOL


@pytest.mark.parametrize("sum_paths", [False, True])
def test_tiny_sum_paths(fc, sum_paths):
    wl = W.tiny()
    wl = dict(wl, lmax=3, channels=8,
              **W.conv_inputs(wl["n_nodes"], wl["edge_index"], 3, 8, 77))
    assert rel_err(gpu_conv(fc, wl, sum_paths), oracle_conv(wl, sum_paths)) <= FWD_TOL


def test_microbench_sampled_receivers(fc, micro):
    """Full-size launch (1024 receivers x 128 neighbours x 128 channels,
    rank 3); receivers compared one by one against the oracle."""
    z = gpu_conv(fc, micro)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1023], rng.choice(1024, 4, replace=False)]))
    m = np.zeros(1024, np.uint8)
    m[rows] = 1
    ref = oracle_conv(micro, recv_mask=m)
    assert rel_err(z[rows], ref[rows]) <= FWD_TOL
    assert np.isfinite(z).all()


def test_microbench_edge_order_invariance(fc, micro):
    """Permuting edges inside every receiver changes only rounding."""
    z = gpu_conv(fc, micro)
    E = micro["edge_index"].shape[1]
    rng = np.random.default_rng(1)
    perm = np.argsort(micro["edge_index"][0] * 4.0 + rng.random(E), kind="stable")
    wl2 = dict(micro, edge_index=micro["edge_index"][:, perm],
               edge_vec=micro["edge_vec"][perm], w=micro["w"][perm])
    assert rel_err(gpu_conv(fc, wl2), z) <= FWD_TOL


def test_microbench_rotation_equivariance(fc, micro):
    L, C = 3, 128
    rng = np.random.default_rng(2)
    q, r = np.linalg.qr(rng.normal(size=(3, 3)))
    R = q * np.sign(np.diag(r))
    D = rot_matrices(R, L)
    z = gpu_conv(fc, micro)
    xr = rotate_rows(D, micro["x"], node_blocks(L), C).astype(np.float32)
    evr = (micro["edge_vec"].astype(np.float64) @ R.T).astype(np.float32)
    zr = gpu_conv(fc, dict(micro, x=xr, edge_vec=evr))
    assert rel_err(zr, rotate_rows(D, z, out_blocks(L), C)) <= 1e-5


def test_microbench_rank4_sampled(fc):
    wl = W.microbench(lmax=4, weight_seed=32)
    z = gpu_conv(fc, wl)
    rows = np.array([3, 511, 1000])
    m = np.zeros(1024, np.uint8)
    m[rows] = 1
    ref = oracle_conv(wl, recv_mask=m)
    assert rel_err(z[rows], ref[rows]) <= FWD_TOL


@pytest.mark.parametrize("L,C", [(1, 8), (1, 64), (2, 4), (3, 40), (3, 200), (4, 12), (5, 8)])
def test_ragged_degrees_and_channel_tails(fc, L, C):
    degrees = [0, 1, 31, 32, 33, 64, 65, 0, 7, 70, 2, 0]
    ei, ev = ragged_graph(len(degrees) + 60, degrees + [3] * 60, 6.0, L * 1000 + C)
    wl = dict(n_nodes=len(degrees) + 60, lmax=L, channels=C, edge_index=ei,
              edge_vec=ev, **W.conv_inputs(len(degrees) + 60, ei, L, C, C))
    z = gpu_conv(fc, wl)
    ref = oracle_conv(wl)
    assert rel_err(z, ref) <= FWD_TOL
    zero_rows = [i for i, k in enumerate(degrees) if k == 0]
    assert np.all(z[zero_rows] == 0)


def test_empty_graph(fc):
    N, L, C = 5, 3, 8
    ei = np.zeros((2, 0), np.int32)
    ev = np.zeros((0, 3), np.float32)
    wl = dict(n_nodes=N, lmax=L, channels=C, edge_index=ei, edge_vec=ev,
              x=np.ones((N, 16 * C), np.float32), w=np.zeros((0, 23, C), np.float32))
    z = gpu_conv(fc, wl)
    assert z.shape == (N, 99 * C) and np.all(z == 0)


def test_graph_validation(fc):
    ei = dev(np.array([[0, 1, 1], [1, 0, 2]], np.int32))
    ev = dev(np.ones((3, 3), np.float32))
    assert fc.build_rowptr(ei, ev, 3).cpu().tolist() == [0, 1, 3, 3]
    with pytest.raises(fc.FlashCartError) as e:      # unsorted receivers
        fc.build_rowptr(dev(np.array([[1, 0, 1], [0, 1, 2]], np.int32)), ev, 3)
    assert e.value.status == 2
    with pytest.raises(fc.FlashCartError) as e:      # sender out of range
        fc.build_rowptr(dev(np.array([[0, 1, 1], [1, 0, 3]], np.int32)), ev, 3)
    assert e.value.status == 2
    with pytest.raises(fc.FlashCartError) as e:      # receiver out of range
        fc.build_rowptr(dev(np.array([[0, 1, 5], [1, 0, 2]], np.int32)), ev, 3)
    assert e.value.status == 2
    bad = np.ones((3, 3), np.float32)
    bad[1] = 0
    with pytest.raises(fc.FlashCartError) as e:      # zero-length edge vector
        fc.build_rowptr(ei, dev(bad), 3)
    assert e.value.status == 3
    assert fc.build_rowptr(dev(np.zeros((2, 0), np.int32)), None, 4).cpu().tolist() == [0] * 5


@pytest.mark.parametrize("sum_paths", [False, True])
def test_envelope_forward(fc, sum_paths):
    """Cosine radial envelope: equal to scaling every weight of edge e by
    s(|r_e|) (bilinearity); some edges lie beyond the cutoff."""
    wl = W.tiny()
    wl = dict(wl, lmax=3, **W.conv_inputs(wl["n_nodes"], wl["edge_index"], 3, 8, 91))
    r_cut, scale = 2.5, 0.7
    s, _, _ = O.envelope(wl["edge_vec"], r_cut, scale)
    assert (s == 0).any() and (s > 0).any()
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    z = fc.edge_conv(3, rowptr, ei, ev, dev(wl["x"]), dev(wl["w"]), sum_paths=sum_paths,
                     envelope=(r_cut, scale)).cpu().numpy()
    ref = O.edge_conv(3, 3, 3, 8, wl["edge_index"], wl["edge_vec"], wl["x"],
                      wl["w"] * s[:, None, None], wl["n_nodes"], sum_paths=sum_paths)
    assert rel_err(z, ref) <= FWD_TOL


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5])
def test_half_warp_pairs_c64(fc, L):
    """C = 64 runs two receivers per warp, one per half-warp.  An odd receiver
    count leaves the last warp's second half without a receiver; paired
    receivers of different degree (0 beside 33, 64 beside 65, 16 beside 17,
    ...) walk their edges in step, the shorter one sitting out.  Rank 5 is
    checked on a receiver sample (the FP64 oracle is slow there)."""
    degrees = [0, 33, 1, 0, 31, 64, 65, 2, 16, 17, 15, 0, 70, 3, 5]
    N = len(degrees) + 60                                   # 75 receivers
    ei, ev = ragged_graph(N, degrees + [4] * 60, 6.0, 500 + L)
    wl = dict(n_nodes=N, lmax=L, channels=64, edge_index=ei, edge_vec=ev,
              **W.conv_inputs(N, ei, L, 64, 64 + L))
    z = gpu_conv(fc, wl)
    rows = list(range(N)) if L <= 4 else [0, 1, 2, 7, 8, 9, N - 2, N - 1]
    m = np.zeros(N, np.uint8)
    m[rows] = 1
    ref = oracle_conv(wl, recv_mask=m)
    assert rel_err(z[rows], ref[rows]) <= FWD_TOL
    zero_rows = [i for i, k in enumerate(degrees) if k == 0]
    assert np.all(z[zero_rows] == 0)


@pytest.mark.parametrize("sum_paths", [False, True])
def test_half_warp_pairs_c64_envelope(fc, sum_paths):
    """The C = 64 pairing with the cosine envelope and with path sums."""
    degrees = [5, 0, 12, 40, 41, 3, 1] + [2] * 44
    N = len(degrees)                                        # 51 receivers
    ei, ev = ragged_graph(N, degrees, 3.0, 77)
    inp = W.conv_inputs(N, ei, 3, 64, 78, sum_paths=sum_paths)
    r_cut, scale = 2.5, 0.7
    s, _, _ = O.envelope(ev, r_cut, scale)
    assert (s == 0).any() and (s > 0).any()
    rowptr = fc.build_rowptr(dev(ei), dev(ev), N)
    z = fc.edge_conv(3, rowptr, dev(ei), dev(ev), dev(inp["x"]), dev(inp["w"]), sum_paths=sum_paths,
                     envelope=(r_cut, scale)).cpu().numpy()
    ref = O.edge_conv(3, 3, 3, 64, ei, ev, inp["x"], inp["w"] * s[:, None, None], N,
                      sum_paths=sum_paths)
    assert rel_err(z, ref) <= FWD_TOL
