"""GPU parity of the odd-J (Levi-Civita) path convolution and its VJP
(FlashCart App. B, paragraph after Eq. B1; Sec. 7; Eq. 1 and App. C Eq. C1
summed as in Algorithms 1 and 2) against the FP64 oracle, through the C ABI.
Tolerances: 1e-5 forward, 1e-4 VJP (normwise max relative error)."""
import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import FWD_TOL, VJP_TOL, ragged_graph, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def odd_inputs(n, ei, L, C, seed, sum_paths=False):
    g = np.random.default_rng(seed)
    P = len(O.paths(L, L, L, odd=True))
    x = g.standard_normal((n, (L + 1) ** 2 * C)).astype(np.float32)
    w = (g.standard_normal((ei.shape[1], P, C)) / np.sqrt(P)).astype(np.float32)
    zr = O.zrow(L, L, L, sum_paths, odd=True)
    gz = g.standard_normal((n, zr * C)).astype(np.float32)
    return x, w, gz


def run(fc, L, ei, ev, n, x, w, gz, sum_paths):
    dei, dev_ = dev(ei), dev(ev)
    rp = fc.build_rowptr(dei, dev_, n)
    z = fc.edge_conv(L, rp, dei, dev_, dev(x), dev(w), sum_paths=sum_paths, odd=True)
    vj = fc.edge_conv_vjp(L, rp, dei, dev_, dev(x), dev(w), dev(gz), sum_paths=sum_paths, odd=True)
    torch.cuda.synchronize()
    return z.cpu().numpy(), [t.cpu().numpy() for t in vj]


@pytest.mark.parametrize("L,C,sum_paths", [(1, 8, False), (2, 8, False), (3, 8, False),
                                           (4, 8, False), (3, 8, True), (2, 128, False),
                                           (3, 128, False), (4, 128, True), (3, 40, False),
                                           (2, 200, True)])
def test_odd_conv_ragged(fc, L, C, sum_paths):
    degrees = [0, 1, 31, 32, 33, 64, 65, 0, 7, 2] + [3] * 20
    n = len(degrees)
    ei, ev = ragged_graph(n, degrees, 6.0, 900 + 10 * L + C)
    x, w, gz = odd_inputs(n, ei, L, C, 17 * L + C, sum_paths)
    z, (xb, wb, rb) = run(fc, L, ei, ev, n, x, w, gz, sum_paths)
    ref = O.edge_conv(L, L, L, C, ei, ev, x, w, n, sum_paths=sum_paths, odd=True)
    assert rel_err(z, ref) <= FWD_TOL
    assert np.all(z[[i for i, k in enumerate(degrees) if k == 0]] == 0)
    rx, rw, rr = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, gz, n, sum_paths=sum_paths, odd=True)
    for name, a, b in (("x_bar", xb, rx), ("w_bar", wb, rw), ("r_bar", rb, rr)):
        e = rel_err(a.reshape(b.shape), b)
        assert e <= VJP_TOL, "%s rel err %g" % (name, e)


def test_odd_conv_microbench_sampled_receivers(fc):
    """Full-size rank-3 launch on the microbenchmark graph (1024 receivers x
    128 neighbours x 128 channels), sampled receivers compared one by one;
    the VJP with the upstream gradient kept on those receivers."""
    mb = W.microbench()
    ei, ev, N, L, C = mb["edge_index"], mb["edge_vec"], 1024, 3, 128
    x, w, gz = odd_inputs(N, ei, L, C, 5)
    rows = np.array([0, 300, 1023])
    keep = np.zeros((N, 1), np.float32)
    keep[rows] = 1
    gz = gz * keep
    z, (xb, wb, rb) = run(fc, L, ei, ev, N, x, w, gz, False)
    m = np.zeros(N, np.uint8)
    m[rows] = 1
    ref = O.edge_conv(L, L, L, C, ei, ev, x, w, N, recv_mask=m, odd=True)
    assert rel_err(z[rows], ref[rows]) <= FWD_TOL
    em = m[ei[0]]
    rx, rw, rr = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, gz, N, edge_mask=em, odd=True)
    assert rel_err(xb, rx) <= VJP_TOL
    assert rel_err(wb.reshape(rw.shape), rw) <= VJP_TOL
    assert rel_err(rb, rr) <= VJP_TOL


def test_odd_rank5_is_refused(fc):
    t = W.tiny()
    ei, ev = dev(t["edge_index"]), dev(t["edge_vec"])
    rp = fc.build_rowptr(ei, ev, t["n_nodes"])
    import ctypes as ct
    d = fc.conv_desc(5, 4)
    x = torch.zeros((t["n_nodes"], 36 * 4), device="cuda")
    z = torch.zeros((t["n_nodes"], 4096), device="cuda")
    st = fc.lib().fc_edge_conv_odd(ct.byref(d), t["n_nodes"], ei.shape[1], fc._ptr(rp), fc._ptr(ei),
                                   fc._ptr(ev), fc._ptr(x), fc._ptr(x), fc._ptr(z), None)
    assert st == 4


@pytest.mark.parametrize("L,sum_paths", [(1, False), (2, True), (3, False), (4, False)])
def test_odd_conv_half_warp_pairs_c64(fc, L, sum_paths):
    """C = 64 runs two receivers per warp, one per half-warp, for the odd-J
    paths too: an odd receiver count and paired receivers of unequal degree
    (0 beside 33, 40 beside 2, 16 beside 17), forward and VJP."""
    degrees = [0, 33, 1, 0, 31, 40, 2, 16, 17] + [3] * 40
    n = len(degrees)                                        # 49 receivers
    C = 64
    ei, ev = ragged_graph(n, degrees, 6.0, 950 + L)
    x, w, gz = odd_inputs(n, ei, L, C, 960 + L, sum_paths)
    z, (xb, wb, rb) = run(fc, L, ei, ev, n, x, w, gz, sum_paths)
    ref = O.edge_conv(L, L, L, C, ei, ev, x, w, n, sum_paths=sum_paths, odd=True)
    assert rel_err(z, ref) <= FWD_TOL
    assert np.all(z[[i for i, k in enumerate(degrees) if k == 0]] == 0)
    rx, rw, rr = O.edge_conv_vjp(L, L, L, C, ei, ev, x, w, gz, n, sum_paths=sum_paths, odd=True)
    for name, a, b in (("x_bar", xb, rx), ("w_bar", wb, rw), ("r_bar", rb, rr)):
        e = rel_err(a.reshape(b.shape), b)
        assert e <= VJP_TOL, "%s rel err %g" % (name, e)
