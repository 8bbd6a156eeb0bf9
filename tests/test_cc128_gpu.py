"""GPU parity of the 128-channel kernel instantiations against the FP64 oracle.

At C = 128 the convolution, its VJP and its VJP-of-VJP launch a separate
compile-time-channel specialisation of their kernels (every row offset an
immediate), so each rank's 128-channel code path is compared here with the
oracle, element by element: forward (FlashCart Sec. 4 Eq. 1, Algorithm 1),
VJP (App. C Eq. C1, Algorithm 2) and VJP-of-VJP (App. C Eq. C2,
Algorithm 3) at ranks 1, 2, 4 and 5 (rank 3 is covered at full size in the
other files).  The graphs are ragged: in-degrees 0, 1, 31-33 (one past the
32-edge index window) and 64-65, plus the full-size rank-4 microbenchmark
launch with sampled receivers.  Tolerances: 1e-5 forward, 1e-4 VJPs
(normwise max relative error per output tensor).
"""
import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import FWD_TOL, VJP_TOL, ragged_graph, rel_err

pytestmark = pytest.mark.gpu

C = 128
DEGREES = [0, 1, 31, 32, 33, 64, 65, 0, 7, 2]
DEGREES_R5 = [0, 1, 33, 65, 2]     # the rank-5 oracle forward is slow: fewer edges


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def dev(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def ragged_case(L, seed, sum_paths=False):
    degrees = DEGREES_R5 + [1] * 6 if L == 5 else DEGREES + [2] * 30
    n = len(degrees)
    ei, ev = ragged_graph(n, degrees, 6.0, 500 + 10 * L + seed)
    d = W.conv_inputs(n, ei, L, C, 600 + 10 * L + seed, with_grad=True, sum_paths=sum_paths)
    cot = W.cotangents(n, ei.shape[1], L, C, 700 + 10 * L + seed, ev)
    zero_rows = [i for i, k in enumerate(degrees) if k == 0]
    return dict(lmax=L, channels=C, n_nodes=n, edge_index=ei, edge_vec=ev,
                zero_rows=zero_rows, **d, **cot)


def rowptr_of(fc, wl):
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    return ei, ev, fc.build_rowptr(ei, ev, wl["n_nodes"])


def check(names, got, ref, tol):
    for name, a, b in zip(names, got, ref):
        if a is None or b is None:
            continue
        e = rel_err(np.asarray(a).reshape(b.shape), b)
        assert e <= tol, "%s rel err %g" % (name, e)


@pytest.mark.parametrize("L,sum_paths", [(1, False), (2, False), (2, True), (4, False),
                                         (4, True), (5, False)])
def test_forward_c128_ragged(fc, L, sum_paths):
    wl = ragged_case(L, 1, sum_paths)
    ei, ev, rp = rowptr_of(fc, wl)
    z = fc.edge_conv(L, rp, ei, ev, dev(wl["x"]), dev(wl["w"]), sum_paths=sum_paths)
    torch.cuda.synchronize()
    z = z.cpu().numpy()
    ref = O.edge_conv(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"],
                      wl["n_nodes"], sum_paths=sum_paths)
    assert rel_err(z, ref) <= FWD_TOL
    assert np.all(z[wl["zero_rows"]] == 0)


@pytest.mark.parametrize("L,sum_paths", [(1, False), (2, False), (4, False), (4, True),
                                         (5, False)])
def test_vjp_c128_ragged(fc, L, sum_paths):
    wl = ragged_case(L, 2, sum_paths)
    ei, ev, rp = rowptr_of(fc, wl)
    got = fc.edge_conv_vjp(L, rp, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(wl["g"]),
                           sum_paths=sum_paths)
    torch.cuda.synchronize()
    got = [t.cpu().numpy() for t in got]
    ref = O.edge_conv_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"],
                          wl["g"], wl["n_nodes"], sum_paths=sum_paths)
    check(("x_bar", "w_bar", "r_bar"), got, ref, VJP_TOL)


@pytest.mark.parametrize("L,sum_paths", [(1, False), (2, False), (2, True), (4, False),
                                         (4, True)])
def test_vjp_of_vjp_c128_ragged(fc, L, sum_paths):
    wl = ragged_case(L, 3, sum_paths)
    ei, ev, rp = rowptr_of(fc, wl)
    got = fc.edge_conv_vjp_vjp(L, rp, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(wl["g"]),
                               v_x=dev(wl["vx"]), v_w=dev(wl["vw"]), v_r=dev(wl["vr"]),
                               sum_paths=sum_paths)
    torch.cuda.synchronize()
    got = [t.cpu().numpy() for t in got]
    ref = O.edge_conv_vjp_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"],
                              wl["g"], wl["vx"], wl["vw"], wl["vr"], wl["n_nodes"],
                              sum_paths=sum_paths)
    check(("g_hat", "x_hat", "w_hat", "r_hat"), got, ref, VJP_TOL)
    assert np.all(got[0][wl["zero_rows"]] == 0)


@pytest.fixture(scope="module")
def micro_r4():
    return W.microbench_grad(lmax=4, weight_seed=32)


def test_microbench_rank4_vjp_sampled_receivers(fc, micro_r4):
    """Full-size rank-4 launch (1024 receivers x 128 neighbours x 128
    channels, the timed rank-4 VJP row).  The upstream gradient is kept on a
    few receivers only, so every entry of x_bar, w_bar and r_bar can be
    compared with the oracle over those receivers' edges."""
    wl = micro_r4
    rows = np.array([0, 77, 1023])
    g = np.zeros_like(wl["g"])
    g[rows] = wl["g"][rows]
    ei, ev, rp = rowptr_of(fc, wl)
    got = fc.edge_conv_vjp(4, rp, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(g))
    torch.cuda.synchronize()
    got = [t.cpu().numpy() for t in got]
    em = np.isin(wl["edge_index"][0], rows).astype(np.uint8)
    ref = O.edge_conv_vjp(4, 4, 4, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"], g,
                          wl["n_nodes"], edge_mask=em)
    check(("x_bar", "w_bar", "r_bar"), got, ref, VJP_TOL)


def test_microbench_rank4_vjp_dense_gradient_samples(fc, micro_r4):
    """Dense upstream gradient at full size, rank 4: w_bar and r_bar on the
    edges of sampled receivers, x_bar on sampled senders."""
    wl = micro_r4
    ei, ev, rp = rowptr_of(fc, wl)
    xb, wb, rb = fc.edge_conv_vjp(4, rp, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(wl["g"]))
    torch.cuda.synchronize()
    xb, wb, rb = xb.cpu().numpy(), wb.cpu().numpy(), rb.cpu().numpy()
    recv, send = wl["edge_index"]
    em = np.isin(recv, [5, 700]).astype(np.uint8)
    _, wref, rref = O.edge_conv_vjp(4, 4, 4, C, wl["edge_index"], wl["edge_vec"], wl["x"],
                                    wl["w"], wl["g"], wl["n_nodes"], edge_mask=em)
    sel = em.astype(bool)
    assert rel_err(wb[sel], wref[sel]) <= VJP_TOL
    assert rel_err(rb[sel], rref[sel]) <= VJP_TOL
    senders = np.array([12, 901])
    sm = np.isin(send, senders).astype(np.uint8)
    xref, _, _ = O.edge_conv_vjp(4, 4, 4, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"],
                                 wl["g"], wl["n_nodes"], edge_mask=sm)
    assert rel_err(xb[senders], xref[senders]) <= VJP_TOL


def test_microbench_rank4_vjp_of_vjp_sampled_receivers(fc, micro_r4):
    """Full-size rank-4 VJP-of-VJP launch; g kept on sampled receivers, so
    their g_hat rows and every entry of x_hat, w_hat, r_hat are comparable
    with the oracle over their incoming edges."""
    wl = micro_r4
    ei_np = wl["edge_index"]
    cot = W.cotangents(1024, ei_np.shape[1], 4, C, 62, wl["edge_vec"])
    rows = np.array([1, 640])
    keep = np.zeros((1024, 1), np.float32)
    keep[rows] = 1
    g = wl["g"] * keep
    ei, ev, rp = rowptr_of(fc, wl)
    got = fc.edge_conv_vjp_vjp(4, rp, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(g),
                               v_x=dev(cot["vx"]), v_w=dev(cot["vw"]), v_r=dev(cot["vr"]))
    torch.cuda.synchronize()
    got = [t.cpu().numpy() for t in got]
    em = np.isin(ei_np[0], rows).astype(np.uint8)
    ref = O.edge_conv_vjp_vjp(4, 4, 4, C, ei_np, wl["edge_vec"], wl["x"], wl["w"], g,
                              cot["vx"], cot["vw"], cot["vr"], 1024, edge_mask=em)
    got[0] = got[0].reshape(ref[0].shape)[rows]
    ref = (ref[0][rows],) + tuple(ref[1:])
    check(("g_hat", "x_hat", "w_hat", "r_hat"), got, ref, VJP_TOL)
