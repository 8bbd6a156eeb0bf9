"""GPU parity of fc_edge_conv_vjp (FlashCart App. C Eq. C1, Algorithm 2)
against the FP64 oracle, through the C ABI.  Tolerance: max relative error
1e-4 per output tensor."""
import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import VJP_TOL, ragged_graph, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_vjp(fc, wl, g, sum_paths=False, want=("x", "w", "r")):
    L = wl["lmax"]
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    out = fc.edge_conv_vjp(L, rowptr, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(g),
                           sum_paths=sum_paths, want=want)
    torch.cuda.synchronize()
    return tuple(None if t is None else t.cpu().numpy() for t in out)


def oracle_vjp(wl, g, sum_paths=False, edge_mask=None):
    L, C = wl["lmax"], wl["channels"]
    return O.edge_conv_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"],
                           wl["w"], g, wl["n_nodes"], sum_paths=sum_paths,
                           edge_mask=edge_mask)


def check_all(got, ref):
    names = ("x_bar", "w_bar", "r_bar")
    for name, a, b in zip(names, got, ref):
        if a is None:
            continue
        e = rel_err(a.reshape(b.shape), b)
        assert e <= VJP_TOL, "%s rel err %g" % (name, e)


def test_tiny_vjp(fc):
    wl = W.tiny()
    g = np.random.default_rng(5).standard_normal(
        (wl["n_nodes"], O.zrow(2, 2, 2) * wl["channels"])).astype(np.float32)
    check_all(gpu_vjp(fc, wl, g), oracle_vjp(wl, g))


def test_tiny_rank4_vjp(fc):
    """Rank 4 on the tiny graph, upstream gradient N(0,1)."""
    wl = W.tiny_r4()
    check_all(gpu_vjp(fc, wl, wl["g"]), oracle_vjp(wl, wl["g"]))


@pytest.mark.parametrize("sum_paths", [True])
def test_tiny_vjp_sum_paths(fc, sum_paths):
    wl = W.tiny()
    wl = dict(wl, lmax=3, **W.conv_inputs(wl["n_nodes"], wl["edge_index"], 3, 8, 78))
    g = np.random.default_rng(6).standard_normal((wl["n_nodes"], 16 * 8)).astype(np.float32)
    check_all(gpu_vjp(fc, wl, g, sum_paths=True), oracle_vjp(wl, g, sum_paths=True))


def test_vjp_optional_outputs(fc):
    wl = W.tiny()
    g = np.random.default_rng(7).standard_normal(
        (wl["n_nodes"], O.zrow(2, 2, 2) * wl["channels"])).astype(np.float32)
    ref = oracle_vjp(wl, g)
    for want in (("x",), ("w",), ("r",), ("x", "r")):
        got = gpu_vjp(fc, wl, g, want=want)
        check_all(got, ref)
        for k, t in zip("xwr", got):
            assert (t is None) == (k not in want)


@pytest.fixture(scope="module")
def micro_grad():
    wl = W.microbench_grad(lmax=3)
    return wl


def test_microbench_vjp_sampled_receivers(fc, micro_grad):
    """Full-size launch; the upstream gradient is nonzero only on a few
    receivers, so every entry of x_bar, w_bar and r_bar can be compared with
    an oracle run over those receivers' edges."""
    wl = micro_grad
    rows = np.array([0, 77, 512, 1023])
    g = np.zeros_like(wl["g"])
    g[rows] = wl["g"][rows]
    edge_mask = np.isin(wl["edge_index"][0], rows).astype(np.uint8)
    check_all(gpu_vjp(fc, wl, g), oracle_vjp(wl, g, edge_mask=edge_mask))


def test_microbench_vjp_dense_gradient_samples(fc, micro_grad):
    """Dense upstream gradient at full size: w_bar and r_bar compared on the
    edges of sampled receivers (they depend on that edge only), x_bar on
    sampled senders (the oracle sums every edge they send on)."""
    wl = micro_grad
    xb, wb, rb = gpu_vjp(fc, wl, wl["g"])
    recv, send = wl["edge_index"]
    rows = np.array([3, 600])
    em = np.isin(recv, rows).astype(np.uint8)
    _, wref, rref = oracle_vjp(wl, wl["g"], edge_mask=em)
    sel = em.astype(bool)
    assert rel_err(wb[sel], wref[sel]) <= VJP_TOL
    assert rel_err(rb[sel], rref[sel]) <= VJP_TOL
    senders = np.array([10, 900])
    sm = np.isin(send, senders).astype(np.uint8)
    xref, _, _ = oracle_vjp(wl, wl["g"], edge_mask=sm)
    assert rel_err(xb[senders], xref[senders]) <= VJP_TOL
    # T depends on the edge direction only: r_bar is orthogonal to r
    r = wl["edge_vec"].astype(np.float64)
    dots = np.abs((rb * r).sum(1)) / (np.linalg.norm(rb, axis=1) * np.linalg.norm(r, axis=1) + 1e-30)
    assert dots.max() < 1e-3


@pytest.mark.parametrize("L,C", [(1, 8), (1, 64), (2, 4), (3, 40), (3, 200), (4, 12), (5, 8)])
def test_vjp_ragged_and_channel_tails(fc, L, C):
    degrees = [0, 1, 31, 32, 33, 40, 2, 0] + [3] * 40
    N = len(degrees)
    ei, ev = ragged_graph(N, degrees, 6.0, 7 * L + C)
    wl = dict(n_nodes=N, lmax=L, channels=C, edge_index=ei, edge_vec=ev,
              **W.conv_inputs(N, ei, L, C, 31 + C, with_grad=True))
    check_all(gpu_vjp(fc, wl, wl["g"]), oracle_vjp(wl, wl["g"]))


@pytest.mark.parametrize("sum_paths", [False, True])
def test_envelope_vjp(fc, sum_paths):
    """With the envelope s(|r|): x_bar as for weights w s, w_bar = s <g, f>,
    and r_bar gains s'(|r|) r_hat sum_{p,k} w <g, f>."""
    wl = W.tiny()
    wl = dict(wl, lmax=3, **W.conv_inputs(wl["n_nodes"], wl["edge_index"], 3, 8, 92,
                                         with_grad=True, sum_paths=sum_paths))
    r_cut, scale = 2.5, 0.7
    s, sp, r = O.envelope(wl["edge_vec"], r_cut, scale)
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    xb, wb, rb = fc.edge_conv_vjp(3, rowptr, ei, ev, dev(wl["x"]), dev(wl["w"]), dev(wl["g"]),
                                  sum_paths=sum_paths, envelope=(r_cut, scale))
    w_eff = wl["w"] * s[:, None, None]
    rxb, rwb, rrb = O.edge_conv_vjp(3, 3, 3, 8, wl["edge_index"], wl["edge_vec"], wl["x"], w_eff,
                                    wl["g"], wl["n_nodes"], sum_paths=sum_paths)
    ev64 = wl["edge_vec"].astype(np.float64)
    rrb = rrb + ((rwb * wl["w"]).sum((1, 2)) * sp)[:, None] * ev64 / r[:, None]
    check_all((xb.cpu().numpy(), wb.cpu().numpy(), rb.cpu().numpy()),
              (rxb, rwb * s[:, None, None], rrb))


@pytest.mark.parametrize("L", [1, 2, 3, 4])
def test_vjp_half_warp_pairs_c64(fc, L):
    """C = 64 runs two receivers per warp, one per half-warp: an odd receiver
    count leaves the last warp's second half without a receiver, and paired
    receivers of unequal degree (0 beside 33, 64 beside 65, 16 beside 17)
    walk their edges in step; the edge-vector gradient is reduced over each
    half's 16 lanes."""
    degrees = [0, 33, 1, 0, 31, 64, 65, 2, 16, 17, 15, 0, 70, 3, 5] + [3] * 60
    N = len(degrees)                                        # 75 receivers
    ei, ev = ragged_graph(N, degrees, 6.0, 900 + L)
    wl = dict(n_nodes=N, lmax=L, channels=64, edge_index=ei, edge_vec=ev,
              **W.conv_inputs(N, ei, L, 64, 910 + L, with_grad=True))
    check_all(gpu_vjp(fc, wl, wl["g"]), oracle_vjp(wl, wl["g"]))


def test_vjp_half_warp_pairs_c64_sum_paths_envelope(fc):
    """The C = 64 pairing with path sums and the cosine envelope."""
    degrees = [5, 0, 12, 40, 41, 3, 1] + [2] * 44
    N = len(degrees)                                        # 51 receivers
    ei, ev = ragged_graph(N, degrees, 3.0, 79)
    inp = W.conv_inputs(N, ei, 3, 64, 80, with_grad=True, sum_paths=True)
    r_cut, scale = 2.5, 0.7
    s, sp, r = O.envelope(ev, r_cut, scale)
    rowptr = fc.build_rowptr(dev(ei), dev(ev), N)
    xb, wb, rb = fc.edge_conv_vjp(3, rowptr, dev(ei), dev(ev), dev(inp["x"]), dev(inp["w"]),
                                  dev(inp["g"]), sum_paths=True, envelope=(r_cut, scale))
    rxb, rwb, rrb = O.edge_conv_vjp(3, 3, 3, 64, ei, ev, inp["x"], inp["w"] * s[:, None, None],
                                    inp["g"], N, sum_paths=True)
    rrb = rrb + ((rwb * inp["w"]).sum((1, 2)) * sp)[:, None] * ev.astype(np.float64) / r[:, None]
    check_all((xb.cpu().numpy(), wb.cpu().numpy(), rb.cpu().numpy()),
              (rxb, rwb * s[:, None, None], rrb))
