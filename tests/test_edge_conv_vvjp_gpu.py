"""GPU parity of fc_edge_conv_vjp_vjp (FlashCart App. C Eq. C2, Algorithm 3)
against the FP64 oracle, through the C ABI.  Tolerance: max relative error
1e-4 per output tensor (the VJP tolerance)."""
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
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def case(L, C, ei, ev, n_nodes, seed, sum_paths=False):
    d = W.conv_inputs(n_nodes, ei, L, C, seed, with_grad=True, sum_paths=sum_paths)
    cot = W.cotangents(n_nodes, ei.shape[1], L, C, seed + 1, ev)
    return dict(lmax=L, channels=C, n_nodes=n_nodes, edge_index=ei, edge_vec=ev, **d, **cot)


def gpu_vvjp(fc, wl, sum_paths=False, use=("vx", "vw", "vr")):
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    out = fc.edge_conv_vjp_vjp(wl["lmax"], rowptr, ei, ev, dev(wl["x"]), dev(wl["w"]),
                               dev(wl["g"]), dev(wl["vx"] if "vx" in use else None),
                               dev(wl["vw"] if "vw" in use else None),
                               dev(wl["vr"] if "vr" in use else None), sum_paths=sum_paths)
    torch.cuda.synchronize()
    assert fc.device_error() == 0
    return tuple(t.cpu().numpy() for t in out)


def oracle_vvjp(wl, sum_paths=False, use=("vx", "vw", "vr"), edge_mask=None, g=None):
    L, C = wl["lmax"], wl["channels"]
    return O.edge_conv_vjp_vjp(L, L, L, C, wl["edge_index"], wl["edge_vec"], wl["x"], wl["w"],
                               wl["g"] if g is None else g,
                               wl["vx"] if "vx" in use else None,
                               wl["vw"] if "vw" in use else None,
                               wl["vr"] if "vr" in use else None, wl["n_nodes"],
                               sum_paths=sum_paths, edge_mask=edge_mask)


def check_all(got, ref, rows=None):
    for name, a, b in zip(("g_hat", "x_hat", "w_hat", "r_hat"), got, ref):
        a = a.reshape(b.shape)
        if rows is not None and name == "g_hat":
            a, b = a[rows], b[rows]
        e = rel_err(a, b)
        assert e <= VJP_TOL, "%s rel err %g" % (name, e)


def test_tiny_rank2(fc):
    t = W.tiny()
    wl = case(2, 8, t["edge_index"], t["edge_vec"], t["n_nodes"], 41)
    check_all(gpu_vvjp(fc, wl), oracle_vvjp(wl))


def test_tiny_rank4(fc):
    t = W.tiny()
    wl = case(4, 8, t["edge_index"], t["edge_vec"], t["n_nodes"], 43)
    check_all(gpu_vvjp(fc, wl), oracle_vvjp(wl))


@pytest.mark.parametrize("use", [("vx",), ("vw",), ("vr",), ("vx", "vr")])
def test_single_cotangents(fc, use):
    t = W.tiny()
    wl = case(3, 8, t["edge_index"], t["edge_vec"], t["n_nodes"], 45)
    check_all(gpu_vvjp(fc, wl, use=use), oracle_vvjp(wl, use=use))


@pytest.mark.parametrize("L,C,sum_paths", [(1, 8, False), (1, 64, True), (3, 40, False), (3, 40, True), (2, 200, False),
                                           (4, 12, True)])
def test_ragged_degrees_and_channel_tails(fc, L, C, sum_paths):
    degrees = [0, 1, 31, 32, 33, 64, 65, 0, 7, 70, 2, 0]
    n = len(degrees) + 40
    ei, ev = ragged_graph(n, degrees + [3] * 40, 6.0, 7 * L + C)
    wl = case(L, C, ei, ev, n, L * 100 + C, sum_paths)
    got = gpu_vvjp(fc, wl, sum_paths)
    check_all(got, oracle_vvjp(wl, sum_paths))
    zero_rows = [i for i, k in enumerate(degrees) if k == 0]
    assert np.all(got[0][zero_rows] == 0)


def test_forward_identity_only_vx(fc):
    """With only vx, g_hat is the forward convolution of vx (both on the GPU)."""
    t = W.tiny()
    wl = case(3, 8, t["edge_index"], t["edge_vec"], t["n_nodes"], 47)
    gh = gpu_vvjp(fc, wl, use=("vx",))[0]
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    z = fc.edge_conv(3, rowptr, ei, ev, dev(wl["vx"]), dev(wl["w"])).cpu().numpy()
    assert rel_err(gh, z) <= 1e-5


def test_microbench_sampled_receivers(fc):
    """Full-size launch (1024 receivers x 128 neighbours x 128 channels,
    rank 3).  g is kept only on sampled receivers, which makes g_hat rows
    of those receivers and every entry of x_hat, w_hat, r_hat comparable
    with the oracle run over their incoming edges."""
    mb = W.microbench_grad(lmax=3)
    ei, ev = mb["edge_index"], mb["edge_vec"]
    cot = W.cotangents(1024, ei.shape[1], 3, 128, 61, ev)
    rows = np.array([0, 517, 1023])
    keep = np.zeros((1024, 1), np.float32)
    keep[rows] = 1
    g = mb["g"] * keep
    wl = dict(lmax=3, channels=128, n_nodes=1024, edge_index=ei, edge_vec=ev, x=mb["x"],
              w=mb["w"], g=g, **cot)
    got = gpu_vvjp(fc, wl)
    emask = np.isin(ei[0], rows).astype(np.uint8)
    ref = oracle_vvjp(wl, edge_mask=emask)
    check_all(got, ref, rows=rows)
    assert np.all(np.isfinite(got[0]))


@pytest.mark.parametrize("C,degrees", [(4, None), (8, None), (128, [0, 1, 33, 2, 1, 1, 1, 1])])
def test_rank5_split_launches(fc, C, degrees):
    """Rank 5 runs one launch per path group (52 groups, each its own
    kernel); every output against the oracle, on the tiny graph and, at
    C = 128 (the compile-time-channel kernels), on a small ragged graph."""
    if degrees is None:
        t = W.tiny()
        ei, ev, n = t["edge_index"], t["edge_vec"], t["n_nodes"]
    else:
        n = len(degrees) + 4
        ei, ev = ragged_graph(n, degrees + [1] * 4, 6.0, 555)
    wl = case(5, C, ei, ev, n, 57 + C)
    got = gpu_vvjp(fc, wl)
    check_all(got, oracle_vvjp(wl))


def test_envelope_is_refused_and_empty_graph(fc):
    t = W.tiny()
    wl = case(2, 8, t["edge_index"], t["edge_vec"], t["n_nodes"], 49)
    ei, ev = dev(wl["edge_index"]), dev(wl["edge_vec"])
    rowptr = fc.build_rowptr(ei, ev, wl["n_nodes"])
    import ctypes as ct
    d = fc.conv_desc(2, 8, False, (2.0, 1.0))
    st = fc.lib().fc_edge_conv_vjp_vjp(ct.byref(d), wl["n_nodes"], ei.shape[1], fc._ptr(rowptr),
                                       fc._ptr(ei), fc._ptr(ev), fc._ptr(dev(wl["x"])),
                                       fc._ptr(dev(wl["w"])), fc._ptr(dev(wl["g"])), None, None,
                                       None, None, None, None, None, None)
    assert st == 1      # FC_ERR_ARG
    # a graph without edges: g_hat and x_hat are zero
    N = 5
    e0 = torch.zeros((2, 0), dtype=torch.int32, device="cuda")
    v0 = torch.zeros((0, 3), dtype=torch.float32, device="cuda")
    rp = fc.build_rowptr(e0, v0, N)
    x = torch.ones((N, 9 * 4), device="cuda")
    g = torch.ones((N, O.zrow(2, 2, 2) * 4), device="cuda")
    w = torch.zeros((0, 11, 4), device="cuda")
    gh, xh, wh, rh = fc.edge_conv_vjp_vjp(2, rp, e0, v0, x, w, g, v_x=x)
    torch.cuda.synchronize()
    assert torch.all(gh == 0) and torch.all(xh == 0) and wh.numel() == 0 and rh.numel() == 0


@pytest.mark.parametrize("L,sum_paths", [(1, False), (2, True), (3, False), (3, True), (4, False)])
def test_half_warp_pairs_c64(fc, L, sum_paths):
    """C = 64 runs two receivers per warp, one per half-warp: an odd receiver
    count leaves the last warp's second half without a receiver, and paired
    receivers of unequal degree (0 beside 33, 16 beside 17, 40 beside 2) walk
    their edges in step; the 12 u-space numbers of r_hat are reduced over each
    half's 16 lanes."""
    degrees = [0, 33, 1, 0, 31, 40, 2, 16, 17, 15, 0, 3] + [3] * 25
    N = len(degrees)                                        # 37 receivers
    ei, ev = ragged_graph(N, degrees, 6.0, 300 + L)
    wl = case(L, 64, ei, ev, N, 310 + L, sum_paths=sum_paths)
    check_all(gpu_vvjp(fc, wl, sum_paths=sum_paths), oracle_vvjp(wl, sum_paths=sum_paths))
