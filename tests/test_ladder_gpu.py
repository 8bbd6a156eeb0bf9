"""GPU parity of fc_product_ladder / fc_product_ladder_vjp (FlashCart Sec. 5
Eq. 2 with path-reduced products and per-rank channel mixing) against the
FP64 oracle, through the C ABI.  Tolerances: 1e-5 forward, 1e-4 VJP."""
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


def run_gpu(fc, wl, gz=None):
    L, order = wl["lmax"], wl["order"]
    A1, pw, mw = dev(wl["A1"]), dev(wl["path_w"]), dev(wl["mix_w"])
    states, z = fc.product_ladder(L, order, A1, pw, mw)
    out = [states.cpu().numpy(), z.cpu().numpy()]
    if gz is not None:
        a1b, pwb, mwb = fc.product_ladder_vjp(L, order, A1, pw, mw, states, dev(gz))
        out += [a1b.cpu().numpy(), pwb.cpu().numpy(), mwb.cpu().numpy()]
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("L,C,order,N", [(1, 8, 5, 30), (2, 8, 4, 24), (3, 8, 4, 20), (3, 12, 3, 17),
                                         (4, 4, 3, 9), (3, 40, 5, 10), (3, 64, 4, 45), (2, 96, 3, 20)])
def test_small_ladder_full(fc, L, C, order, N):
    wl = dict(lmax=L, channels=C, order=order,
              **W.ladder_inputs(N, L, C, order, 1000 + 10 * L + C))
    states, z, a1b, pwb, mwb = run_gpu(fc, wl, wl["gz"])
    rs, rz = O.ladder(L, C, order, wl["A1"], wl["path_w"], wl["mix_w"])
    assert rel_err(z, rz) <= FWD_TOL
    for v in range(order - 1):
        assert rel_err(states[v], rs[v]) <= FWD_TOL
    ra, rp, rm = O.ladder_vjp(L, C, order, wl["A1"], wl["path_w"], wl["mix_w"], wl["gz"])
    assert rel_err(a1b, ra) <= VJP_TOL
    for v in range(order - 1):
        assert rel_err(pwb[v], rp[v]) <= VJP_TOL
        assert rel_err(mwb[v], rm[v]) <= VJP_TOL


@pytest.mark.parametrize("L,order,N", [(1, 4, 90), (2, 3, 50), (3, 4, 37), (4, 3, 21), (3, 3, 1200)])
def test_tensor_core_mix_c128(fc, L, order, N):
    """C = 128 takes the tcgen05 mix (three-term TF32 split): ragged last
    tiles of every rank; N = 1200 at rank 3 gives 152 tiles, so some CTAs
    walk two tiles and cross a rank boundary."""
    C = 128
    wl = dict(lmax=L, channels=C, order=order, **W.ladder_inputs(N, L, C, order, 2000 + L + N))
    states, z, a1b, pwb, mwb = run_gpu(fc, wl, wl["gz"])
    assert fc.device_error() == 0
    rs, rz = O.ladder(L, C, order, wl["A1"], wl["path_w"], wl["mix_w"])
    assert rel_err(z, rz) <= FWD_TOL
    for v in range(order - 1):
        assert rel_err(states[v], rs[v]) <= FWD_TOL
    ra, rp, rm = O.ladder_vjp(L, C, order, wl["A1"], wl["path_w"], wl["mix_w"], wl["gz"])
    assert rel_err(a1b, ra) <= VJP_TOL
    for v in range(order - 1):
        assert rel_err(pwb[v], rp[v]) <= VJP_TOL
        assert rel_err(mwb[v], rm[v]) <= VJP_TOL


@pytest.mark.parametrize("L,order,N", [(1, 3, 70), (2, 2, 33), (3, 4, 37), (3, 2, 300), (4, 3, 21)])
def test_tensor_core_forward_c256(fc, L, order, N):
    """C = 256: the forward's tcgen05 maps take K = 256 inputs per row and
    split each rank's 256 x 256 matrix into two maps of 128 output channels
    (ragged last tiles; N = 300 gives three tiles per component); the VJP
    runs the FP32 kernels at this width."""
    C = 256
    wl = dict(lmax=L, channels=C, order=order, **W.ladder_inputs(N, L, C, order, 2500 + L + N))
    states, z, a1b, pwb, mwb = run_gpu(fc, wl, wl["gz"])
    assert fc.device_error() == 0
    rs, rz = O.ladder(L, C, order, wl["A1"], wl["path_w"], wl["mix_w"])
    assert rel_err(z, rz) <= FWD_TOL
    for v in range(order - 1):
        assert rel_err(states[v], rs[v]) <= FWD_TOL
    ra, rp, rm = O.ladder_vjp(L, C, order, wl["A1"], wl["path_w"], wl["mix_w"], wl["gz"])
    assert rel_err(a1b, ra) <= VJP_TOL
    for v in range(order - 1):
        assert rel_err(pwb[v], rp[v]) <= VJP_TOL
        assert rel_err(mwb[v], rm[v]) <= VJP_TOL


def test_caller_workspace_too_small_is_refused(fc):
    """A caller-provided scratch buffer is passed with its real size; one
    byte short of the query is refused on the host (FC_ERR_WORKSPACE)."""
    L, C, order, N = 3, 128, 3, 40
    wl = W.ladder_inputs(N, L, C, order, 77)
    A1, pw, mw = dev(wl["A1"]), dev(wl["path_w"]), dev(wl["mix_w"])
    need = fc.ladder_workspace_bytes(L, C, order, N)
    short = torch.empty(need // 4 - 1, device="cuda")
    with pytest.raises(fc.FlashCartError) as e:
        fc.product_ladder(L, order, A1, pw, mw, workspace=short)
    assert e.value.status == 7
    states, z = fc.product_ladder(L, order, A1, pw, mw, workspace=torch.empty(need // 4, device="cuda"))
    need_v = fc.ladder_workspace_bytes(L, C, order, N, vjp=True)
    with pytest.raises(fc.FlashCartError) as e:
        fc.product_ladder_vjp(L, order, A1, pw, mw, states, dev(wl["gz"]),
                              workspace=torch.empty(need_v // 4 - 1, device="cuda"))
    assert e.value.status == 7
    torch.cuda.synchronize()


def test_order_one_is_copy(fc):
    wl = dict(lmax=3, channels=8, order=1, **W.ladder_inputs(6, 3, 8, 1, 5))
    wl["path_w"] = np.zeros((1, 23, 8), np.float32)
    wl["mix_w"] = np.zeros((1, 4, 8, 8), np.float32)
    states, z, a1b, pwb, mwb = run_gpu(fc, wl, wl["gz"])
    np.testing.assert_array_equal(z, wl["A1"])
    np.testing.assert_array_equal(a1b, wl["gz"])


@pytest.fixture(scope="module")
def lad():
    return W.ladder()


def test_ladder_4096_sampled_nodes(fc, lad):
    """Full-size launch (4096 nodes x 128 channels, rank 3, order 4).  The
    forward is node-local, so sampled nodes are exact; for the VJP the
    upstream gradient is kept only on the sampled nodes, which makes every
    entry of A1_bar, path_w_bar and mix_w_bar comparable with the oracle run
    over those nodes."""
    L, C, order = lad["lmax"], lad["channels"], lad["order"]
    nodes = np.array([0, 1, 2047, 4095])
    mask = np.zeros(lad["n_nodes"], np.uint8)
    mask[nodes] = 1
    gz = lad["gz"] * mask[:, None]
    states, z, a1b, pwb, mwb = run_gpu(fc, lad, gz)
    rs, rz = O.ladder(L, C, order, lad["A1"], lad["path_w"], lad["mix_w"], node_mask=mask)
    assert rel_err(z[nodes], rz[nodes]) <= FWD_TOL
    for v in range(order - 1):
        assert rel_err(states[v][nodes], rs[v][nodes]) <= FWD_TOL
    ra, rp, rm = O.ladder_vjp(L, C, order, lad["A1"], lad["path_w"], lad["mix_w"], gz,
                              node_mask=mask)
    assert rel_err(a1b, ra) <= VJP_TOL
    assert rel_err(pwb, rp) <= VJP_TOL
    assert rel_err(mwb, rm) <= VJP_TOL
    assert np.isfinite(z).all()
    assert fc.device_error() == 0
