"""GPU parity of fc_full_ladder (FlashCart Sec. 5 Eq. 2: path-separated
products with per-rank path+channel maps) against the FP64 oracle, through
the C ABI.  Tolerance: max relative error 1e-5."""
import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from oracle import oracle as O
from parity import FWD_TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# C = 128 runs the tensor-core maps: node counts whose rank blocks span
# several 128-row tiles and end in a ragged tile, order 1 (phi_1 alone)
@pytest.mark.parametrize("L,C,order,N", [(1, 8, 4, 33), (2, 8, 3, 20), (3, 12, 4, 13),
                                         (3, 128, 3, 9), (4, 4, 3, 7), (3, 40, 1, 11),
                                         (1, 128, 4, 70), (2, 128, 3, 100), (3, 128, 2, 150),
                                         (4, 128, 3, 40), (3, 128, 1, 50)])
def test_full_ladder_small(fc, L, C, order, N):
    d = W.full_ladder_inputs(N, L, C, order, 300 + 10 * L + C)
    st, z = fc.full_ladder(L, order, dev(d["A"]), dev(d["W1"]), dev(d["Wq"]))
    torch.cuda.synchronize()
    rs, rz = O.full_ladder(L, C, order, d["A"], d["W1"], d["Wq"])
    assert rel_err(z.cpu().numpy(), rz) <= FWD_TOL
    for q in range(order):
        assert rel_err(st[q].cpu().numpy(), rs[q]) <= FWD_TOL


def test_full_ladder_4096_sampled_nodes(fc):
    """The benchmark shape (4096 nodes x 128 channels, rank 3, order 4); the
    ladder is node-local, so sampled nodes are exact."""
    L, C, order, N = 3, 128, 4, 4096
    d = W.full_ladder_inputs(N, L, C, order, 44)
    st, z = fc.full_ladder(L, order, dev(d["A"]), dev(d["W1"]), dev(d["Wq"]))
    torch.cuda.synchronize()
    nodes = np.array([0, 1, 2047, 4095])
    m = np.zeros(N, np.uint8)
    m[nodes] = 1
    rs, rz = O.full_ladder(L, C, order, d["A"], d["W1"], d["Wq"], node_mask=m)
    assert rel_err(z.cpu().numpy()[nodes], rz[nodes]) <= FWD_TOL
    for q in range(order):
        assert rel_err(st[q].cpu().numpy()[nodes], rs[q][nodes]) <= FWD_TOL
    assert np.isfinite(z.cpu().numpy()).all()


@pytest.mark.parametrize("L,C,order,N", [(3, 128, 3, 40), (3, 128, 1, 40), (2, 8, 3, 20)])
def test_workspace_refusal_and_error_word(fc, L, C, order, N):
    """One float short of the queried workspace is refused on the host
    (FC_ERR_WORKSPACE = 7), on the tensor-core path (C = 128, which needs
    scratch at order 1 too) and on the SIMT path; a run with the exact size
    matches the oracle and leaves the bounded-wait error word clear."""
    import ctypes as ct
    d = W.full_ladder_inputs(N, L, C, order, 90 + C + order)
    A, W1, Wq = dev(d["A"]), dev(d["W1"]), dev(d["Wq"])
    need = fc.lib().fc_full_ladder_workspace_size(ct.byref(fc.LadderDesc(L, C, order)), N)
    assert need > 0 and need % 4 == 0
    with pytest.raises(fc.FlashCartError) as e:
        fc.full_ladder(L, order, A, W1, Wq, workspace=torch.empty(need // 4 - 1, device="cuda"))
    assert e.value.status == 7
    st, z = fc.full_ladder(L, order, A, W1, Wq, workspace=torch.empty(need // 4, device="cuda"))
    torch.cuda.synchronize()
    assert fc.device_error() == 0
    _, rz = O.full_ladder(L, C, order, d["A"], d["W1"], d["Wq"])
    assert rel_err(z.cpu().numpy(), rz) <= FWD_TOL


def test_no_nodes(fc):
    """Zero nodes: FC_OK, nothing launched, empty outputs."""
    d = W.full_ladder_inputs(3, 3, 128, 3, 5)
    A = dev(d["A"])[:0]
    st, z = fc.full_ladder(3, 3, A, dev(d["W1"]), dev(d["Wq"]))
    torch.cuda.synchronize()
    assert st.shape == (3, 0, 16 * 128) and z.shape == (0, 16 * 128)
    assert fc.device_error() == 0


# ---------------------------------------------------------------------------
# VJP of the full ladder (reverse accumulation, App. C Eq. C1 per product)
# ---------------------------------------------------------------------------

def check_vjp(got, ref):
    from parity import VJP_TOL
    for name, a, b in zip(("A_bar", "W1_bar", "Wq_bar"), got, ref):
        if b.size == 0:
            continue
        e = rel_err(a.cpu().numpy().reshape(b.shape), b)
        assert e <= VJP_TOL, "%s rel err %g" % (name, e)


@pytest.mark.parametrize("L,C,order,N", [(1, 8, 4, 33), (2, 8, 3, 20), (3, 12, 4, 13),
                                         (4, 4, 3, 7), (3, 40, 1, 11), (3, 128, 3, 70),
                                         (2, 128, 4, 100), (4, 128, 2, 30), (1, 200, 3, 17)])
def test_full_ladder_vjp_small(fc, L, C, order, N):
    d = W.full_ladder_inputs(N, L, C, order, 400 + 10 * L + C)
    A, W1, Wq, gz = dev(d["A"]), dev(d["W1"]), dev(d["Wq"]), dev(d["gz"])
    st, _ = fc.full_ladder(L, order, A, W1, Wq)
    got = fc.full_ladder_vjp(L, order, A, W1, Wq, st, gz)
    torch.cuda.synchronize()
    ref = O.full_ladder_vjp(L, C, order, d["A"], d["W1"], d["Wq"], d["gz"])
    check_vjp(got, ref)


def test_full_ladder_vjp_4096_masked_gradient(fc):
    """The benchmark shape (4096 nodes x 128 channels, rank 3, order 4) at
    full size.  The upstream gradient is kept on sampled nodes only, so
    A_bar (zero elsewhere) and every entry of W1_bar and Wq_bar can be
    compared with the oracle run over those nodes."""
    L, C, order, N = 3, 128, 4, 4096
    d = W.full_ladder_inputs(N, L, C, order, 44)
    nodes = np.array([0, 1, 2047, 4095])
    m = np.zeros(N, np.uint8)
    m[nodes] = 1
    gz = d["gz"] * m[:, None]
    A, W1, Wq = dev(d["A"]), dev(d["W1"]), dev(d["Wq"])
    st, _ = fc.full_ladder(L, order, A, W1, Wq)
    got = fc.full_ladder_vjp(L, order, A, W1, Wq, st, dev(gz))
    torch.cuda.synchronize()
    ref = O.full_ladder_vjp(L, C, order, d["A"], d["W1"], d["Wq"], gz, node_mask=m)
    check_vjp(got, ref)
    assert np.isfinite(got[0].cpu().numpy()).all()


def test_full_ladder_vjp_workspace_refusal_and_no_nodes(fc):
    import ctypes as ct
    L, C, order, N = 2, 8, 3, 9
    d = W.full_ladder_inputs(N, L, C, order, 77)
    A, W1, Wq, gz = dev(d["A"]), dev(d["W1"]), dev(d["Wq"]), dev(d["gz"])
    st, _ = fc.full_ladder(L, order, A, W1, Wq)
    need = fc.lib().fc_full_ladder_vjp_workspace_size(ct.byref(fc.LadderDesc(L, C, order)), N)
    with pytest.raises(fc.FlashCartError) as e:
        fc.full_ladder_vjp(L, order, A, W1, Wq, st, gz,
                           workspace=torch.empty(need // 4 - 1, device="cuda"))
    assert e.value.status == 7
    # zero nodes: the weight gradients are zero
    Ab, W1b, Wqb = fc.full_ladder_vjp(L, order, A[:0], W1, Wq, st[:, :0].contiguous(), gz[:0])
    torch.cuda.synchronize()
    assert Ab.numel() == 0 and torch.all(W1b == 0) and torch.all(Wqb == 0)
