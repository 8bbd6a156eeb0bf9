"""The give-up path of the tensor-core kernels' bounded barrier waits.

The ladder's tcgen05 kernels (the per-rank mix of the forward, the mix and
the weight gradient of the VJP) wait on mbarriers.  Every wait is bounded:
when it runs out, the CTA lets the copies and MMAs it already started
finish, skips the rest of its work, sets the library's sticky error word and
exits instead of hanging.  Here the bound is set to 1 ns, so the waits run
out without any fault being provoked: the calls must return, the error
word must read 1, and after the default bound is restored the same calls
must again match the FP64 oracle (FlashCart Sec. 5 Eq. 2) with the word at 0.
"""
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


def test_waits_give_up_then_recover(fc):
    L, C, order, N = 3, 128, 3, 600
    lad = W.ladder_inputs(N, L, C, order, 23)
    A1, pw, mw, gz = (torch.from_numpy(lad[k]).cuda() for k in ("A1", "path_w", "mix_w", "gz"))
    assert fc.device_error() == 0
    fc.set_wait_timeout(1)
    try:
        states, _ = fc.product_ladder(L, order, A1, pw, mw)
        fc.product_ladder_vjp(L, order, A1, pw, mw, states, gz)
        torch.cuda.synchronize()
        flag = fc.device_error()
    finally:
        fc.set_wait_timeout(0)
    assert flag == 1
    assert fc.device_error() == 0          # the word was cleared by the read

    states, z = fc.product_ladder(L, order, A1, pw, mw)
    a1b, pwb, mwb = fc.product_ladder_vjp(L, order, A1, pw, mw, states, gz)
    torch.cuda.synchronize()
    assert fc.device_error() == 0
    _, rz = O.ladder(L, C, order, lad["A1"], lad["path_w"], lad["mix_w"])
    ra, rp, rm = O.ladder_vjp(L, C, order, lad["A1"], lad["path_w"], lad["mix_w"], lad["gz"])
    assert rel_err(z.cpu().numpy(), rz) <= FWD_TOL
    for got, ref in ((a1b, ra), (pwb, rp), (mwb, rm)):
        assert rel_err(got.cpu().numpy().reshape(ref.shape), ref) <= VJP_TOL
