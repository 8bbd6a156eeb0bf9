"""The allocation-free ladder entry point (fc_product_ladder_noalloc) against
the workspace entry point (fc_product_ladder), through the C ABI.

It serves callers that cannot allocate device memory (inside another
framework's memory pool, or in latency-critical loops where cudaMalloc may
synchronise the device): its scratch is a fixed 16 MiB array inside the
library.  Two calls in a row must each match the workspace entry within the
forward tolerance, the second one reusing the array the first one left
behind; a size beyond the array is refused before anything runs."""
import ctypes as ct

import numpy as np
import pytest
import torch

from cartesian_tensor_products_b200 import workloads as W
from parity import FWD_TOL, rel_err

pytestmark = pytest.mark.gpu


def test_noalloc_ladder_matches_workspace_entry_twice():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart as fc
    lib = fc.lib()
    f = lib.fc_product_ladder_noalloc
    f.restype = ct.c_int
    f.argtypes = [ct.POINTER(fc.LadderDesc), ct.c_int] + [ct.c_void_p] * 6

    L, C, order, N = 3, 128, 4, 512          # 4.5 MiB of scratch (tensor-core path)
    wl = W.ladder_inputs(N, L, C, order, 2024)
    dev = torch.device("cuda:0")
    A1 = torch.from_numpy(wl["A1"]).to(dev)
    pw = torch.from_numpy(wl["path_w"]).to(dev)
    mw = torch.from_numpy(wl["mix_w"]).to(dev)
    ref_states, ref_z = fc.product_ladder(L, order, A1, pw, mw)
    torch.cuda.synchronize()
    ref_states, ref_z = ref_states.cpu().numpy(), ref_z.cpu().numpy()

    d = fc.LadderDesc(L, C, order)
    stream = ct.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        states = torch.full((order - 1, N, 16 * C), float("nan"), device=dev)
        z = torch.full((N, 16 * C), float("nan"), device=dev)
        st = f(ct.byref(d), N, ct.c_void_p(A1.data_ptr()), ct.c_void_p(pw.data_ptr()),
               ct.c_void_p(mw.data_ptr()), ct.c_void_p(states.data_ptr()),
               ct.c_void_p(z.data_ptr()), stream)
        assert st == 0, lib.fc_status_string(st)
        torch.cuda.synchronize()
        assert rel_err(z.cpu().numpy(), ref_z) <= FWD_TOL
        for v in range(order - 1):
            assert rel_err(states[v].cpu().numpy(), ref_states[v]) <= FWD_TOL

    # beyond the 16 MiB array: refused on the host (FC_ERR_WORKSPACE)
    big = 4096                               # 32.5 MiB of scratch
    st = f(ct.byref(d), big, ct.c_void_p(A1.data_ptr()), ct.c_void_p(pw.data_ptr()),
           ct.c_void_p(mw.data_ptr()), ct.c_void_p(states.data_ptr()),
           ct.c_void_p(z.data_ptr()), stream)
    assert st == 7
