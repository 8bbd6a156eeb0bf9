"""Workspace-size queries of the ladder entry points (host logic, no GPU).

The sizes follow the scratch layouts the header states:

* tensor-core path (C = 128): the product as FP32 tiles of 128 nodes per
  rank and component, with K = 128 P_l inputs per row for the full ladder
  (Sec. 5 Eq. 2, every path kept) or K = 128 for the path-reduced ladder;
  plus one step's maps as TF32 hi and lo; the path-reduced ladder's forward
  also at C = 256 (K = 256, two 128-row maps per rank);
* ladder VJP: four product states, plus at C = 128 the gradient as split
  tiles and one step's split matrices;
* SIMT path: one product state (full ladder: the convolution's output row
  of sum_l (2l+1) P_l slots; ladder: (L+1)^2 slots), none at order 1 for
  the full ladder;
* unsupported descriptors: 0.
"""
import ctypes as ct

import pytest

from cartesian_tensor_products_b200 import workloads as W


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def blocks(N):
    return (N + 127) // 128


def query(fc, fn, L, C, order, N):
    return getattr(fc.lib(), fn)(ct.byref(fc.LadderDesc(L, C, order)), N)


@pytest.mark.parametrize("L", [1, 2, 3, 4])
@pytest.mark.parametrize("N", [1, 127, 128, 129, 4096])
def test_full_ladder_tensor_core(fc, L, N):
    Pl = W.paths_per_rank(L, L, L)
    product = sum((2 * l + 1) * blocks(N) * 128 * (128 * Pl[l]) for l in range(L + 1))
    maps = 2 * 128 * sum(Pl) * 128
    for order in (1, 2, 4):
        assert query(fc, "fc_full_ladder_workspace_size", L, 128, order, N) == 4 * (product + maps)


@pytest.mark.parametrize("L,C", [(1, 8), (3, 64), (4, 256)])
def test_full_ladder_simt(fc, L, C):
    Pl = W.paths_per_rank(L, L, L)
    row = sum((2 * l + 1) * p for l, p in enumerate(Pl))
    N = 37
    assert query(fc, "fc_full_ladder_workspace_size", L, C, 1, N) == 0
    assert query(fc, "fc_full_ladder_workspace_size", L, C, 3, N) == 4 * N * row * C


@pytest.mark.parametrize("L", [1, 2, 3, 4])
@pytest.mark.parametrize("N", [1, 128, 129, 4096])
def test_ladder_forward(fc, L, N):
    NY = (L + 1) ** 2
    product = NY * blocks(N) * 128 * 128
    maps = (L + 1) * 2 * 128 * 128
    assert query(fc, "fc_product_ladder_workspace_size", L, 128, 4, N) == 4 * (product + maps)
    assert query(fc, "fc_product_ladder_workspace_size", L, 64, 4, N) == 4 * N * NY * 64
    # C = 256: K = 256 inputs per row, each rank's matrix as two 128-row maps
    product = NY * blocks(N) * 128 * 256
    maps = (L + 1) * 2 * 256 * 256
    assert query(fc, "fc_product_ladder_workspace_size", L, 256, 4, N) == 4 * (product + maps)


@pytest.mark.parametrize("L", [1, 2, 3, 4])
@pytest.mark.parametrize("N", [1, 128, 129, 4096])
def test_ladder_vjp(fc, L, N):
    """Four product states; at C = 128 also the gradient as split tiles of
    128 rows per rank (rows n (2l+1) + c, hi and lo) and one step's split
    matrices.  The weight gradient reads the FP32 rows and needs nothing."""
    NY = (L + 1) ** 2
    tiles = sum((N * (2 * l + 1) + 127) // 128 for l in range(L + 1))
    states = 4 * N * NY * 128
    split = tiles * 2 * 128 * 128 + (L + 1) * 2 * 128 * 128
    assert query(fc, "fc_product_ladder_vjp_workspace_size", L, 128, 4, N) == 4 * (states + split)
    assert query(fc, "fc_product_ladder_vjp_workspace_size", L, 64, 4, N) == 4 * 4 * N * NY * 64
    # C = 256: the gradient as FP32 tiles of K = 256 and the transposed maps
    tiles256 = NY * ((N + 127) // 128) * 128 * 256
    assert query(fc, "fc_product_ladder_vjp_workspace_size", L, 256, 4, N) == \
        4 * (4 * N * NY * 256 + tiles256 + (L + 1) * 2 * 256 * 256)


def test_unsupported_descriptors_need_nothing(fc):
    assert query(fc, "fc_full_ladder_workspace_size", 5, 128, 3, 10) == 0    # rank 5
    assert query(fc, "fc_full_ladder_workspace_size", 3, 6, 3, 10) == 0      # C not a multiple of 4
    assert query(fc, "fc_full_ladder_workspace_size", 3, 128, 0, 10) == 0    # order 0
    assert query(fc, "fc_full_ladder_workspace_size", 3, 128, 3, -1) == 0    # negative count
    assert query(fc, "fc_product_ladder_workspace_size", 0, 128, 3, 10) == 0
