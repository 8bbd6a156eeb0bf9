"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/*.h declares, and its descriptor queries agree
with the path rules of FlashCart Sec. 2 as the oracle lists them."""
import ctypes as ct
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fc():
    from cartesian_tensor_products_b200 import build
    build.build()
    from cartesian_tensor_products_b200 import flashcart
    return flashcart


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(fc_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("fc_edge_conv", "fc_build_rowptr", "fc_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(fc):
    lib = ct.CDLL(fc.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(fc):
    lib = fc.lib()
    for s in range(0, 8):
        assert lib.fc_status_string(s)
    assert b"unknown" in lib.fc_status_string(99)
    assert lib.fc_version() >= 100


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5])
def test_descriptor_queries_match_oracle_paths(fc, L):
    from oracle import oracle as O
    assert fc.paths(L) == O.paths(L, L, L)
    assert fc.num_paths(L) == len(O.paths(L, L, L))
    assert fc.out_row(L) == O.zrow(L, L, L)
    assert fc.out_row(L, sum_paths=True) == (L + 1) ** 2


def test_descriptor_rejections(fc):
    lib = fc.lib()
    bad = [fc.ConvDesc(0, 0, 0, 8, 0),      # unsupported rank (1..4 are built)
           fc.ConvDesc(6, 6, 6, 8, 0),      # unsupported rank
           fc.ConvDesc(3, 2, 3, 8, 0),      # mixed ranks
           fc.ConvDesc(3, 3, 3, 6, 0),      # channels not multiple of 4
           fc.ConvDesc(3, 3, 3, 0, 0),      # no channels
           fc.ConvDesc(3, 3, 3, 8, 2)]      # bad flag
    for d in bad:
        assert lib.fc_conv_num_paths(ct.byref(d)) == -1
    # the compute entry rejects them before touching the GPU
    d = fc.ConvDesc(3, 3, 3, 6, 0)
    st = lib.fc_edge_conv(ct.byref(d), 4, 0, None, None, None, None, None, None, None)
    assert st == 5
    d = fc.ConvDesc(6, 6, 6, 8, 0)
    st = lib.fc_edge_conv(ct.byref(d), 4, 0, None, None, None, None, None, None, None)
    assert st == 4
    d = fc.ConvDesc(3, 3, 3, 8, 0)
    st = lib.fc_edge_conv(ct.byref(d), 4, 0, None, None, None, None, None, None, None)
    assert st == 1
    # misaligned pointers are caught on the host
    st = lib.fc_edge_conv(ct.byref(d), 1, 0, ct.c_void_p(16), None, None,
                          ct.c_void_p(20), None, ct.c_void_p(32), None)
    assert st == 5


@pytest.mark.parametrize("L", [1, 2, 3, 4])
def test_odd_path_queries_match_oracle(fc, L):
    """Odd-J (Levi-Civita) path list and output row of the library against
    the oracle's odd path rule (App. B, paragraph after Eq. B1)."""
    from oracle import oracle as O
    assert fc.odd_paths(L) == O.paths(L, L, L, odd=True)
    assert fc.odd_out_row(L) == O.zrow(L, L, L, odd=True)
    assert fc.odd_out_row(L, sum_paths=True) == (L + 1) ** 2
