"""The C-ABI library loads, exports every symbol include/da2.h declares, and
rejects bad arguments before touching a device (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import oracle as O
from video_dit_sparse_da2_b200 import da2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "da2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(da2_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 10
    L = da2.lib()
    for n in names:
        assert hasattr(L, n), n
    assert sorted(da2.EXPORTS) == names


def test_status_strings():
    L = da2.lib()
    for code in (0, -1, -2, -3, -4):
        assert L.da2_status_string(code)
    assert L.da2_status_string(-4).decode().startswith("a bounded")


def test_create_rejects_bad_shapes_without_device():
    L = da2.lib()
    h = ctypes.c_void_p()
    assert L.da2_create(None, ctypes.byref(h)) == da2.ERR_ARG
    for bad in [(1, 1, 96, 1, 8, 8, 64), (1, 1, 64, 1, 8, 8, 32), (0, 1, 64, 1, 8, 8, 64), (1, 1, 64, 1, 0, 8, 64)]:
        s = da2.Shape(*bad)
        assert L.da2_create(ctypes.byref(s), ctypes.byref(h)) == da2.ERR_ARG
    assert L.da2_destroy(None) == da2.OK
    assert L.da2_prepare(None, None, None, None, None, None, None) == da2.ERR_ARG
    assert L.da2_plan(None, None, None, None, None) == da2.ERR_ARG
    assert L.da2_attention(None, None, None, None, None, None) == da2.ERR_ARG


@pytest.mark.parametrize("geom", [(4, 16, 16), (21, 30, 52), (13, 60, 90), (33, 45, 80), (21, 45, 80), (3, 9, 13),
                                  (2, 1, 1), (1, 7, 100), (5, 31, 7)])
def test_library_partition_matches_oracle(geom):
    # The library's host partition and the oracle's are independent
    # implementations of the same reading of App. C.2; they must agree exactly.
    st, na = da2.partition(*geom)
    ost, ona = O.slot_tokens(*geom)
    assert np.array_equal(st, ost) and np.array_equal(na, ona)


def test_partition_rejects_bad_sizes():
    assert da2.lib().da2_partition(0, 4, 4, None, None) == da2.ERR_ARG
    assert da2.lib().da2_partition(1, 0, 4, None, None) == da2.ERR_ARG


def test_budget_struct_layout_matches_header():
    # da2_budget in include/da2.h: int bp_fp8, int bp_fp4, double lambda, int per_row
    import ctypes

    from video_dit_sparse_da2_b200 import da2
    B = da2.Budget
    assert [B.bp_fp8.offset, B.bp_fp4.offset, B.lam.offset, B.per_row.offset] == [0, 4, 8, 16]
    assert ctypes.sizeof(B) == 24
