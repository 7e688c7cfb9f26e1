"""da2_plan_static: routing for callers that cannot allocate device memory
(for example code that records a CUDA graph by stream capture, where
cudaMalloc is not allowed, or hosts that own all device memory and forbid
plugins to allocate).  Its working memory is a fixed array inside the
library.  It must give exactly what da2_plan gives with a caller-provided
scratch buffer -- the routing outputs are compared bit for bit, as every
routing test here does -- on two calls in a row (the second call finds the
first call's leftovers in the array), and it must refuse shapes whose working
memory exceeds the array.  Both ranking modes are covered: per head, and
per query block (which runs a different routing kernel on the same array).

This file sorts last so that a run stopping at the first failure has run
every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from video_dit_sparse_da2_b200 import da2, layouts
from video_dit_sparse_da2_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, d, F, Hv, Wv, bp8, bp4, lam): the second needs ~27 MB of working memory
    (1, 2, 64, 4, 16, 16, 2500, 2500, 0.2),
    (1, 12, 128, 21, 30, 52, 1000, 3000, 0.2),
]


def _plan_bytes(plan, B, H, R, list_bytes):
    g = layouts.plan_to_logical(plan.bufs, B, H, R)
    g["kidx_flat"] = g["kidx_flat"][: list_bytes // 2]
    return {k: np.ascontiguousarray(v).view(np.uint8).copy() for k, v in g.items()}


@pytest.mark.parametrize("per_row", [False, True], ids=["per-head", "per-row"])
@pytest.mark.parametrize("case", CASES, ids=["tiny", "wan2.1-1.3b-480p"])
def test_plan_static_matches_plan_twice(case, per_row):
    B, H, d, F, Hv, Wv, bp8, bp4, lam = case
    m = da2.DA2(B, H, d, F, Hv, Wv)
    assert m.sizes.plan_scratch <= (32 << 20)
    q, k, v = (t.cuda() for t in make_qkv(B, H, F * Hv * Wv, d, seed=11))
    prep = m.alloc_prepared()
    m.prepare(q, k, v, prep)
    nlist = m.list_bytes(bp8, bp4, per_row)
    ref = m.alloc_plan(budget=(bp8, bp4, per_row))
    m.plan(prep, ref, bp8, bp4, lam, per_row=per_row)
    torch.cuda.synchronize()
    want = _plan_bytes(ref, B, H, m.R, nlist)
    for call in range(2):
        got_plan = m.alloc_plan(budget=(bp8, bp4, per_row))
        for t in got_plan.bufs.values():
            t.fill_(0xA5)  # outputs start as garbage: everything must be written
        m.plan_static(prep, got_plan, bp8, bp4, lam, per_row=per_row)
        torch.cuda.synchronize()
        m.check_status()
        got = _plan_bytes(got_plan, B, H, m.R, nlist)
        R = m.R
        cnt = want["cnt"].view(np.int32).reshape(2, B, H, R)
        n = (cnt[0] + cnt[1])[..., None]
        listed = np.arange(R)[None, None, None, :] < n
        for key in ("A", "prec", "cnt", "off", "kidx_flat"):
            assert np.array_equal(got[key], want[key]), (call, key)
        gk = got["kidx"].view(np.uint16).reshape(B, H, R, R)
        wk = want["kidx"].view(np.uint16).reshape(B, H, R, R)
        assert np.array_equal(np.where(listed, gk, 0), np.where(listed, wk, 0)), (call, "kidx")
    m.close()


def test_plan_static_refuses_large_shapes():
    m = da2.DA2(1, 24, 128, 33, 45, 80)  # needs ~680 MB of working memory
    assert m.sizes.plan_scratch > (32 << 20)
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    p = small.data_ptr()
    ptrs = da2.PreparedPtrs(*([p] * 12))
    b = da2.Budget(1000, 1000, 0.2)
    rc = da2.lib().da2_plan_static(m.handle, ctypes.byref(ptrs), ctypes.byref(b), p, p, p, p, p, None)
    assert rc == da2.ERR_ARG
    torch.cuda.synchronize()
    assert not small.any()  # nothing was enqueued
    m.close()
