"""GPU parity of the per-query-row ranking option (budget.per_row = 1): the
precision map, counts and lists equal the oracle's per-row assignment bit for
bit, and the attention on such a plan matches the oracle."""
import numpy as np
import pytest

from oracle import oracle as O
from tests.gpu_common import SMALL, bf16_round, gpu_run, inputs, rel_l2
from tests.test_gpu_plan import _check_plan
from video_dit_sparse_da2_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

BUDGETS = [(2500, 2500), (0, 10000), (10000, 0), (1000, 3000), (700, 600), (0, 0)]


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("bp", BUDGETS)
def test_plan_rows_bit_exact_small(name, bp):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, *bp, per_row=True)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, *bp, per_row=True))


def test_plan_rows_ties_by_key_block():
    F, Hv, Wv = 4, 16, 16
    q, k, v = make_qkv(1, 2, F * Hv * Wv, 64, 9)
    st, na = O.slot_tokens(F, Hv, Wv)
    for t in (q, k):
        base = t[:, :, st[:64]].clone()
        for a in range(len(na)):
            t[:, :, st[a * 64:(a + 1) * 64]] = base
    res = gpu_run(1, 2, 64, F, Hv, Wv, 2500, 2500, qkv=(q, k, v), per_row=True)
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, 2500, 2500, per_row=True))


@pytest.mark.parametrize("shape,bp", [((1, 12, 128, 21, 30, 52), (1000, 3000)),
                                      ((1, 24, 128, 33, 45, 80), (500, 2500))],
                         ids=["wan2.1-1.3b-480p", "hunyuanvideo-720p"])
def test_plan_rows_bit_exact_full_size(shape, bp):
    B, H, d, F, Hv, Wv = shape
    res = gpu_run(B, H, d, F, Hv, Wv, *bp, per_row=True)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, *bp, per_row=True))


@pytest.mark.parametrize("name", ["tiny", "ragged128"])
def test_attention_on_row_plan(name):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, 2500, 2500, per_row=True)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    _, _, _, ref = O.run(q, k, v, F, Hv, Wv, 2500, 2500, 0.2, per_row=True)
    ref16 = bf16_round(ref)
    err = rel_l2(res["out"], ref16)
    mx = np.abs(res["out"] - ref16).max()
    assert err <= 2e-3 and mx <= 1e-2, (err, mx)
