"""GPU parity: draft map, ranking, quotas, precision map and per-row lists
against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import SMALL, check_compact_lists, gpu_run, inputs
from video_dit_sparse_da2_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def _check_plan(got, A, plan):
    assert np.array_equal(got["A"].view(np.uint64), A.view(np.uint64)), "draft map differs"
    assert np.array_equal(got["prec"], plan.prec)
    assert np.array_equal(got["cnt"], plan.cnt)
    check_compact_lists(got, plan.cnt, plan.kidx)
    B, H, R, _ = A.shape
    for b in range(B):
        for h in range(H):
            for a in range(R):
                n = plan.cnt[0, b, h, a] + plan.cnt[1, b, h, a]
                assert np.array_equal(got["kidx"][b, h, a, :n], plan.kidx[b, h, a, :n])


BUDGETS = [(2500, 2500), (0, 0), (10000, 0), (0, 10000), (1000, 3000), (1, 9998), (3333, 3333)]


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("bp", BUDGETS)
def test_plan_bit_exact_small(name, bp):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, *bp)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    prep = O.prepare(q, k, v, F, Hv, Wv)
    A = O.draft(prep.desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, *bp))


@pytest.mark.parametrize("lam", [0.0, 1.0])
def test_plan_lambda_extremes(lam):
    B, H, d, F, Hv, Wv = SMALL["ragged64"]
    res = gpu_run(B, H, d, F, Hv, Wv, 1500, 3500, lam=lam)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, lam)
    _check_plan(res["plan"], A, O.assign(A, 1500, 3500))


def test_plan_ties_by_pair_index():
    # identical regions: every draft score ties, the pair index decides
    F, Hv, Wv = 4, 16, 16
    q, k, v = make_qkv(1, 2, F * Hv * Wv, 64, 9)
    st, na = O.slot_tokens(F, Hv, Wv)
    for t in (q, k):
        base = t[:, :, st[:64]].clone()
        for a in range(len(na)):
            t[:, :, st[a * 64:(a + 1) * 64]] = base
    res = gpu_run(1, 2, 64, F, Hv, Wv, 2500, 2500, qkv=(q, k, v))
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, 2500, 2500))


def test_plan_bit_exact_wan13b():
    B, H, d, F, Hv, Wv = 1, 12, 128, 21, 30, 52
    res = gpu_run(B, H, d, F, Hv, Wv, 1000, 3000)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, 1000, 3000))


@pytest.mark.parametrize("d", [64, 128])
def test_plan_max_branch_exact_path_and_fp64_fallback(d):
    # The max-pool branch's logits of blocks whose channel maxima span at most
    # a few binades come from exact integer tensor-core products, the others
    # from the fp64 chain; both must give the defining fp64 values.  Frames 0-1
    # (Q) and 5 (K) get one channel scaled by 2^-10, which widens those blocks'
    # range past the exact one; frame 7 gets an all-negative Q channel (a
    # negative maximum); R = 300 spans three 128-block tiles, mixing tiles with
    # and without such blocks.
    B, H, F, Hv, Wv = 1, 2, 12, 30, 52
    q, k, v = make_qkv(B, H, F * Hv * Wv, d, seed=4)
    fr = Hv * Wv
    q[:, :, 0:2 * fr, 0] *= 2.0 ** -10
    k[:, :, 5 * fr:6 * fr, 3] *= 2.0 ** -10
    q[:, :, 7 * fr:8 * fr, 2] = -(q[:, :, 7 * fr:8 * fr, 2].abs() + 1.0)
    res = gpu_run(B, H, d, F, Hv, Wv, 1000, 3000, qkv=(q, k, v))
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    _check_plan(res["plan"], A, O.assign(A, 1000, 3000))
