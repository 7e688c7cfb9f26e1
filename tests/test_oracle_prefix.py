"""Pins of the oracle's prefix (text) tokens (DraftAttention2 App. C.1: the
budget covers video-region pairs only; every video query block also sees every
valid prefix key and every prefix query sees all keys).  Readings: the P
prefix tokens come first in the sequence and are packed into ceil(P/64) blocks
after the video blocks; prefix interactions run on the 16-bit path.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from video_dit_sparse_da2_b200.inputs import make_qkv

F, HV, WV = 3, 9, 13   # 3 frames of 9 x 13: ragged video blocks


def _qkv(P, seed=0, H=2, d=64):
    return make_qkv(1, H, P + F * HV * WV, d, seed)


def _dense_mask(q, k, v, mask):
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    s = np.einsum("bhud,bhtd->bhut", qn, kn) / math.sqrt(qn.shape[-1])
    s = np.where(mask, s, -np.inf)
    m = s.max(-1, keepdims=True)
    p = np.exp(s - np.where(np.isfinite(m), m, 0.0))
    l = p.sum(-1, keepdims=True)
    return np.where(l > 0, np.einsum("bhut,bhtd->bhud", p, vn) / np.where(l > 0, l, 1), 0.0)


@pytest.mark.parametrize("P", [0, 1, 64, 100, 200])
def test_slot_tables_put_the_prefix_blocks_last(P):
    st, na = O.slot_tokens(F, HV, WV, P)
    st0, na0 = O.slot_tokens(F, HV, WV)
    Rv = len(na0)
    Rp = -(-P // 64)
    assert len(na) == Rv + Rp
    vs = st[:64 * Rv]
    assert np.array_equal(vs, np.where(st0 >= 0, st0 + P, -1))
    assert np.array_equal(na[:Rv], na0)
    for i in range(Rp):
        cnt = min(64, P - 64 * i)
        assert na[Rv + i] == cnt
        blk = st[64 * (Rv + i):64 * (Rv + i + 1)]
        assert np.array_equal(blk[:cnt], np.arange(64 * i, 64 * i + cnt)) and np.all(blk[cnt:] == -1)


def test_no_prefix_equals_the_plain_pipeline():
    q, k, v = _qkv(0, 1)
    _, _, _, ref = O.run(q, k, v, F, HV, WV, 2000, 3000, bp16=1000)
    _, _, _, got = O.run_prefix(q, k, v, F, HV, WV, 0, 2000, 3000, bp16=1000)
    assert np.array_equal(got, ref)


def _kept_mask(plan, P, h):
    """Dense [N, N] mask of the kept pairs of head h under the prefix rule."""
    st, na = O.slot_tokens(F, HV, WV, P)
    Rt = len(na)
    N = P + F * HV * WV
    mask = np.zeros((N, N), bool)
    for a in range(Rt):
        qa = st[64 * a:64 * a + na[a]]
        n = plan.cnt[0, 0, h, a] + plan.cnt[1, 0, h, a] + plan.cnt[2, 0, h, a]
        for b in plan.kidx[0, h, a, :n]:
            mask[np.ix_(qa, st[64 * b:64 * b + na[b]])] = True
    return mask


@pytest.mark.parametrize("P,bp", [(100, (1000, 2000, 1000)), (64, (0, 3000, 2000)), (200, (2500, 0, 2500)),
                                  (37, (0, 0, 0))])
def test_prefix_rule_unquantized_is_dense_on_its_mask(P, bp):
    # without quantization (flags 0 and 4, the units exact inverses) every row
    # is softmax attention over its kept keys; prefix rows keep every key and
    # video rows keep every prefix key besides their budgeted video blocks
    bp16, bp8, bp4 = bp
    q, k, v = _qkv(P, 1)
    st, na = O.slot_tokens(F, HV, WV, P)
    for flags in (0, 4):
        prep, A, plan, out = O.run_prefix(q, k, v, F, HV, WV, P, bp8, bp4, flags=flags, bp16=bp16)
        for h in range(2):
            mask = _kept_mask(plan, P, h)
            assert mask[:P].all()                # prefix queries: non-sparse
            assert mask[:, :P].all()             # every query keeps the prefix keys
            ref = _dense_mask(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], mask[None, None])
            np.testing.assert_allclose(out[0, h], ref[0, 0], rtol=0, atol=1e-12)


def test_prefix_plan_lists():
    P = 150
    q, k, v = _qkv(P, 2)
    prep, A, plan, out = O.run_prefix(q, k, v, F, HV, WV, P, 1500, 2500, bp16=1000)
    Rv = A.shape[-1]
    Rp = 3
    video = O.tiers_plan(A, 1500, 2500, bp16=1000)
    for h in range(2):
        for a in range(Rv + Rp):
            n8, n4, n16 = (int(plan.cnt[t, 0, h, a]) for t in range(3))
            lst = list(plan.kidx[0, h, a, :n8 + n4 + n16])
            if a < Rv:
                v8, v4, v16 = (int(video.cnt[t, 0, h, a]) for t in range(3))
                vl = list(video.kidx[0, h, a, :v8 + v4 + v16])
                assert (n8, n4, n16) == (v8, v4, v16 + Rp)
                assert lst == vl[:v16] + list(range(Rv, Rv + Rp)) + vl[v16:]
            else:
                assert (n8, n4, n16) == (0, 0, Rv + Rp) and lst == list(range(Rv + Rp))


def test_prefix_rows_closed_form_uniform_scores():
    # K = 0: all scores of a row tie (p = 1); a prefix row's weights are then
    # bf16(1) = 1 on every key, so its output is the exact mean of V over all
    # tokens, whatever the budgets of the video pairs
    P = 90
    q, k, v = _qkv(P, 3)
    k = torch.zeros_like(k)
    _, _, _, out = O.run_prefix(q, k, v, F, HV, WV, P, 2000, 3000, flags=7, bp16=1000)
    mean = v.double().numpy().mean(axis=2)
    for h in range(2):
        np.testing.assert_allclose(out[0, h, :P], np.broadcast_to(mean[0, h], (P, mean.shape[-1])), rtol=0,
                                   atol=1e-12)
