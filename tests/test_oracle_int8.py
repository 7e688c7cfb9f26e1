"""Pins of the oracle's INT8 QK^T path (DraftAttention2 App. C.1: the 8-bit
path computes Q K^T from INT8 operands and P V from FP8 ones).
Reading of the unstated scale: symmetric per 64-token tile, s = amax/127,
code = clamp(RNE(x * (127/amax)), -127, 127), zero tile -> s = 0, codes 0.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.test_oracle_attention import F, HV, WV, _dequant_tables, _qkv


@pytest.mark.parametrize("x,want", [(2.5, 2), (3.5, 4), (-2.5, -2), (0.49, 0), (-0.5, 0), (126.6, 127), (127.4, 127),
                                    (300.0, 127), (-300.0, -127), (0.0, 0), (1.5, 2)])
def test_int8_codec_hand_table(x, want):
    assert O.int8_encode(x) == want


def _tile_of(values, F=1, Hv=8, Wv=8, d=64):
    """One 8x8 frame (a single 64-token block) whose Q tile holds `values`."""
    q = torch.tensor(values, dtype=torch.float32).reshape(1, 1, 64, d).to(torch.bfloat16)
    return q, q.clone()


def test_int8_hand_built_tile():
    # amax = 4 -> s = 4/127, inv = 127/4 = 31.75: x = 1 -> 31.75 -> 32; x = -2 -> -63.5 -> -64 (even);
    # x = 4 -> 127; x = 0.5 -> 15.875 -> 16; x = 0.015625 -> 0.49609375 -> 0
    vals = np.zeros(64 * 64, np.float32)
    vals[:5] = [1.0, -2.0, 4.0, 0.5, 0.015625]
    q, k = _tile_of(vals)
    st, na = O.slot_tokens(1, 8, 8)
    q8i, k8i, si8 = O.prepare_int8(q, k, 1, 8, 8)
    assert si8[0, 0, 0, 0] == np.float32(4.0) / np.float32(127.0)
    # slot order follows the partition: find where token 0..4 landed
    pos = {int(t): i for i, t in enumerate(st[:64]) if t >= 0}
    codes = [int(q8i[0, 0, 0, pos[0], c]) for c in range(5)]
    assert codes == [32, -64, 127, 16, 0]
    assert not q8i[0, 0, 0][:, 5:].any()


def test_int8_zero_tile_and_error_bound():
    q, k, v = _qkv(8)
    k = torch.zeros_like(k)
    q8i, k8i, si8 = O.prepare_int8(q, k, F, HV, WV)
    assert not k8i.any() and not si8[1].any()
    st, na = O.slot_tokens(F, HV, WV)
    qn = q.float().numpy()
    for h in range(2):
        for a in range(len(na)):
            toks = st[a * 64:a * 64 + na[a]]
            x = qn[0, h, toks].astype(np.float64)
            sc = float(si8[0, 0, h, a])
            deq = q8i[0, h, a, :na[a]].astype(np.float64) * sc
            # half a step, plus the fp32 rounding of 127/amax and of amax/127
            # (each within 2^-24 relative) acting on |x| <= amax
            assert np.all(np.abs(deq - x) <= 0.5 * sc + np.abs(x) * 2.0 ** -22)


def test_int8_qk_exact_weights_match_numpy():
    # quantized operands with exact weights (flags 1 | 8): the 8-bit pairs'
    # logits come from the INT8-dequantized Q and K, the values stay FP8 and
    # the NVFP4 pairs are unchanged; recomputed block by block in numpy
    q, k, v = _qkv(9)
    prep = O.prepare(q, k, v, F, HV, WV)
    A = O.draft(prep.desc, 0.2)
    plan = O.assign(A, 2500, 2500)
    i8 = O.prepare_int8(q, k, F, HV, WV)
    out = O.attention(q, k, v, F, HV, WV, prep, plan, flags=1, int8=i8)
    q8i, k8i, si8 = i8
    e4, e2 = _dequant_tables()
    st, na = O.slot_tokens(F, HV, WV)
    R, d = len(na), q.shape[-1]
    for h in range(2):
        deq = {}
        for b in range(R):
            s8 = prep.s8[:, 0, h, b].astype(np.float64)
            g4 = prep.g4[:, 0, h, b].astype(np.float64)
            deq[8, b] = (q8i[0, h, b] * float(si8[0, 0, h, b]), k8i[0, h, b] * float(si8[1, 0, h, b]),
                         e4[prep.v8t[0, h, b]].T * s8[2])
            sq = np.repeat(e4[prep.sfq[0, h, b]], 16, 1)
            sk = np.repeat(e4[prep.sfk[0, h, b]], 16, 1)
            sv = np.repeat(e4[prep.sfv[0, h, b]], 16, 1)
            deq[4, b] = (e2[prep.q4[0, h, b]] * sq * g4[0], e2[prep.k4[0, h, b]] * sk * g4[1],
                         (e2[prep.v4t[0, h, b]] * sv).T * g4[2])
        for a in range(R):
            nq = na[a]
            logits, vals = [], []
            for b in range(R):
                p = plan.prec[0, h, a, b]
                if p:
                    logits.append(deq[p, a][0][:nq] @ deq[p, b][1][:na[b]].T / math.sqrt(d))
                    vals.append(deq[p, b][2][:na[b]])
            toks = st[a * 64:a * 64 + nq]
            s = np.concatenate(logits, 1)
            pm = np.exp(s - s.max(1, keepdims=True))
            ref = (pm @ np.concatenate(vals, 0)) / pm.sum(1, keepdims=True)
            np.testing.assert_allclose(out[0, h, toks], ref, rtol=0, atol=1e-12)


def test_int8_qk_leaves_uniform_scores_unchanged():
    # K = 0: every score is 0 in both 8-bit formats, so the INT8 QK^T path gives
    # exactly the FP8 path's output (the weights and the FP8 PV do not change)
    q, k, v = _qkv(10)
    k = torch.zeros_like(k)
    _, _, _, ref = O.run(q, k, v, F, HV, WV, 3000, 2000, flags=7)
    _, _, _, got = O.run(q, k, v, F, HV, WV, 3000, 2000, flags=7, int8=True)
    assert np.array_equal(got, ref)


def test_int8_qk_changes_only_8_bit_pairs():
    # with no 8-bit pairs the INT8 operands are never used
    q, k, v = _qkv(11)
    _, _, _, ref = O.run(q, k, v, F, HV, WV, 0, 5000, flags=7)
    _, _, _, got = O.run(q, k, v, F, HV, WV, 0, 5000, flags=7, int8=True)
    assert np.array_equal(got, ref)
    _, _, _, ref8 = O.run(q, k, v, F, HV, WV, 5000, 0, flags=7)
    _, _, _, got8 = O.run(q, k, v, F, HV, WV, 5000, 0, flags=7, int8=True)
    assert not np.array_equal(got8, ref8)
    assert np.abs(got8 - ref8).max() < 0.05
