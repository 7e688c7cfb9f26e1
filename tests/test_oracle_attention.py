"""Pins for the oracle's block-sparse mixed-precision attention
("DraftAttention2", App. B.3-B.4, C.1; Sec. 3.3 cross-precision accumulation).

flags: bit0 quantize Q/K/V, bit1 quantize the weights, bit2 phase units.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from video_dit_sparse_da2_b200.inputs import make_qkv

F, HV, WV = 4, 16, 16


def _qkv(seed=0, H=2, d=64, F=F, Hv=HV, Wv=WV):
    return make_qkv(1, H, F * Hv * Wv, d, seed)


def _dense_np(q, k, v, mask=None):
    """Brute-force softmax attention in numpy float64; mask[u, t] False drops key t."""
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    d = qn.shape[-1]
    s = np.einsum("bhud,bhtd->bhut", qn, kn) / math.sqrt(d)
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    m = s.max(-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m)
    l = p.sum(-1, keepdims=True)
    o = np.einsum("bhut,bhtd->bhud", p, vn)
    return np.where(l > 0, o / np.where(l > 0, l, 1), 0.0)


@pytest.mark.parametrize("flags", [0, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_all_kept_unquantized_equals_dense(flags, d):
    # Everything kept at full precision must equal dense attention (1e-12);
    # the unit changes of Eq. 8 are exact inverses (App. B.3).
    q, k, v = _qkv(0, 2, d)
    for bp8, bp4 in ((10000, 0), (0, 10000), (3000, 7000)):
        prep, A, plan, out = O.run(q, k, v, F, HV, WV, bp8, bp4, flags=flags)
        ref = _dense_np(q, k, v)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_dense_oracle_helper_agrees_with_numpy():
    q, k, v = _qkv(7, 1, 64, 2, 8, 8)
    np.testing.assert_allclose(O.dense(q, k, v), _dense_np(q, k, v), rtol=0, atol=1e-12)


def _token_mask(plan, st, na, N, h):
    """Dense mask [N, N] of the kept (query token, key token) pairs of head h."""
    R = len(na)
    mask = np.zeros((N, N), bool)
    for a in range(R):
        qa = st[a * 64:a * 64 + na[a]]
        for b in range(R):
            if plan.prec[0, h, a, b]:
                mask[np.ix_(qa, st[b * 64:b * 64 + na[b]])] = True
    return mask


def test_skipped_blocks_follow_the_mask_and_the_sparsification_bound():
    # Quantization off, half of the pairs skipped: the output is dense
    # attention restricted to the kept blocks, and it obeys the closed-form
    # bound ||O_dense - O_u|| <= 2 max_v ||V_v|| delta_u (Eq. 5 with no
    # quantization term; proof in App. B.4).
    q, k, v = _qkv(1)
    prep, A, plan, out = O.run(q, k, v, F, HV, WV, 2500, 2500, flags=4)
    st, na = O.slot_tokens(F, HV, WV)
    N = q.shape[2]
    masks = np.stack([_token_mask(plan, st, na, N, h) for h in range(2)])[None]
    ref = _dense_np(q, k, v, masks)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    dense = _dense_np(q, k, v)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    s = np.einsum("bhud,bhtd->bhut", qn, kn) / 8.0
    P = np.exp(s - s.max(-1, keepdims=True))
    P /= P.sum(-1, keepdims=True)
    delta = np.where(masks, 0.0, P).sum(-1)
    vmax = np.linalg.norm(vn, axis=-1).max(-1)[..., None]
    err = np.linalg.norm(dense - out, axis=-1)
    assert np.all(err <= 2 * vmax * delta + 1e-12)


def test_empty_rows_return_zero():
    # App. C.1: a row with no retained valid key returns zero.
    q, k, v = _qkv(2)
    prep, A, plan, out = O.run(q, k, v, F, HV, WV, 0, 0)
    assert not out.any()
    prep, A, plan, out = O.run(q, k, v, F, HV, WV, 100, 0)
    kept_rows = plan.cnt[0, 0].sum(0) + plan.cnt[1, 0].sum(0)
    assert (plan.cnt[0, 0] + plan.cnt[1, 0] == 0).any()
    st, na = O.slot_tokens(F, HV, WV)
    for h in range(2):
        for a in range(len(na)):
            toks = st[a * 64:a * 64 + na[a]]
            if plan.cnt[0, 0, h, a] + plan.cnt[1, 0, h, a] == 0:
                assert not out[0, h, toks].any()
            else:
                assert np.abs(out[0, h, toks]).sum() > 0


def _dequant_tables():
    e4 = np.array([O.e4m3_decode(c) for c in range(256)])
    e2 = np.array([O.e2m1_decode(c) for c in range(16)])
    return e4, e2


@pytest.mark.parametrize("flags", [1, 5])
def test_quantized_operands_exact_weights(flags):
    # With the weights exact, the output is softmax attention over the kept
    # blocks computed from the dequantized operands of each pair's precision
    # (codes * scales, App. C.1), here recomputed block by block in numpy.
    q, k, v = _qkv(3)
    prep, A, plan, out = O.run(q, k, v, F, HV, WV, 2500, 2500, flags=flags)
    e4, e2 = _dequant_tables()
    st, na = O.slot_tokens(F, HV, WV)
    R, d = len(na), q.shape[-1]
    for h in range(2):
        deq = {}
        for b in range(R):
            s8 = prep.s8[:, 0, h, b].astype(np.float64)
            g4 = prep.g4[:, 0, h, b].astype(np.float64)
            deq[8, b] = (e4[prep.q8[0, h, b]] * s8[0], e4[prep.k8[0, h, b]] * s8[1], e4[prep.v8t[0, h, b]].T * s8[2])
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
                if not p:
                    continue
                Qd, Kd, Vd = deq[p, a][0], deq[p, b][1], deq[p, b][2]
                logits.append(Qd[:nq] @ Kd[:na[b]].T / math.sqrt(d))
                vals.append(Vd[:na[b]])
            toks = st[a * 64:a * 64 + nq]
            if not logits:
                assert not out[0, h, toks].any()
                continue
            s = np.concatenate(logits, 1)
            pm = np.exp(s - s.max(1, keepdims=True))
            ref = (pm @ np.concatenate(vals, 0)) / pm.sum(1, keepdims=True)
            np.testing.assert_allclose(out[0, h, toks], ref, rtol=0, atol=1e-12)


def test_quantized_weights_stay_close():
    # Quantizing the weights (FP8 e4m3, and NVFP4 with e4m3 scales per 16
    # keys) keeps the output near the exact-weight output: a wrong unit,
    # scale or grouping moves it by a large factor instead.
    q, k, v = _qkv(4)
    for bp8, bp4 in ((10000, 0), (0, 10000), (2500, 2500)):
        _, _, _, o7 = O.run(q, k, v, F, HV, WV, bp8, bp4, flags=7)
        _, _, _, o5 = O.run(q, k, v, F, HV, WV, bp8, bp4, flags=5)
        rel = np.linalg.norm(o7 - o5) / np.linalg.norm(o5)
        lim = 0.05 if bp4 == 0 else 0.25
        assert rel < lim, (bp8, bp4, rel)
    # FP8 weights: each weight is within half an e4m3 step, so each output row
    # moves by at most 2^-4 * sum_v w_v |code_v| * unit / l <= 2^-4 * max|V| * (1 + ...)
    _, _, _, o7 = O.run(q, k, v, F, HV, WV, 10000, 0, flags=7)
    _, _, _, o5 = O.run(q, k, v, F, HV, WV, 10000, 0, flags=5)
    vabs = np.abs(v.double().numpy()).max()
    assert np.abs(o7 - o5).max() <= (2.0 ** -4 + 1e-3) * vabs


def test_zero_values_give_zero_output():
    q, k, v = _qkv(5)
    v = torch.zeros_like(v)
    _, _, _, out = O.run(q, k, v, F, HV, WV, 2500, 2500)
    assert not out.any()


@pytest.mark.parametrize("bp8,bp4", [(10000, 0), (0, 10000), (2500, 2500), (1000, 3000)])
def test_quantized_weights_closed_form_uniform_scores(bp8, bp4):
    # K = 0: every score of a row ties, so p = 1 for every valid key.  One
    # entry of +8 in every V tile gives every tile the head's maximum amax,
    # so every tile scale equals the head maximum: s8_V = vmax8 and g4_V =
    # vmax4, hence ratio8 = s8/sigma8 ~ 448 and ratio4 = g4/sigma4 ~ 2688
    # with sigma8 = vmax8/448, sigma4 = vmax4/2688 (reading 9).  The weights
    # of p = 1 then follow from the formats alone: FP8 e4m3(ratio8) = 448
    # (the largest e4m3 value); NVFP4: the group scale e4m3(ratio4/6) = 448
    # and e2m1(ratio4 * (1/448)) = 6, so the weight is 6 * 448 = 2688.  Each
    # output is (f8 * sum of the FP8-kept dequantized values + f4 * sum of the
    # NVFP4-kept ones) / (number of kept valid keys), f8 = 448 sigma8 / s8 and
    # f4 = 2688 sigma4 / g4 (both 1 up to one fp32 rounding), across the
    # phase switch and its change of units.
    f32 = np.float32
    q, k, v = _qkv(6)
    k = torch.zeros_like(k)
    st, na = O.slot_tokens(F, HV, WV)
    R, d = len(na), q.shape[-1]
    for a in range(R):
        v[:, :, st[a * 64], 0] = 8.0
    assert float(v.float().abs().max()) == 8.0
    prep, A, plan, out = O.run(q, k, v, F, HV, WV, bp8, bp4, flags=7)
    e4, e2 = _dequant_tables()
    for h in range(2):
        s8 = f32(prep.s8[2, 0, h, 0])
        g4 = f32(prep.g4[2, 0, h, 0])
        assert np.all(prep.s8[2, 0, h] == s8) and np.all(prep.g4[2, 0, h] == g4)
        sig8, sig4 = f32(prep.vmax[0, 0, h]) / f32(448), f32(prep.vmax[1, 0, h]) / f32(2688)
        r8, r4 = f32(s8 / sig8), f32(g4 / sig4)
        assert O.e4m3_decode(O.e4m3_encode(float(r8))) == 448.0
        assert O.e4m3_decode(O.e4m3_encode(float(f32(r4 / f32(6))))) == 448.0
        assert O.e2m1_decode(O.e2m1_encode(float(f32(r4 * f32(1.0 / 448.0))))) == 6.0
        f8 = 448.0 * float(sig8) / float(s8)
        f4 = 2688.0 * float(sig4) / float(g4)
        dq = {}
        for b in range(R):
            dq[8, b] = (e4[prep.v8t[0, h, b]] * float(s8)).T[:na[b]]
            sv = np.repeat(e4[prep.sfv[0, h, b]], 16, 1)
            dq[4, b] = ((e2[prep.v4t[0, h, b]] * sv) * float(g4)).T[:na[b]]
        for a in range(R):
            toks = st[a * 64:a * 64 + na[a]]
            num, cnt = np.zeros(d), 0
            for b in range(R):
                p = plan.prec[0, h, a, b]
                if p == 8:
                    num += f8 * dq[8, b].sum(0)
                elif p == 4:
                    num += f4 * dq[4, b].sum(0)
                if p:
                    cnt += na[b]
            ref = num / cnt if cnt else np.zeros(d)
            np.testing.assert_allclose(out[0, h, toks], np.broadcast_to(ref, (len(toks), d)), rtol=1e-12, atol=1e-12)
