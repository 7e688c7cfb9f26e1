"""Pins of the oracle's 16-bit tier (DraftAttention2 Table 1's 0 / 4 / 8 / 16-bit
allocations; App. B.6: the 16-bit path takes the largest draft masses, the
8-bit path the next, NVFP4 the rest; Sec. 3.3 "Phased execution", Eq. 7:
at most two phase switches).  Readings: cumulative quotas C16, C8, Ck over the
same ranking; phases 16 -> 8 -> 4; the 16-bit path multiplies the bf16
inputs as they are, with bf16(p) weights in unit 1; O changes units by
u_old / u_new at each switch.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.test_oracle_attention import F, HV, WV, _dense_np, _dequant_tables, _qkv, _token_mask


# ---------------------------------------------------------------- bf16 rounding
@pytest.mark.parametrize("x,want", [
    (1.0, 1.0),
    (1.0 + 2.0 ** -8, 1.0),                      # tie, to the even significand
    (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),       # tie, to the even significand
    (1.0 + 3 * 2.0 ** -9, 1.0 + 2.0 ** -7),       # nearest
    (0.3, 0.30078125),                           # 0.3 = 1.2 * 2^-2 -> 1.203125 * 2^-2
    (2.0 ** -130, 2.0 ** -130),                  # a bf16 subnormal
    (3 * 2.0 ** -134, 2.0 ** -132),              # tie between subnormals 2^-133 and 2^-132
    (0.0, 0.0),
])
def test_bf16_round_hand_table(x, want):
    assert O.bf16_round(x) == want


def test_bf16_round_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.rand(4000, generator=g), torch.rand(4000, generator=g) * 1e-30,
                   torch.randn(2000, generator=g) * 100])
    want = x.to(torch.bfloat16).double().numpy()
    got = np.array([O.bf16_round(float(t)) for t in x.double().numpy()])
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- tiers
def _brute_tiers(A, bp16, bp8, bp4, per_row):
    B, H, R, _ = A.shape
    prec = np.zeros(A.shape, np.uint8)
    for b in range(B):
        for h in range(H):
            sets = [[(a, bb) for bb in range(R)] for a in range(R)] if per_row else \
                [[(a, bb) for a in range(R) for bb in range(R)]]
            for pairs in sets:
                n = len(pairs)
                c16, c8, ck = n * bp16 // 10000, n * (bp16 + bp8) // 10000, n * (bp16 + bp8 + bp4) // 10000
                order = sorted(pairs, key=lambda ab: (-A[b, h, ab[0], ab[1]], ab[0] * R + ab[1]))
                for r, (a, bb) in enumerate(order):
                    prec[b, h, a, bb] = 16 if r < c16 else 8 if r < c8 else 4 if r < ck else 0
    return prec


TIER_BUDGETS = [(2000, 1000, 3000), (10000, 0, 0), (3333, 3333, 3334), (500, 0, 4000), (1, 1, 1), (0, 2500, 2500)]


@pytest.mark.parametrize("per_row", [False, True])
@pytest.mark.parametrize("bp", TIER_BUDGETS)
def test_tiers_match_brute_force_and_quotas(bp, per_row):
    q, k, v = _qkv(1)
    A = O.draft(O.prepare(q, k, v, F, HV, WV).desc, 0.2)
    bp16, bp8, bp4 = bp
    plan = O.assign(A, bp8, bp4, per_row=per_row, bp16=bp16) if bp16 else O.assign(A, bp8, bp4, per_row)
    assert np.array_equal(plan.prec, _brute_tiers(A, bp16, bp8, bp4, per_row))
    R = A.shape[-1]
    n = R if per_row else R * R
    c16, c8, ck = n * bp16 // 10000, n * (bp16 + bp8) // 10000, n * (bp16 + bp8 + bp4) // 10000
    axes = (-1,) if per_row else (-2, -1)
    for val, want in ((16, c16), (8, c8 - c16), (4, ck - c8)):
        assert np.all((plan.prec == val).sum(axis=axes) == want)
    # lists: 16-bit, then 8-bit, then 4-bit key blocks, each ascending
    if bp16:
        for h in range(2):
            for a in range(R):
                row = plan.prec[0, h, a]
                want = [b for t in (16, 8, 4) for b in range(R) if row[b] == t]
                n16, n8, n4 = plan.cnt[2, 0, h, a], plan.cnt[0, 0, h, a], plan.cnt[1, 0, h, a]
                assert (n16, n8, n4) == tuple(int((row == t).sum()) for t in (16, 8, 4))
                assert list(plan.kidx[0, h, a, :n16 + n8 + n4]) == want


def test_tiers_without_16_bit_equal_two_tier_assignment():
    q, k, v = _qkv(2)
    A = O.draft(O.prepare(q, k, v, F, HV, WV).desc, 0.2)
    for per_row in (False, True):
        two = O.assign(A, 1500, 3500, per_row)
        lib = O.lib()
        B, H, R, _ = A.shape
        prec = np.zeros((B, H, R, R), np.uint8)
        cnt = np.zeros((3, B, H, R), np.int32)
        kidx = np.zeros((B, H, R, R), np.uint16)
        assert lib.oracle_assign_tiers(B * H, R, O._p(np.ascontiguousarray(A)), 0, 1500, 3500, int(per_row),
                                       O._p(prec), O._p(cnt), O._p(kidx)) == 0
        assert np.array_equal(prec, two.prec) and np.array_equal(cnt[:2], two.cnt) and not cnt[2].any()
        assert np.array_equal(kidx, two.kidx)


def test_tiers_monotone_in_draft_mass():
    # App. B.6: larger mass -> higher precision (ties by pair index only)
    q, k, v = _qkv(3)
    A = O.draft(O.prepare(q, k, v, F, HV, WV).desc, 0.2)
    plan = O.assign(A, 2000, 2000, bp16=2000)
    for h in range(2):
        a, p = A[0, h], plan.prec[0, h]
        assert a[p == 16].min() >= a[p == 8].max() >= a[p == 4].max()
        assert a[p == 4].min() >= a[p == 0].max()


# ---------------------------------------------------------------- attention
@pytest.mark.parametrize("d", [64, 128])
def test_all_16_bit_exact_weights_equals_dense(d):
    # every pair at 16 bits, weights not rounded (flags 5: quantized 8/4-bit
    # operands, which this budget never uses; units on): dense attention
    q, k, v = _qkv(4, d=d)
    _, _, _, out = O.run(q, k, v, F, HV, WV, 0, 0, flags=5, bp16=10000)
    np.testing.assert_allclose(out, _dense_np(q, k, v), rtol=0, atol=1e-12)


def test_all_16_bit_weights_rounded_to_bf16_stay_close():
    # bf16(p) differs from p by at most 2^-9 p, so every output moves by at
    # most 2^-9 max|V| (the weights are renormalized by the exact l)
    q, k, v = _qkv(5)
    _, _, _, out = O.run(q, k, v, F, HV, WV, 0, 0, flags=7, bp16=10000)
    dense = _dense_np(q, k, v)
    assert np.abs(out - dense).max() <= 2.0 ** -9 * float(v.float().abs().max())
    assert np.abs(out - dense).max() > 0  # the rounding is applied


@pytest.mark.parametrize("bp", [(2000, 1000, 3000), (3000, 0, 3000), (2500, 2500, 0)])
def test_three_phases_unquantized_equal_dense_on_kept_mask(bp):
    # without any quantization the unit changes are exact inverses: the three
    # phases give softmax attention restricted to the kept pairs
    q, k, v = _qkv(6)
    bp16, bp8, bp4 = bp
    st, na = O.slot_tokens(F, HV, WV)
    N = q.shape[2]
    for flags in (0, 4):
        prep, A, plan, out = O.run(q, k, v, F, HV, WV, bp8, bp4, flags=flags, bp16=bp16)
        for h in range(2):
            mask = _token_mask(plan, st, na, N, h)
            ref = _dense_np(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], mask[None, None])
            rows = mask.any(1)
            np.testing.assert_allclose(out[0, h][rows], ref[0, 0][rows], rtol=0, atol=1e-12)


@pytest.mark.parametrize("bp", [(2000, 1000, 3000), (2000, 0, 3000), (3000, 3000, 0)])
def test_three_phases_closed_form_uniform_scores(bp):
    # K = 0 makes every score of a row tie, so p = 1 for every valid key; one
    # +8 per V tile puts every tile at the head maximum.  The weights then
    # follow from the formats: 16-bit bf16(1) = 1; FP8 e4m3(448) = 448;
    # NVFP4 e2m1(6) * 448 = 2688.  Each output is the mean, over the kept
    # valid keys, of the exact V (16-bit), of f8 * the dequantized FP8 values
    # and of f4 * the dequantized NVFP4 values (f8, f4 = 1 up to one fp32
    # rounding), across both changes of units.
    f32 = np.float32
    bp16, bp8, bp4 = bp
    q, k, v = _qkv(7)
    k = torch.zeros_like(k)
    st, na = O.slot_tokens(F, HV, WV)
    R, d = len(na), q.shape[-1]
    for a in range(R):
        v[:, :, st[a * 64], 0] = 8.0
    prep, A, plan, out = O.run(q, k, v, F, HV, WV, bp8, bp4, flags=7, bp16=bp16)
    assert (plan.prec == 16).any()
    e4, e2 = _dequant_tables()
    vx = v.double().numpy()
    for h in range(2):
        s8 = f32(prep.s8[2, 0, h, 0])
        g4 = f32(prep.g4[2, 0, h, 0])
        sig8, sig4 = f32(prep.vmax[0, 0, h]) / f32(448), f32(prep.vmax[1, 0, h]) / f32(2688)
        f8 = 448.0 * float(sig8) / float(s8)
        f4 = 2688.0 * float(sig4) / float(g4)
        dq = {}
        for b in range(R):
            dq[16, b] = vx[0, h, st[b * 64:b * 64 + na[b]]]
            dq[8, b] = (e4[prep.v8t[0, h, b]] * float(s8)).T[:na[b]]
            sv = np.repeat(e4[prep.sfv[0, h, b]], 16, 1)
            dq[4, b] = ((e2[prep.v4t[0, h, b]] * sv) * float(g4)).T[:na[b]]
        for a in range(R):
            toks = st[a * 64:a * 64 + na[a]]
            num, cnt = np.zeros(d), 0
            for b in range(R):
                p = int(plan.prec[0, h, a, b])
                if p:
                    num += {16: 1.0, 8: f8, 4: f4}[p] * dq[p, b].sum(0)
                    cnt += na[b]
            ref = num / cnt if cnt else np.zeros(d)
            np.testing.assert_allclose(out[0, h, toks], np.broadcast_to(ref, (len(toks), d)), rtol=1e-12, atol=1e-12)
