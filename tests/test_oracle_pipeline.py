"""Pins for the oracle's partition, pooling, draft map, ranking and
quantization, each checked against something other than the oracle itself:
the properties the pages state, closed forms, brute force, and numbers
computed by hand.  Citations are to "DraftAttention2" (paperpeel.com/paper/
2609.32628.md).
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from video_dit_sparse_da2_b200.inputs import make_qkv

SHAPES = [(16, 16), (30, 52), (60, 90), (45, 80), (1, 1), (7, 13), (3, 100), (9, 9), (8, 8), (11, 64)]


def _connected(mask):
    ys, xs = np.nonzero(mask)
    if len(ys) == 0:
        return False
    seen = {(ys[0], xs[0])}
    stack = [(ys[0], xs[0])]
    cells = set(zip(ys.tolist(), xs.tolist()))
    while stack:
        y, x = stack.pop()
        for n in ((y + 1, x), (y - 1, x), (y, x + 1), (y, x - 1)):
            if n in cells and n not in seen:
                seen.add(n)
                stack.append(n)
    return len(seen) == len(cells)


@pytest.mark.parametrize("Hv,Wv", SHAPES)
def test_partition_properties(Hv, Wv):
    # Sec. 3.3: connected regions, balanced counts bounded by the block
    # capacity, the minimum number of blocks, less than one block of padding.
    reg, slot, na = O.partition(Hv, Wv)
    n = Hv * Wv
    Rf = len(na)
    assert Rf == math.ceil(n / 64)
    assert Rf * 64 - n < 64
    assert na.max() - na.min() <= 1 and na.max() <= 64 and na.sum() == n
    g = reg.reshape(Hv, Wv)
    for j in range(Rf):
        m = g == j
        assert m.sum() == na[j]
        assert sorted(slot[reg == j].tolist()) == list(range(na[j]))
        if n > 1:
            assert _connected(m), f"region {j} not connected"


def test_partition_tiny_is_8x8_patches():
    reg, _, na = O.partition(16, 16)
    g = reg.reshape(16, 16)
    for j in range(4):
        ys, xs = np.nonzero(g == j)
        assert ys.max() - ys.min() == 7 and xs.max() - xs.min() == 7


def _tiny(seed=0, B=1, H=2, d=64, F=4, Hv=16, Wv=16):
    q, k, v = make_qkv(B, H, F * Hv * Wv, d, seed)
    return q, k, v, (F, Hv, Wv)


def _regions(F, Hv, Wv):
    st, na = O.slot_tokens(F, Hv, Wv)
    R = len(na)
    return [st[a * 64:a * 64 + na[a]] for a in range(R)]


@pytest.mark.parametrize("geom", [(4, 16, 16), (2, 9, 13), (3, 5, 30)])
def test_descriptors_mean_max_and_bilinearity(geom):
    F, Hv, Wv = geom
    q, k, v, _ = _tiny(1, 1, 2, 32, F, Hv, Wv)
    prep = O.prepare(q, k, v, F, Hv, Wv)
    regs = _regions(F, Hv, Wv)
    qn = q.double().numpy()
    kn = k.double().numpy()
    for h in range(2):
        for a, toks in enumerate(regs):
            np.testing.assert_allclose(prep.desc[0, 0, h, a], qn[0, h, toks].mean(0), rtol=0, atol=1e-14)
            assert np.array_equal(prep.desc[1, 0, h, a], qn[0, h, toks].max(0))
            assert np.array_equal(prep.desc[3, 0, h, a], kn[0, h, toks].max(0))
        # Sec. 3.1: by bilinearity Qbar_a . Kbar_b equals the mean token-pair logit
        for a in (0, len(regs) - 1):
            for b in (0, 3, len(regs) - 1):
                lhs = prep.desc[0, 0, h, a] @ prep.desc[2, 0, h, b]
                rhs = (qn[0, h, regs[a]] @ kn[0, h, regs[b]].T).mean()
                assert abs(lhs - rhs) < 1e-12


def _softmax(x):
    x = x - x.max(-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(-1, keepdims=True)


@pytest.mark.parametrize("lam", [0.0, 0.2, 1.0])
def test_draft_map_closed_form(lam):
    # Eq. 3 with both branches normalized over key regions (App. C.1).
    q, k, v, (F, Hv, Wv) = _tiny(2)
    prep = O.prepare(q, k, v, F, Hv, Wv)
    A = O.draft(prep.desc, lam)
    d = q.shape[-1]
    for h in range(2):
        sa = _softmax(prep.desc[0, 0, h] @ prep.desc[2, 0, h].T / math.sqrt(d))
        sm = _softmax(prep.desc[1, 0, h] @ prep.desc[3, 0, h].T / math.sqrt(d))
        ref = (1 - lam) * sa + lam * sm
        np.testing.assert_allclose(A[0, h], ref, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(A[0, h].sum(-1), 1.0, rtol=0, atol=1e-13)


def _brute_assign(A, bp8, bp4):
    R = A.shape[0]
    order = sorted(range(R * R), key=lambda i: (-A.flat[i], i))
    T8 = (R * R * bp8) // 10000
    Tk = (R * R * (bp8 + bp4)) // 10000
    prec = np.zeros(R * R, np.uint8)
    for r, i in enumerate(order):
        prec[i] = 8 if r < T8 else (4 if r < Tk else 0)
    return prec.reshape(R, R)


@pytest.mark.parametrize("bp8,bp4", [(2500, 2500), (0, 0), (10000, 0), (0, 10000), (1000, 3000), (1, 9998)])
def test_assign_matches_brute_force_sort(bp8, bp4):
    q, k, v, (F, Hv, Wv) = _tiny(3, 1, 2, 64, 6, 16, 16)
    prep = O.prepare(q, k, v, F, Hv, Wv)
    A = O.draft(prep.desc, 0.2)
    plan = O.assign(A, bp8, bp4)
    R = A.shape[-1]
    for h in range(2):
        ref = _brute_assign(A[0, h], bp8, bp4)
        assert np.array_equal(plan.prec[0, h], ref)
        assert (ref == 8).sum() == (R * R * bp8) // 10000
        assert (ref == 4).sum() == (R * R * (bp8 + bp4)) // 10000 - (R * R * bp8) // 10000
        for a in range(R):
            n8, n4 = plan.cnt[0, 0, h, a], plan.cnt[1, 0, h, a]
            row = plan.kidx[0, h, a]
            assert list(row[:n8]) == list(np.nonzero(ref[a] == 8)[0])
            assert list(row[n8:n8 + n4]) == list(np.nonzero(ref[a] == 4)[0])
        # precision-by-mass ordering (Sec. 3.2 theorem, App. B.6) as an invariant
        Ah = A[0, h]
        if (ref == 8).any() and (ref == 4).any():
            assert Ah[ref == 8].min() >= Ah[ref == 4].max()
        if (ref == 4).any() and (ref == 0).any():
            assert Ah[ref == 4].min() >= Ah[ref == 0].max()


def test_assign_ties_resolved_by_pair_index():
    # All regions identical -> every draft score ties; App. C.1 resolves ties
    # by region-pair index, so the lowest indices win the higher precisions.
    F, Hv, Wv = 4, 16, 16
    q, k, v = make_qkv(1, 1, F * Hv * Wv, 64, 4)
    regs = _regions(F, Hv, Wv)
    for t in (q, k):
        base = t[0, 0, regs[0]].clone()
        for toks in regs:
            t[0, 0, toks] = base
    prep = O.prepare(q, k, v, F, Hv, Wv)
    A = O.draft(prep.desc, 0.2)
    assert np.all(A[0, 0] == A[0, 0, 0, 0])
    plan = O.assign(A, 2500, 2500)
    R = A.shape[-1]
    flat = plan.prec[0, 0].reshape(-1)
    T8, Tk = R * R * 2500 // 10000, R * R * 5000 // 10000
    assert np.all(flat[:T8] == 8) and np.all(flat[T8:Tk] == 4) and np.all(flat[Tk:] == 0)


def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def test_quantization_hand_example():
    """A hand-built tile: amax 6, so the FP8 scale is 6/448 and the NVFP4 tile
    scale is 6/2688; channel group 0 has amax 6 (group scale 448), group 1 has
    amax 0.75 (group scale 56, so the group step is 8 x 6/2688 x 56/448 ...)."""
    F, Hv, Wv, d = 1, 8, 8, 32
    q = torch.zeros(1, 1, 64, d, dtype=torch.bfloat16)
    row0 = [6, 4, 3, 2, 1.5, 1, 0.5, 0, -0.5, -1, -6, 5.2, 2.4, 0.2, 0.8, -3]
    row1 = [0.75, 0.5, 0.25, 0.125, 0.0625, 0.1875, 0.375, -0.75, 0, 0, 0, 0, 0, 0, 0, -0.0625]
    q[0, 0, 0, :16] = _bf16(row0)
    q[0, 0, 0, 16:] = _bf16(row1)
    k = q.clone()
    v = q.clone()
    prep = O.prepare(q, k, v, F, Hv, Wv)
    st, _ = O.slot_tokens(F, Hv, Wv)
    slot = int(np.nonzero(st == 0)[0][0])  # slot of token 0
    # FP8: scale amax/448, codes e4m3(x*448/6)
    assert prep.s8[0, 0, 0, 0] == np.float32(6) / np.float32(448)
    exp8 = {6: 0x7E, 4: 0x79, 1: 0x69, 0.5: 0x61, 0: 0x00, -6: 0xFE, 0.75: 0x66}
    for c, x in enumerate(row0 + row1):
        if x in exp8:
            assert prep.q8[0, 0, 0, slot, c] == exp8[x], (c, x)
    # NVFP4 group scales: ue4m3(6 * 448/6) = 448, ue4m3(0.75 * 448/6) = 56
    assert prep.sfq[0, 0, 0, slot, 0] == 0x7E and prep.sfq[0, 0, 0, slot, 1] == 0x66
    assert prep.g4[0, 0, 0, 0] == np.float32(6) / np.float32(2688)
    codes0 = [0x7, 0x6, 0x5, 0x4, 0x3, 0x2, 0x1, 0x0, 0x9, 0xA, 0xF, 0x7, 0x4, 0x0, 0x2, 0xD]
    codes1 = [0x7, 0x6, 0x4, 0x2, 0x1, 0x3, 0x5, 0xF, 0, 0, 0, 0, 0, 0, 0, 0x9]
    assert list(prep.q4[0, 0, 0, slot, :16]) == codes0
    assert list(prep.q4[0, 0, 0, slot, 16:]) == codes1
    # every other slot of the tile is zero: zero codes, and its groups get scale 0
    others = [s for s in range(64) if s != slot]
    assert not prep.q4[0, 0, 0, others].any() and not prep.sfq[0, 0, 0, others].any()
    # the value path is the transpose: V^T row c holds channel c over the slots
    assert prep.v8t[0, 0, 0, 0, slot] == 0x7E and prep.v4t[0, 0, 0, 16, slot] == 0x7


def test_quantization_error_bounds():
    q, k, v, (F, Hv, Wv) = _tiny(5)
    prep = O.prepare(q, k, v, F, Hv, Wv)
    st, na = O.slot_tokens(F, Hv, Wv)
    e4 = np.array([O.e4m3_decode(c) for c in range(256)])
    e2 = np.array([O.e2m1_decode(c) for c in range(16)])
    qn = q.double().numpy()[0, 0]
    for a in range(0, len(na), 5):
        toks = st[a * 64:(a + 1) * 64]
        x = np.zeros((64, 64))
        x[toks >= 0] = qn[toks[toks >= 0]]
        s = float(prep.s8[0, 0, 0, a])
        xh = e4[prep.q8[0, 0, a]] * s
        # e4m3 relative step is 2^-3 in the normal range; subnormal step 2^-9
        assert np.all(np.abs(xh - x) <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s) * (1 + 1e-6))
        g = float(prep.g4[0, 0, 0, a])
        sf = e4[prep.sfq[0, 0, a]]  # [64, d/16]
        x4 = e2[prep.q4[0, 0, a]] * np.repeat(sf, 16, axis=1) * g
        # e2m1 half-step is at most 1 (between 4 and 6) in units of the group scale,
        # plus the group scale's own rounding (relative 2^-4) at saturation
        bound = np.repeat(sf, 16, axis=1) * g * 1.0 + np.abs(x) * 2.0 ** -4 + 1e-12
        assert np.all(np.abs(x4 - x) <= bound)


def _brute_assign_rows(A, bp8, bp4):
    R = A.shape[0]
    T8, Tk = R * bp8 // 10000, R * (bp8 + bp4) // 10000
    prec = np.zeros((R, R), np.uint8)
    for a in range(R):
        order = sorted(range(R), key=lambda b: (-A[a, b], b))
        for r, b in enumerate(order):
            prec[a, b] = 8 if r < T8 else (4 if r < Tk else 0)
    return prec


@pytest.mark.parametrize("bp8,bp4", [(2500, 2500), (0, 0), (10000, 0), (0, 10000), (1000, 3000), (700, 600)])
def test_assign_rows_matches_brute_force_sort(bp8, bp4):
    q, k, v, (F, Hv, Wv) = _tiny(3, 1, 2, 64, 6, 16, 16)
    prep = O.prepare(q, k, v, F, Hv, Wv)
    A = O.draft(prep.desc, 0.2)
    plan = O.assign(A, bp8, bp4, per_row=True)
    R = A.shape[-1]
    for h in range(2):
        ref = _brute_assign_rows(A[0, h], bp8, bp4)
        assert np.array_equal(plan.prec[0, h], ref)
        for a in range(R):
            # per-row quotas, exact
            assert (ref[a] == 8).sum() == R * bp8 // 10000
            assert (ref[a] == 4).sum() == R * (bp8 + bp4) // 10000 - R * bp8 // 10000
            n8, n4 = plan.cnt[0, 0, h, a], plan.cnt[1, 0, h, a]
            row = plan.kidx[0, h, a]
            assert list(row[:n8]) == list(np.nonzero(ref[a] == 8)[0])
            assert list(row[n8:n8 + n4]) == list(np.nonzero(ref[a] == 4)[0])
            # precision by mass inside each row
            Ar = A[0, h, a]
            if (ref[a] == 8).any() and (ref[a] == 4).any():
                assert Ar[ref[a] == 8].min() >= Ar[ref[a] == 4].max()
            if (ref[a] == 4).any() and (ref[a] == 0).any():
                assert Ar[ref[a] == 4].min() >= Ar[ref[a] == 0].max()


def test_assign_rows_ties_resolved_by_key_block():
    F, Hv, Wv = 4, 16, 16
    q, k, v = make_qkv(1, 1, F * Hv * Wv, 64, 4)
    regs = _regions(F, Hv, Wv)
    for t in (q, k):
        base = t[0, 0, regs[0]].clone()
        for toks in regs:
            t[0, 0, toks] = base
    prep = O.prepare(q, k, v, F, Hv, Wv)
    A = O.draft(prep.desc, 0.2)
    plan = O.assign(A, 2500, 2500, per_row=True)
    R = A.shape[-1]
    T8, Tk = R * 2500 // 10000, R * 5000 // 10000
    for a in range(R):
        row = plan.prec[0, 0, a]
        assert np.all(row[:T8] == 8) and np.all(row[T8:Tk] == 4) and np.all(row[Tk:] == 0)
