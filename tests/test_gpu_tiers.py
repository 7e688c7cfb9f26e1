"""GPU parity of the 16-bit tier (DraftAttention2 Table 1's 16-bit share; App.
B.6 ordering; Sec. 3.3 phased execution with up to two phase switches): the
bf16 operand tiles, the three-tier precision map, counts and lists bit for bit,
and the three-phase attention within the output tolerance of the oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import SMALL, bf16_round, check_compact_lists, gpu_run, inputs, rel_l2
from video_dit_sparse_da2_b200 import da2

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS = 1e-2
# (bp16, bp8, bp4): all three tiers, 16/4 only, 16/8 only, 16-bit only, a sliver of 16-bit
TIERS = [(1500, 1500, 2000), (3000, 0, 3000), (2500, 2500, 0), (10000, 0, 0), (300, 1000, 3000)]


@pytest.mark.parametrize("name", ["tiny", "ragged128", "oddR128", "ragged64"])
def test_bf16_tiles_are_the_inputs(name):
    B, H, d, F, Hv, Wv = SMALL[name]
    res = gpu_run(B, H, d, F, Hv, Wv, 1000, 1000, bp16=1000)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    st, na = O.slot_tokens(F, Hv, Wv)
    R = len(na)
    g = res["prep"]
    bits = {n: t.contiguous().view(torch.int16).numpy().view(np.uint16) for n, t in (("q", q), ("k", k), ("v", v))}
    for a in range(R):
        toks = st[a * 64:(a + 1) * 64]
        valid = toks >= 0
        for n, key in (("q", "q16"), ("k", "k16")):
            want = np.zeros((B, H, 64, d), np.uint16)
            want[:, :, valid] = bits[n][:, :, toks[valid]]
            assert np.array_equal(g[key][:, :, a], want), (key, a)
        want = np.zeros((B, H, 64, d), np.uint16)
        want[:, :, valid] = bits["v"][:, :, toks[valid]]
        assert np.array_equal(g["v16t"][:, :, a], np.swapaxes(want, -1, -2)), ("v16t", a)


@pytest.mark.parametrize("per_row", [False, True], ids=["per-head", "per-row"])
@pytest.mark.parametrize("bp", TIERS)
@pytest.mark.parametrize("name", ["tiny", "ragged128", "oddR128"])
def test_three_tier_plan_bit_exact(name, bp, per_row):
    B, H, d, F, Hv, Wv = SMALL[name]
    bp16, bp8, bp4 = bp
    res = gpu_run(B, H, d, F, Hv, Wv, bp8, bp4, bp16=bp16, per_row=per_row)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    A = O.draft(O.prepare(q, k, v, F, Hv, Wv).desc, 0.2)
    plan = O.assign(A, bp8, bp4, per_row=per_row, bp16=bp16)
    got = res["plan"]
    assert np.array_equal(got["A"].view(np.uint64), A.view(np.uint64))
    assert np.array_equal(got["prec"], plan.prec)
    assert np.array_equal(got["cnt"], plan.cnt[:2]) and np.array_equal(got["cnt16"], plan.cnt[2])
    check_compact_lists(got, plan.cnt, plan.kidx)


@pytest.mark.parametrize("bp", TIERS)
@pytest.mark.parametrize("name", list(SMALL))
def test_three_phase_attention_within_tolerance(name, bp):
    B, H, d, F, Hv, Wv = SMALL[name]
    bp16, bp8, bp4 = bp
    res = gpu_run(B, H, d, F, Hv, Wv, bp8, bp4, bp16=bp16)
    q, k, v = inputs(B, H, d, F, Hv, Wv)
    _, _, _, ref = O.run(q, k, v, F, Hv, Wv, bp8, bp4, 0.2, bp16=bp16)
    r16 = bf16_round(ref)
    err, mx = rel_l2(res["out"], r16), np.abs(res["out"] - r16).max()
    assert err <= REL_L2 and mx <= MAX_ABS, (err, mx)


def test_16_bit_plan_without_bf16_operands_is_reported():
    B, H, d, F, Hv, Wv = SMALL["tiny"]
    q, k, v = (t.cuda() for t in inputs(B, H, d, F, Hv, Wv))
    m = da2.DA2(B, H, d, F, Hv, Wv)
    prep = m.alloc_prepared(with16=False)
    plan = m.alloc_plan(budget=(1000, 1000, False, 1000))
    out = torch.empty_like(q)
    m.prepare(q, k, v, prep)
    m.plan(prep, plan, 1000, 1000, bp16=1000)
    m.attention(prep, plan, out)
    torch.cuda.synchronize()
    assert m.status() == da2.ERR_ARG
    m.close()
