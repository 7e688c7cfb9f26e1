"""GPU parity of the prefix (text) tokens (DraftAttention2 App. C.1: the budget
covers video-region pairs only; every video query block also sees every valid
prefix key and every prefix query sees all keys): slot tables, the plan
(precision map of the video pairs, counts, offsets and lists over every block)
bit for bit, and the attention within the output tolerance of the oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import bf16_round, check_compact_lists, rel_l2
from video_dit_sparse_da2_b200 import da2, layouts
from video_dit_sparse_da2_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

SHAPES = {"tiny": (1, 2, 64, 4, 16, 16), "ragged128": (2, 3, 128, 3, 9, 13)}
CASES = [(100, (1500, 2500, 1000)), (1, (1000, 2000, 0)), (64, (2500, 2500, 0)), (200, (0, 3000, 2000))]


def _run(name, P, bp, int8_qk=False):
    B, H, d, F, Hv, Wv = SHAPES[name]
    bp8, bp4, bp16 = bp
    q, k, v = make_qkv(B, H, P + F * Hv * Wv, d, seed=5)
    m = da2.DA2(B, H, d, F, Hv, Wv, P)
    out, prep, plan = m.forward(q.cuda(), k.cuda(), v.cuda(), bp8, bp4, 0.2, bp16=bp16, int8_qk=int8_qk)
    torch.cuda.synchronize()
    m.check_status()
    got = {"out": out.double().cpu().numpy(), "plan": layouts.plan_to_logical(plan.bufs, B, H, m.R, m.Rv),
           "tables": m.tables(), "R": m.R, "Rv": m.Rv}
    m.close()
    return (q, k, v), got


@pytest.mark.parametrize("P", [1, 64, 100, 200])
def test_prefix_slot_tables(P):
    B, H, d, F, Hv, Wv = SHAPES["ragged128"]
    m = da2.DA2(B, H, d, F, Hv, Wv, P)
    st, na = m.tables()
    ost, ona = O.slot_tokens(F, Hv, Wv, P)
    assert np.array_equal(st, ost) and np.array_equal(na, ona)
    m.close()


@pytest.mark.parametrize("P,bp", CASES)
@pytest.mark.parametrize("name", list(SHAPES))
def test_prefix_plan_bit_exact(name, P, bp):
    B, H, d, F, Hv, Wv = SHAPES[name]
    bp8, bp4, bp16 = bp
    (q, k, v), got = _run(name, P, bp)
    prep = O.prepare(q, k, v, F, Hv, Wv, P)
    Rv = got["Rv"]
    A = O.draft(np.ascontiguousarray(prep.desc[:, :, :, :Rv]), 0.2)
    video = O.tiers_plan(A, bp8, bp4, bp16=bp16)
    plan = O.prefix_plan(video, got["R"] - Rv)
    g = got["plan"]
    assert np.array_equal(g["A"].view(np.uint64), A.view(np.uint64))
    assert np.array_equal(g["prec"], video.prec)
    assert np.array_equal(g["cnt"], plan.cnt[:2]) and np.array_equal(g["cnt16"], plan.cnt[2])
    check_compact_lists(g, plan.cnt, plan.kidx)


@pytest.mark.parametrize("int8_qk", [False, True], ids=["fp8-qk", "int8-qk"])
@pytest.mark.parametrize("P,bp", CASES)
@pytest.mark.parametrize("name", list(SHAPES))
def test_prefix_attention_within_tolerance(name, P, bp, int8_qk):
    B, H, d, F, Hv, Wv = SHAPES[name]
    bp8, bp4, bp16 = bp
    (q, k, v), got = _run(name, P, bp, int8_qk)
    _, _, _, ref = O.run_prefix(q, k, v, F, Hv, Wv, P, bp8, bp4, 0.2, bp16=bp16, int8=int8_qk)
    r16 = bf16_round(ref)
    err, mx = rel_l2(got["out"], r16), np.abs(got["out"] - r16).max()
    assert err <= 2e-3 and mx <= 1e-2, (err, mx)


def test_capture_shaped_workload_full_size():
    # full size, in the configuration the benchmark runs: the plan bit for bit
    # on every head, the output on a seeded sample of query blocks (video and
    # prefix) of every head
    from video_dit_sparse_da2_b200.inputs import CAPTURE as w
    q, k, v = make_qkv(w.B, w.H, w.N, w.d, seed=0)
    m = da2.DA2(w.B, w.H, w.d, w.F, w.Hv, w.Wv, w.P)
    out, prep, plan = m.forward(q.cuda(), k.cuda(), v.cuda(), w.bp8, w.bp4, w.lam)
    torch.cuda.synchronize()
    m.check_status()
    R, Rv = m.R, m.Rv
    g = layouts.plan_to_logical(plan.bufs, w.B, w.H, R, Rv)
    got = out.double().cpu().numpy()
    st, na = m.tables()
    del out, prep, plan
    m.close()
    torch.cuda.empty_cache()
    ref_prep = O.prepare(q, k, v, w.F, w.Hv, w.Wv, w.P)
    A = O.draft(np.ascontiguousarray(ref_prep.desc[:, :, :, :Rv]), w.lam)
    assert np.array_equal(g["A"].view(np.uint64), A.view(np.uint64))
    rplan = O.prefix_plan(O.tiers_plan(A, w.bp8, w.bp4), R - Rv)
    assert np.array_equal(g["prec"], rplan.prec)
    assert np.array_equal(g["cnt"], rplan.cnt[:2]) and np.array_equal(g["cnt16"], rplan.cnt[2])
    check_compact_lists(g, rplan.cnt, rplan.kidx)
    rng = np.random.default_rng(2)
    sel = np.zeros((w.B, w.H, R), np.uint8)
    for h in range(w.H):
        sel[0, h, rng.choice(Rv, 3, replace=False)] = 1
        sel[0, h, Rv + rng.integers(R - Rv)] = 1  # a prefix block
    ref = O.attention_prefix(q, k, v, w.F, w.Hv, w.Wv, w.P, ref_prep, rplan, blocks=sel)
    mask = np.zeros((w.B, w.H, w.N), bool)
    for h in range(w.H):
        for a in np.nonzero(sel[0, h])[0]:
            mask[0, h, st[a * 64:a * 64 + na[a]]] = True
    r16 = bf16_round(ref[mask])
    err, mx = rel_l2(got[mask], r16), np.abs(got[mask] - r16).max()
    assert err <= 2e-3 and mx <= 1e-2, (err, mx)
