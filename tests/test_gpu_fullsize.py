"""GPU parity at the full sizes of the five workloads, in the launch
configuration the benchmark times: prepared operands, draft map, precision
map and lists bit for bit on every head; the attention output on a seeded
sample of query blocks (all heads), which the oracle computes block by block.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.gpu_common import bf16_round, check_compact_lists, rel_l2
from video_dit_sparse_da2_b200 import da2, layouts
from video_dit_sparse_da2_b200.inputs import ALL, workload_qkv

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS = 1e-2
# query blocks checked per head: 16 on the two largest workloads (among them
# each head's block with the longest list), 3 on the others
BLOCKS_PER_HEAD = {"hunyuanvideo-720p": 16, "cogvideox": 16}

FULL = [w for w in ALL if w.name != "tiny"]


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_parity(w):
    q, k, v = workload_qkv(w, seed=0)
    m = da2.DA2(w.B, w.H, w.d, w.F, w.Hv, w.Wv)
    out, prep, plan = m.forward(q.cuda(), k.cuda(), v.cuda(), w.bp8, w.bp4, w.lam)
    torch.cuda.synchronize()
    m.check_status()
    R = m.R
    gp = layouts.prepared_to_logical(prep.bufs, w.B, w.H, R, w.d)
    gl = layouts.plan_to_logical(plan.bufs, w.B, w.H, R)
    got = out.float().cpu().double().numpy()
    del out, prep, plan
    torch.cuda.empty_cache()

    ref_prep = O.prepare(q, k, v, w.F, w.Hv, w.Wv)
    for f in ("desc", "q8", "k8", "v8t", "s8", "q4", "k4", "v4t", "sfq", "sfk", "sfv", "g4", "vmax"):
        a, b = gp[f], getattr(ref_prep, f)
        same = np.array_equal(a.view(np.uint8), np.ascontiguousarray(b).view(np.uint8)) if a.dtype.kind == "f" \
            else np.array_equal(a, b)
        assert same, f
    A = O.draft(ref_prep.desc, w.lam)
    assert np.array_equal(gl["A"].view(np.uint64), A.view(np.uint64)), "draft map"
    ref_plan = O.assign(A, w.bp8, w.bp4)
    assert np.array_equal(gl["prec"], ref_plan.prec), "precision map"
    assert np.array_equal(gl["cnt"], ref_plan.cnt), "row counts"
    cnt = ref_plan.cnt[0] + ref_plan.cnt[1]
    ar = np.arange(R)
    listed = ar[None, None, None, :] < cnt[..., None]
    assert np.array_equal(np.where(listed, gl["kidx"], 0), np.where(listed, ref_plan.kidx, 0)), "block lists"
    check_compact_lists(gl, ref_plan.cnt, ref_plan.kidx)

    rng = np.random.default_rng(1)
    nblk = BLOCKS_PER_HEAD.get(w.name, 3)
    sel = np.zeros((w.B, w.H, R), np.uint8)
    for b in range(w.B):
        for h in range(w.H):
            sel[b, h, rng.choice(R, nblk, replace=False)] = 1
            if nblk > 3:
                sel[b, h, int(np.argmax(cnt[b, h]))] = 1  # the longest list of the head
    ref = O.attention(q, k, v, w.F, w.Hv, w.Wv, ref_prep, ref_plan, blocks=sel)
    st, na = m.tables()
    toks = np.concatenate([st[a * 64:a * 64 + na[a]] for a in range(R)])
    # rows of the sampled blocks
    mask = np.zeros((w.B, w.H, w.N), bool)
    for b in range(w.B):
        for h in range(w.H):
            for a in np.nonzero(sel[b, h])[0]:
                mask[b, h, st[a * 64:a * 64 + na[a]]] = True
    r16 = bf16_round(ref[mask])
    g = got[mask]
    err, mx = rel_l2(g, r16), np.abs(g - r16).max()
    m.close()
    assert err <= REL_L2 and mx <= MAX_ABS, (err, mx)
