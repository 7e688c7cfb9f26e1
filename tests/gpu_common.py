"""Shared helpers of the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import functools

import numpy as np
import torch

from oracle import oracle as O
from video_dit_sparse_da2_b200 import da2, layouts
from video_dit_sparse_da2_b200.inputs import make_qkv

# (name, B, H, d, F, Hv, Wv) -- small shapes that span several tiles and have
# ragged regions, an odd number of blocks and both head dims.
SMALL = {
    "tiny": (1, 2, 64, 4, 16, 16),
    "ragged128": (2, 3, 128, 3, 9, 13),
    "ragged64": (1, 3, 64, 5, 11, 10),
    "oddR128": (1, 2, 128, 7, 8, 8),
}


def rel_l2(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    den = np.linalg.norm(y)
    return np.linalg.norm(x - y) / (den if den > 0 else 1.0)


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


@functools.lru_cache(maxsize=16)
def inputs(B, H, d, F, Hv, Wv, seed=0):
    return make_qkv(B, H, F * Hv * Wv, d, seed)


def gpu_run(B, H, d, F, Hv, Wv, bp8, bp4, lam=0.2, seed=0, qkv=None, per_row=False, bp16=0, int8_qk=False):
    q, k, v = qkv if qkv is not None else inputs(B, H, d, F, Hv, Wv, seed)
    m = da2.DA2(B, H, d, F, Hv, Wv)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, prep, plan = m.forward(qd, kd, vd, bp8, bp4, lam, per_row=per_row, bp16=bp16, int8_qk=int8_qk)
    torch.cuda.synchronize()
    m.check_status()
    res = {
        "out": out.float().cpu().double().numpy(),
        "prep": layouts.prepared_to_logical(prep.bufs, B, H, m.R, d),
        "plan": layouts.plan_to_logical(plan.bufs, B, H, m.R),
    }
    m.close()
    return res


def expected_compact_lists(cnt: np.ndarray, kidx: np.ndarray):
    """The compact list layout of include/da2.h built from the oracle's per-row
    counts cnt[2,B,H,R] and fixed-stride lists kidx[B,H,R,R]: offsets
    off[B,H,R+1] (head (b,h) starts at (b*H+h)*K, K = pairs a head keeps) and
    the concatenated lists.  Pure re-layout, no arithmetic of the method."""
    _, B, H, R = cnt.shape
    n = cnt.sum(axis=0).astype(np.int64)
    per_head = n.sum(axis=-1)
    K = int(per_head.flat[0]) if per_head.size else 0
    assert np.all(per_head == K), "every head keeps the same number of pairs"
    off = np.zeros((B, H, R + 1), np.int64)
    flat = []
    for b in range(B):
        for h in range(H):
            off[b, h, 0] = (b * H + h) * K
            off[b, h, 1:] = off[b, h, 0] + np.cumsum(n[b, h])
            for a in range(R):
                flat.append(kidx[b, h, a, : n[b, h, a]])
    return off, (np.concatenate(flat).astype(np.uint16) if flat else np.zeros(0, np.uint16))


def check_compact_lists(got_plan: dict, cnt: np.ndarray, kidx: np.ndarray):
    """Offsets and compact lists of a device plan equal the oracle's, bit for bit."""
    off, flat = expected_compact_lists(cnt, kidx)
    assert np.array_equal(got_plan["off"], off), "list offsets"
    assert np.array_equal(got_plan["kidx_flat"][: flat.size], flat), "compact lists"
