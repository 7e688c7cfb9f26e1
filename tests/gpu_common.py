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


def gpu_run(B, H, d, F, Hv, Wv, bp8, bp4, lam=0.2, seed=0, qkv=None, per_row=False):
    q, k, v = qkv if qkv is not None else inputs(B, H, d, F, Hv, Wv, seed)
    m = da2.DA2(B, H, d, F, Hv, Wv)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, prep, plan = m.forward(qd, kd, vd, bp8, bp4, lam, per_row=per_row)
    torch.cuda.synchronize()
    m.check_status()
    res = {
        "out": out.float().cpu().double().numpy(),
        "prep": layouts.prepared_to_logical(prep.bufs, B, H, m.R, d),
        "plan": layouts.plan_to_logical(plan.bufs, B, H, m.R),
    }
    m.close()
    return res
