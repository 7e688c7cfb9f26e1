"""Seeded synthetic inputs shaped like video-DiT attention operands.

This module holds no arithmetic of the method: it only draws random numbers
and names the workloads.  Both the CUDA path's tests and the oracle's tests
use it, so that both sides see the same bf16 tensors.

Recipe: Q, K, V ~ i.i.d. N(0, 1), drawn in float32 with a CPU
``torch.Generator`` seeded with ``seed``, in the order Q, K, V, each of
shape [B, H, N, d], then rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    F: int
    Hv: int
    Wv: int
    bp8: int   # basis points of the R^2 region pairs of a head kept in FP8
    bp4: int   # basis points kept in NVFP4; the rest are skipped
    lam: float = 0.2
    P: int = 0  # prefix (text) tokens before the video tokens

    @property
    def N(self) -> int:
        return self.P + self.F * self.Hv * self.Wv


# The five workload shapes (video latent geometry, head count and dim, budgets).
TINY = Workload("tiny", 1, 2, 64, 4, 16, 16, 2500, 2500)
WAN13B = Workload("wan2.1-1.3b-480p", 1, 12, 128, 21, 30, 52, 1000, 3000)
COGVIDEOX = Workload("cogvideox", 1, 48, 64, 13, 60, 90, 1500, 3500)
HUNYUAN = Workload("hunyuanvideo-720p", 1, 24, 128, 33, 45, 80, 500, 2500)


def wan14b(bp4: int) -> Workload:
    return Workload(f"wan2.1-14b-720p-fp4-{bp4 // 100}", 1, 40, 128, 21, 45, 80, 1000, bp4)


WAN14B_SWEEP = [wan14b(b) for b in (0, 2000, 4000, 6000)]
ALL = [TINY, WAN13B, COGVIDEOX, HUNYUAN] + WAN14B_SWEEP
# Shaped like the captured video-attention input of the pages' error analysis
# (N = 109,376 tokens, 56 heads, d = 128, average-only draft guidance).  The
# pages give no frame geometry: 256 prefix tokens + 31 frames of 44 x 80 is a
# synthetic geometry with that token count.  Budgets: 10 / 30 / 60 %.
CAPTURE = Workload("capture-shaped-109k", 1, 56, 128, 31, 44, 80, 1000, 3000, lam=0.0, P=256)
BY_NAME = {w.name: w for w in ALL + [CAPTURE]}


def make_qkv(B: int, H: int, N: int, d: int, seed: int = 0):
    """bf16 Q, K, V of shape [B, H, N, d] on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out = []
    for _ in range(3):
        out.append(torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16))
    return tuple(out)


def workload_qkv(w: Workload, seed: int = 0):
    return make_qkv(w.B, w.H, w.N, w.d, seed)
