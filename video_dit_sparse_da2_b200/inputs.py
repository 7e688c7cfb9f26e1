"""Seeded synthetic inputs shaped like video-DiT attention operands.

This module holds no arithmetic of the method: it only draws random numbers
and names the workloads.  Both the CUDA path's tests and the oracle's tests
use it, so that both sides see the same bf16 tensors.

Recipe: Q, K, V ~ i.i.d. N(0, 1), drawn in float32 with a CPU
``torch.Generator`` seeded with ``seed``, in the order Q, K, V, each of
shape [B, H, N, d], then rounded to bf16 (round to nearest even).

Second, structured set (``make_qkv_structured``, seed 1): the same i.i.d.
draw, then Q and K (video tokens only) get an added smooth per-frame field,
x += 2 f(frame, y/Hv, x/Wv), where per (batch, head, channel) f is half the sum
of 4 cosines of low spatial frequency (integer wave numbers 0..2 along each
axis, random phase) whose phases drift slowly from frame to frame; the draft
map of such inputs is far from uniform, like that of video latents.
"""
from __future__ import annotations

import math
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


def make_qkv_structured(B: int, H: int, d: int, F: int, Hv: int, Wv: int, P: int = 0, seed: int = 1):
    """bf16 Q, K, V of shape [B, H, P + F*Hv*Wv, d] on the CPU: the second,
    structured input set of the module docstring."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    N = P + F * Hv * Wv
    qkv = [torch.randn((B, H, N, d), generator=g, dtype=torch.float32) for _ in range(3)]
    xx = (torch.arange(Wv, dtype=torch.float32) / Wv).view(1, 1, 1, Wv)
    yy = (torch.arange(Hv, dtype=torch.float32) / Hv).view(1, 1, Hv, 1)
    for t in qkv[:2]:
        kx = torch.randint(0, 3, (B, H, 4, d), generator=g).float()
        ky = torch.randint(0, 3, (B, H, 4, d), generator=g).float()
        ph = torch.rand((B, H, 4, d), generator=g) * (2 * math.pi)
        dr = (torch.rand((B, H, 4, d), generator=g) - 0.5) * 0.2
        for b in range(B):
            for h in range(H):
                # spatial phase [4, d, Hv, Wv]
                sp = 2 * math.pi * (kx[b, h, :, :, None, None] * xx + ky[b, h, :, :, None, None] * yy) \
                    + ph[b, h, :, :, None, None]
                for f in range(F):
                    field = 0.5 * torch.cos(sp + dr[b, h, :, :, None, None] * f).sum(0)  # [d, Hv, Wv]
                    t[b, h, P + f * Hv * Wv:P + (f + 1) * Hv * Wv, :] += 2.0 * field.reshape(d, Hv * Wv).T
    return tuple(x.to(torch.bfloat16) for x in qkv)


def workload_qkv(w: Workload, seed: int = 0, structured: bool = False):
    if structured:
        return make_qkv_structured(w.B, w.H, w.d, w.F, w.Hv, w.Wv, w.P, seed)
    return make_qkv(w.B, w.H, w.N, w.d, seed)
