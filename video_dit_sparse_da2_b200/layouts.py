"""Decoders from the device layouts of include/da2.h to plain logical arrays.

Host-side inspection helpers (numpy) for tests and debugging: they reorder
bytes, they compute nothing of the method.
"""
from __future__ import annotations

import numpy as np


def untile_kmajor(buf: np.ndarray, rows: int, row_bytes: int) -> np.ndarray:
    """[..., rows*row_bytes] K-major no-swizzle tiles -> [..., rows, row_bytes].

    Byte (r, c) sits at ((r//8)*(row_bytes//16) + c//16)*128 + (r%8)*16 + c%16."""
    lead = buf.shape[:-1]
    t = buf.reshape(*lead, rows // 8, row_bytes // 16, 8, 16)
    t = np.swapaxes(t, -3, -2)  # [..., rows/8, 8, row_bytes/16, 16]
    return t.reshape(*lead, rows, row_bytes)


def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    """[..., n] bytes -> [..., 2n] e2m1 codes (low nibble first)."""
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def sfk_atoms_to_logical(atoms: np.ndarray, d: int) -> np.ndarray:
    """[..., 512] K scale atoms -> [..., 64, d/16] (key slot, channel group)."""
    out = np.zeros(atoms.shape[:-1] + (64, d // 16), np.uint8)
    for n in range(64):
        for g in range(d // 16):
            c = 16 * g
            out[..., n, g] = atoms[..., 16 * (n % 32) + 4 * (2 * (c // 64) + n // 32) + (c % 64) // 16]
    return out


def sfv_atoms_to_logical(atoms: np.ndarray, d: int) -> np.ndarray:
    """[..., 512] V^T scale atoms -> [..., d, 4] (channel, slot group)."""
    out = np.zeros(atoms.shape[:-1] + (d, 4), np.uint8)
    for c in range(d):
        for j in range(4):
            out[..., c, j] = atoms[..., 16 * (c % 32) + 4 * (c // 32) + j]
    return out


def prepared_to_logical(bufs: dict, B: int, H: int, R: int, d: int) -> dict:
    """Device prepared operands (uint8 tensors) -> the oracle's logical arrays."""
    g = {k: v.cpu().numpy() for k, v in bufs.items()}
    BH = B * H
    out = {}
    out["desc"] = g["desc"][: 4 * BH * R * d * 8].view(np.float64).reshape(4, B, H, R, d)
    out["q8"] = untile_kmajor(g["q8"].reshape(B, H, R, 64 * d), 64, d)
    out["k8"] = untile_kmajor(g["k8"].reshape(B, H, R, 64 * d), 64, d)
    out["v8t"] = untile_kmajor(g["v8"].reshape(B, H, R, 64 * d), d, 64)
    out["q4"] = unpack_nibbles(untile_kmajor(g["q4"].reshape(B, H, R, 32 * d), 64, d // 2))
    out["k4"] = unpack_nibbles(untile_kmajor(g["k4"].reshape(B, H, R, 32 * d), 64, d // 2))
    out["v4t"] = unpack_nibbles(untile_kmajor(g["v4"].reshape(B, H, R, 32 * d), d, 32))
    out["sfq"] = g["sfq"][: BH * R * 64 * (d // 16)].reshape(B, H, R, 64, d // 16)
    out["sfk"] = sfk_atoms_to_logical(g["sfk"][: BH * R * 512].reshape(B, H, R, 512), d)
    out["sfv"] = sfv_atoms_to_logical(g["sfv"][: BH * R * 512].reshape(B, H, R, 512), d)
    sc = g["scale"][: 6 * BH * R * 4].view(np.float32).reshape(6, B, H, R)
    out["s8"], out["g4"] = sc[:3], sc[3:]
    out["vmax"] = g["vmax"][: 2 * BH * 4].view(np.float32).reshape(2, B, H)
    if "q8i" in g:
        out["q8i"] = untile_kmajor(g["q8i"].reshape(B, H, R, 64 * d), 64, d).view(np.int8)
        out["k8i"] = untile_kmajor(g["k8i"].reshape(B, H, R, 64 * d), 64, d).view(np.int8)
        out["si8"] = g["si8"][: 2 * BH * R * 4].view(np.float32).reshape(2, B, H, R)
    if "q16" in g:
        # bf16 tiles of the 16-bit path, as uint16 bit patterns
        def untile16(buf, rows, row_bytes):
            return np.ascontiguousarray(untile_kmajor(buf.reshape(B, H, R, rows * row_bytes), rows,
                                                      row_bytes)).view(np.uint16)
        out["q16"] = untile16(g["q16"], 64, 2 * d)
        out["k16"] = untile16(g["k16"], 64, 2 * d)
        out["v16t"] = untile16(g["v16"], d, 128)
    return out


def plan_to_logical(bufs: dict, B: int, H: int, R: int, Rv: int = None) -> dict:
    """Device plan buffers -> logical arrays; the compact lists are unpacked
    into fixed-stride rows kidx[B,H,R,R] (entries past a row's count are 0).
    R counts every block, Rv the video blocks (prec and A; default R)."""
    Rv = R if Rv is None else Rv
    g = {k: v.cpu().numpy() for k, v in bufs.items() if k != "scratch"}
    BH = B * H
    off = g["off"][: BH * (R + 1) * 8].view(np.int64).reshape(B, H, R + 1)
    flat = g["kidx"].view(np.uint16)
    kidx = np.zeros((B, H, R, R), np.uint16)
    for b in range(B):
        for h in range(H):
            for a in range(R):
                lo, hi = int(off[b, h, a]), int(off[b, h, a + 1])
                kidx[b, h, a, : hi - lo] = flat[lo:hi]
    return {
        "prec": g["prec"][: BH * Rv * Rv].reshape(B, H, Rv, Rv),
        "cnt": g["cnt"][: 2 * BH * R * 4].view(np.int32).reshape(2, B, H, R),
        "cnt16": g["cnt"][2 * BH * R * 4: 3 * BH * R * 4].view(np.int32).reshape(B, H, R),
        "off": off,
        "kidx": kidx,
        "kidx_flat": flat,
        "A": g["A"][: BH * Rv * Rv * 8].view(np.float64).reshape(B, H, Rv, Rv),
    }
