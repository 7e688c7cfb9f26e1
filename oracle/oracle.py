"""ctypes wrapper around ``da2_oracle.c`` (argument marshalling only).

TEST INFRASTRUCTURE ONLY.  Every arithmetic step lives in the C file, which
cites the passages of "DraftAttention2" it restates.  The shared library is
compiled on first use (or by ``build()``) with gcc, OpenMP and
``-ffp-contract=off``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "da2_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")
BLOCK = 64


def build(force: bool = False) -> str:
    """Compile the oracle shared library if it is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_exp.restype = ctypes.c_double
        L.oracle_exp.argtypes = [ctypes.c_double]
        L.oracle_partition.argtypes = [i, i, i, P, P, P]
        L.oracle_slot_tokens.argtypes = [i, i, i, P, P]
        L.oracle_prepare.argtypes = [i] * 6 + [P] * 3 + [P] * 13
        L.oracle_draft.argtypes = [i, i, i, P, ctypes.c_double, P]
        L.oracle_assign.argtypes = [i, i, P, i, i, P, P, P]
        L.oracle_assign_rows.argtypes = [i, i, P, i, i, P, P, P]
        L.oracle_assign_tiers.argtypes = [i, i, P, i, i, i, i, P, P, P]
        L.oracle_attention_tiers.argtypes = [i] * 6 + [P] * 3 + [P] * 14 + [i, P, P]
        L.oracle_int8_encode.restype = ctypes.c_int8
        L.oracle_int8_encode.argtypes = [ctypes.c_float]
        L.oracle_prepare_int8.argtypes = [i] * 6 + [P] * 5
        L.oracle_prepare_int8_p.argtypes = [i] * 7 + [P] * 5
        L.oracle_prepare_p.argtypes = [i] * 7 + [P] * 3 + [P] * 13
        L.oracle_slot_tokens_p.argtypes = [i, i, i, i, P, P]
        L.oracle_prefix_plan.argtypes = [i, i, i, P, P, P, P]
        L.oracle_attention_p.argtypes = [i] * 7 + [P] * 3 + [P] * 14 + [i, P, P, P, P, P]
        L.oracle_attention_int8.argtypes = [i] * 6 + [P] * 3 + [P] * 13 + [i, P, i, P, P, P, P, P]
        L.oracle_bf16_round.restype = ctypes.c_double
        L.oracle_bf16_round.argtypes = [ctypes.c_double]
        L.oracle_attention.argtypes = [i] * 6 + [P] * 3 + [P] * 14 + [i, P, P]
        L.oracle_dense.argtypes = [i, i, i, P, P, P, P]
        L.oracle_num_threads.restype = i
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def e4m3_encode(x: float) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def e4m3_decode(c: int) -> float:
    return float(lib().oracle_e4m3_decode(int(c)))


def e2m1_encode(x: float) -> int:
    return int(lib().oracle_e2m1_encode(float(x)))


def e2m1_decode(c: int) -> float:
    return float(lib().oracle_e2m1_decode(int(c)))


def int8_encode(x: float) -> int:
    return int(lib().oracle_int8_encode(float(x)))


def prepare_int8(q, k, F: int, Hv: int, Wv: int, P: int = 0):
    """INT8 tiles of Q and K (s8 [B,H,R,64,d] each) and their tile scales f32 [2,B,H,R]."""
    qb, kb = _bits(q), _bits(k)
    B, H, N, d = qb.shape
    R = F * (-(-(Hv * Wv) // BLOCK)) + -(-P // BLOCK)
    q8i = np.zeros((B, H, R, BLOCK, d), np.int8)
    k8i = np.zeros((B, H, R, BLOCK, d), np.int8)
    si8 = np.zeros((2, B, H, R), np.float32)
    if lib().oracle_prepare_int8_p(B, H, d, F, Hv, Wv, int(P), _p(qb), _p(kb), _p(q8i), _p(k8i), _p(si8)):
        raise ValueError("oracle_prepare_int8 failed")
    return q8i, k8i, si8


def bf16_round(x: float) -> float:
    return float(lib().oracle_bf16_round(float(x)))


def exp(x: float) -> float:
    return float(lib().oracle_exp(float(x)))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def partition(Hv: int, Wv: int, C: int = BLOCK):
    """Region index and in-region slot of every cell of an Hv x Wv frame (row-major)."""
    n = Hv * Wv
    region_of = np.zeros(n, np.int32)
    slot_of = np.zeros(n, np.int32)
    n_a = np.zeros(n, np.int32)
    Rf = lib().oracle_partition(Hv, Wv, C, _p(region_of), _p(slot_of), _p(n_a))
    if Rf <= 0:
        raise ValueError("bad partition arguments")
    return region_of, slot_of, n_a[:Rf].copy()


def slot_tokens(F: int, Hv: int, Wv: int, P: int = 0):
    """Token index held by each packed slot (-1 = padding) and valid counts per
    block; with P prefix tokens the prefix blocks follow the video blocks."""
    n = Hv * Wv
    Rf = -(-n // BLOCK)
    R = F * Rf + -(-P // BLOCK)
    st = np.zeros(R * BLOCK, np.int32)
    na = np.zeros(R, np.int32)
    if lib().oracle_slot_tokens_p(F, Hv, Wv, int(P), _p(st), _p(na)) != R:
        raise ValueError("bad shape")
    return st, na


@dataclass
class Prepared:
    desc: np.ndarray   # f64 [4,B,H,R,d]  Qbar, Qmax, Kbar, Kmax
    q8: np.ndarray     # u8 [B,H,R,64,d]
    k8: np.ndarray
    v8t: np.ndarray    # u8 [B,H,R,d,64]
    s8: np.ndarray     # f32 [3,B,H,R]
    q4: np.ndarray     # u8 [B,H,R,64,d] one e2m1 code per byte
    k4: np.ndarray
    v4t: np.ndarray    # u8 [B,H,R,d,64]
    sfq: np.ndarray    # u8 [B,H,R,64,d/16]
    sfk: np.ndarray
    sfv: np.ndarray    # u8 [B,H,R,d,4]
    g4: np.ndarray     # f32 [3,B,H,R]
    vmax: np.ndarray   # f32 [2,B,H]


def _bits(x) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16
    return x


def prepare(q, k, v, F: int, Hv: int, Wv: int, P: int = 0) -> Prepared:
    """Prepared operands of every block: the video blocks, then (P > 0) the
    prefix blocks."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, N, d = qb.shape
    R = F * (-(-(Hv * Wv) // BLOCK)) + -(-P // BLOCK)
    assert N == P + F * Hv * Wv
    out = Prepared(
        desc=np.zeros((4, B, H, R, d), np.float64),
        q8=np.zeros((B, H, R, BLOCK, d), np.uint8), k8=np.zeros((B, H, R, BLOCK, d), np.uint8),
        v8t=np.zeros((B, H, R, d, BLOCK), np.uint8), s8=np.zeros((3, B, H, R), np.float32),
        q4=np.zeros((B, H, R, BLOCK, d), np.uint8), k4=np.zeros((B, H, R, BLOCK, d), np.uint8),
        v4t=np.zeros((B, H, R, d, BLOCK), np.uint8),
        sfq=np.zeros((B, H, R, BLOCK, d // 16), np.uint8), sfk=np.zeros((B, H, R, BLOCK, d // 16), np.uint8),
        sfv=np.zeros((B, H, R, d, 4), np.uint8), g4=np.zeros((3, B, H, R), np.float32),
        vmax=np.zeros((2, B, H), np.float32))
    rc = lib().oracle_prepare_p(B, H, d, F, Hv, Wv, int(P), _p(qb), _p(kb), _p(vb), _p(out.desc), _p(out.q8), _p(out.k8),
                              _p(out.v8t), _p(out.s8), _p(out.q4), _p(out.k4), _p(out.v4t), _p(out.sfq),
                              _p(out.sfk), _p(out.sfv), _p(out.g4), _p(out.vmax))
    if rc:
        raise ValueError("oracle_prepare failed")
    return out


def draft(desc: np.ndarray, lam: float = 0.2) -> np.ndarray:
    """Draft map A, f64 [B,H,R,R]."""
    desc = np.ascontiguousarray(desc, np.float64)
    _, B, H, R, d = desc.shape
    A = np.zeros((B, H, R, R), np.float64)
    lib().oracle_draft(B * H, R, d, _p(desc), float(lam), _p(A))
    return A


@dataclass
class Plan:
    prec: np.ndarray   # u8 [B,H,R,R] in {0,4,8} (and 16 with the 16-bit tier)
    cnt: np.ndarray    # i32 [2,B,H,R] (8-bit, 4-bit) or [3,B,H,R] (8-bit, 4-bit, 16-bit) kept blocks per row
    kidx: np.ndarray   # u16 [B,H,R,R] row a: (16-bit blocks asc,) 8-bit blocks asc, then 4-bit blocks asc


def assign(A: np.ndarray, bp8: int, bp4: int, per_row: bool = False, bp16: int = 0) -> Plan:
    """Precision of every pair: ranking of all R^2 pairs of a head (the pages),
    or with per_row of the R key blocks of each query block.  With bp16 > 0
    the three-tier assignment (cnt gets a third plane, the 16-bit counts)."""
    A = np.ascontiguousarray(A, np.float64)
    B, H, R, _ = A.shape
    tiers = 3 if bp16 else 2
    plan = Plan(prec=np.zeros((B, H, R, R), np.uint8), cnt=np.zeros((tiers, B, H, R), np.int32),
                kidx=np.zeros((B, H, R, R), np.uint16))
    if bp16:
        rc = lib().oracle_assign_tiers(B * H, R, _p(A), int(bp16), int(bp8), int(bp4), int(bool(per_row)),
                                       _p(plan.prec), _p(plan.cnt), _p(plan.kidx))
    else:
        fn = lib().oracle_assign_rows if per_row else lib().oracle_assign
        rc = fn(B * H, R, _p(A), int(bp8), int(bp4), _p(plan.prec), _p(plan.cnt), _p(plan.kidx))
    if rc:
        raise ValueError("bad budget")
    return plan


def prefix_plan(plan: Plan, Rp: int) -> Plan:
    """The plan over the video and the Rp prefix blocks (App. C.1 prefix rule,
    reading in da2_oracle.c item 4d) from a three-plane video plan."""
    assert plan.cnt.shape[0] == 3, "needs the three-tier plan (assign with bp16, or tiers_plan)"
    _, B, H, Rv = plan.cnt.shape
    Rt = Rv + Rp
    out = Plan(prec=plan.prec, cnt=np.zeros((3, B, H, Rt), np.int32), kidx=np.zeros((B, H, Rt, Rt), np.uint16))
    if lib().oracle_prefix_plan(B * H, Rv, Rp, _p(np.ascontiguousarray(plan.cnt)),
                                _p(np.ascontiguousarray(plan.kidx)), _p(out.cnt), _p(out.kidx)):
        raise ValueError("oracle_prefix_plan failed")
    return out


def tiers_plan(A: np.ndarray, bp8: int, bp4: int, per_row: bool = False, bp16: int = 0) -> Plan:
    """The three-plane (three-tier) plan, also when bp16 = 0."""
    A = np.ascontiguousarray(A, np.float64)
    B, H, R, _ = A.shape
    plan = Plan(prec=np.zeros((B, H, R, R), np.uint8), cnt=np.zeros((3, B, H, R), np.int32),
                kidx=np.zeros((B, H, R, R), np.uint16))
    if lib().oracle_assign_tiers(B * H, R, _p(A), int(bp16), int(bp8), int(bp4), int(bool(per_row)),
                                 _p(plan.prec), _p(plan.cnt), _p(plan.kidx)):
        raise ValueError("bad budget")
    return plan


def attention_prefix(q, k, v, F, Hv, Wv, P, prep: Prepared, plan: Plan, flags: int = 7, blocks=None,
                     int8=None) -> np.ndarray:
    """Attention with P prefix tokens (plan from prefix_plan), f64 [B,H,N,d]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, N, d = qb.shape
    out = np.zeros((B, H, N, d), np.float64)
    sel = None if blocks is None else np.ascontiguousarray(blocks, np.uint8)
    q8i, k8i, si8 = (None, None, None) if int8 is None else (np.ascontiguousarray(x) for x in int8)
    rc = lib().oracle_attention_p(B, H, d, F, Hv, Wv, int(P), _p(qb), _p(kb), _p(vb), _p(prep.q8), _p(prep.k8),
                                  _p(prep.v8t), _p(prep.s8), _p(prep.q4), _p(prep.k4), _p(prep.v4t),
                                  _p(prep.sfq), _p(prep.sfk), _p(prep.sfv), _p(prep.g4), _p(prep.vmax),
                                  _p(plan.cnt), _p(plan.kidx), int(flags), None if sel is None else _p(sel),
                                  None if q8i is None else _p(q8i), None if k8i is None else _p(k8i),
                                  None if si8 is None else _p(si8), _p(out))
    if rc:
        raise ValueError(f"oracle_attention_p failed ({rc})")
    return out


def run_prefix(q, k, v, F, Hv, Wv, P, bp8, bp4, lam=0.2, flags=7, per_row=False, bp16=0, int8=False):
    """Whole pipeline with P prefix tokens: prepare (all blocks) -> draft and
    assign over the video blocks -> prefix plan -> attention."""
    prep = prepare(q, k, v, F, Hv, Wv, P)
    Rv = F * (-(-(Hv * Wv) // BLOCK))
    A = draft(np.ascontiguousarray(prep.desc[:, :, :, :Rv]), lam)
    plan = prefix_plan(tiers_plan(A, bp8, bp4, per_row, bp16), -(-P // BLOCK))
    i8 = prepare_int8(q, k, F, Hv, Wv, P) if int8 else None
    out = attention_prefix(q, k, v, F, Hv, Wv, P, prep, plan, flags, int8=i8)
    return prep, A, plan, out


def attention(q, k, v, F, Hv, Wv, prep: Prepared, plan: Plan, flags: int = 7, blocks=None, int8=None) -> np.ndarray:
    """Block-sparse mixed-precision attention, f64 [B,H,N,d] in token order.

    blocks: optional boolean [B,H,R] selecting the query blocks to compute
    (the other tokens stay 0).  int8: optional (q8i, k8i, si8) of
    prepare_int8, for the 8-bit phase's QK^T in INT8."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, N, d = qb.shape
    out = np.zeros((B, H, N, d), np.float64)
    sel = None if blocks is None else np.ascontiguousarray(blocks, np.uint8)
    if int8 is not None:
        q8i, k8i, si8 = (np.ascontiguousarray(x) for x in int8)
        rc = lib().oracle_attention_int8(B, H, d, F, Hv, Wv, _p(qb), _p(kb), _p(vb), _p(prep.q8), _p(prep.k8),
                                         _p(prep.v8t), _p(prep.s8), _p(prep.q4), _p(prep.k4), _p(prep.v4t),
                                         _p(prep.sfq), _p(prep.sfk), _p(prep.sfv), _p(prep.g4), _p(prep.vmax),
                                         _p(plan.cnt), int(plan.cnt.shape[0]), _p(plan.kidx), int(flags),
                                         None if sel is None else _p(sel), _p(q8i), _p(k8i), _p(si8), _p(out))
        if rc:
            raise ValueError(f"oracle_attention_int8 failed ({rc})")
        return out
    fn = lib().oracle_attention_tiers if plan.cnt.shape[0] == 3 else lib().oracle_attention
    rc = fn(B, H, d, F, Hv, Wv, _p(qb), _p(kb), _p(vb), _p(prep.q8), _p(prep.k8),
                                _p(prep.v8t), _p(prep.s8), _p(prep.q4), _p(prep.k4), _p(prep.v4t),
                                _p(prep.sfq), _p(prep.sfk), _p(prep.sfv), _p(prep.g4), _p(prep.vmax),
                                _p(plan.cnt), _p(plan.kidx), int(flags),
                                None if sel is None else _p(sel), _p(out))
    if rc:
        raise ValueError(f"oracle_attention failed ({rc})")
    return out


def dense(q, k, v) -> np.ndarray:
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, N, d = qb.shape
    out = np.zeros((B, H, N, d), np.float64)
    lib().oracle_dense(B * H, N, d, _p(qb), _p(kb), _p(vb), _p(out))
    return out


def run(q, k, v, F, Hv, Wv, bp8, bp4, lam=0.2, flags=7, per_row=False, bp16=0, int8=False):
    """Whole pipeline: prepare -> draft -> assign -> attention (int8: the
    8-bit phase's QK^T in INT8)."""
    prep = prepare(q, k, v, F, Hv, Wv)
    A = draft(prep.desc, lam)
    plan = assign(A, bp8, bp4, per_row, bp16)
    out = attention(q, k, v, F, Hv, Wv, prep, plan, flags, int8=prepare_int8(q, k, F, Hv, Wv) if int8 else None)
    return prep, A, plan, out
