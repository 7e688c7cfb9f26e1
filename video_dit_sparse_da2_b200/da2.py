"""Python binding of libda2 (include/da2.h): argument marshalling only.

Every step of the hot path runs in the CUDA kernels behind the C ABI;
PyTorch supplies device memory and streams.  Importing this module loads the
in-tree ``libda2.so`` and raises if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libda2.so")

OK, ERR_ARG, ERR_ARCH, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4

# Every symbol include/da2.h declares.
EXPORTS = ("da2_create", "da2_destroy", "da2_partition", "da2_sizes", "da2_tables", "da2_prepare", "da2_plan",
           "da2_plan_static", "da2_list_bytes", "da2_attention",
           "da2_check_device_status", "da2_set_wait_limit", "da2_selftest_wait_timeout", "da2_status_string",
           "da2_last_cuda_error")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("F", ctypes.c_int),
                ("Hv", ctypes.c_int), ("Wv", ctypes.c_int), ("C", ctypes.c_int), ("P", ctypes.c_int)]


class Budget(ctypes.Structure):
    _fields_ = [("bp_fp8", ctypes.c_int), ("bp_fp4", ctypes.c_int), ("lam", ctypes.c_double),
                ("per_row", ctypes.c_int), ("bp_fp16", ctypes.c_int)]


_SIZE_FIELDS = ("desc", "q8", "k8", "v8", "q4", "k4", "v4", "sfq", "sfk", "sfv", "scale", "vmax",
                "prec", "cnt", "off", "kidx", "A", "plan_scratch", "q16", "k16", "v16", "q8i", "k8i", "si8")


class Sizes(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int), ("Rf", ctypes.c_int), ("Npad", ctypes.c_int)] + \
               [(f, ctypes.c_size_t) for f in _SIZE_FIELDS] + [("Rv", ctypes.c_int), ("Rp", ctypes.c_int)]


_PREP_FIELDS = ("desc", "q8", "k8", "v8", "q4", "k4", "v4", "sfq", "sfk", "sfv", "scale", "vmax")
_PREP16_FIELDS = ("q16", "k16", "v16")  # optional operands of the 16-bit path
_PREPI8_FIELDS = ("q8i", "k8i", "si8")   # optional INT8 operands of the 8-bit phase's QK^T
_PLAN_FIELDS = ("prec", "cnt", "off", "kidx", "A", "scratch")


class PreparedPtrs(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _PREP_FIELDS + _PREP16_FIELDS + _PREPI8_FIELDS]


class PlanPtrs(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _PLAN_FIELDS]


class DA2Error(RuntimeError):
    pass


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libda2 (raises when the CUDA library has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DA2Error(f"CUDA library not built: {LIB_PATH} is missing (run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        L.da2_create.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(P)]
        L.da2_destroy.argtypes = [P]
        L.da2_partition.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.da2_sizes.argtypes = [P, ctypes.POINTER(Sizes)]
        L.da2_tables.argtypes = [P, P, P]
        L.da2_prepare.argtypes = [P, P, P, P, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(PreparedPtrs), P]
        L.da2_plan.argtypes = [P, ctypes.POINTER(PreparedPtrs), ctypes.POINTER(Budget), ctypes.POINTER(PlanPtrs), P]
        L.da2_plan_static.argtypes = [P, ctypes.POINTER(PreparedPtrs), ctypes.POINTER(Budget), P, P, P, P, P, P]
        L.da2_list_bytes.argtypes = [P, ctypes.POINTER(Budget), ctypes.POINTER(ctypes.c_size_t)]
        L.da2_attention.argtypes = [P, ctypes.POINTER(PreparedPtrs), ctypes.POINTER(PlanPtrs), P,
                                    ctypes.POINTER(ctypes.c_int64), P]
        L.da2_check_device_status.argtypes = [P, P]
        L.da2_set_wait_limit.argtypes = [P, ctypes.c_uint64]
        L.da2_selftest_wait_timeout.argtypes = [P, ctypes.c_uint64, P]
        L.da2_status_string.restype = ctypes.c_char_p
        L.da2_status_string.argtypes = [ctypes.c_int]
        L.da2_last_cuda_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != OK:
        msg = lib().da2_status_string(rc).decode()
        if rc == ERR_CUDA:
            msg += ": " + lib().da2_last_cuda_error().decode()
        raise DA2Error(f"{what} failed: {msg} ({rc})")


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _strides(t: torch.Tensor):
    return (ctypes.c_int64 * 4)(*t.stride())


@dataclass
class Prepared:
    """Caller-owned prepared operands (uint8 device tensors, layouts in da2.h)."""
    bufs: dict

    def ptrs(self) -> PreparedPtrs:
        return PreparedPtrs(**{f: (self.bufs[f].data_ptr() if f in self.bufs else None)
                               for f in _PREP_FIELDS + _PREP16_FIELDS + _PREPI8_FIELDS})


@dataclass
class Plan:
    bufs: dict

    def ptrs(self) -> PlanPtrs:
        return PlanPtrs(**{f: self.bufs[f].data_ptr() for f in _PLAN_FIELDS})


def partition(F: int, Hv: int, Wv: int):
    """Host partition of a shape: (slot_token[64 R], n_a[R]) as numpy int32 arrays."""
    import numpy as np
    R = F * (-(-(Hv * Wv) // 64))
    st = np.zeros(64 * R, np.int32)
    na = np.zeros(R, np.int32)
    rc = lib().da2_partition(F, Hv, Wv, st.ctypes.data_as(ctypes.c_void_p), na.ctypes.data_as(ctypes.c_void_p))
    if rc != R:
        _check(rc if rc < 0 else ERR_ARG, "da2_partition")
    return st, na


class DA2:
    """One shape: its partition tables and helpers to run the three steps."""

    def __init__(self, B: int, H: int, d: int, F: int, Hv: int, Wv: int, P: int = 0):
        """P prefix (text) tokens before the F*Hv*Wv video tokens (0 = none)."""
        self.shape = Shape(B, H, d, F, Hv, Wv, 64, P)
        h = ctypes.c_void_p()
        _check(lib().da2_create(ctypes.byref(self.shape), ctypes.byref(h)), "da2_create")
        self.handle = h
        self.sizes = Sizes()
        _check(lib().da2_sizes(h, ctypes.byref(self.sizes)), "da2_sizes")
        self.R, self.Npad = self.sizes.R, self.sizes.Npad
        self.Rv, self.Rp = self.sizes.Rv, self.sizes.Rp

    def close(self):
        if self.handle:
            lib().da2_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def tables(self):
        import numpy as np
        st = np.zeros(self.Npad, np.int32)
        na = np.zeros(self.R, np.int32)
        _check(lib().da2_tables(self.handle, st.ctypes.data_as(ctypes.c_void_p), na.ctypes.data_as(ctypes.c_void_p)),
               "da2_tables")
        return st, na

    def _alloc(self, fields, device, override=None):
        override = override or {}

        def nbytes(f):
            return override.get(f, int(getattr(self.sizes, f if f != "scratch" else "plan_scratch")))
        return {f: torch.empty(max(nbytes(f), 16), dtype=torch.uint8, device=device) for f in fields}

    def list_bytes(self, bp8: int, bp4: int, per_row: bool = False, bp16: int = 0) -> int:
        """Exact byte size of the compact block lists under a budget (da2_list_bytes)."""
        b = Budget(int(bp8), int(bp4), 0.0, int(bool(per_row)), int(bp16))
        n = ctypes.c_size_t()
        _check(lib().da2_list_bytes(self.handle, ctypes.byref(b), ctypes.byref(n)), "da2_list_bytes")
        return int(n.value)

    def alloc_prepared(self, device="cuda", with16: bool = False, int8_qk: bool = False) -> Prepared:
        """Prepared-operand buffers; with16 adds the bf16 tiles of the 16-bit
        path, int8_qk the INT8 Q/K tiles (the 8-bit phase's QK^T in INT8)."""
        fields = _PREP_FIELDS + (_PREP16_FIELDS if with16 else ()) + (_PREPI8_FIELDS if int8_qk else ())
        return Prepared(self._alloc(fields, device))

    def alloc_plan(self, device="cuda", budget=None) -> Plan:
        """Plan buffers; with budget = (bp8, bp4[, per_row[, bp16]]) the lists get
        their exact compact size, otherwise the size of the largest budget."""
        override = {"kidx": self.list_bytes(*budget)} if budget is not None else None
        return Plan(self._alloc(_PLAN_FIELDS, device, override))

    def prepare(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, prep: Prepared, stream=None):
        assert q.dtype == k.dtype == v.dtype == torch.bfloat16
        assert q.stride() == k.stride() == v.stride()
        _check(lib().da2_prepare(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), _strides(q),
                                 ctypes.byref(prep.ptrs()), _stream_ptr(stream)), "da2_prepare")

    def plan(self, prep: Prepared, plan: Plan, bp8: int, bp4: int, lam: float = 0.2, stream=None,
             per_row: bool = False, bp16: int = 0):
        b = Budget(int(bp8), int(bp4), float(lam), int(bool(per_row)), int(bp16))
        _check(lib().da2_plan(self.handle, ctypes.byref(prep.ptrs()), ctypes.byref(b), ctypes.byref(plan.ptrs()),
                              _stream_ptr(stream)), "da2_plan")

    def plan_static(self, prep: Prepared, plan: Plan, bp8: int, bp4: int, lam: float = 0.2, stream=None,
                    per_row: bool = False, bp16: int = 0):
        """Routing without a caller scratch buffer (da2_plan_static): for callers
        that cannot allocate device memory, e.g. while capturing a CUDA graph.
        Writes plan.bufs' prec / cnt / off / kidx / A; plan.bufs["scratch"] is unused."""
        need = int(self.sizes.plan_scratch)
        limit = 32 << 20
        if need > limit:
            raise DA2Error(f"da2_plan_static: this shape needs {need} bytes of working memory, "
                           f"more than the library's fixed {limit} bytes; use plan() with a scratch buffer")
        b = Budget(int(bp8), int(bp4), float(lam), int(bool(per_row)), int(bp16))
        bufs = plan.bufs
        _check(lib().da2_plan_static(self.handle, ctypes.byref(prep.ptrs()), ctypes.byref(b), bufs["prec"].data_ptr(),
                                     bufs["cnt"].data_ptr(), bufs["off"].data_ptr(), bufs["kidx"].data_ptr(),
                                     bufs["A"].data_ptr(), _stream_ptr(stream)), "da2_plan_static")

    def attention(self, prep: Prepared, plan: Plan, out: torch.Tensor, stream=None):
        assert out.dtype == torch.bfloat16
        _check(lib().da2_attention(self.handle, ctypes.byref(prep.ptrs()), ctypes.byref(plan.ptrs()),
                                   out.data_ptr(), _strides(out), _stream_ptr(stream)), "da2_attention")

    def check_status(self, stream=None):
        _check(lib().da2_check_device_status(self.handle, _stream_ptr(stream)), "device status")

    def status(self, stream=None) -> int:
        """da2_check_device_status's return code (synchronizes the stream, clears the flag)."""
        return int(lib().da2_check_device_status(self.handle, _stream_ptr(stream)))

    def set_wait_limit(self, ns: int):
        """Limit of the kernels' bounded device-side waits (0 = the default 4 s)."""
        _check(lib().da2_set_wait_limit(self.handle, int(ns)), "da2_set_wait_limit")

    def selftest_wait_timeout(self, ns: int, stream=None):
        """Enqueue the failure-path self-test kernel (a bounded wait that runs out)."""
        _check(lib().da2_selftest_wait_timeout(self.handle, int(ns), _stream_ptr(stream)),
               "da2_selftest_wait_timeout")

    def forward(self, q, k, v, bp8, bp4, lam=0.2, out=None, prep=None, plan=None, stream=None, per_row=False,
                bp16=0, int8_qk=False):
        """prepare -> plan -> attention; returns (out, prep, plan)."""
        prep = prep or self.alloc_prepared(q.device, with16=bp16 > 0 or self.Rp > 0, int8_qk=int8_qk)
        plan = plan or self.alloc_plan(q.device, (bp8, bp4, per_row, bp16))
        out = torch.empty_like(q) if out is None else out
        self.prepare(q, k, v, prep, stream)
        self.plan(prep, plan, bp8, bp4, lam, stream, per_row, bp16)
        self.attention(prep, plan, out, stream)
        return out, prep, plan
