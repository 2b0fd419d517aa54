"""Python binding of the CPU oracle (oracle.cpp) of the MoE layer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU baseline leg use this module. The product path (the package
``combine_softmax_top_b200``) never imports it, and this module imports
nothing from the product path.

Arrays are numpy. bf16 data is carried as ``uint16`` bit patterns and e4m3
data as ``uint8`` codes, the same bytes the GPU library reads and writes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Mapping, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32, BF16, E4M3, E2M1 = 0, 1, 2, 3
OK, BAD_ARG, NONFINITE = 0, 1, 6


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so beside it (g++, OpenMP)."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(_SRC):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c++17",
                               "-o", tmp, _SRC])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int32
        sigs = {
            "oracle_e4m3_encode": [P, P, I64],
            "oracle_e4m3_decode": [P, P, I64],
            "oracle_e2m1_decode": [P, P, I64],
            "oracle_ue8m0_decode": [P, P, I64],
            "oracle_bf16_round": [P, P, I64],
            "oracle_pow2_scale": [P, P, I64],
            "oracle_route": [I64, I64, I64, I32, P, P, P],
            "oracle_counts": [I64, I64, I64, P, P],
            "oracle_quantize_rows": [I64, I64, P, P, P],
            "oracle_expert_rows": [P, I64, P, P, P, P, P, P],
            "oracle_combine": [I64, I64, I64, I32, P, P, I32, P],
            "oracle_moe_layer": [P, P, P, I64, I64, P, P, P, P, P, P],
            "oracle_set_threads": [I32],
        }
        for name, args in sigs.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
    return _lib


def set_threads(n: int) -> int:
    """Limit the oracle's OpenMP loops to n threads (timing only); returns the
    count in force."""
    return int(lib().oracle_set_threads(int(n)))


class OracleError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code}")
        self.code = code


def _ptr(a: np.ndarray | None) -> ctypes.c_void_p:
    if a is None:
        return ctypes.c_void_p(0)
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _call(name: str, *args) -> None:
    rc = getattr(lib(), name)(*args)
    if rc != OK:
        raise OracleError(name, rc)


class _Problem(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("E", ctypes.c_int64),
        ("k", ctypes.c_int64), ("I", ctypes.c_int64),
        ("x_dtype", ctypes.c_int32), ("xq_dtype", ctypes.c_int32),
        ("w_dtype", ctypes.c_int32), ("h_dtype", ctypes.c_int32),
        ("y_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
        ("renorm", ctypes.c_int32), ("identity", ctypes.c_int32), ("shared", ctypes.c_int32),
        ("w_gate", ctypes.POINTER(ctypes.c_void_p)), ("w_up", ctypes.POINTER(ctypes.c_void_p)),
        ("w_down", ctypes.POINTER(ctypes.c_void_p)),
        ("s_gate", ctypes.POINTER(ctypes.c_void_p)), ("s_up", ctypes.POINTER(ctypes.c_void_p)),
        ("s_down", ctypes.POINTER(ctypes.c_void_p)),
    ]


ExpertWeights = Mapping[int, np.ndarray] | np.ndarray | None


class Problem:
    """Shapes, dtypes and expert weights of one MoE layer.

    Weights are either full arrays ([E, I, H] gate/up, [E, H, I] down, e4m3
    scales [E, I/128, H/128] / [E, H/128, I/128]; e2m1 weights packed two per
    byte, [E, I, H/2] / [E, H, I/2], element 2i in the low nibble, with UE8M0
    scale bytes [E, I, H/32] / [E, H, I/32]) or mappings from expert index to
    that expert's matrix, for checks that touch only a few experts. With
    shared=1 the arrays hold E + 1 experts: expert E is the shared expert that
    every token also goes through, added with weight 1.
    """

    def __init__(self, T, H, E, k, I, *, x_dtype, xq_dtype, w_dtype, h_dtype, y_dtype,
                 out_dtype, renorm=1, identity=0, shared=0, w_gate: ExpertWeights = None,
                 w_up: ExpertWeights = None, w_down: ExpertWeights = None,
                 s_gate: ExpertWeights = None, s_up: ExpertWeights = None,
                 s_down: ExpertWeights = None):
        self.T, self.H, self.E, self.k, self.I = int(T), int(H), int(E), int(k), int(I)
        self.x_dtype, self.xq_dtype, self.w_dtype = x_dtype, xq_dtype, w_dtype
        self.h_dtype, self.y_dtype, self.out_dtype = h_dtype, y_dtype, out_dtype
        self.renorm, self.identity, self.shared = int(renorm), int(identity), int(shared)
        self.nw = self.E + self.shared     # experts with weights
        self._keep = []
        tabs = []
        for w in (w_gate, w_up, w_down, s_gate, s_up, s_down):
            tabs.append(self._table(w))
        s = _Problem()
        s.T, s.H, s.E, s.k, s.I = self.T, self.H, self.E, self.k, self.I
        s.x_dtype, s.xq_dtype, s.w_dtype = x_dtype, xq_dtype, w_dtype
        s.h_dtype, s.y_dtype, s.out_dtype = h_dtype, y_dtype, out_dtype
        s.renorm, s.identity, s.shared = self.renorm, self.identity, self.shared
        s.w_gate, s.w_up, s.w_down, s.s_gate, s.s_up, s.s_down = tabs
        self._s = s

    def _table(self, w: ExpertWeights):
        arr = (ctypes.c_void_p * self.nw)()
        if w is None:
            pass
        elif isinstance(w, np.ndarray):
            assert w.shape[0] == self.nw and w.flags["C_CONTIGUOUS"]
            self._keep.append(w)
            for e in range(self.nw):
                arr[e] = w[e].ctypes.data
        else:
            for e, m in w.items():
                m = np.ascontiguousarray(m)
                self._keep.append(m)
                arr[int(e)] = m.ctypes.data
        self._keep.append(arr)
        return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))

    @property
    def ref(self):
        return ctypes.byref(self._s)


_NP = {F32: np.float32, BF16: np.uint16, E4M3: np.uint8}


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint8)
    _call("oracle_e4m3_encode", _ptr(v), _ptr(out), v.size)
    return out


def e4m3_decode(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    out = np.empty(q.shape, np.float64)
    _call("oracle_e4m3_decode", _ptr(q), _ptr(out), q.size)
    return out


def e2m1_decode(q: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes (one per uint8, low nibble) -> float64 values."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    out = np.empty(q.shape, np.float64)
    _call("oracle_e2m1_decode", _ptr(q), _ptr(out), q.size)
    return out


def ue8m0_decode(b: np.ndarray) -> np.ndarray:
    """UE8M0 scale bytes -> float64 powers of two (255 -> NaN)."""
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, np.float64)
    _call("oracle_ue8m0_decode", _ptr(b), _ptr(out), b.size)
    return out


def bf16_round(v: np.ndarray) -> np.ndarray:
    """float32 values -> bf16 bit patterns (uint16), nearest-even."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint16)
    _call("oracle_bf16_round", _ptr(v), _ptr(out), v.size)
    return out


def pow2_scale(amax: np.ndarray) -> np.ndarray:
    amax = np.ascontiguousarray(amax, dtype=np.float64)
    out = np.empty(amax.shape, np.float64)
    _call("oracle_pow2_scale", _ptr(amax), _ptr(out), amax.size)
    return out


def route(logits: np.ndarray, k: int, renorm: int = 1):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _call("oracle_route", T, E, k, int(renorm), _ptr(logits), _ptr(idx), _ptr(w))
    return idx, w


def counts(idx: np.ndarray, E: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    c = np.empty(E, np.int32)
    _call("oracle_counts", T, E, k, _ptr(idx), _ptr(c))
    return c


def quantize_rows(x: np.ndarray):
    """[rows, H] float32 -> (e4m3 codes [rows, H], scales [rows, H/128])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, H = x.shape
    q = np.empty((rows, H), np.uint8)
    s = np.empty((rows, H // 128), np.float32)
    _call("oracle_quantize_rows", rows, H, _ptr(x), _ptr(q), _ptr(s))
    return q, s


def expert_rows(p: Problem, expert: np.ndarray, xq: np.ndarray, xs: np.ndarray | None = None):
    """Experts applied to rows already stored as xq_dtype. Returns (h, hs, y)."""
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    rows = expert.shape[0]
    xq = np.ascontiguousarray(xq)
    h = np.empty((rows, p.I), _NP[p.h_dtype])
    hs = np.empty((rows, p.I // 128), np.float32) if p.h_dtype == E4M3 else None
    y = np.empty((rows, p.H), _NP[p.y_dtype])
    if xs is not None:
        xs = np.ascontiguousarray(xs, dtype=np.float32)
    _call("oracle_expert_rows", p.ref, rows, _ptr(expert), _ptr(xq), _ptr(xs), _ptr(h),
          _ptr(hs), _ptr(y))
    return h, hs, y


def combine(y_pairs: np.ndarray, w: np.ndarray, y_dtype: int, out_dtype: int) -> np.ndarray:
    """y_pairs [T*k, H] (pair order t*k+j), w [T, k] -> out [T, H]."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    T, k = w.shape
    y_pairs = np.ascontiguousarray(y_pairs)
    H = y_pairs.shape[1]
    out = np.empty((T, H), _NP[out_dtype])
    _call("oracle_combine", T, k, H, y_dtype, _ptr(y_pairs), _ptr(w), out_dtype, _ptr(out))
    return out


def moe_layer(p: Problem, x: np.ndarray, logits: np.ndarray, t0: int = 0, t1: int | None = None,
              want_intermediates: bool = False):
    """Whole layer for tokens [t0, t1). Returns dict with idx, w (the k routed
    slots), out (and xq, xs, y_pairs when want_intermediates; y_pairs has
    k + shared rows per token, the shared expert's last)."""
    t1 = p.T if t1 is None else t1
    n = t1 - t0
    x = np.ascontiguousarray(x)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    idx = np.empty((p.T, p.k), np.int32)
    w = np.empty((p.T, p.k), np.float32)
    out = np.empty((n, p.H), _NP[p.out_dtype])
    xq = xs = yp = None
    if want_intermediates:
        xq = np.empty((n, p.H), _NP[p.xq_dtype])
        xs = np.empty((n, p.H // 128), np.float32) if p.xq_dtype == E4M3 else None
        yp = None if p.identity else np.empty((n * (p.k + p.shared), p.H), _NP[p.y_dtype])
    _call("oracle_moe_layer", p.ref, _ptr(x), _ptr(logits), t0, t1, _ptr(idx), _ptr(w),
          _ptr(out), _ptr(xq), _ptr(xs), _ptr(yp))
    res = {"idx": idx, "w": w, "out": out}
    if want_intermediates:
        res.update(xq=xq, xs=xs, y_pairs=yp)
    return res


__all__ = [
    "F32", "BF16", "E4M3", "Problem", "OracleError", "build", "lib", "e4m3_encode",
    "e4m3_decode", "bf16_round", "pow2_scale", "route", "counts", "quantize_rows",
    "expert_rows", "combine", "moe_layer",
]
