"""CPU oracle for the virtual-rank all-reduce (ctypes wrapper over liboracle.so).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg may use it; the product path never does. It is
independent of the CUDA library (no shared code, headers or constants).

Arrays are numpy: bf16 and fp16 data travel as ``uint16`` bit patterns, fp32
as ``float32``. A "rank list" is a list of P one-dimensional arrays.

What each function computes, and which source passage it follows, is stated in
oracle.cpp next to the C++ that does it. ``Oracle(path)`` wraps any build of
that file (the tests also load deliberately broken builds to show that the
pins catch planted mistakes); the module-level functions use the normal build.
"""

from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

ALGOS = ("oneshot", "twostage", "twostage_write", "rd", "hier", "rd_fp32wire", "hier_fp32wire",
         "oneshot_fp8", "twostage_fp8", "twostage_write_fp8")
_NP = {"bf16": np.uint16, "fp16": np.uint16, "fp32": np.float32}


def _ptrs(arrs):
    return (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])


def _check(arrs, dtype, n=None):
    want = _NP[dtype]
    out = []
    for a in arrs:
        a = np.ascontiguousarray(a)
        if a.dtype != want:
            raise TypeError(f"expected {np.dtype(want)} arrays for {dtype}, got {a.dtype}")
        if a.ndim != 1 or (n is not None and a.shape[0] != n):
            raise ValueError("each rank buffer must be 1-D with the stated length")
        out.append(a)
    return out


class Oracle:
    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        i64, vp, cp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_char_p
        pp = ctypes.POINTER(ctypes.c_void_p)
        L.oracle_bf16_round.argtypes = [vp, vp, i64]
        L.oracle_bf16_round.restype = None
        L.oracle_bf16_widen.argtypes = [vp, vp, i64]
        L.oracle_bf16_widen.restype = None
        L.oracle_fp16_round.argtypes = [vp, vp, i64]
        L.oracle_fp16_round.restype = None
        L.oracle_fp16_widen.argtypes = [vp, vp, i64]
        L.oracle_fp16_widen.restype = None
        L.oracle_allreduce.argtypes = [cp, pp, pp, ctypes.c_int, i64, cp, ctypes.c_int, ctypes.c_int]
        L.oracle_allreduce.restype = ctypes.c_int
        L.oracle_reduce_scatter.argtypes = [pp, pp, ctypes.c_int, i64, cp]
        L.oracle_reduce_scatter.restype = ctypes.c_int
        L.oracle_all_gather.argtypes = [pp, pp, ctypes.c_int, i64, cp]
        L.oracle_all_gather.restype = ctypes.c_int
        L.oracle_fp64_reference.argtypes = [pp, ctypes.c_int, i64, cp, vp, vp]
        L.oracle_fp64_reference.restype = ctypes.c_int
        L.oracle_e4m3_round.argtypes = [vp, vp, i64]
        L.oracle_e4m3_round.restype = None
        L.oracle_fp8_wire.argtypes = [vp, i64]
        L.oracle_fp8_wire.restype = None
        self.lib = L
        self.path = path

    def bf16_round(self, x: np.ndarray) -> np.ndarray:
        """float32 -> bf16 bit patterns, round to nearest even (NaN -> 0x7FC0)."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        y = np.empty(x.shape, np.uint16)
        self.lib.oracle_bf16_round(x.ctypes.data, y.ctypes.data, x.size)
        return y

    def bf16_widen(self, h: np.ndarray) -> np.ndarray:
        """bf16 bit patterns -> float32 (exact)."""
        h = np.ascontiguousarray(h, dtype=np.uint16)
        y = np.empty(h.shape, np.float32)
        self.lib.oracle_bf16_widen(h.ctypes.data, y.ctypes.data, h.size)
        return y

    def fp16_round(self, x: np.ndarray) -> np.ndarray:
        """float32 -> fp16 bit patterns, round to nearest even (NaN -> 0x7E00)."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        y = np.empty(x.shape, np.uint16)
        self.lib.oracle_fp16_round(x.ctypes.data, y.ctypes.data, x.size)
        return y

    def fp16_widen(self, h: np.ndarray) -> np.ndarray:
        """fp16 bit patterns -> float32 (exact)."""
        h = np.ascontiguousarray(h, dtype=np.uint16)
        y = np.empty(h.shape, np.float32)
        self.lib.oracle_fp16_widen(h.ctypes.data, y.ctypes.data, h.size)
        return y

    def e4m3_round(self, x: np.ndarray) -> np.ndarray:
        """float32 -> the nearest OCP FP8 E4M3 value (ties to even, saturating at 448), as float32."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        y = np.empty(x.shape, np.float32)
        self.lib.oracle_e4m3_round(x.ctypes.data, y.ctypes.data, x.size)
        return y

    def fp8_wire(self, x: np.ndarray) -> np.ndarray:
        """float32 values after the fp8 wire: groups of 8 from index 0, each with
        scale amax / 448, quantised to E4M3 and dequantised."""
        y = np.array(x, dtype=np.float32, copy=True).ravel()
        self.lib.oracle_fp8_wire(y.ctypes.data, y.size)
        return y

    def allreduce(self, algo: str, xs, dtype: str = "bf16", L: int = 8, chunks: int = 4):
        """All P outputs of one all-reduce with algorithm ``algo``."""
        if algo not in ALGOS:
            raise ValueError(f"unknown algorithm {algo!r}")
        P = len(xs)
        n = int(np.asarray(xs[0]).shape[0])
        xs = _check(xs, dtype, n)
        outs = [np.zeros(n, _NP[dtype]) for _ in range(P)]
        rc = self.lib.oracle_allreduce(algo.encode(), _ptrs(xs), _ptrs(outs), P, n, dtype.encode(), L, chunks)
        if rc != 0:
            raise ValueError(f"oracle_allreduce({algo}, P={P}, n={n}, L={L}) returned {rc}")
        return outs

    def reduce_scatter(self, xs, dtype: str = "bf16"):
        """``xs``: P buffers of n elements; returns P slices of n/P."""
        P = len(xs)
        n = int(np.asarray(xs[0]).shape[0])
        xs = _check(xs, dtype, n)
        outs = [np.zeros(n // P, _NP[dtype]) for _ in range(P)]
        rc = self.lib.oracle_reduce_scatter(_ptrs(xs), _ptrs(outs), P, n, dtype.encode())
        if rc != 0:
            raise ValueError(f"oracle_reduce_scatter(P={P}, n={n}) returned {rc}")
        return outs

    def all_gather(self, xs, dtype: str = "bf16"):
        """``xs``: P slices of n/P elements; returns P buffers of n."""
        P = len(xs)
        m = int(np.asarray(xs[0]).shape[0])
        xs = _check(xs, dtype, m)
        n = m * P
        outs = [np.zeros(n, _NP[dtype]) for _ in range(P)]
        rc = self.lib.oracle_all_gather(_ptrs(xs), _ptrs(outs), P, n, dtype.encode())
        if rc != 0:
            raise ValueError(f"oracle_all_gather(P={P}, n={n}) returned {rc}")
        return outs

    def fp64_reference(self, xs, dtype: str = "bf16"):
        """(S, A): the fp64 sum over ranks and the sum of magnitudes, per element."""
        P = len(xs)
        n = int(np.asarray(xs[0]).shape[0])
        xs = _check(xs, dtype, n)
        S = np.empty(n, np.float64)
        A = np.empty(n, np.float64)
        rc = self.lib.oracle_fp64_reference(_ptrs(xs), P, n, dtype.encode(), S.ctypes.data, A.ctypes.data)
        if rc != 0:
            raise ValueError("oracle_fp64_reference failed")
        return S, A

    def to_float(self, x: np.ndarray, dtype: str) -> np.ndarray:
        """Rank-buffer values as float64 (16-bit patterns widened exactly)."""
        if dtype == "bf16":
            return self.bf16_widen(x).astype(np.float64)
        if dtype == "fp16":
            return self.fp16_widen(x).astype(np.float64)
        return np.asarray(x, np.float64)


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def allreduce(algo, xs, dtype="bf16", L=8, chunks=4):
    return default().allreduce(algo, xs, dtype, L, chunks)


def reduce_scatter(xs, dtype="bf16"):
    return default().reduce_scatter(xs, dtype)


def all_gather(xs, dtype="bf16"):
    return default().all_gather(xs, dtype)


def fp64_reference(xs, dtype="bf16"):
    return default().fp64_reference(xs, dtype)


def bf16_round(x):
    return default().bf16_round(x)


def bf16_widen(h):
    return default().bf16_widen(h)


def fp16_round(x):
    return default().fp16_round(x)


def fp16_widen(h):
    return default().fp16_widen(h)


def to_float(x, dtype):
    return default().to_float(x, dtype)


def e4m3_round(x):
    return default().e4m3_round(x)


def fp8_wire(x):
    return default().fp8_wire(x)


__all__ = ["ALGOS", "Oracle", "default", "allreduce", "reduce_scatter", "all_gather",
           "fp64_reference", "bf16_round", "bf16_widen", "fp16_round", "fp16_widen", "to_float", "e4m3_round",
           "fp8_wire"]
