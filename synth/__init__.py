"""Seeded synthetic inputs for the virtual-rank all-reduce.

This module only draws numbers. It holds none of the all-reduce arithmetic: no
sums, no reduction order, no rounding rule of the method. Both the CPU oracle
(through the tests) and the CUDA path (through the tests and the benchmark)
take their inputs from here, so that the two sides see the same bits.

Generator (counter-based, so any element can be drawn on its own):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014). ``mix`` is its output finaliser; the j-th draw of
  a stream with state ``s`` is ``mix(s + (j + 1) * GAMMA)`` mod 2**64.
* The stream of virtual rank ``r`` under seed ``seed`` starts from
  ``s = mix(((seed << 32) | r) + GAMMA)``, the first output of SplitMix64
  seeded with ``(seed << 32) | r``.
* A 53-bit uniform is ``(draw >> 11) * 2**-53``.

Distributions (element i of rank r):

* ``int8`` : integers -8..8 inclusive, ``((draw_i >> 11) mod 17) - 8``.
* ``uniform(a, b)`` : ``a + (b - a) * U_i`` in float64.
* ``normal(mu, sigma)`` : Box-Muller in float64 from draws ``2i`` and ``2i+1``:
  ``U1 = ((d >> 11) + 1) * 2**-53`` in (0, 1], ``U2 = (d >> 11) * 2**-53``,
  ``z = sqrt(-2 ln U1) * cos(2 pi U2)``, value ``mu + sigma * z``.

The float64 value is then rounded to float32 (round to nearest even) and, for
bf16 or fp16 tensors, from float32 to that type (round to nearest even).
Integer values in -8..8 are exact in all three types.

Everything is written with int64 torch ops (two's-complement wrap-around
stands in for unsigned 64-bit arithmetic), so it runs unchanged on the CPU or
on a CUDA device.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = [
    "Dist",
    "INT8",
    "normal",
    "uniform",
    "draws",
    "rank_values",
    "make_inputs",
    "parse_dist",
]

_M64 = (1 << 64) - 1


def _s64(u: int) -> int:
    """An unsigned 64-bit constant as the int64 with the same bits."""
    u &= _M64
    return u - (1 << 64) if u >= (1 << 63) else u


GAMMA = _s64(0x9E3779B97F4A7C15)
_C1 = _s64(0xBF58476D1CE4E5B9)
_C2 = _s64(0x94D049BB133111EB)


def _srl(x: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bits (torch's >> is arithmetic)."""
    return (x >> k) & ((1 << (64 - k)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _C1
    z = (z ^ _srl(z, 27)) * _C2
    return z ^ _srl(z, 31)


def _mix_int(z: int) -> int:
    """Same finaliser on a Python int (used for the per-stream start state)."""
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def stream_state(seed: int, rank: int) -> int:
    """Start state (as unsigned int) of rank ``rank``'s stream under ``seed``."""
    if not (0 <= seed < (1 << 32) and 0 <= rank < (1 << 32)):
        raise ValueError("seed and rank must fit in 32 bits")
    return _mix_int(((seed << 32) | rank) + 0x9E3779B97F4A7C15)


def draws(seed: int, rank: int, j: torch.Tensor) -> torch.Tensor:
    """Raw 64-bit draws (as int64 bits) at draw indices ``j`` (int64 tensor)."""
    s = _s64(stream_state(seed, rank))
    return _mix(s + (j + 1) * GAMMA)


def _u53(d: torch.Tensor) -> torch.Tensor:
    return _srl(d, 11).to(torch.float64) * (2.0 ** -53)


@dataclass(frozen=True)
class Dist:
    kind: str  # "int8", "uniform", "normal"
    a: float = 0.0  # uniform low / normal mean
    b: float = 1.0  # uniform high / normal sigma

    def describe(self) -> str:
        if self.kind == "int8":
            return "integers -8..8"
        if self.kind == "uniform":
            return f"uniform({self.a:g},{self.b:g})"
        return f"N({self.a:g},{self.b:g})"


INT8 = Dist("int8")


def normal(mu: float = 0.0, sigma: float = 1.0) -> Dist:
    return Dist("normal", mu, sigma)


def uniform(a: float = -1.0, b: float = 1.0) -> Dist:
    return Dist("uniform", a, b)


def parse_dist(s: str) -> Dist:
    """``"int8"``, ``"normal:0,0.02"``, ``"uniform:-1,1"``."""
    if s == "int8":
        return INT8
    kind, _, args = s.partition(":")
    a, b = (float(t) for t in args.split(",")) if args else (None, None)
    if kind == "normal":
        return normal(0.0 if a is None else a, 1.0 if b is None else b)
    if kind == "uniform":
        return uniform(-1.0 if a is None else a, 1.0 if b is None else b)
    raise ValueError(f"unknown distribution {s!r}")


def rank_values(dist: Dist, seed: int, rank: int, idx: torch.Tensor) -> torch.Tensor:
    """float64 values of rank ``rank`` at element indices ``idx`` (int64)."""
    if dist.kind == "int8":
        d = draws(seed, rank, idx)
        return (torch.remainder(_srl(d, 11), 17) - 8).to(torch.float64)
    if dist.kind == "uniform":
        u = _u53(draws(seed, rank, idx))
        return dist.a + (dist.b - dist.a) * u
    if dist.kind == "normal":
        d1 = draws(seed, rank, 2 * idx)
        d2 = draws(seed, rank, 2 * idx + 1)
        u1 = (_srl(d1, 11) + 1).to(torch.float64) * (2.0 ** -53)
        u2 = _u53(d2)
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
        return dist.a + dist.b * z
    raise ValueError(dist.kind)


def to_dtype(v64: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    """float64 -> float32 (RNE) -> dtype (RNE); bf16, fp16 and fp32."""
    v32 = v64.to(torch.float32)
    if dtype == torch.float32:
        return v32
    if dtype in (torch.bfloat16, torch.float16):
        return v32.to(dtype)
    raise ValueError(f"unsupported dtype {dtype}")


def make_inputs(P: int, n: int, dtype: torch.dtype, dist: Dist, seed: int = 0,
                device: str | torch.device = "cpu", block: int = 1 << 24) -> list[torch.Tensor]:
    """P rank buffers of n elements each, drawn on ``device`` in blocks."""
    out = []
    for r in range(P):
        t = torch.empty(n, dtype=dtype, device=device)
        for lo in range(0, n, block):
            hi = min(n, lo + block)
            idx = torch.arange(lo, hi, dtype=torch.int64, device=device)
            t[lo:hi] = to_dtype(rank_values(dist, seed, r, idx), dtype)
        out.append(t)
    return out
