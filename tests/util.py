"""Helpers shared by the tests: seeded inputs as numpy arrays, bit views, fixtures."""

from __future__ import annotations

import json
import os

import numpy as np
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}
NP_DT = {"bf16": np.uint16, "fp16": np.uint16, "fp32": np.float32}


def to_np(t: torch.Tensor) -> np.ndarray:
    """A CPU tensor's elements as numpy: bf16 / fp16 as uint16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def from_np(a: np.ndarray, dtype: str) -> torch.Tensor:
    """numpy rank buffer (uint16 patterns for 16-bit types) -> CPU tensor of that dtype."""
    if dtype in ("bf16", "fp16"):
        return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16).copy()).view(TORCH_DT[dtype])
    return torch.from_numpy(np.ascontiguousarray(a, np.float32).copy())


def gen(P: int, n: int, dtype: str, dist, seed: int = 0) -> list[np.ndarray]:
    """P seeded rank buffers of n elements, as numpy (CPU generation)."""
    return [to_np(t) for t in synth.make_inputs(P, n, TORCH_DT[dtype], dist, seed)]


def hexvals(strs, dtype: str) -> np.ndarray:
    """Hex-float strings -> a numpy rank buffer of the given dtype (exact)."""
    f = np.array([float.fromhex(s) for s in strs], np.float64)
    f32 = f.astype(np.float32)
    assert (f32.astype(np.float64) == f).all(), "fixture value not exact in fp32"
    if dtype == "fp32":
        return f32
    if dtype == "fp16":
        h = f32.astype(np.float16)
        assert (h.astype(np.float64) == f).all(), "fixture value not exact in fp16"
        return h.view(np.uint16)
    bits = f32.view(np.uint32)
    assert (bits & 0xFFFF == 0).all(), "fixture value not exact in bf16"
    return (bits >> 16).astype(np.uint16)


def bits_of(a: np.ndarray) -> np.ndarray:
    """Raw bits of a rank buffer (so that +0 and -0 differ)."""
    return a.view(np.uint16) if a.dtype == np.uint16 else a.view(np.uint32)


def load_golden(name: str = "order_cases.json"):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def parse_algo(spec: str):
    """"hier:L=4" -> ("hier", 4); "rd" -> ("rd", None)."""
    if ":" in spec:
        algo, arg = spec.split(":", 1)
        return algo, int(arg.split("=", 1)[1])
    return spec, None
