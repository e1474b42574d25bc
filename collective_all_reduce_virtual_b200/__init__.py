"""Python binding of libvrar (virtual-rank all-reduce on one GPU).

Argument marshalling only: every step of an all-reduce runs in the library's
CUDA kernels. torch provides device memory and streams. The C ABI and the
meaning of every argument are documented in include/vrar.h.

There is no fallback: if libvrar.so is missing or cannot be loaded, importing
this package raises ImportError (build it with ``python
collective_all_reduce_virtual_b200/build.py`` or ``__graft_entry__.build()``).
"""

from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvrar.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libvrar.so not found at {LIB_PATH}; build it first "
                      "(python collective_all_reduce_virtual_b200/build.py)")
_lib = ctypes.CDLL(LIB_PATH)

OK, EINVAL, ENOTSUP, ENOMEM, ECUDA, ETIMEDOUT, ETOOBIG = 0, -1, -2, -3, -4, -5, -6
NOALLOC_SCRATCH_BYTES = 16 << 20
MAX_RANKS = 32

DTYPES = {torch.bfloat16: 0, torch.float32: 1, torch.float16: 2}
ALGOS = {"auto": 0, "oneshot": 1, "twostage": 2, "twostage_write": 3, "rd": 4, "hier": 5}
ALGO_NAMES = {v: k for k, v in ALGOS.items()}

# Every symbol include/vrar.h declares, with its ctypes signature.
_i, _u32, _u64, _sz, _vp = ctypes.c_int, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p
_pp = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "vrar_allreduce": ([_pp, _pp, _i, _sz, _i, _i, _vp], _i),
    "vrar_reduce_scatter": ([_pp, _pp, _i, _sz, _i, _vp], _i),
    "vrar_all_gather": ([_pp, _pp, _i, _sz, _i, _vp], _i),
    "vrar_select_algo": ([_i, _sz, _i], _i),
    "vrar_kernel_name": ([_i, _sz, _i, _i], ctypes.c_char_p),
    "vrar_set_group_size": ([_i], _i),
    "vrar_get_group_size": ([], _i),
    "vrar_set_rd_chunks": ([_i], _i),
    "vrar_get_rd_chunks": ([], _i),
    "vrar_set_payload_wire": ([_i], _i),
    "vrar_get_payload_wire": ([], _i),
    "vrar_set_fp8_quant": ([_i], _i),
    "vrar_get_fp8_quant": ([], _i),
    "vrar_set_edge_sync": ([_i], _i),
    "vrar_get_edge_sync": ([], _i),
    "vrar_set_max_ctas": ([_i], _i),
    "vrar_get_max_ctas": ([], _i),
    "vrar_set_spin_timeout_ns": ([_u64], _i),
    "vrar_get_spin_timeout_ns": ([], _u64),
    "vrar_query_status": ([_vp, ctypes.POINTER(_u32)], _i),
    "vrar_reserve": ([_sz], _i),
    "vrar_workspace_bytes": ([_i, _sz, _i, _i], _sz),
    "vrar_reset": ([], _i),
    "vrar_set_spin_stats": ([_i], _i),
    "vrar_get_spin_stats": ([ctypes.POINTER(_u64), _i], _i),
    "vrar_debug_set_fault_mask": ([_u32], _i),
    "vrar_allreduce_rd_noalloc": ([_pp, _pp, _i, _sz, _i, _vp], _i),
    "vrar_strerror": ([_i], ctypes.c_char_p),
    "vrar_version": ([], _i),
}
for _name, (_args, _res) in SIGNATURES.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class VrarError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_lib.vrar_strerror(code).decode()} ({code})")


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise VrarError(rc, what)
    return rc


def lib() -> ctypes.CDLL:
    """The loaded libvrar (for callers that pass raw pointers)."""
    return _lib


def ptr_array(ptrs: Sequence[int]):
    """A C array of device pointers (ints) for the raw entry points."""
    return (ctypes.c_void_p * len(ptrs))(*ptrs)


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _rank_tensors(ts: Sequence[torch.Tensor], numel: int | None, what: str):
    if not 1 <= len(ts) <= MAX_RANKS:
        raise ValueError(f"{what}: need 1..{MAX_RANKS} rank tensors, got {len(ts)}")
    dt = ts[0].dtype
    if dt not in DTYPES:
        raise TypeError(f"{what}: dtype must be bfloat16, float16 or float32, got {dt}")
    dev = ts[0].device
    if dev.type != "cuda":
        raise ValueError(f"{what}: tensors must be on a CUDA device")
    for t in ts:
        if t.dtype != dt or t.device != dev:
            raise ValueError(f"{what}: all rank tensors must share dtype and device")
        if not t.is_contiguous():
            raise ValueError(f"{what}: rank tensors must be contiguous")
        if numel is not None and t.numel() != numel:
            raise ValueError(f"{what}: expected {numel} elements per rank, got {t.numel()}")
    return dt, dev


def all_reduce(inputs: Sequence[torch.Tensor], outputs: Sequence[torch.Tensor] | None = None,
               algo: str = "auto", stream=None) -> list[torch.Tensor]:
    """All-reduce P rank tensors (same shape) into P outputs (allocated if None)."""
    n = inputs[0].numel()
    dt, dev = _rank_tensors(inputs, n, "all_reduce inputs")
    if outputs is None:
        outputs = [torch.empty_like(t) for t in inputs]
    _rank_tensors(outputs, n, "all_reduce outputs")
    P = len(inputs)
    with torch.cuda.device(dev):
        rc = _lib.vrar_allreduce(ptr_array([t.data_ptr() for t in inputs]),
                                 ptr_array([t.data_ptr() for t in outputs]),
                                 P, n, DTYPES[dt], ALGOS[algo], _stream_handle(stream))
    _check(rc, f"vrar_allreduce({algo}, P={P}, n={n})")
    return list(outputs)


def reduce_scatter(inputs: Sequence[torch.Tensor], outputs: Sequence[torch.Tensor] | None = None,
                   stream=None) -> list[torch.Tensor]:
    """P inputs of n elements -> P outputs of n/P elements (slice p of the sum)."""
    n = inputs[0].numel()
    P = len(inputs)
    dt, dev = _rank_tensors(inputs, n, "reduce_scatter inputs")
    if n % P:
        raise ValueError("reduce_scatter: n must be a multiple of P")
    if outputs is None:
        outputs = [torch.empty(n // P, dtype=dt, device=dev) for _ in inputs]
    _rank_tensors(outputs, n // P, "reduce_scatter outputs")
    with torch.cuda.device(dev):
        rc = _lib.vrar_reduce_scatter(ptr_array([t.data_ptr() for t in inputs]),
                                      ptr_array([t.data_ptr() for t in outputs]),
                                      P, n, DTYPES[dt], _stream_handle(stream))
    _check(rc, f"vrar_reduce_scatter(P={P}, n={n})")
    return list(outputs)


def all_gather(inputs: Sequence[torch.Tensor], outputs: Sequence[torch.Tensor] | None = None,
               stream=None) -> list[torch.Tensor]:
    """P inputs of m elements -> P outputs of P*m elements (the concatenation)."""
    m = inputs[0].numel()
    P = len(inputs)
    dt, dev = _rank_tensors(inputs, m, "all_gather inputs")
    if outputs is None:
        outputs = [torch.empty(m * P, dtype=dt, device=dev) for _ in inputs]
    _rank_tensors(outputs, m * P, "all_gather outputs")
    with torch.cuda.device(dev):
        rc = _lib.vrar_all_gather(ptr_array([t.data_ptr() for t in inputs]),
                                  ptr_array([t.data_ptr() for t in outputs]),
                                  P, m * P, DTYPES[dt], _stream_handle(stream))
    _check(rc, f"vrar_all_gather(P={P}, n={m * P})")
    return list(outputs)


def select_algo(P: int, n: int, dtype: torch.dtype = torch.bfloat16) -> str:
    return ALGO_NAMES[_check(_lib.vrar_select_algo(P, n, DTYPES[dtype]), "vrar_select_algo")]


def kernel_name(P: int, n: int, dtype: torch.dtype = torch.bfloat16, algo: str = "auto") -> str:
    """Base name of the kernel all_reduce(P buffers of n, dtype, algo) would launch."""
    name = _lib.vrar_kernel_name(P, n, DTYPES[dtype], ALGOS[algo])
    if name is None:
        raise VrarError(EINVAL, "vrar_kernel_name")
    return name.decode()


def set_group_size(L: int) -> None:
    _check(_lib.vrar_set_group_size(L), "vrar_set_group_size")


def get_group_size() -> int:
    return _lib.vrar_get_group_size()


def set_rd_chunks(C: int) -> None:
    _check(_lib.vrar_set_rd_chunks(C), "vrar_set_rd_chunks")


def get_rd_chunks() -> int:
    return _lib.vrar_get_rd_chunks()


WIRE_ELEMENT, WIRE_FP32 = 0, 1


def set_payload_wire(wire: str) -> None:
    """'element' (default) or 'fp32': what RD / HIER payload words carry."""
    _check(_lib.vrar_set_payload_wire({"element": WIRE_ELEMENT, "fp32": WIRE_FP32}[wire]), "vrar_set_payload_wire")


def get_payload_wire() -> str:
    return "fp32" if _lib.vrar_get_payload_wire() == WIRE_FP32 else "element"


def set_fp8_quant(on: bool) -> None:
    """fp8 payloads of the custom all-reduce algorithms (see vrar_set_fp8_quant)."""
    _check(_lib.vrar_set_fp8_quant(1 if on else 0), "vrar_set_fp8_quant")


def get_fp8_quant() -> bool:
    return bool(_lib.vrar_get_fp8_quant())


def set_edge_sync(on: bool) -> None:
    _check(_lib.vrar_set_edge_sync(1 if on else 0), "vrar_set_edge_sync")


def get_edge_sync() -> bool:
    return bool(_lib.vrar_get_edge_sync())


def set_max_ctas(n: int) -> None:
    """Cap the CTAs a call launches (0 = as many as fit)."""
    _check(_lib.vrar_set_max_ctas(n), "vrar_set_max_ctas")


def get_max_ctas() -> int:
    return _lib.vrar_get_max_ctas()


def set_spin_timeout_ns(ns: int) -> None:
    _check(_lib.vrar_set_spin_timeout_ns(ns), "vrar_set_spin_timeout_ns")


def get_spin_timeout_ns() -> int:
    return _lib.vrar_get_spin_timeout_ns()


def query_status(stream=None) -> tuple[int, list[int]]:
    """(code, info): waits for the stream, returns and clears the status word."""
    info = (ctypes.c_uint32 * 4)()
    rc = _lib.vrar_query_status(_stream_handle(stream), info)
    return rc, list(info)


def reserve(nbytes: int) -> None:
    _check(_lib.vrar_reserve(nbytes), "vrar_reserve")


def workspace_bytes(P: int, n: int, dtype: torch.dtype, algo: str) -> int:
    return _lib.vrar_workspace_bytes(P, n, DTYPES[dtype], ALGOS[algo])


def reset() -> None:
    _check(_lib.vrar_reset(), "vrar_reset")


def set_spin_stats(on: bool) -> None:
    _check(_lib.vrar_set_spin_stats(1 if on else 0), "vrar_set_spin_stats")


SPIN_STAT_KEYS = ("waits", "polls", "max_polls", "long_waits", "timeouts")


def get_spin_stats(reset: bool = False) -> dict:
    """Spin statistics of the current device (waits for the device)."""
    out = (ctypes.c_uint64 * 5)()
    _check(_lib.vrar_get_spin_stats(out, 1 if reset else 0), "vrar_get_spin_stats")
    return dict(zip(SPIN_STAT_KEYS, (int(v) for v in out)))


def debug_set_fault_mask(mask: int) -> None:
    _check(_lib.vrar_debug_set_fault_mask(mask), "vrar_debug_set_fault_mask")


def strerror(code: int) -> str:
    return _lib.vrar_strerror(code).decode()


def version() -> int:
    return _lib.vrar_version()


__all__ = ["all_reduce", "reduce_scatter", "all_gather", "select_algo", "kernel_name", "set_group_size",
           "get_group_size", "set_rd_chunks", "get_rd_chunks", "set_payload_wire", "get_payload_wire", "set_fp8_quant",
           "get_fp8_quant", "set_edge_sync", "get_edge_sync",
           "set_max_ctas", "get_max_ctas", "set_spin_timeout_ns", "get_spin_timeout_ns", "query_status", "reserve",
           "workspace_bytes", "reset", "set_spin_stats", "get_spin_stats", "debug_set_fault_mask", "strerror", "version", "VrarError",
           "ALGOS", "DTYPES", "SIGNATURES", "LIB_PATH", "lib", "ptr_array"]
