"""The C-ABI library on the CPU: it loads, exports every symbol include/vrar.h
declares, and rejects bad arguments on the host before touching a device.

No compute call reaches a kernel here. The pointers below are fake device
addresses; every call that uses them fails its host-side checks first, except
the one test that needs "no device" and is skipped when a GPU is present.
"""

import ctypes
import os
import re

import pytest
import torch

import collective_all_reduce_virtual_b200 as vrar

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "vrar.h")
L = vrar.lib()


def header_functions():
    src = open(HEADER).read()
    return set(re.findall(r"^VRAR_API\s+[\w\s\*]+?\b(vrar_\w+)\(", src, flags=re.M))


def test_every_declared_symbol_is_exported_and_bound():
    declared = header_functions()
    assert len(declared) >= 19
    assert declared == set(vrar.SIGNATURES), "binding signatures and header declarations differ"
    for name in declared:
        assert hasattr(L, name), f"{name} not exported by libvrar.so"


def test_version_and_strerror():
    assert vrar.version() == 1
    for code, word in ((0, "success"), (-1, "invalid"), (-2, "not supported"), (-3, "allocation"),
                       (-4, "CUDA"), (-5, "timed out"), (-99, "unknown")):
        assert word in vrar.strerror(code)


def _ptrs(base, P, stride=1 << 20):
    return vrar.ptr_array([base + p * stride for p in range(P)])


IN, OUT = 0x7F0000000000, 0x7F1000000000


def call_ar(ins, outs, P, n, dtype=0, algo=1):
    return L.vrar_allreduce(ins, outs, P, n, dtype, algo, None)


def test_rejects_bad_rank_counts_and_dtypes():
    assert call_ar(_ptrs(IN, 1), _ptrs(OUT, 1), 0, 16) == vrar.EINVAL
    assert call_ar(_ptrs(IN, 33), _ptrs(OUT, 33), 33, 16) == vrar.EINVAL
    assert call_ar(_ptrs(IN, 2), _ptrs(OUT, 2), 2, 16, dtype=7) == vrar.EINVAL
    assert call_ar(_ptrs(IN, 2), _ptrs(OUT, 2), 2, 16, algo=9) == vrar.EINVAL
    assert L.vrar_allreduce(None, _ptrs(OUT, 2), 2, 16, 0, 1, None) == vrar.EINVAL


def test_rejects_null_and_misaligned_pointers():
    ins = vrar.ptr_array([IN, 0])
    assert call_ar(ins, _ptrs(OUT, 2), 2, 16) == vrar.EINVAL
    ins = vrar.ptr_array([IN, IN + (1 << 20) + 8])  # 8-byte aligned only
    assert call_ar(ins, _ptrs(OUT, 2), 2, 16) == vrar.EINVAL


def test_rejects_overlap():
    # out[1] overlaps in[0]
    outs = vrar.ptr_array([OUT, IN + 16])
    assert call_ar(_ptrs(IN, 2), outs, 2, 64) == vrar.EINVAL
    # two outputs overlap each other
    outs = vrar.ptr_array([OUT, OUT + 32])
    assert call_ar(_ptrs(IN, 2), outs, 2, 64) == vrar.EINVAL


def test_shape_errors():
    assert call_ar(_ptrs(IN, 3), _ptrs(OUT, 3), 3, 16, algo=4) == vrar.ENOTSUP  # RD needs 2^k
    vrar.set_group_size(4)
    try:
        assert call_ar(_ptrs(IN, 12), _ptrs(OUT, 12), 12, 16, algo=5) == vrar.ENOTSUP  # G = 3
        assert call_ar(_ptrs(IN, 6), _ptrs(OUT, 6), 6, 16, algo=5) == vrar.ENOTSUP  # 4 does not divide 6
    finally:
        vrar.set_group_size(8)
    # reduce-scatter / all-gather need n % P == 0
    assert L.vrar_reduce_scatter(_ptrs(IN, 3), _ptrs(OUT, 3), 3, 10, 0, None) == vrar.EINVAL
    assert L.vrar_all_gather(_ptrs(IN, 3), _ptrs(OUT, 3), 3, 10, 0, None) == vrar.EINVAL


def test_zero_length_is_a_no_op():
    assert call_ar(_ptrs(IN, 4), _ptrs(OUT, 4), 4, 0) == vrar.OK


# These calls pass every host check, so on a machine with a GPU they would
# launch a kernel on fake addresses: they run only where there is no device.
@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a GPU")
def test_valid_call_without_device_reports_cuda_error():
    assert call_ar(_ptrs(IN, 2), _ptrs(OUT, 2), 2, 64) == vrar.ECUDA
    # adjacent, non-overlapping ranges pass the overlap check
    assert call_ar(vrar.ptr_array([IN, IN + 128]), _ptrs(OUT, 2), 2, 64) == vrar.ECUDA
    # largest request the fixed scratch holds at P = 8, bf16: passes the size check
    assert L.vrar_allreduce_rd_noalloc(_ptrs(IN, 8), _ptrs(OUT, 8), 8, 174_760, 0, None) == vrar.ECUDA


def test_noalloc_rejects_requests_beyond_its_fixed_scratch():
    """The allocation-free entry point refuses, on the host, any request whose
    payload slots would not fit its fixed array (fake pointers: nothing runs)."""
    f = L.vrar_allreduce_rd_noalloc
    assert f(_ptrs(IN, 8), _ptrs(OUT, 8), 8, 174_760 + 8, 0, None) == vrar.ETOOBIG
    # 2^24 fp32 per rank at P = 2: 256 MiB of slots (buffers 1 GiB apart, no overlap)
    assert f(_ptrs(IN, 2, 1 << 30), _ptrs(OUT, 2, 1 << 30), 2, 1 << 24, 1, None) == vrar.ETOOBIG
    assert f(_ptrs(IN, 3), _ptrs(OUT, 3), 3, 64, 0, None) == vrar.ENOTSUP
    assert f(_ptrs(IN, 8), _ptrs(OUT, 8), 8, 0, 0, None) == vrar.OK
    assert "fixed scratch" in vrar.strerror(vrar.ETOOBIG)


def test_settings_round_trip_and_ranges():
    assert vrar.get_group_size() == 8 and vrar.get_rd_chunks() == 4 and not vrar.get_edge_sync()
    for bad in (0, 33):
        with pytest.raises(vrar.VrarError):
            vrar.set_group_size(bad)
    for bad in (0, 9):
        with pytest.raises(vrar.VrarError):
            vrar.set_rd_chunks(bad)
    with pytest.raises(vrar.VrarError):
        vrar.set_spin_timeout_ns(10)
    t = vrar.get_spin_timeout_ns()
    vrar.set_spin_timeout_ns(5_000_000)
    assert vrar.get_spin_timeout_ns() == 5_000_000
    vrar.set_spin_timeout_ns(t)
    vrar.set_edge_sync(True)
    assert vrar.get_edge_sync()
    vrar.set_edge_sync(False)


def test_selector_is_defined_for_every_shape():
    for P in range(1, 33):
        for n in (1, 1000, 65536, 1 << 20, 117440512):
            for dt in (torch.bfloat16, torch.float32, torch.float16):
                a = vrar.select_algo(P, n, dt)
                assert a in ("oneshot", "twostage", "twostage_write", "rd", "hier")
                if a == "rd":
                    assert P & (P - 1) == 0


def test_selector_table_entries():
    """A few entries of the measured per-shape table (bytes per rank)."""
    bf = torch.bfloat16
    assert vrar.select_algo(1, 1 << 20, bf) == "oneshot"            # a copy
    assert vrar.select_algo(2, 1 << 19, bf) == "oneshot"            # 1 MiB at 2 ranks
    assert vrar.select_algo(2, 1 << 20, bf) == "twostage_write"     # 2 MiB at 2 ranks (batched write kernel)
    assert vrar.kernel_name(2, 1 << 20, bf, "auto") == "k_twostage_write_batched"  # 2 MiB at 2 ranks
    assert vrar.kernel_name(32, 8 << 20, bf, "auto") == "k_twostage_write"        # 16 MiB at 32 ranks
    assert vrar.kernel_name(4, 32 << 20, bf, "auto") == "k_twostage_write_batched"  # 64 MiB at 4 ranks
    assert vrar.kernel_name(2, 16 << 20, bf, "auto") == "k_twostage_write_async"    # 32 MiB at 2 ranks
    assert vrar.select_algo(2, 4 << 20, bf) == "twostage_write"     # 8 MiB at 2 ranks
    assert vrar.select_algo(8, 524288, bf) == "twostage_write"      # 1 MiB at 8 ranks (the decode shape)
    assert vrar.select_algo(8, 117440512, bf) == "twostage_write"   # prefill
    assert vrar.select_algo(32, 16384, bf) == "twostage_write"      # 32 KiB at 32 ranks
    assert vrar.select_algo(8, 524288, torch.float16) == "twostage_write"


def test_kernel_name():
    """Which kernel a call launches: write mode has four kernels with one result."""
    bf = torch.bfloat16
    if os.environ.get("VRAR_WRITE_KERNEL") or os.environ.get("VRAR_ALGO"):
        pytest.skip("an override is set in the environment")
    assert vrar.kernel_name(8, 524288, bf, "oneshot") == "k_oneshot"
    assert vrar.kernel_name(8, 524288, bf, "twostage") == "k_twostage"
    assert vrar.kernel_name(8, 524288, bf, "rd") == "k_rd"
    assert vrar.kernel_name(32, 524288, bf, "hier") == "k_hier"
    assert vrar.kernel_name(8, 524288, bf, "auto") == "k_twostage_write_async"       # the decode shape
    assert vrar.kernel_name(8, 117440512, bf, "auto") == "k_twostage_write"          # prefill
    assert vrar.kernel_name(8, 8 << 20, bf, "auto") == "k_twostage_write_staged"     # 16 MiB at 8 ranks
    assert vrar.kernel_name(1, 1000, bf, "auto") == "k_oneshot"
    for P in (1, 2, 3, 8, 13, 32):
        for n in (0, 1, 65536, 524288, 1 << 24):
            for dt in (bf, torch.float16, torch.float32):
                assert vrar.kernel_name(P, n, dt, "twostage_write").startswith("k_twostage_write")
    vrar.set_payload_wire("fp32")
    try:
        assert vrar.kernel_name(8, 524288, bf, "rd") == "k_rd_wide"
        assert vrar.kernel_name(8, 524288, torch.float32, "rd") == "k_rd"   # fp32 data already travels as fp32
    finally:
        vrar.set_payload_wire("element")
    for bad in ((0, 10), (33, 10)):
        with pytest.raises(vrar.VrarError):
            vrar.kernel_name(bad[0], bad[1], bf, "auto")


def test_fp8_write_kernel_table():
    """With fp8 payloads on, the write kernel comes from its own measured table
    (the arithmetic, not memory, bounds it); the algorithm AUTO runs does not
    change (one-shot and write mode pass different values through the wire)."""
    bf = torch.bfloat16
    if os.environ.get("VRAR_WRITE_KERNEL") or os.environ.get("VRAR_ALGO"):
        pytest.skip("an override is set in the environment")
    algos = {(P, n): vrar.select_algo(P, n, bf) for P in (2, 4, 8, 32) for n in (1 << 14, 1 << 20, 1 << 24)}
    vrar.set_fp8_quant(True)
    try:
        assert vrar.kernel_name(32, 1 << 20, bf, "twostage_write") == "k_twostage_write"          # 32 x 2 MiB
        assert vrar.kernel_name(32, 1 << 16, bf, "twostage_write") == "k_twostage_write_async"    # 32 x 128 KiB
        assert vrar.kernel_name(8, 1 << 19, bf, "twostage_write") == "k_twostage_write"           # 8 x 1 MiB
        assert vrar.kernel_name(8, 1 << 20, bf, "twostage_write") == "k_twostage_write_batched"   # 8 x 2 MiB
        assert vrar.kernel_name(8, 1 << 21, bf, "twostage_write") == "k_twostage_write_async"     # 8 x 4 MiB
        assert vrar.kernel_name(4, 1 << 23, bf, "twostage_write") == "k_twostage_write_staged"    # 4 x 16 MiB
        assert vrar.kernel_name(8, 117440512, bf, "auto") == "k_twostage_write_async"             # prefill
        assert {(P, n): vrar.select_algo(P, n, bf) for P, n in algos} == algos
    finally:
        vrar.set_fp8_quant(False)
    assert vrar.kernel_name(8, 117440512, bf, "auto") == "k_twostage_write"


def test_payload_wire_setting():
    assert vrar.get_payload_wire() == "element"
    assert L.vrar_set_payload_wire(7) == vrar.EINVAL
    vrar.set_payload_wire("fp32")
    try:
        assert vrar.get_payload_wire() == "fp32"
        # fp32 partials of bf16: twice the slot bytes; fp32 elements unchanged; one-shot needs none
        # (no device here: the bound for any grid, twice the one-round size)
        if not torch.cuda.is_available():
            assert vrar.workspace_bytes(8, 1 << 20, torch.bfloat16, "rd") == 2 * 2 * 8 * 3 * 131072 * 32
            assert vrar.workspace_bytes(8, 1 << 20, torch.float32, "rd") == 2 * 8 * 3 * 262144 * 32
            assert vrar.workspace_bytes(32, 1 << 20, torch.float16, "hier") == 2 * 2 * 32 * 2 * 16384 * 32
        assert vrar.workspace_bytes(8, 1 << 20, torch.bfloat16, "oneshot") == 0
        # the allocation-free entry point's limit halves for bf16 with fp32 partials
        f = L.vrar_allreduce_rd_noalloc
        assert f(_ptrs(IN, 8), _ptrs(OUT, 8), 8, 87_380 + 8, 0, None) == vrar.ETOOBIG
    finally:
        vrar.set_payload_wire("element")


@pytest.mark.skipif(torch.cuda.is_available(), reason="the device-independent bound applies without a GPU")
def test_workspace_bytes_without_a_device():
    """Without a device the slot bytes of a shape are bounded for any grid:
    one round over the whole message takes P x steps x items x 32 bytes, and
    several rounds take two slot sets of fewer slots, so twice that."""
    # RD at P=8 on 2 MiB of bf16 per rank: 8 ranks x 3 steps x 131072 items x 32 bytes, twice
    assert vrar.workspace_bytes(8, 1 << 20, torch.bfloat16, "rd") == 2 * 8 * 3 * 131072 * 32
    # HIER 4 x 8 on 2 MiB: 32 ranks x 2 steps x (131072 / 8) items x 32 bytes, twice
    assert vrar.workspace_bytes(32, 1 << 20, torch.bfloat16, "hier") == 2 * 32 * 2 * 16384 * 32


def test_workspace_bytes_of_algorithms_without_payloads():
    assert vrar.workspace_bytes(8, 1 << 20, torch.bfloat16, "oneshot") == 0
    assert vrar.workspace_bytes(3, 1 << 20, torch.bfloat16, "rd") == 0
