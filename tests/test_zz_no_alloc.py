"""The allocation-free entry point, vrar_allreduce_rd_noalloc, on the GPU.

It is for callers that cannot let the library allocate device memory (their
own allocator owns the GPU's memory, or they must not wait on the
synchronisation an allocation can imply): its scratch is a fixed array inside
the library. It must give exactly what vrar_allreduce with the
recursive-doubling algorithm gives. This file is named so that pytest
collects it last; it also passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from util import bits_of, from_np, gen, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import collective_all_reduce_virtual_b200 as vrar
else:  # collected on the CPU machine, never run there
    vrar = None

RTOL = {"bf16": 1e-2, "fp32": 1e-5, "fp16": 5e-3}
DT = {"bf16": 0, "fp32": 1, "fp16": 2}

# (P, n, dtype, wire): a tiny ragged case, the P=2 128 KiB shape, a several-CTA
# ragged case, and the largest request the fixed scratch holds at P = 8
# (8 * 3 * ceil(n / e) * 32 * w + 256 <= 16 MiB: n <= 174,760 bf16, 87,380 fp32,
# 87,376 bf16 with fp32 partials on the wire).
CASES = [(4, 7, "bf16", "element"), (2, 65_536, "bf16", "element"), (8, 100_003, "bf16", "element"),
         (8, 174_760, "bf16", "element"), (4, 7, "fp32", "element"), (2, 65_536, "fp32", "element"),
         (8, 50_003, "fp32", "element"), (8, 87_380, "fp32", "element"), (8, 50_001, "fp16", "element"),
         (8, 87_376, "bf16", "fp32")]  # fp32 partials of bf16: twice the slot bytes per item


@pytest.mark.parametrize("P,n,dtype,wire", CASES)
def test_noalloc_matches_allocating_rd_on_two_calls(P, n, dtype, wire):
    lib = vrar.lib()
    vrar.set_payload_wire(wire)
    xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=900 + P)
    d_in = [from_np(x, dtype).cuda() for x in xs]
    ref = vrar.all_reduce(d_in, algo="rd")
    rc, info = vrar.query_status()
    assert rc == 0, info
    ref_np = [to_np(t) for t in ref]
    S, A = oracle.fp64_reference(xs, dtype)
    outs = [torch.full_like(t, float("nan")) for t in d_in]
    ins_arr = vrar.ptr_array([t.data_ptr() for t in d_in])
    outs_arr = vrar.ptr_array([t.data_ptr() for t in outs])
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        for t in outs:
            t.fill_(float("nan"))
        rc = lib.vrar_allreduce_rd_noalloc(ins_arr, outs_arr, P, n, DT[dtype], stream)
        assert rc == vrar.OK, vrar.strerror(rc)
        torch.cuda.synchronize()
        for p in range(P):
            got = to_np(outs[p])
            assert np.array_equal(bits_of(got), bits_of(ref_np[p])), f"call {call} rank {p}"
            y = oracle.to_float(got, dtype)
            assert (np.abs(y - S) <= RTOL[dtype] * A).all(), f"call {call} rank {p}: tolerance"
    vrar.set_payload_wire("element")

