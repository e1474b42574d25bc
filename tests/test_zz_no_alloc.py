"""The allocation-free entry point, vrar_allreduce_rd_noalloc, on the GPU.

It is for callers that cannot let the library allocate device memory (their
own allocator owns the GPU's memory, or they must not wait on the
synchronisation an allocation can imply): its scratch is a fixed array inside
the library. It must give exactly what the oracle's recursive doubling gives,
and exactly what vrar_allreduce with the recursive-doubling algorithm gives.
This file is named so that pytest collects it last; it also passes on its own
in a fresh process.
"""

import os
import subprocess
import sys
import textwrap

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

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RTOL = {"bf16": 1e-2, "fp32": 1e-5, "fp16": 5e-3}
DT = {"bf16": 0, "fp32": 1, "fp16": 2}


@pytest.fixture(autouse=True)
def _defaults():
    yield
    if vrar is not None:
        vrar.set_payload_wire("element")
        vrar.set_max_ctas(0)
        vrar.set_spin_timeout_ns(2_000_000_000)
        vrar.debug_set_fault_mask(0)


def _noalloc(d_in, outs, P, n, dtype, stream=None):
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return vrar.lib().vrar_allreduce_rd_noalloc(vrar.ptr_array([t.data_ptr() for t in d_in]),
                                                vrar.ptr_array([t.data_ptr() for t in outs]), P, n, DT[dtype], s)


# (P, n, dtype, wire, CTA budget): a tiny ragged case, the P=2 128 KiB shape, a
# several-CTA ragged case, the largest request the fixed scratch holds at P = 8
# (256 + 8 * 3 * ceil(n / e) * 32 * w <= 16 MiB: n <= 174,760 bf16, 87,380
# fp32, 87,376 bf16 with fp32 partials on the wire), and calls whose CTA budget
# makes the grid too small for one round, so that the slots are reused round
# by round; and 2 ranks with fp32 partials at the limit (256 + 2 * 1 * 131,070
# * 64 bytes), which needs several rounds.
CASES = [(4, 7, "bf16", "element", 0), (2, 65_536, "bf16", "element", 0), (8, 100_003, "bf16", "element", 0),
         (8, 174_760, "bf16", "element", 0), (4, 7, "fp32", "element", 0), (2, 65_536, "fp32", "element", 0),
         (8, 50_003, "fp32", "element", 0), (8, 87_380, "fp32", "element", 0), (8, 50_001, "fp16", "element", 0),
         (8, 87_376, "bf16", "fp32", 0),
         (8, 100_003, "bf16", "element", 16), (16, 60_001, "fp16", "element", 16), (8, 87_376, "bf16", "fp32", 16),
         (2, 1_048_560, "bf16", "fp32", 0)]  # several rounds at the limit: both slot sets within it


@pytest.mark.parametrize("P,n,dtype,wire,budget", CASES)
def test_noalloc_matches_oracle_and_allocating_rd_on_two_calls(P, n, dtype, wire, budget):
    vrar.set_payload_wire(wire)
    vrar.set_max_ctas(budget)
    xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=900 + P)
    want = oracle.allreduce("rd_fp32wire" if wire == "fp32" else "rd", xs, dtype)
    S, A = oracle.fp64_reference(xs, dtype)
    d_in = [from_np(x, dtype).cuda() for x in xs]
    ref = vrar.all_reduce(d_in, algo="rd")
    rc, info = vrar.query_status()
    assert rc == 0, info
    ref_np = [to_np(t) for t in ref]
    outs = [torch.empty_like(t) for t in d_in]
    for call in range(2):
        for t in outs:
            t.fill_(float("nan"))
        rc = _noalloc(d_in, outs, P, n, dtype)
        assert rc == vrar.OK, vrar.strerror(rc)
        rc, info = vrar.query_status()
        assert rc == 0, (call, info)
        for p in range(P):
            got = to_np(outs[p])
            assert np.array_equal(bits_of(got), bits_of(want[p])), f"call {call} rank {p}: differs from the oracle"
            assert np.array_equal(bits_of(got), bits_of(ref_np[p])), f"call {call} rank {p}: differs from vrar_allreduce"
            y = oracle.to_float(got, dtype)
            assert (np.abs(y - S) <= RTOL[dtype] * A).all(), f"call {call} rank {p}: tolerance"


@pytest.mark.parametrize("P,n,dtype,wire", [(8, 174_761, "bf16", "element"), (8, 87_381, "fp32", "element"),
                                            (8, 87_377, "bf16", "fp32"), (32, 26_209, "fp16", "element"),
                                            (2, 1_048_561, "bf16", "fp32")])
def test_noalloc_rejects_one_past_the_limit_and_queues_nothing(P, n, dtype, wire):
    """One element past the limit (for 32 ranks: 256 + 32 * 5 * 3277 * 32 > 16 MiB)
    is refused before anything is queued: the outputs keep their contents."""
    vrar.set_payload_wire(wire)
    d_in = [torch.ones(n, dtype=getattr(torch, {"bf16": "bfloat16", "fp32": "float32", "fp16": "float16"}[dtype]),
                       device="cuda") for _ in range(P)]
    outs = [torch.full_like(t, 7.0) for t in d_in]
    assert _noalloc(d_in, outs, P, n, dtype) == vrar.ETOOBIG
    torch.cuda.synchronize()
    for o in outs:
        assert bool((o == 7.0).all())
    assert vrar.query_status()[0] == 0


def test_noalloc_timeout_is_reported_and_the_next_call_is_correct():
    """A rank that never sends (host-set fault mask) makes its partners' waits
    run out; the timeout is recorded in the fixed array and vrar_query_status
    reports and clears it; the next call is bit-exact again."""
    P, n, dtype = 4, 40_000, "bf16"
    xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=77)
    want = oracle.allreduce("rd", xs, dtype)
    d_in = [from_np(x, dtype).cuda() for x in xs]
    outs = [torch.empty_like(t) for t in d_in]
    vrar.set_spin_timeout_ns(20_000_000)
    vrar.debug_set_fault_mask(1 << 1)
    assert _noalloc(d_in, outs, P, n, dtype) == vrar.OK
    rc, info = vrar.query_status()
    assert rc == vrar.ETIMEDOUT, (rc, info)
    assert info[1] == 4, info  # the payload phase
    assert vrar.query_status()[0] == 0, "the status must be cleared by the query"
    vrar.debug_set_fault_mask(0)
    assert _noalloc(d_in, outs, P, n, dtype) == vrar.OK
    assert vrar.query_status()[0] == 0
    for p in range(P):
        assert np.array_equal(to_np(outs[p]), want[p]), f"rank {p} after the timeout"


FRESH = textwrap.dedent("""
    import ctypes, sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import numpy as np
    import torch
    import collective_all_reduce_virtual_b200 as vrar
    import oracle, synth
    from util import from_np, gen, to_np

    import json
    lib = vrar.lib()
    stages = {{}}
    cases = [(8, 100_003, "bf16", 1), (2, 65_536, "fp32", 1), (8, 174_760, "bf16", 2), (4, 9, "fp16", 1)]
    data = []
    for P, n, dtype, seed in cases:
        xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=seed)
        d_in = [from_np(x, dtype).cuda() for x in xs]
        outs = [torch.empty_like(t) for t in d_in]
        data.append((P, n, dtype, xs, d_in, outs))
    torch.cuda.synchronize()
    stages["inputs"] = torch.cuda.mem_get_info()[0]
    # The driver sets a context up further at its first kernel launch, whoever
    # launches it; one unrelated kernel takes that out of the measurement.
    torch.ones(1024, device="cuda").add_(1)
    torch.cuda.synchronize()
    stages["first_kernel"] = torch.cuda.mem_get_info()[0]
    # Start this library's CUDA runtime (with CUDA_MODULE_LOADING=EAGER its
    # module, fixed array included, is loaded here) without allocating anything.
    assert lib.vrar_query_status(None, None) == 0
    side = torch.cuda.Stream()  # created non-blocking: not ordered with the legacy default stream
    torch.cuda.synchronize()
    stages["runtime"] = free0 = torch.cuda.mem_get_info()[0]
    for k, (P, n, dtype, xs, d_in, outs) in enumerate(data):
        rc = lib.vrar_allreduce_rd_noalloc(vrar.ptr_array([t.data_ptr() for t in d_in]),
                                           vrar.ptr_array([t.data_ptr() for t in outs]), P, n,
                                           {{"bf16": 0, "fp32": 1, "fp16": 2}}[dtype], side.cuda_stream)
        assert rc == 0, (k, rc)
        side.synchronize()
        stages[f"call{{k}}"] = torch.cuda.mem_get_info()[0]
    print(json.dumps(stages))
    for k in range(len(data)):
        assert stages[f"call{{k}}"] == free0, ("device memory changed", k, stages)
    rc, info = vrar.query_status()
    assert rc == 0, info
    for P, n, dtype, xs, d_in, outs in data:
        want = oracle.allreduce("rd", xs, dtype)
        for p in range(P):
            assert np.array_equal(to_np(outs[p]), want[p]), (P, n, dtype, p)
    print("ok")
""")


def test_noalloc_first_call_in_a_fresh_process_on_a_side_stream_allocates_nothing():
    """In a fresh process, the first call (which sets the device up) runs on a
    non-blocking stream, and neither it nor the calls after it change the
    device's free memory; all of them match the oracle. The driver's own
    set-up of the context at its first kernel launch is taken out first (one
    unrelated kernel), and the library's code is loaded eagerly, because
    neither is an allocation this entry point makes."""
    code = FRESH.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]
