"""Property test of the C ABI's host-side argument checks (CPU only).

Hypothesis draws rank counts, sizes, element types, the entry point
(all-reduce, reduce-scatter, all-gather) and fake 16-byte-aligned addresses
packed into a small range, so that overlaps are common, and sometimes a
misaligned pointer. The expected return code comes from a plain interval
model of the header's rules: a misaligned pointer, or an output that
overlaps any input or another output, is VRAR_EINVAL (inputs may overlap
each other: they are only read); anything else passes the host checks and,
with no device present, fails as VRAR_ECUDA when the call looks for one.

These calls would launch kernels on fake addresses on a machine with a GPU,
so they run only where there is none.
"""

import pytest
import torch
from hypothesis import event, given, settings
from hypothesis import strategies as st

import collective_all_reduce_virtual_b200 as vrar

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a GPU")

L = vrar.lib()
ESZ = {0: 2, 1: 4, 2: 2}  # VRAR_BF16, VRAR_FP32, VRAR_FP16
BASE = 1 << 40


def _overlap(a, alen, b, blen):
    return a < b + blen and b < a + alen


def expected(ins, outs, in_bytes, out_bytes):
    if any(p % 16 for p in ins + outs):
        return vrar.EINVAL
    for q, o in enumerate(outs):
        if any(_overlap(o, out_bytes, i, in_bytes) for i in ins):
            return vrar.EINVAL
        if any(_overlap(o, out_bytes, o2, out_bytes) for o2 in outs[q + 1:]):
            return vrar.EINVAL
    return vrar.ECUDA


@settings(max_examples=500, derandomize=True, deadline=None)
@given(data=st.data())
def test_host_checks_follow_the_interval_rules(data):
    P = data.draw(st.integers(1, 8), label="P")
    dt = data.draw(st.sampled_from([0, 1, 2]), label="dtype")
    kind = data.draw(st.sampled_from(["allreduce", "reduce_scatter", "all_gather"]), label="kind")
    if kind == "allreduce":
        n = data.draw(st.integers(1, 300), label="n")
    else:
        n = P * data.draw(st.integers(1, 40), label="n/P")
    in_elems = n // P if kind == "all_gather" else n
    out_elems = n // P if kind == "reduce_scatter" else n
    in_bytes, out_bytes = in_elems * ESZ[dt], out_elems * ESZ[dt]
    if data.draw(st.booleans(), label="disjoint layout"):
        # Buffers end to end with random gaps, in a random order; then maybe one
        # output shifted back by a few 16-byte units onto whatever precedes it.
        order = data.draw(st.permutations(list(range(2 * P))), label="order")
        gaps = data.draw(st.lists(st.integers(0, 3), min_size=2 * P, max_size=2 * P), label="gaps")
        addrs, at = [0] * (2 * P), BASE
        for k, g in zip(order, gaps):
            at += 16 * g
            addrs[k] = at
            at += -(-(in_bytes if k < P else out_bytes) // 16) * 16
        if data.draw(st.booleans(), label="shift an output"):
            k = data.draw(st.integers(P, 2 * P - 1), label="which output")
            addrs[k] -= 16 * data.draw(st.integers(1, 4), label="units")
    else:
        # Random slots in a range of 1x - 64x the total size, in 16-byte units.
        spread = data.draw(st.sampled_from([1, 4, 16, 64]), label="spread")
        span = max(1, spread * P * (in_bytes + out_bytes) // 16)
        slots = data.draw(st.lists(st.integers(0, span), min_size=2 * P, max_size=2 * P), label="slots")
        addrs = [BASE + 16 * s for s in slots]
    if data.draw(st.integers(0, 9), label="misalign?") == 0:
        k = data.draw(st.integers(0, 2 * P - 1), label="which")
        addrs[k] += data.draw(st.sampled_from([2, 4, 8]), label="by")
    ins, outs = addrs[:P], addrs[P:]
    if kind == "allreduce":
        rc = L.vrar_allreduce(vrar.ptr_array(ins), vrar.ptr_array(outs), P, n, dt, 0, None)
    elif kind == "reduce_scatter":
        rc = L.vrar_reduce_scatter(vrar.ptr_array(ins), vrar.ptr_array(outs), P, n, dt, None)
    else:
        rc = L.vrar_all_gather(vrar.ptr_array(ins), vrar.ptr_array(outs), P, n, dt, None)
    assert rc == expected(ins, outs, in_bytes, out_bytes), (kind, P, n, dt, ins, outs)
    event(f"{kind}: {'EINVAL' if rc == vrar.EINVAL else 'passes the checks' if rc == vrar.ECUDA else rc}")
