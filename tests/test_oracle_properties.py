"""Property tests of the CPU oracle on random inputs (Hypothesis).

The fixed-input pins (tests/pins.py) use seeded normal and integer data. Here
Hypothesis draws rank counts, lengths, element types and raw values,
subnormals, signed zeros and large exponents included (bounded so that no sum
can overflow), and checks what must hold for any input:

* every rank's output is the same, and one-shot, 2-stage and write mode agree
  bit for bit (one fixed order);
* the special shapes reduce to the simpler algorithms: P <= 2 recursive
  doubling is one-shot, a single group is one-shot, groups of one are
  recursive doubling, and the chunk count changes nothing;
* every result is within the error bound of the exact sum (math.fsum):
  |y - S| <= rtol * A + 8 * (the type's smallest subnormal);
* the reduction is elementwise: rotating every rank's vector by k rotates the
  outputs by k (a slice, chunk or group boundary that mixed up indices would
  break this).
"""

from __future__ import annotations

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from util import bits_of

RTOL = {"bf16": 1e-2, "fp32": 1e-5, "fp16": 5e-3}
TINY = {"bf16": 2.0 ** -133, "fp32": 2.0 ** -149, "fp16": 2.0 ** -24}


def _values(dtype, n):
    if dtype == "fp32":
        val = st.floats(min_value=-2.0 ** 100, max_value=2.0 ** 100, allow_nan=False, allow_infinity=False, width=32)
        return st.lists(val, min_size=n, max_size=n).map(lambda v: np.array(v, np.float32))
    if dtype == "bf16":  # exponent field <= 0xF0: |x| < 2^114, so 32 of them stay finite in fp32
        pat = st.integers(0, 0xFFFF).filter(lambda b: ((b >> 7) & 0xFF) <= 0xF0)
    else:  # fp16: exponent field <= 0x17 (|x| < 512), so 32 of them stay below 65504
        pat = st.integers(0, 0xFFFF).filter(lambda b: ((b >> 10) & 0x1F) <= 0x17)
    return st.lists(pat, min_size=n, max_size=n).map(lambda v: np.array(v, np.uint16))


@st.composite
def cases(draw):
    dtype = draw(st.sampled_from(["bf16", "fp32", "fp16"]))
    P = draw(st.sampled_from([1, 2, 3, 4, 5, 8, 16, 32]))
    n = draw(st.integers(1, 40))
    xs = [draw(_values(dtype, n)) for _ in range(P)]
    return dtype, P, n, xs


def _same(a, b):
    return np.array_equal(bits_of(a), bits_of(b))


@settings(max_examples=150, derandomize=True, deadline=None)
@given(cases())
def test_orders_agree_and_special_shapes_reduce(case):
    dtype, P, n, xs = case
    one = oracle.allreduce("oneshot", xs, dtype)
    assert all(_same(o, one[0]) for o in one)
    for algo in ("twostage", "twostage_write"):
        outs = oracle.allreduce(algo, xs, dtype)
        assert all(_same(o, one[0]) for o in outs), algo
    if P & (P - 1) == 0:
        rd = oracle.allreduce("rd", xs, dtype, chunks=1)
        assert all(_same(o, rd[0]) for o in rd)
        assert _same(oracle.allreduce("rd", xs, dtype, chunks=5)[0], rd[0]), "rd depends on the chunk count"
        assert _same(oracle.allreduce("hier", xs, dtype, L=P)[0], one[0]), "one group is one-shot"
        assert _same(oracle.allreduce("hier", xs, dtype, L=1)[0], rd[0]), "groups of one are rd"
        if P <= 2:
            assert _same(rd[0], one[0]), "P <= 2: rd is one add and one rounding"


@settings(max_examples=150, derandomize=True, deadline=None)
@given(cases())
def test_results_are_within_the_error_bound(case):
    dtype, P, n, xs = case
    f = np.stack([oracle.to_float(x, dtype) for x in xs])
    S = np.array([math.fsum(f[:, k]) for k in range(n)])
    A = np.array([math.fsum(np.abs(f[:, k])) for k in range(n)])
    algos = [("oneshot", 8)] + ([("rd", 8), ("hier", max(1, P // 2))] if P & (P - 1) == 0 else [])
    for algo, L in algos:
        y = oracle.to_float(oracle.allreduce(algo, xs, dtype, L=L)[0], dtype)
        assert (np.abs(y - S) <= RTOL[dtype] * A + 8 * TINY[dtype]).all(), (algo, L)


@settings(max_examples=100, derandomize=True, deadline=None)
@given(cases(), st.integers(0, 39))
def test_the_reduction_is_elementwise(case, k):
    dtype, P, n, xs = case
    k %= n
    rolled = [np.roll(x, k) for x in xs]
    algos = ["oneshot", "twostage_write"] + (["rd", "hier"] if P & (P - 1) == 0 else [])
    for algo in algos:
        L = max(1, P // 2)
        a = oracle.allreduce(algo, xs, dtype, L=L)[0]
        b = oracle.allreduce(algo, rolled, dtype, L=L)[0]
        assert _same(np.roll(a, k), b), (algo, k)
