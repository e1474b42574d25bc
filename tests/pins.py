"""Checks that pin the CPU oracle to facts other than itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with what the mathematics or the sources fix:

* torch's float32 -> bfloat16 conversion (a library routine for the textbook
  round-to-nearest-even) on every bf16 boundary pattern, and numpy's
  float32 -> float16 conversion on every tie point of every binary16 value;
* exact integer sums (every algorithm must return the exact sum of small
  integers, which bf16 and fp32 hold exactly) by brute force;
* closed forms of a periodic integer pattern;
* hand-derived results on inputs chosen so that the summation order, the
  recursive-doubling pairing, the group mapping and ties each change the bits
  (tests/golden/order_cases.json, derivations included);
* the error bound against math.fsum;
* numpy's sequential float32 accumulate (a library left fold);
* invariants the sources imply (all ranks equal; one-shot = 2-stage; chunk
  count and special shapes reduce to the simpler algorithms).

The same checks run against deliberately broken builds of the oracle, each of
which must fail at least one of them.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import synth
from util import bits_of, gen, hexvals, load_golden, parse_algo, to_np

POW2 = (1, 2, 4, 8, 16, 32)


def _all_equal(outs):
    b0 = bits_of(outs[0])
    return all((bits_of(o) == b0).all() for o in outs)


def _algos_for(P):
    """(algo, L) pairs defined for P ranks."""
    out = [("oneshot", 8), ("twostage", 8), ("twostage_write", 8)]
    if P & (P - 1) == 0:
        out += [("rd", 8), ("rd_fp32wire", 8)]
        L = 1
        while L <= P:
            out += [("hier", L), ("hier_fp32wire", L)]
            L *= 2
    return out


def pin_bf16_round_vs_torch(o):
    hi = np.arange(65536, dtype=np.uint32) << 16
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF], np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    rng = np.random.default_rng(12345)
    bits = np.concatenate([bits, rng.integers(0, 2**32, 300_000, dtype=np.uint64).astype(np.uint32)])
    f = bits.view(np.float32)
    ours = o.bf16_round(f)
    ref = to_np(torch.from_numpy(f.copy()).to(torch.bfloat16))
    nan = np.isnan(f)
    assert (ours[~nan] == ref[~nan]).all(), "bf16 rounding differs from torch on finite/inf inputs"
    assert (ours[nan] == 0x7FC0).all(), "NaN must round to 0x7FC0"


def pin_bf16_round_hand(o):
    cases = [
        (1.0, 0x3F80),
        (1.0 + 2**-8, 0x3F80),            # tie -> even (down)
        (1.0 + 3 * 2**-8, 0x3F82),        # tie -> even (up)
        (1.0 + 2**-8 + 2**-20, 0x3F81),   # above the tie
        (-(1.0 + 2**-8), 0xBF80),
        (2**-30, 0x3080),
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (float("inf"), 0x7F80),
        (-float("inf"), 0xFF80),
        (3.3895313892515355e38, 0x7F7F),  # largest finite bf16
        (2**-133, 0x0001),                # smallest bf16 subnormal
    ]
    x = np.array([c[0] for c in cases], np.float32)
    want = np.array([c[1] for c in cases], np.uint16)
    assert (o.bf16_round(x) == want).all()
    # half way between the largest finite bf16 (odd significand) and 2^128 -> infinity
    edge = np.array([0x7F7F8000], np.uint32).view(np.float32)
    assert o.bf16_round(edge)[0] == 0x7F80


def pin_bf16_widen(o):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = o.bf16_widen(h).view(np.uint32)
    ref = torch.from_numpy(h.view(np.int16).copy()).view(torch.bfloat16).to(torch.float32).numpy().view(np.uint32)
    fin = ~np.isnan(ours.view(np.float32))
    assert (ours[fin] == ref[fin]).all()
    assert (ours == (h.astype(np.uint32) << 16)).all(), "widening appends 16 zero bits"


def pin_fp16_round_vs_numpy(o):
    """Every tie point and its neighbours for every finite binary16 value (both
    signs), plus random binary32 patterns, against numpy's float32 -> float16
    conversion (a library routine for round-to-nearest-even)."""
    h = np.arange(0x7C00, dtype=np.uint32).astype(np.uint16)            # finite, positive
    lo = h.view(np.float16).astype(np.float32)
    hi = (h.astype(np.uint32) + 1).astype(np.uint16).view(np.float16).astype(np.float32)
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) / 2            # exact in binary32
    mid32 = mid.astype(np.float32)
    assert (mid32.astype(np.float64) == mid).all()
    pts = [lo, mid32, np.nextafter(mid32, np.float32(0)), np.nextafter(mid32, np.float32(np.inf))]
    x = np.concatenate(pts)
    x = np.concatenate([x, -x])
    rng = np.random.default_rng(7)
    x = np.concatenate([x, rng.integers(0, 2**32, 500_000, dtype=np.uint64).astype(np.uint32).view(np.float32)])
    with np.errstate(over="ignore", invalid="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    ours = o.fp16_round(x)
    nan = np.isnan(x)
    assert (ours[~nan] == ref[~nan]).all(), "fp16 rounding differs from numpy"
    assert (ours[nan] == 0x7E00).all()


def pin_fp16_widen(o):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = o.fp16_widen(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert (ours.view(np.uint32)[~nan] == ref.view(np.uint32)[~nan]).all()


def pin_fp16_round_hand(o):
    cases = [(1.0, 0x3C00), (1.0 + 2**-11, 0x3C00), (1.0 + 3 * 2**-11, 0x3C02), (65504.0, 0x7BFF),
             (65519.0, 0x7BFF), (65520.0, 0x7C00), (2**-24, 0x0001), (2**-25, 0x0000), (3 * 2**-26, 0x0001),
             (1.5 * 2**-24, 0x0002), (2**-14, 0x0400), (2**-14 - 2**-25, 0x0400), (-0.0, 0x8000),
             (-(1.0 + 2**-11), 0xBC00)]
    x = np.array([c[0] for c in cases], np.float32)
    want = np.array([c[1] for c in cases], np.uint16)
    assert (o.fp16_round(x) == want).all()


def pin_integer_sums(o, n_values=tuple(range(1, 68)), P_values=(1, 2, 3, 4, 5, 8, 16, 32)):
    for dtype in ("bf16", "fp32", "fp16"):
        for P in P_values:
            for n in n_values:
                xs = gen(P, n, dtype, synth.INT8, seed=1000 + P * 97 + n)
                ints = np.stack([o.to_float(x, dtype) for x in xs]).astype(np.int64)
                exact = ints.sum(axis=0)
                for algo, L in _algos_for(P):
                    if algo == "hier" and L > P:
                        continue
                    outs = o.allreduce(algo, xs, dtype, L=L, chunks=3)
                    assert _all_equal(outs), f"{algo} L={L} P={P} n={n}: ranks differ"
                    got = o.to_float(outs[0], dtype)
                    assert (got == exact).all(), f"{algo} L={L} P={P} n={n} {dtype}: not the exact integer sum"


def pin_closed_form(o):
    """x_p[i] = ((7p + i) mod 17) - 8. Over a full period of 17 ranks the values
    are a permutation of -8..8 (7 is invertible mod 17) and sum to 0, so:
    P=2: (i mod 17) + ((7 + i) mod 17) - 16;
    P=16 = 17 - 1: minus the p=16 term = 8 - ((112 + i) mod 17) = 8 - ((10 + i) mod 17);
    P=32 = 17 + 15: minus the p=15 and p=16 terms of a second period
          = 16 - ((3 + i) mod 17) - ((10 + i) mod 17)."""
    n = 40
    i = np.arange(n)
    closed = {
        2: (i % 17) + ((7 + i) % 17) - 16,
        16: 8 - ((10 + i) % 17),
        32: 16 - ((3 + i) % 17) - ((10 + i) % 17),
    }
    for dtype in ("bf16", "fp32", "fp16"):
        for P, want in closed.items():
            vals = [(((7 * p + i) % 17) - 8).astype(np.float32) for p in range(P)]
            xs = [(v.view(np.uint32) >> 16).astype(np.uint16) if dtype == "bf16"
                  else v.astype(np.float16).view(np.uint16) if dtype == "fp16" else v for v in vals]
            for algo, L in _algos_for(P):
                outs = o.allreduce(algo, xs, dtype, L=L)
                got = o.to_float(outs[0], dtype)
                assert (got == want).all(), f"{algo} L={L} P={P}: closed form"
                assert _all_equal(outs)


def pin_golden_order(o):
    g = load_golden()
    for case in g["cases"]:
        dt = case["dtype"]
        xs = [hexvals(row, dt) for row in case["inputs"]]
        for spec, want_strs in case["expect"].items():
            algo, L = parse_algo(spec)
            want = hexvals(want_strs, dt)
            outs = o.allreduce(algo, xs, dt, L=L if L is not None else 8, chunks=1)
            for r, out in enumerate(outs):
                assert (bits_of(out) == bits_of(want)).all(), \
                    f"{case['name']} {spec} rank {r}: got {o.to_float(out, dt)} want {o.to_float(want, dt)}"


def pin_error_bound(o):
    """|y - S| <= rtol * A with S, A from math.fsum (independent of the oracle's
    own fp64 helper, which is checked here too)."""
    rtol = {"bf16": 1e-2, "fp32": 1e-5, "fp16": 5e-3}
    for dtype in ("bf16", "fp32", "fp16"):
        for P in (2, 8, 32):
            n = 300
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=7 + P)
            f = np.stack([o.to_float(x, dtype) for x in xs])
            S = np.array([math.fsum(f[:, k]) for k in range(n)])
            A = np.array([math.fsum(np.abs(f[:, k])) for k in range(n)])
            S2, A2 = o.fp64_reference(xs, dtype)
            assert np.array_equal(S, S2) and np.array_equal(A, A2), "fp64 reference is not the exact sum"
            for algo, L in _algos_for(P):
                outs = o.allreduce(algo, xs, dtype, L=L)
                y = o.to_float(outs[0], dtype)
                assert (np.abs(y - S) <= rtol[dtype] * A).all(), f"{algo} L={L} P={P} {dtype}: outside error bound"
                # The result is also close in the normwise sense.
                assert np.linalg.norm(y - S) <= rtol[dtype] * np.linalg.norm(A)


def pin_fp32_left_fold(o):
    """fp32 one-shot equals numpy's sequential float32 accumulate over ranks."""
    for P in (2, 3, 8, 32):
        xs = gen(P, 257, "fp32", synth.normal(0.0, 1.0), seed=P)
        fold = np.add.accumulate(np.stack(xs).astype(np.float32), axis=0, dtype=np.float32)[-1]
        for algo in ("oneshot", "twostage", "twostage_write"):
            outs = o.allreduce(algo, xs, "fp32")
            assert (outs[0].view(np.uint32) == fold.view(np.uint32)).all(), f"{algo} P={P}: not the left fold"


def pin_invariants(o):
    for dtype in ("bf16", "fp32", "fp16"):
        for P in (1, 2, 4, 8, 32):
            n = 531  # several 16-byte vectors, a ragged tail
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=40 + P)
            one = o.allreduce("oneshot", xs, dtype)
            assert _all_equal(one)
            for algo in ("twostage", "twostage_write"):
                outs = o.allreduce(algo, xs, dtype)
                assert _all_equal(outs) and (bits_of(outs[0]) == bits_of(one[0])).all(), f"{algo} != oneshot"
            rd = [o.allreduce("rd", xs, dtype, chunks=c) for c in (1, 2, 4, 7)]
            for outs in rd:
                assert _all_equal(outs) and (bits_of(outs[0]) == bits_of(rd[0][0])).all(), "rd depends on chunks"
            assert (bits_of(o.allreduce("hier", xs, dtype, L=P)[0]) == bits_of(one[0])).all(), "hier G=1 != oneshot"
            assert (bits_of(o.allreduce("hier", xs, dtype, L=1)[0]) == bits_of(rd[0][0])).all(), "hier L=1 != rd"
            rd32 = o.allreduce("rd_fp32wire", xs, dtype)
            assert _all_equal(rd32)
            assert (bits_of(o.allreduce("hier_fp32wire", xs, dtype, L=1)[0]) == bits_of(rd32[0])).all()
            assert (bits_of(o.allreduce("hier_fp32wire", xs, dtype, L=P)[0]) == bits_of(one[0])).all(), \
                "one group with fp32 partials is the one-shot fold"
            if dtype == "fp32":
                assert (bits_of(rd32[0]) == bits_of(rd[0][0])).all(), "fp32 elements: the wires agree"
            if P <= 2:
                assert (bits_of(rd32[0]) == bits_of(one[0])).all(), "P<=2: one add, one rounding"
            if P <= 2:
                assert (bits_of(rd[0][0]) == bits_of(one[0])).all(), "P<=2: rd != oneshot"
            if P == 1:
                assert (bits_of(one[0]) == bits_of(xs[0])).all(), "P=1 must copy"
            # A real reduction happened (P >= 2): outputs differ from the inputs.
            if P >= 2:
                assert not (bits_of(one[0]) == bits_of(xs[0])).all()


def pin_rs_ag(o):
    for dtype in ("bf16", "fp32", "fp16"):
        for P in (1, 2, 3, 8, 32):
            m = 37
            n = m * P
            xs = gen(P, n, dtype, synth.INT8, seed=500 + P)
            ints = np.stack([o.to_float(x, dtype) for x in xs]).astype(np.int64).sum(axis=0)
            rs = o.reduce_scatter(xs, dtype)
            for p in range(P):
                assert (o.to_float(rs[p], dtype) == ints[p * m:(p + 1) * m]).all(), "reduce-scatter slice"
            xn = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=600 + P)
            rs = o.reduce_scatter(xn, dtype)
            one = o.allreduce("oneshot", xn, dtype)
            for p in range(P):
                assert (bits_of(rs[p]) == bits_of(one[0][p * m:(p + 1) * m])).all(), "RS != slice of one-shot"
            sl = gen(P, m, dtype, synth.normal(0.0, 1.0), seed=700 + P)
            ag = o.all_gather(sl, dtype)
            cat = np.concatenate(sl)
            for p in range(P):
                assert (bits_of(ag[p]) == bits_of(cat)).all(), "all-gather is not the concatenation"


def pin_shape_errors(o):
    xs = gen(3, 16, "bf16", synth.INT8)
    for algo, L in (("rd", 8), ("hier", 1)):
        try:
            o.allreduce(algo, xs, "bf16", L=L)
        except ValueError:
            pass
        else:
            raise AssertionError(f"{algo} with P=3 must be rejected")
    xs = gen(12, 16, "bf16", synth.INT8)
    try:
        o.allreduce("hier", xs, "bf16", L=4)  # G = 3 is not a power of two
    except ValueError:
        pass
    else:
        raise AssertionError("hier with G=3 must be rejected")


ALL_PINS = [
    pin_bf16_round_vs_torch,
    pin_bf16_round_hand,
    pin_bf16_widen,
    pin_fp16_round_vs_numpy,
    pin_fp16_widen,
    pin_fp16_round_hand,
    pin_integer_sums,
    pin_closed_form,
    pin_golden_order,
    pin_error_bound,
    pin_fp32_left_fold,
    pin_invariants,
    pin_rs_ag,
    pin_shape_errors,
]
