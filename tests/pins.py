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
  count and special shapes reduce to the simpler algorithms);
* for the fp8 payloads (the reading of the custom all-reduce's ca_fp8_quant
  flag): E4M3 rounding against a brute-force search over every finite E4M3
  value decoded from the format's definition (exact fractions) and against
  torch's float8_e4m3fn cast, the group scaling and both fp8 algorithms
  against a numpy restatement, the hand-derived case in
  tests/golden/fp8_cases.json, exact power-of-two scale invariance and an
  error bound.

The same checks run against deliberately broken builds of the oracle, each of
which must fail at least one of them.
"""

from __future__ import annotations

import math
from fractions import Fraction

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


# ---- fp8 payloads: OCP FP8 E4M3, one binary32 scale per group of 8 -------------------------

def _e4m3_values():
    """Every finite non-negative E4M3 value with its code, decoded from the
    format: 1 sign bit, 4 exponent bits biased by 7, 3 fraction bits; exponent
    field 0 holds the subnormals frac/8 * 2^-6; code 0x7F (all ones) is NaN and
    there are no infinities."""
    out = []
    for code in range(0x7F):
        e, f = code >> 3, code & 7
        v = Fraction(f, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(f, 8)) * Fraction(2) ** (e - 7)
        out.append((v, code))
    return out


_E4M3 = _e4m3_values()


def e4m3_brute(x: float) -> float:
    """Nearest E4M3 value to x by exhaustive search over the finite values
    (saturating past the largest, 448); ties go to the even code."""
    a = Fraction(abs(float(x)))
    best = min(_E4M3, key=lambda vc: (abs(vc[0] - a), vc[1] & 1))
    v = float(best[0])
    return -v if math.copysign(1.0, float(x)) < 0 else v


def _e4m3_torch(t32: np.ndarray) -> np.ndarray:
    """torch's float32 -> float8_e4m3fn cast (round to nearest even) and back."""
    return torch.from_numpy(t32).to(torch.float8_e4m3fn).to(torch.float32).numpy()


def fp8_wire_numpy(x32: np.ndarray) -> np.ndarray:
    """The fp8 wire restated in numpy: groups of 8 from index 0; s = amax / 448
    in binary32 (1 if that is 0); q = E4M3(x / s) with torch's cast; q * s in
    binary32. A binary32 quotient or product formed in float64 and then
    rounded to binary32 is the correctly rounded binary32 result (53 >= 2*24+2
    bits), so these match IEEE binary32 division and multiplication."""
    x = np.asarray(x32, np.float32)
    out = np.empty_like(x)
    for g in range(0, x.size, 8):
        grp = x[g:g + 8]
        amax = np.float32(np.max(np.abs(grp))) if grp.size else np.float32(0)
        s = np.float32(np.float64(amax) / 448.0)
        if s == 0:
            s = np.float32(1.0)
        t = (grp.astype(np.float64) / np.float64(s)).astype(np.float32)
        q = _e4m3_torch(t)
        out[g:g + 8] = (q.astype(np.float64) * np.float64(s)).astype(np.float32)
    return out


def _to32(x, dtype):
    if dtype == "bf16":
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x.view(np.float16).astype(np.float32)


def _round_to(y32, dtype):
    if dtype == "bf16":
        return to_np(torch.from_numpy(np.ascontiguousarray(y32)).to(torch.bfloat16))
    return np.ascontiguousarray(y32).astype(np.float16).view(np.uint16)


def pin_e4m3_round_brute(o):
    pts = []
    vals = sorted(v for v, _ in _E4M3)
    for a, b in zip(vals, vals[1:]):
        mid = (a + b) / 2
        m = np.float32(float(mid))
        assert Fraction(float(m)) == mid, "E4M3 midpoints are exact in binary32"
        pts += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9)), np.float32(float(a))]
    pts += [np.float32(v) for v in (448.0, 450.0, 463.99, 464.0, 470.0, 480.0, 1e4, 3e38, 0.0, 2.0**-10,
                                     2.0**-11, 3 * 2.0**-10, 2.0**-9, 2.0**-20, 1e-40)]
    rng = np.random.default_rng(8)
    pts += list((2.0 ** rng.uniform(-14, 9.2, 1500)).astype(np.float32))
    x = np.array(pts, np.float32)
    x = np.concatenate([x, -x])
    got = o.e4m3_round(x)
    want = np.array([e4m3_brute(v) for v in x], np.float32)
    bad = np.nonzero(got.view(np.uint32) != want.view(np.uint32))[0]
    assert bad.size == 0, f"E4M3 rounding differs at {x[bad[:5]]}: {got[bad[:5]]} vs {want[bad[:5]]}"


def pin_e4m3_round_vs_torch(o):
    rng = np.random.default_rng(9)
    x = (rng.uniform(-1, 1, 200_000) * 2.0 ** rng.uniform(-16, 8.85, 200_000)).astype(np.float32)
    x = x[np.abs(x) < 464]  # torch's cast gives NaN from the rounding boundary past 448 on; ours saturates
    got, want = o.e4m3_round(x), _e4m3_torch(x)
    assert (got.view(np.uint32) == want.view(np.uint32)).all(), "E4M3 rounding differs from torch's cast"


def pin_fp8_wire_numpy(o):
    rng = np.random.default_rng(10)
    cases = [rng.normal(0, 1, 531).astype(np.float32),
             (rng.normal(0, 1, 64) * 2.0 ** rng.integers(-30, 30, 64)).astype(np.float32),
             np.zeros(16, np.float32), np.array([-0.0] * 5 + [1e-3] * 3, np.float32),
             np.array([448.0, 1e-6, -2e-5, 3e-4, 0, 5, 6, 7, 1e-30, 2e-30, -3e-30], np.float32)]
    bits = rng.integers(0, 1 << 16, 200, dtype=np.uint32)          # raw bf16 patterns, incl. subnormals
    bits = bits[(bits & 0x7F80) != 0x7F80]                          # finite ones
    cases.append((bits << 16).view(np.float32))
    for x in cases:
        got, want = o.fp8_wire(x), fp8_wire_numpy(x)
        assert (got.view(np.uint32) == want.view(np.uint32)).all(), "fp8 wire differs from the numpy restatement"


def pin_fp8_allreduce_numpy(o):
    for dtype in ("bf16", "fp16"):
        for P in (1, 2, 3, 8):
            n = 531
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=800 + P)
            wired = [fp8_wire_numpy(_to32(x, dtype)) for x in xs]
            acc = wired[0].copy()
            for w in wired[1:]:
                acc = (acc + w).astype(np.float32)  # one binary32 add per element, ascending rank order
            one = _round_to(acc, dtype)
            two = _round_to(fp8_wire_numpy(acc), dtype)
            for algo, want in (("oneshot_fp8", one), ("twostage_fp8", two), ("twostage_write_fp8", two)):
                outs = o.allreduce(algo, xs, dtype)
                assert _all_equal(outs), f"{algo}: ranks differ"
                assert (bits_of(outs[0]) == bits_of(want)).all(), f"{algo} {dtype} P={P}: differs from numpy"


def pin_fp8_golden(o):
    for c in load_golden("fp8_cases.json")["cases"]:
        xs = [hexvals(r, c["dtype"]) for r in c["inputs"]]
        for algo, key in (("oneshot_fp8", "oneshot_fp8"), ("twostage_fp8", "twostage_fp8"),
                          ("twostage_write_fp8", "twostage_fp8")):
            want = hexvals(c[key], c["dtype"])
            for p, out in enumerate(o.allreduce(algo, xs, c["dtype"])):
                assert (bits_of(out) == bits_of(want)).all(), f"{c['name']} {algo} rank {p}"


def pin_fp8_invariants(o):
    rng = np.random.default_rng(11)
    x = rng.normal(0, 1, 1000).astype(np.float32)
    base = o.fp8_wire(x)
    for k in (-20, -7, -1, 1, 5, 20):  # power-of-two scaling is exact at every step
        scaled = o.fp8_wire((x * np.float32(2.0 ** k)).astype(np.float32))
        assert (scaled == (base * np.float32(2.0 ** k)).astype(np.float32)).all(), f"not scale invariant (2^{k})"
    # Groups whose largest magnitude is 448 and whose values are E4M3 values
    # have scale 1 and pass unchanged, so one-shot over them is the plain one-shot.
    vals = np.array(sorted({float(v) for v, _ in _E4M3}), np.float32)
    for dtype in ("bf16", "fp16"):
        xs = []
        for p in range(4):
            g = rng.choice(np.concatenate([vals, -vals]), size=(40, 8)).astype(np.float32)
            g[:, rng.integers(0, 8)] = 448.0 * (1 if p % 2 else -1)
            xs.append(_round_to(g.ravel(), dtype))
        assert (bits_of(o.allreduce("oneshot_fp8", xs, dtype)[0]) == bits_of(o.allreduce("oneshot", xs, dtype)[0])).all()
    # Error bound: each dequantised value is within 2^-4 of its input relative
    # (E4M3 keeps 4 significant bits) plus 2^-10 of the group scale (the
    # subnormal spacing), and the fp32 adds and the final rounding add less
    # than 2^-8 of the magnitudes; the 2-stage wire adds the same again on the sum.
    xs = gen(8, 4099, "bf16", synth.normal(0.0, 1.0), seed=12)
    S, A = o.fp64_reference(xs, "bf16")
    amax_sum = sum(np.repeat(np.abs(_to32(x, "bf16")).reshape(-1, 1)[:4096].reshape(-1, 8).max(axis=1), 8)[:4096]
                   for x in xs)
    y1 = o.to_float(o.allreduce("oneshot_fp8", xs, "bf16")[0], "bf16")[:4096]
    y2 = o.to_float(o.allreduce("twostage_fp8", xs, "bf16")[0], "bf16")[:4096]
    bound1 = (2.0**-4 + 2.0**-8) * A[:4096] + 2.0**-10 / 448 * 1.01 * amax_sum
    assert (np.abs(y1 - S[:4096]) <= bound1).all(), "oneshot_fp8 outside its error bound"
    assert (np.abs(y2 - S[:4096]) <= 2 * bound1 + 2.0**-4 * np.abs(S[:4096])).all(), "twostage_fp8 outside its bound"
    for algo in ("oneshot_fp8", "twostage_fp8"):
        try:
            o.allreduce(algo, gen(2, 8, "fp32", synth.INT8), "fp32")
        except ValueError:
            pass
        else:
            raise AssertionError(f"{algo} must reject fp32 elements")


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
    pin_e4m3_round_brute,
    pin_e4m3_round_vs_torch,
    pin_fp8_wire_numpy,
    pin_fp8_allreduce_numpy,
    pin_fp8_golden,
    pin_fp8_invariants,
]
