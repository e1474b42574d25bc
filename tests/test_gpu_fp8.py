"""fp8 payloads of the custom all-reduce (vrar_set_fp8_quant) against the CPU
oracle, bit for bit, through the C ABI.

The reading of the ca_fp8_quant flag (ROCm/ATOM pull request 1681 page) that
both sides implement: OCP FP8 E4M3 with one binary32 scale amax / 448 per group
of 8 elements; one-shot passes the inputs through it once, the 2-stage variants
pass the inputs and then the reduced binary32 slice. The oracle's side is
pinned in tests/pins.py; the GPU side rounds with the hardware's E4M3
conversion and must agree everywhere, ties and subnormals included.
"""

from __future__ import annotations

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
import synth
from util import bits_of, from_np, gen, hexvals, load_golden, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import collective_all_reduce_virtual_b200 as vrar
else:  # collected on the CPU machine, never run there
    vrar = None

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_NAME = {"oneshot": "oneshot_fp8", "twostage": "twostage_fp8", "twostage_write": "twostage_write_fp8",
               "auto": None}


@pytest.fixture(autouse=True)
def _fp8_on():
    if vrar is not None:
        vrar.set_fp8_quant(True)
    yield
    if vrar is not None:
        vrar.set_fp8_quant(False)
        vrar.set_edge_sync(False)
        vrar.set_max_ctas(0)


def _run(algo, xs, dtype):
    outs = vrar.all_reduce([from_np(x, dtype).cuda() for x in xs], algo=algo)
    rc, info = vrar.query_status()
    assert rc == 0, (rc, info)
    return [to_np(o) for o in outs]


def _want(algo, xs, dtype):
    P, n = len(xs), xs[0].size
    if algo == "auto":
        algo = vrar.select_algo(P, n, {"bf16": torch.bfloat16, "fp16": torch.float16}[dtype])
    return oracle.allreduce(ORACLE_NAME[algo], xs, dtype)


def _assert_bits(got, want, what, dtype=None):
    """Bit for bit; with dtype given, NaNs compare by NaN-ness (a group whose
    binary32 sum overflows comes back as NaN on both sides, in each side's
    canonical NaN encoding)."""
    for p, (g, w) in enumerate(zip(got, want)):
        if dtype is not None:
            gn, wn = np.isnan(oracle.to_float(g, dtype)), np.isnan(oracle.to_float(w, dtype))
            assert (gn == wn).all(), f"{what}: rank {p} NaN at {np.nonzero(gn != wn)[0][:8]}"
            g, w = g[~gn], w[~wn]
        if not np.array_equal(bits_of(g), bits_of(w)):
            bad = np.nonzero(bits_of(g) != bits_of(w))[0]
            raise AssertionError(f"{what}: rank {p} differs at {bad[:8]} (of {bad.size})")


SHAPES = [(P, n) for P in (1, 2, 3, 5, 8) for n in (1, 7, 9, 4099, 100_003)] + \
         [(P, n) for P in (16, 32) for n in (9, 20_011)]


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("P,n", SHAPES)
def test_fp8_matches_oracle(P, n, dtype):
    xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=P * 7 + n)
    for algo in ("oneshot", "twostage", "twostage_write", "auto"):
        _assert_bits(_run(algo, xs, dtype), _want(algo, xs, dtype), f"{algo} P={P} n={n} {dtype}")


def test_fp8_golden_on_the_gpu():
    for c in load_golden("fp8_cases.json")["cases"]:
        xs = [hexvals(r, c["dtype"]) for r in c["inputs"]]
        for algo, key in (("oneshot", "oneshot_fp8"), ("twostage", "twostage_fp8"),
                          ("twostage_write", "twostage_fp8")):
            want = hexvals(c[key], c["dtype"])
            _assert_bits(_run(algo, xs, c["dtype"]), [want] * len(xs), f"{c['name']} {algo}")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_fp8_special_values(dtype):
    """Raw bit patterns: subnormals, signed zeros, values whose quotient by the
    scale lands on E4M3 ties and on the subnormal E4M3 range; groups of zeros;
    sums that overflow binary32 (their group is NaN after the 2-stage's second
    quantisation, whose scale is then infinite)."""
    rng = np.random.default_rng(21)
    P, n = 4, 8 * 997 + 3
    xs = []
    for p in range(P):
        bits = rng.integers(0, 1 << 16, n, dtype=np.uint32).astype(np.uint16)
        if dtype == "bf16":
            bits[(bits & 0x7F80) == 0x7F80] &= 0x3FFF   # no inf / NaN
        else:
            bits[(bits & 0x7C00) == 0x7C00] &= 0x3FFF
        bits[: 8 * 5] = 0                                 # whole groups of zeros
        bits[8 * 5: 8 * 6] = 0x8000                       # a group of negative zeros
        xs.append(bits)
    for algo in ("oneshot", "twostage", "twostage_write"):
        _assert_bits(_run(algo, xs, dtype), _want(algo, xs, dtype), f"{algo} {dtype} special values", dtype)


def test_fp8_with_barriers_and_a_cta_budget():
    xs = gen(8, 300_007, "bf16", synth.normal(0.0, 1.0), seed=5)
    for edge, cap in ((True, 0), (False, 16), (True, 40)):
        vrar.set_edge_sync(edge)
        vrar.set_max_ctas(cap)
        for algo in ("oneshot", "twostage", "twostage_write"):
            _assert_bits(_run(algo, xs, "bf16"), _want(algo, xs, "bf16"), f"{algo} edge={edge} budget={cap}")


def test_fp8_rejects_what_it_does_not_define():
    for dtype, algo in (("fp32", "oneshot"), ("fp32", "twostage_write"), ("bf16", "rd"), ("bf16", "hier")):
        xs = [from_np(x, dtype).cuda() for x in gen(8, 64, dtype, synth.INT8)]
        with pytest.raises(vrar.VrarError) as e:
            vrar.all_reduce(xs, algo=algo)
        assert e.value.code == vrar.ENOTSUP, (dtype, algo)


def test_fp8_error_bound_and_not_the_plain_sum():
    """Within the bound the format gives (2^-4 of each magnitude, 2^-10 of the
    group scale, and the binary32 adds and final rounding), and different from
    the plain all-reduce: a real quantisation happened."""
    P, n = 8, 65_536
    xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=6)
    S, A = oracle.fp64_reference(xs, "bf16")
    amax = sum(np.repeat(np.abs(oracle.to_float(x, "bf16")).reshape(-1, 8).max(axis=1), 8) for x in xs)
    bound = (2.0 ** -4 + 2.0 ** -8) * A + 2.0 ** -10 / 448 * 1.01 * amax
    one = oracle.to_float(_run("oneshot", xs, "bf16")[0], "bf16")
    assert (np.abs(one - S) <= bound).all()
    two = oracle.to_float(_run("twostage_write", xs, "bf16")[0], "bf16")
    assert (np.abs(two - S) <= 2 * bound + 2.0 ** -4 * np.abs(S)).all()
    vrar.set_fp8_quant(False)
    plain = oracle.to_float(_run("oneshot", xs, "bf16")[0], "bf16")
    assert (plain != one).mean() > 0.5


CHILD = textwrap.dedent("""
    import sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import numpy as np
    import collective_all_reduce_virtual_b200 as vrar
    import oracle, synth
    from util import from_np, gen, to_np, bits_of
    vrar.set_fp8_quant(True)
    for dtype in ("bf16", "fp16"):
        for P, n in ((2, 7), (8, 9), (8, 300_007), (13, 4_099), (32, 33_333), (8, 4_194_307)):
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=P + n)
            want = oracle.allreduce("twostage_write_fp8", xs, dtype)
            for edge, cap in ((False, 0), (True, 0), (False, 64)):
                vrar.set_edge_sync(edge)
                vrar.set_max_ctas(cap)
                outs = vrar.all_reduce([from_np(x, dtype).cuda() for x in xs], algo="twostage_write")
                rc, info = vrar.query_status()
                assert rc == 0, (rc, info)
                for p in range(P):
                    assert np.array_equal(bits_of(to_np(outs[p])), bits_of(want[p])), (dtype, P, n, edge, cap, p)
            vrar.set_edge_sync(False)
            vrar.set_max_ctas(0)
    print("ok")
""")


@pytest.mark.parametrize("variant", ["plain", "staged", "async", "batched"])
def test_fp8_each_write_kernel(variant):
    env = dict(os.environ, VRAR_WRITE_KERNEL=variant)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]
