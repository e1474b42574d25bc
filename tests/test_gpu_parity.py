"""GPU path against the CPU oracle, through the C ABI (Python binding).

Bit-exact: every algorithm fixes its fp32-accumulate order, and the oracle
restates that order, so outputs must match bit for bit (NaN never appears in
these inputs). The fp64 tolerances (bf16 1e-2, fp32 1e-5, relative to the sum
of magnitudes) are checked as well.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from util import TORCH_DT, bits_of, from_np, gen, hexvals, load_golden, parse_algo, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import collective_all_reduce_virtual_b200 as vrar
else:  # collected on the CPU machine, never run there
    vrar = None

RTOL = {"bf16": 1e-2, "fp32": 1e-5, "fp16": 5e-3}


@pytest.fixture(autouse=True)
def _defaults():
    yield
    if vrar is not None:
        vrar.set_group_size(8)
        vrar.set_rd_chunks(4)
        vrar.set_edge_sync(False)
        vrar.set_spin_timeout_ns(2_000_000_000)
        vrar.debug_set_fault_mask(0)
        vrar.set_max_ctas(0)
        vrar.set_payload_wire("element")


def _dev(xs_np, dtype):
    return [from_np(x, dtype).cuda() for x in xs_np]


def run(algo, xs_np, dtype, L=8, C=4, edge=False):
    """One call through the binding. 'rd_fp32wire' / 'hier_fp32wire' are the
    oracle's names for RD / HIER with fp32 partials on the wire."""
    vrar.set_group_size(L)
    vrar.set_rd_chunks(C)
    vrar.set_edge_sync(edge)
    wire = algo.endswith("_fp32wire")
    vrar.set_payload_wire("fp32" if wire else "element")
    outs = vrar.all_reduce(_dev(xs_np, dtype), algo=algo[: -len("_fp32wire")] if wire else algo)
    rc, info = vrar.query_status()
    assert rc == 0, f"device status {rc} {info}"
    return [to_np(o) for o in outs]


def assert_bits(got, want, what):
    for p, (g, w) in enumerate(zip(got, want)):
        if not np.array_equal(bits_of(g), bits_of(w)):
            bad = np.nonzero(bits_of(g) != bits_of(w))[0]
            raise AssertionError(f"{what}: rank {p} differs at {bad[:8]} (of {bad.size})")


def algos_for(P):
    out = [("oneshot", 8), ("twostage", 8), ("twostage_write", 8)]
    if P & (P - 1) == 0:
        out += [("rd", 8), ("rd_fp32wire", 8)]
        for L in sorted({1, max(1, P // 2), P}):
            out += [("hier", L), ("hier_fp32wire", L)]
    return out


# ---- small shapes: several CTAs' worth of items and a ragged tail ----------------------------

SHAPES = [(P, n) for P in (1, 2, 3, 4, 5, 8) for n in (1, 7, 8, 9, 4099, 100_003)] + \
         [(P, n) for P in (16, 32) for n in (1, 9, 20_011)]


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "fp16"])
@pytest.mark.parametrize("P,n", SHAPES)
def test_parity_small(P, n, dtype):
    xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=P * 1000 + n)
    for algo, L in algos_for(P):
        want = oracle.allreduce(algo, xs, dtype, L=L, chunks=4)
        got = run(algo, xs, dtype, L=L)
        assert_bits(got, want, f"{algo} L={L} P={P} n={n} {dtype}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "fp16"])
def test_integer_inputs_give_exact_sums(dtype):
    for P in (2, 4, 8, 16, 32):
        n = 5003
        xs = gen(P, n, dtype, synth.INT8, seed=P)
        exact = np.stack([oracle.to_float(x, dtype) for x in xs]).astype(np.int64).sum(axis=0)
        for algo, L in algos_for(P):
            got = run(algo, xs, dtype, L=L)
            for p, g in enumerate(got):
                assert (oracle.to_float(g, dtype) == exact).all(), f"{algo} L={L} P={P}"
                # A real reduction happened: a rank's output is not its own input
                # (a one-rank "collective" that copies would pass a same-value check).
                assert (bits_of(g) != bits_of(xs[p])).mean() > 0.5, f"{algo} L={L} P={P} rank {p} copied its input"


def test_golden_order_cases_on_gpu():
    for case in load_golden()["cases"]:
        dt = case["dtype"]
        xs = [hexvals(row, dt) for row in case["inputs"]]
        for spec, want_strs in case["expect"].items():
            algo, L = parse_algo(spec)
            want = hexvals(want_strs, dt)
            got = run(algo, xs, dt, L=L if L is not None else 8)
            assert_bits(got, [want] * len(got), f"{case['name']} {spec}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "fp16"])
def test_fp64_tolerance(dtype):
    for P in (2, 8, 32):
        xs = gen(P, 30_000, dtype, synth.normal(0.0, 1.0), seed=77 + P)
        S, A = oracle.fp64_reference(xs, dtype)
        for algo, L in algos_for(P):
            y = oracle.to_float(run(algo, xs, dtype, L=L)[0], dtype)
            assert (np.abs(y - S) <= RTOL[dtype] * A).all(), f"{algo} L={L} P={P}"


def test_special_values_classes():
    """inf, -inf, subnormals and signed zeros (NaN only as inf - inf)."""
    vals = np.array([np.inf, -np.inf, 1e-40, -1e-40, 0.0, -0.0, 3e38, 3e38], np.float32)
    xs32 = [vals, np.array([1.0, 1.0, 1e-40, 0.0, -0.0, -0.0, 3e38, -3e38], np.float32),
            np.array([-np.inf, 2.0, 0.0, -1e-40, -0.0, -0.0, 0.0, 1.0], np.float32)]
    for dtype in ("fp32", "bf16", "fp16"):
        xs = xs32 if dtype == "fp32" else [oracle.bf16_round(x) if dtype == "bf16" else oracle.fp16_round(x)
                                           for x in xs32]
        for algo in ("oneshot", "twostage", "twostage_write"):
            want = oracle.allreduce(algo, xs, dtype)
            got = run(algo, xs, dtype)
            for g, w in zip(got, want):
                gf, wf = oracle.to_float(g, dtype), oracle.to_float(w, dtype)
                assert np.array_equal(np.isnan(gf), np.isnan(wf))
                fin = ~np.isnan(wf)
                assert np.array_equal(bits_of(g)[fin], bits_of(w)[fin]), f"{algo} {dtype}"


# ---- the workload shapes at full size ---------------------------------------------------------

def test_config_p2_ints_oneshot_and_rd():
    xs = gen(2, 65_536, "bf16", synth.INT8, seed=0)
    exact = np.stack([oracle.to_float(x, "bf16") for x in xs]).astype(np.int64).sum(axis=0)
    for algo in ("oneshot", "rd"):
        got = run(algo, xs, "bf16")
        assert_bits(got, oracle.allreduce(algo, xs, "bf16"), algo)
        assert (oracle.to_float(got[0], "bf16") == exact).all()
        assert_bits(got, [got[0]] * 2, f"{algo} ranks equal")


def test_config_p8_decode_1mib():
    xs = gen(8, 64 * 8192, "bf16", synth.normal(0.0, 1.0), seed=0)
    one = None
    for algo in ("oneshot", "twostage", "twostage_write", "rd", "auto"):
        want = oracle.allreduce(algo if algo != "auto" else vrar.select_algo(8, 64 * 8192), xs, "bf16")
        got = run(algo, xs, "bf16")
        assert_bits(got, want, algo)
        if algo == "oneshot":
            one = got
        elif algo in ("twostage", "twostage_write"):
            assert_bits(got, one, f"{algo} == oneshot")


@pytest.mark.parametrize("n", [65_536, 131_072, 262_144, 524_288, 1_048_576])
def test_config_p8_rd_sweep(n):
    xs = gen(8, n, "bf16", synth.normal(0.0, 1.0), seed=0)
    got = run("rd", xs, "bf16", C=4)
    assert_bits(got, oracle.allreduce("rd", xs, "bf16", chunks=4), f"rd n={n}")


def test_config_p8_rd_1000_calls_reuse_flags():
    n = 262_144
    xs = gen(8, n, "bf16", synth.normal(0.0, 1.0), seed=3)
    want = oracle.allreduce("rd", xs, "bf16", chunks=4)
    d_in = _dev(xs, "bf16")
    outs = [torch.empty_like(t) for t in d_in]
    vrar.set_rd_chunks(4)
    for i in range(1000):
        vrar.all_reduce(d_in, outs, algo="rd")
        if i in (0, 499, 999):
            assert_bits([to_np(o) for o in outs], want, f"call {i}")
    rc, info = vrar.query_status()
    assert rc == 0, info


@pytest.mark.parametrize("edge", [False, True])
def test_cuda_graph_replay_reuses_flags(edge):
    n = 131_072
    xs = gen(8, n, "bf16", synth.normal(0.0, 1.0), seed=4)
    d_in = _dev(xs, "bf16")
    vrar.set_edge_sync(edge)
    for algo in ("rd", "twostage", "oneshot", "twostage_write", "hier"):
        outs = [torch.empty_like(t) for t in d_in]
        want = oracle.allreduce(algo, xs, "bf16")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            vrar.all_reduce(d_in, outs, algo=algo, stream=s)  # sizes the workspace before capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(10):
                vrar.all_reduce(d_in, outs, algo=algo)
        for _ in range(50):
            g.replay()
        torch.cuda.synchronize()
        rc, info = vrar.query_status()
        assert rc == 0, (algo, info)
        assert_bits([to_np(o) for o in outs], want, f"{algo} after 500 graph-replayed calls")
        del g


@pytest.mark.parametrize("n", [131_072, 1_048_576])
def test_config_p32_hier_4x8(n):
    xs = gen(32, n, "bf16", synth.uniform(-1.0, 1.0), seed=0)
    got = run("hier", xs, "bf16", L=8)
    assert_bits(got, oracle.allreduce("hier", xs, "bf16", L=8), f"hier 4x8 n={n}")


# ---- protocol properties ----------------------------------------------------------------------

@pytest.mark.parametrize("algo", ["oneshot", "twostage", "twostage_write", "rd", "hier"])
def test_inputs_written_by_the_previous_kernel(algo):
    """Calls launch with programmatic dependent launch; a kernel that writes the
    inputs right before the call (no host sync in between) must be waited for.
    Integer inputs: after k rounds of `x += 1` on every rank the sum grows by k*P."""
    P, n = 8, 300_001
    xs = gen(P, n, "bf16", synth.INT8, seed=21)
    base = np.stack([oracle.to_float(x, "bf16") for x in xs]).astype(np.int64).sum(axis=0)
    d_in = _dev(xs, "bf16")
    outs = [torch.empty_like(t) for t in d_in]
    vrar.set_group_size(4)
    for k in range(1, 6):
        for t in d_in:
            t.add_(1.0)
        vrar.all_reduce(d_in, outs, algo=algo)
        got = oracle.to_float(to_np(outs[3]), "bf16")
        assert (got == base + k * P).all(), f"{algo} round {k}"
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t in d_in:
            t.add_(1.0)
        vrar.all_reduce(d_in, outs, algo=algo)
    for k in range(6, 11):
        g.replay()
        torch.cuda.synchronize()
        got = oracle.to_float(to_np(outs[5]), "bf16")
        assert (got == base + k * P).all(), f"{algo} graph round {k}"
    rc, info = vrar.query_status()
    assert rc == 0, info


def test_chained_calls_read_the_previous_calls_output():
    """out1 = allreduce(x); out2 = allreduce(out1) back to back: the second
    kernel reads what the first wrote (P * sum for integer inputs)."""
    P, n = 4, 200_003
    xs = gen(P, n, "fp32", synth.INT8, seed=22)
    base = np.stack(xs).astype(np.int64).sum(axis=0)
    d_in = _dev(xs, "fp32")
    mid = [torch.empty_like(t) for t in d_in]
    out = [torch.empty_like(t) for t in d_in]
    for a1 in ("oneshot", "twostage_write", "rd", "twostage"):
        for a2 in ("oneshot", "twostage", "rd", "twostage_write"):
            vrar.all_reduce(d_in, mid, algo=a1)
            vrar.all_reduce(mid, out, algo=a2)
            assert (to_np(out[P - 1]).astype(np.int64) == P * base).all(), (a1, a2)


def test_chunk_count_and_edge_sync_do_not_change_results():
    # Large enough that the grid needs several pieces per thread (a call uses
    # fewer chunks than configured only when threads are to spare).
    xs = gen(8, 1_000_003, "bf16", synth.normal(0.0, 1.0), seed=11)
    ref = run("rd", xs, "bf16", C=1)
    for C in range(2, 9):
        assert_bits(run("rd", xs, "bf16", C=C), ref, f"rd C={C}")
    ref = run("hier", xs, "bf16", L=2, C=1)
    for C in (2, 4, 8):
        assert_bits(run("hier", xs, "bf16", L=2, C=C), ref, f"hier C={C}")
    for algo in ("oneshot", "twostage", "twostage_write"):
        assert_bits(run(algo, xs, "bf16", edge=False), run(algo, xs, "bf16", edge=True), algo)


@pytest.mark.parametrize("budget", [1, 16, 40])
def test_cta_budget_keeps_results(budget):
    """A CTA budget shrinks the grid (down to one CTA per rank); every
    algorithm still matches the oracle."""
    vrar.set_max_ctas(budget)
    try:
        for P, n in ((8, 300_007), (32, 70_001)):
            xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=budget + P)
            for algo, L in algos_for(P):
                if algo == "hier" and L not in (1, P // 2):
                    continue
                assert_bits(run(algo, xs, "bf16", L=L), oracle.allreduce(algo, xs, "bf16", L=L),
                            f"{algo} L={L} P={P} budget={budget}")
    finally:
        vrar.set_max_ctas(0)


def test_shapes_interleaved_across_calls():
    """Flags and payload slots are reused across calls of different P, n and
    algorithm without ever being cleared."""
    plan = [(8, 70_000, "twostage", 8), (32, 40_000, "hier", 8), (2, 9, "rd", 8), (8, 70_000, "rd", 8),
            (4, 100_000, "oneshot", 8), (32, 40_000, "hier", 4), (16, 33_333, "twostage_write", 8),
            (8, 70_000, "twostage", 8)]
    for i, (P, n, algo, L) in enumerate(plan * 2):
        xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=i)
        assert_bits(run(algo, xs, "bf16", L=L), oracle.allreduce(algo, xs, "bf16", L=L), f"step {i} {algo}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "fp16"])
def test_reduce_scatter_and_all_gather(dtype):
    for P in (1, 2, 3, 8, 32):
        for m in (8, 37, 4104, 20_000):
            n = m * P
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=P + m)
            got = [to_np(o) for o in vrar.reduce_scatter(_dev(xs, dtype))]
            assert_bits(got, oracle.reduce_scatter(xs, dtype), f"RS P={P} m={m}")
            sl = gen(P, m, dtype, synth.normal(0.0, 1.0), seed=P * m)
            got = [to_np(o) for o in vrar.all_gather(_dev(sl, dtype))]
            assert_bits(got, oracle.all_gather(sl, dtype), f"AG P={P} m={m}")
    # Many tiles per CTA, with and without a CTA budget (which deepens the
    # stages): 32,768 elements per chunk take the async-copy form (at most
    # 1 MiB per rank), 131,072 the 16-byte plain kernel.
    for P, m in ((8, 32_768), (8, 131_072)):
        xs = gen(P, m * P, dtype, synth.normal(0.0, 1.0), seed=7)
        want = oracle.reduce_scatter(xs, dtype)
        for cap in (0, 16):
            vrar.set_max_ctas(cap)
            try:
                got = [to_np(o) for o in vrar.reduce_scatter(_dev(xs, dtype))]
            finally:
                vrar.set_max_ctas(0)
            assert_bits(got, want, f"RS P={P} m={m} max_ctas={cap}")
    rc, info = vrar.query_status()
    assert rc == 0, info


def test_workspace_growth_between_calls():
    vrar.reset()
    for n in (1000, 300_000, 1_000, 2_000_000):
        xs = gen(8, n, "bf16", synth.normal(0.0, 1.0), seed=n)
        assert_bits(run("rd", xs, "bf16"), oracle.allreduce("rd", xs, "bf16"), f"rd n={n}")


def test_device_argument_errors():
    t = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    ins = [t[:256], t[256:512]]
    outs = [t[512:768], t[520:776]]  # overlapping outputs
    with pytest.raises(vrar.VrarError) as e:
        vrar.all_reduce(ins, outs, algo="oneshot")
    assert e.value.code == vrar.EINVAL
    mis = [t[1:257], t[257:513]]  # 2-byte offset: not 16-byte aligned
    with pytest.raises(vrar.VrarError) as e:
        vrar.all_reduce(mis, algo="oneshot")
    assert e.value.code == vrar.EINVAL
    with pytest.raises(vrar.VrarError) as e:
        vrar.all_reduce([t[:256]] * 3, algo="rd")
    assert e.value.code in (vrar.EINVAL, vrar.ENOTSUP)


# ---- spin statistics ----------------------------------------------------------------------------

def test_spin_stats_counts_every_wait():
    vrar.get_spin_stats(reset=True)
    P, n = 8, 8 * 4096  # 4096 items per rank: one item per thread, one chunk
    xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=31)
    run("rd", xs, "bf16")
    assert vrar.get_spin_stats(reset=True)["waits"] == 0, "statistics must be off by default"
    vrar.set_spin_stats(True)
    try:
        run("rd", xs, "bf16")
        st = vrar.get_spin_stats(reset=True)
        # every thread holding an item waits once per step: P * log2(P) * items
        assert st["waits"] == P * 3 * 4096, st
        assert st["polls"] >= st["waits"] and st["max_polls"] >= 1 and st["timeouts"] == 0, st
        run("twostage", xs, "bf16")  # mid barrier: P polling threads per CTA
        st = vrar.get_spin_stats(reset=True)
        assert st["waits"] > 0 and st["waits"] % P == 0 and st["timeouts"] == 0, st
        assert vrar.get_spin_stats()["waits"] == 0, "reset must clear the counters"
    finally:
        vrar.set_spin_stats(False)


def test_spin_stats_count_timeouts():
    xs = gen(4, 40_000, "bf16", synth.normal(0.0, 1.0), seed=32)
    d_in = _dev(xs, "bf16")
    vrar.get_spin_stats(reset=True)
    vrar.set_spin_stats(True)
    vrar.set_spin_timeout_ns(20_000_000)
    vrar.debug_set_fault_mask(1 << 2)
    try:
        vrar.all_reduce(d_in, algo="rd")
        rc, info = vrar.query_status()
        assert rc == vrar.ETIMEDOUT
        st = vrar.get_spin_stats(reset=True)
        assert st["timeouts"] >= 1 and st["long_waits"] >= 1, st
    finally:
        vrar.set_spin_stats(False)
        vrar.debug_set_fault_mask(0)
    outs = vrar.all_reduce(d_in, algo="rd")
    assert vrar.query_status()[0] == 0
    assert_bits([to_np(o) for o in outs], oracle.allreduce("rd", xs, "bf16"), "rd after the timeout")


# ---- failure detection: bounded waits, no GPU fault ----------------------------------------------

@pytest.mark.parametrize("algo,P,L,edge,phase,n", [
    ("rd_fp32wire", 4, 8, True, 4, 40_000),
    ("oneshot", 4, 8, True, 1, 40_000),
    ("twostage", 4, 8, False, 2, 40_000),
    ("twostage_write", 8, 8, True, 1, 40_000),      # async-copy write kernel
    ("twostage_write", 8, 8, True, 1, 4_194_304),   # 8 MiB per rank: bulk-copy staged kernel
    ("twostage_write", 8, 8, True, 1, 20_000_000),  # 40 MiB per rank: plain kernel
    ("twostage_write", 4, 8, True, 1, 20_000_000),  # 40 MiB per rank at 4 ranks: batched kernel
    ("rd", 4, 8, True, 4, 40_000),
    ("hier", 8, 2, True, 4, 40_000),
    ("hier", 8, 2, True, 4, 600_000),               # above 256 KiB per rank: two CTAs per SM
])
def test_missing_rank_times_out_and_recovers(algo, P, L, edge, phase, n):
    """A rank that never posts (fault mask) makes its peers' waits run out; the
    kernel records VRAR_ETIMEDOUT and exits, and the next call works."""
    xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=5)
    if algo == "twostage_write":  # the case must reach the kernel it is there for
        want_kernel = {(8, 40_000): "k_twostage_write_async", (8, 4_194_304): "k_twostage_write_staged",
                       (8, 20_000_000): "k_twostage_write", (4, 20_000_000): "k_twostage_write_batched"}[(P, n)]
        assert vrar.kernel_name(P, n, torch.bfloat16, algo) == want_kernel
    d_in = _dev(xs, "bf16")
    vrar.set_group_size(L)
    vrar.set_edge_sync(edge)
    vrar.set_spin_timeout_ns(50_000_000)
    wire = algo.endswith("_fp32wire")
    vrar.set_payload_wire("fp32" if wire else "element")
    base = algo[: -len("_fp32wire")] if wire else algo
    vrar.debug_set_fault_mask(1 << 1)
    vrar.all_reduce(d_in, algo=base)
    rc, info = vrar.query_status()
    assert rc == vrar.ETIMEDOUT, (rc, info)
    assert info[1] == phase
    vrar.debug_set_fault_mask(0)
    outs = vrar.all_reduce(d_in, algo=base)
    rc, info = vrar.query_status()
    assert rc == 0, info
    assert_bits([to_np(o) for o in outs], oracle.allreduce(algo, xs, "bf16", L=L), f"{algo} after timeout")


# ---- overlap with compute on another stream ------------------------------------------------------

def test_allreduce_overlapped_with_gemm_on_another_stream():
    """The all-reduce of one micro-batch runs on a side stream while the other
    micro-batch's GEMMs run; every output must still equal the oracle's sum of
    the partials (checked on sampled elements) on both micro-batches."""
    import bench
    m = bench.TboPrefill(torch.device("cuda", 0), P=8, tokens=1024, hidden=2048, layers=3)
    comm = torch.cuda.Stream()
    vrar.set_max_ctas(32)  # a budget leaves SMs to the GEMMs (and selects the deep pipeline)
    try:
        for _ in range(3):
            m.step_overlapped(comm)
        torch.cuda.synchronize()
    finally:
        vrar.set_max_ctas(0)
    assert vrar.query_status()[0] == 0
    rng = np.random.default_rng(5)
    idx = torch.from_numpy(rng.integers(0, m.T * m.H, 50_000)).cuda()
    for u in range(2):
        parts = [to_np(p.reshape(-1)[idx]) for p in m.part[u]]
        want = oracle.allreduce(vrar.select_algo(m.P, m.T * m.H), parts, "bf16")
        assert_bits([to_np(o.reshape(-1)[idx]) for o in m.out[u]], want, f"micro-batch {u}")


# ---- first use of the workspace, and its size ---------------------------------------------------

FIRST_CALL = """
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import numpy as np
import torch
import collective_all_reduce_virtual_b200 as vrar
import oracle, synth
from util import from_np, gen, to_np

side = torch.cuda.Stream()  # created non-blocking: not ordered with the legacy default stream
for algo, P, n in (("rd", 8, 300_001), ("twostage", 8, 300_001), ("hier", 8, 200_003)):
    xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=P + n)
    d_in = [from_np(x, "bf16").cuda() for x in xs]
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        outs = vrar.all_reduce(d_in, algo=algo, stream=side)
    side.synchronize()
    rc, info = vrar.query_status()
    assert rc == 0, (algo, rc, info)
    want = oracle.allreduce(algo, xs, "bf16", L=8)
    for p in range(P):
        assert np.array_equal(to_np(outs[p]), want[p]), (algo, p)
print("ok")
"""


def test_first_calls_of_a_process_on_a_side_stream():
    """The workspace is allocated and zeroed by the first call that needs it;
    that call may come on a non-blocking stream, which is not ordered with the
    zeroing by stream semantics, so the zeroing must be complete before it
    returns. A fresh process makes first calls of three algorithms there (the
    first allocates the control words and the slots, the third grows the
    slots)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = FIRST_CALL.format(root=root, tests=os.path.join(root, "tests"))
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]


def test_payload_slots_are_bounded_by_the_grid():
    """Recursive doubling and the hierarchical algorithm reuse their payload
    slots round by round once the grid cannot cover the message in one round,
    so their slot bytes stop growing with the message."""
    one_round = lambda P, items, steps: P * steps * items * 32  # noqa: E731
    # 8 x 128 KiB: one round, one slot per item
    assert vrar.workspace_bytes(8, 65_536, torch.bfloat16, "rd") == one_round(8, 8192, 3)
    # several rounds: two slot sets of at most one resident grid's slots, whatever the message
    # (rounds are evened out, so the grid, and with it the slots, may shrink a little)
    big = [vrar.workspace_bytes(8, n, torch.bfloat16, "rd") for n in (1 << 22, 1 << 24, 16384 * 7168)]
    assert max(big) <= 64 << 20 and min(big) >= max(big) // 2, big
    assert big[2] < one_round(8, (16384 * 7168) // 8, 3) // 100, big
    h = [vrar.workspace_bytes(32, n, torch.bfloat16, "hier") for n in (1 << 22, 1 << 24)]
    assert max(h) <= 64 << 20 and min(h) >= max(h) // 2, h
    # the full-size prefill through recursive doubling, against the oracle on sampled windows
    P, n = 8, 16384 * 7168
    d_in = synth.make_inputs(P, n, torch.bfloat16, synth.normal(0.0, 0.02), seed=0, device="cuda", block=1 << 25)
    outs = vrar.all_reduce(d_in, algo="rd")
    rc, info = vrar.query_status()
    assert rc == 0, info
    for lo in (0, n // 3 - 4096, n - 8192):
        xs = [to_np(t[lo:lo + 8192]) for t in d_in]
        want = oracle.allreduce("rd", xs, "bf16")
        assert_bits([to_np(o[lo:lo + 8192]) for o in outs], want, f"rd prefill window {lo}")
    del outs, d_in
    torch.cuda.empty_cache()


def test_waits_on_peers_that_cannot_become_resident_end_in_a_timeout():
    """The waits assume that all CTAs of a call are resident together. When
    concurrent work holds SMs, that may not hold: then the waits must end with
    VRAR_ETIMEDOUT, and no output element may ever receive a wrong value. The
    blocker is the allocation-free entry point (its own control words and
    slots, so the two calls share no protocol state) with a CTA budget of 72
    and a rank that never sends: its CTAs hold 72 SMs for its 300 ms limit.
    Meanwhile a full-grid RD call with a 50 ms limit runs on another stream, on
    outputs filled with NaN: every element must end either exact or unwritten
    (a wait that gives up stores nothing), and the status must say a wait ran
    out."""
    P, n = 8, 100_003
    xs = gen(P, n, "bf16", synth.normal(0.0, 1.0), seed=44)
    want = oracle.allreduce("rd", xs, "bf16")
    d_in = _dev(xs, "bf16")
    outs = [torch.empty_like(t) for t in d_in]
    blk_out = [torch.empty_like(t) for t in d_in]
    vrar.all_reduce(d_in, outs, algo="rd")  # sizes the workspace
    for t in outs:
        t.fill_(float("nan"))
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    lib = vrar.lib()
    vrar.set_max_ctas(72)
    vrar.set_spin_timeout_ns(300_000_000)
    vrar.debug_set_fault_mask(1 << 3)
    rc = lib.vrar_allreduce_rd_noalloc(vrar.ptr_array([t.data_ptr() for t in d_in]),
                                       vrar.ptr_array([t.data_ptr() for t in blk_out]), P, n, 0, s1.cuda_stream)
    assert rc == vrar.OK
    vrar.set_max_ctas(0)
    vrar.debug_set_fault_mask(0)
    vrar.set_spin_timeout_ns(50_000_000)
    vrar.all_reduce(d_in, outs, algo="rd", stream=s2)
    torch.cuda.synchronize()
    rc, info = vrar.query_status()
    assert rc == vrar.ETIMEDOUT, (rc, info)
    unwritten = 0
    for p in range(P):
        got = to_np(outs[p])
        nan = np.isnan(oracle.to_float(got, "bf16"))
        unwritten += int(nan.sum())
        assert (got[~nan] == want[p][~nan]).all(), f"rank {p}: a written element is wrong"
    print(f"elements left unwritten by the contended call: {unwritten} of {P * n}")
    # Alone again, the same call is exact.
    outs = vrar.all_reduce(d_in, algo="rd")
    assert vrar.query_status()[0] == 0
    assert_bits([to_np(o) for o in outs], want, "rd after the contention")
