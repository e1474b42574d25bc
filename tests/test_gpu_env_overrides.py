"""The environment switches the library reads once per process, each in a
child process: VRAR_PDL=0 (plain stream-ordered launches instead of
programmatic dependent launch) and VRAR_ALGO (forces the algorithm AUTO
runs). Results must still equal the oracle bit for bit, both as direct calls
and as CUDA-graph replays of back-to-back calls.
"""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import numpy as np, torch
    import collective_all_reduce_virtual_b200 as vrar
    import oracle, synth
    from util import from_np, gen, to_np, bits_of
    algos = {algos!r}
    for dtype in ("bf16", "fp32"):
        for P, n in ((2, 4099), (8, 300_007), (8, 9), (16, 70_001)):
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=P + n)
            d_in = [from_np(x, dtype).cuda() for x in xs]
            for algo in algos:
                # AUTO runs one-shot or write mode here, which share one summation order
                ref = {oracle_algo!r} or ("oneshot" if algo == "auto" else algo)
                want = oracle.allreduce(ref, xs, dtype, L=min(8, P))
                vrar.set_group_size(min(8, P))
                if {forced!r}:
                    assert vrar.kernel_name(P, n, d_in[0].dtype, "auto") == {forced!r}, vrar.kernel_name(P, n, d_in[0].dtype, "auto")
                outs = [torch.empty_like(t) for t in d_in]
                vrar.all_reduce(d_in, outs, algo=algo)
                torch.cuda.synchronize()
                # the same call, 20 times back to back in a CUDA graph
                g = torch.cuda.CUDAGraph()
                outs2 = [torch.empty_like(t) for t in d_in]
                with torch.cuda.graph(g):
                    for _ in range(20):
                        vrar.all_reduce(d_in, outs2, algo=algo, stream=torch.cuda.current_stream())
                g.replay()
                torch.cuda.synchronize()
                rc, info = vrar.query_status()
                assert rc == 0, (algo, rc, info)
                for p in range(P):
                    for o in (outs, outs2):
                        assert np.array_equal(bits_of(to_np(o[p])), bits_of(want[p])), (algo, dtype, P, n, p)
    print("ok")
""")


def _child(env, algos, oracle_algo=None, forced=None):
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), algos=algos, oracle_algo=oracle_algo,
                        forced=forced)
    res = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, **env), capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]


def test_without_programmatic_dependent_launch():
    _child({"VRAR_PDL": "0"}, ["auto", "oneshot", "twostage", "twostage_write", "rd", "hier"])


@pytest.mark.parametrize("algo,kernel", [("rd", "k_rd"), ("twostage", "k_twostage"), ("oneshot", "k_oneshot")])
def test_vrar_algo_forces_what_auto_runs(algo, kernel):
    _child({"VRAR_ALGO": algo}, ["auto"], oracle_algo=algo, forced=kernel)
