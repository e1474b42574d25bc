"""The prefill workload at full size (P = 8 ranks of 16,384 x 7,168 bf16, 1.88 GB
of inputs), every output element checked against the CPU oracle.

Each output element of the custom all-reduce algorithms depends only on the P
inputs at the same index (one ascending-rank fp32 sum, one rounding), so the
oracle runs over contiguous windows of the vectors and its window results are
exactly the full-size results at those indices. Rank 0's output is compared
with the oracle element by element over all 117,440,512 elements; the other
P - 1 outputs are compared with rank 0's, whole, on the device.

The write mode has four kernels; the per-shape table gives this shape to the
plain kernel. The staged, async-copy and register-batched kernels are forced
in child processes (VRAR_WRITE_KERNEL is read once per process), so that every
write kernel is checked at this size.
"""

import os
import subprocess
import sys
import textwrap

import pytest
import torch

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P, N = 8, 16384 * 7168
WINDOW = 1 << 22

CHECK = textwrap.dedent("""
    import sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import numpy as np
    import torch
    import collective_all_reduce_virtual_b200 as vrar
    import oracle, synth

    P, N, WINDOW = {P}, {N}, {WINDOW}
    d_in = synth.make_inputs(P, N, torch.bfloat16, synth.normal(0.0, 0.02), seed=0, device="cuda",
                             block=1 << 25)
    xs = [t.cpu().view(torch.int16).numpy().view(np.uint16) for t in d_in]
    for algo, kernel in {cases!r}:
        got_kernel = vrar.kernel_name(P, N, torch.bfloat16, algo)
        assert got_kernel == kernel, (algo, got_kernel, kernel)
        outs = vrar.all_reduce(d_in, algo=algo)
        rc, info = vrar.query_status()
        assert rc == 0, (algo, rc, info)
        for p in range(1, P):
            assert torch.equal(outs[p].view(torch.int16), outs[0].view(torch.int16)), (algo, "rank", p)
        got = outs[0].cpu().view(torch.int16).numpy().view(np.uint16)
        del outs
        checked = 0
        for lo in range(0, N, WINDOW):
            hi = min(N, lo + WINDOW)
            want = oracle.allreduce("twostage_write" if algo == "auto" else algo, [x[lo:hi] for x in xs],
                                    "bf16")[0]
            if not np.array_equal(got[lo:hi], want):
                bad = np.nonzero(got[lo:hi] != want)[0]
                raise AssertionError(f"{{algo}} ({{kernel}}): {{bad.size}} elements differ in window "
                                     f"[{{lo}}, {{hi}}), first at {{lo + bad[:8]}}")
            checked += hi - lo
        assert checked == N
        torch.cuda.empty_cache()
    print("ok")
""")


def _run(cases, env_extra=None):
    code = CHECK.format(root=ROOT, tests=os.path.join(ROOT, "tests"), P=P, N=N, WINDOW=WINDOW, cases=cases)
    env = dict(os.environ, **(env_extra or {}))
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]


def test_prefill_full_pull_and_plain_write():
    """The pull 2-stage and the write mode as the table picks it (plain kernel)."""
    _run([("twostage", "k_twostage"), ("twostage_write", "k_twostage_write"), ("auto", "k_twostage_write")])


@pytest.mark.parametrize("variant,kernel", [("staged", "k_twostage_write_staged"), ("async", "k_twostage_write_async"),
                                            ("batched", "k_twostage_write_batched")])
def test_prefill_full_other_write_kernels(variant, kernel):
    _run([("twostage_write", kernel)], {"VRAR_WRITE_KERNEL": variant})
