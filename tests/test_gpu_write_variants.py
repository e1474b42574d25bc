"""The four write-mode kernels (plain, bulk-copy staged, per-thread async
copies, register-batched) against the oracle.

The per-shape table sends each shape to one of the kernels, so this test
forces each in turn (VRAR_WRITE_KERNEL is read once per process, hence the
child processes) over shapes with ragged tails, up to 32 ranks, all three
dtypes, with and without the start/end barriers, and with a CTA budget (which
changes the grid and, for the staged and async kernels, the stage depth).
The batched kernel's unguarded passes need 512 items per CTA pass, so the
larger shapes at 13, 16, 24 and 32 ranks run both its paths; 2 ranks x 2 MiB
is a small call that one plain CTA per SM cannot cover in one pass, so the
plain kernel runs its two-CTA-per-SM build there.
"""

import os
import subprocess
import sys
import textwrap

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import numpy as np
    import collective_all_reduce_virtual_b200 as vrar
    import oracle, synth
    from util import from_np, gen, to_np, bits_of
    for dtype in ("bf16", "fp32", "fp16"):
        for P, n in ((1, 1001), (2, 7), (2, 1_048_583), (3, 66_001), (8, 9), (8, 300_007), (13, 4_099), (13, 700_001),
                     (16, 70_001), (24, 50_021), (24, 2_000_003), (32, 33_333), (32, 1_000_003)):
            xs = gen(P, n, dtype, synth.normal(0.0, 1.0), seed=P + n)
            want = oracle.allreduce("twostage_write", xs, dtype)
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
def test_write_kernel_variant_matches_oracle(variant):
    env = dict(os.environ, VRAR_WRITE_KERNEL=variant)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]
