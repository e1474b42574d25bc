"""Maximum sizes: vectors past 2^31 elements and 2^32 bytes per rank.

Two ranks of 2^31 + 29 bf16 elements (4 GiB per buffer, a ragged tail) and of
2^30 + 5 fp32 elements (byte offsets past 2^32) go through every all-reduce
algorithm, and 2^31 + 32 bf16 through the reduce-scatter and all-gather; any
32-bit index or byte offset on the device or the host would land in the wrong
place. Each output element depends only on the inputs at its own index (the
chunking of recursive doubling does not change results), so the oracle on a
window of the inputs gives the exact expected values of that window: windows
at the start, across the 2^31-element (bf16) or 2^30-element (fp32) boundary,
and at the end. About 32 GiB of device memory at the peak (four buffers plus
the payload slots of recursive doubling).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from util import TORCH_DT, bits_of, to_np

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import collective_all_reduce_virtual_b200 as vrar
else:  # collected on the CPU machine, never run there
    vrar = None

W = 4096


def _windows(n: int, edge: int):
    return [(0, W), (edge - W, edge + W), (n - W, n)]


def _slice_np(t: torch.Tensor, a: int, b: int) -> np.ndarray:
    return to_np(t[a:b])


@pytest.fixture(autouse=True)
def _cleanup():
    yield
    if vrar is not None:
        vrar.set_group_size(8)
        vrar.reset()  # give the payload slots back
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype,n,edge", [("bf16", (1 << 31) + 29, 1 << 31), ("fp32", (1 << 30) + 5, 1 << 30)])
def test_allreduce_past_32_bit_offsets(dtype, n, edge):
    P = 2
    xs = synth.make_inputs(P, n, TORCH_DT[dtype], synth.normal(0.0, 1.0), seed=31, device="cuda", block=1 << 26)
    outs = [torch.empty_like(x) for x in xs]
    wins = _windows(n, edge)
    x_win = [[_slice_np(x, a, b) for x in xs] for a, b in wins]
    for algo, L in (("oneshot", 8), ("twostage", 8), ("twostage_write", 8), ("rd", 8), ("hier", 1)):
        vrar.set_group_size(L)
        for o in outs:
            o.zero_()
        vrar.all_reduce(xs, outs, algo=algo)
        rc, info = vrar.query_status()
        assert rc == 0, (algo, rc, info)
        for (a, b), xw in zip(wins, x_win):
            want = oracle.allreduce(algo, xw, dtype, L=L)
            for p in range(P):
                got = _slice_np(outs[p], a, b)
                assert np.array_equal(bits_of(got), bits_of(want[p])), f"{algo} {dtype} rank {p} window {a}"
    del xs, outs


def test_reduce_scatter_and_all_gather_past_32_bit_offsets():
    P, n, dtype = 2, (1 << 31) + 32, "bf16"
    m = n // P
    xs = synth.make_inputs(P, n, TORCH_DT[dtype], synth.normal(0.0, 1.0), seed=32, device="cuda", block=1 << 26)
    rs = vrar.reduce_scatter(xs)
    rc, info = vrar.query_status()
    assert rc == 0, info
    # out[p] holds elements [p*m, (p+1)*m) of the sum, in the order of one-shot.
    for p in range(P):
        for a, b in _windows(m, m // 2):
            want = oracle.allreduce("oneshot", [_slice_np(x, p * m + a, p * m + b) for x in xs], dtype)
            assert np.array_equal(bits_of(_slice_np(rs[p], a, b)), bits_of(want[0])), f"RS rank {p} window {a}"
    del rs
    sl = [x[:m] for x in xs]  # rank c contributes n/P elements
    ag = vrar.all_gather(sl)
    rc, info = vrar.query_status()
    assert rc == 0, info
    for p in range(P):
        for c in range(P):
            for a, b in _windows(m, m // 2):
                assert np.array_equal(bits_of(_slice_np(ag[p], c * m + a, c * m + b)),
                                      bits_of(_slice_np(sl[c], a, b))), f"AG out {p} chunk {c} window {a}"
    del xs, sl, ag
