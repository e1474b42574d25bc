"""The seeded input generator against a plain Python-int SplitMix64 (CPU only)."""

import math

import numpy as np
import torch

import synth

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def _mix(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def _splitmix_stream(state, count):
    """Textbook SplitMix64 next(): state += GAMMA; return mix(state)."""
    out = []
    for _ in range(count):
        state = (state + GAMMA) & M64
        out.append(_mix(state))
    return out


def test_draws_match_sequential_splitmix():
    for seed, rank in ((0, 0), (0, 7), (3, 31), (2**32 - 1, 5)):
        start = _splitmix_stream((seed << 32) | rank, 1)[0]
        seq = _splitmix_stream(start, 50)
        got = synth.draws(seed, rank, torch.arange(50, dtype=torch.int64))
        got_u = [int(v) & M64 for v in got.tolist()]
        assert got_u == seq


def test_int8_range_and_balance():
    v = synth.rank_values(synth.INT8, 0, 0, torch.arange(170_000, dtype=torch.int64))
    assert v.min() == -8 and v.max() == 8
    assert torch.equal(v, v.round())
    counts = torch.bincount((v + 8).to(torch.int64), minlength=17).double()
    assert (counts / counts.mean() - 1).abs().max() < 0.05


def test_normal_moments():
    v = synth.rank_values(synth.normal(0.0, 1.0), 1, 2, torch.arange(400_000, dtype=torch.int64))
    assert abs(v.mean().item()) < 0.01 and abs(v.std().item() - 1.0) < 0.01
    w = synth.rank_values(synth.normal(0.0, 0.02), 1, 2, torch.arange(1000, dtype=torch.int64))
    assert torch.allclose(w, 0.02 * v[:1000], rtol=0, atol=1e-15)


def test_uniform_range():
    v = synth.rank_values(synth.uniform(-1, 1), 4, 1, torch.arange(100_000, dtype=torch.int64))
    assert v.min() >= -1 and v.max() < 1 and abs(v.mean().item()) < 0.01


def test_counter_based_and_blocked_generation_agree():
    whole = synth.make_inputs(3, 1000, torch.bfloat16, synth.normal(), seed=9)
    blocked = synth.make_inputs(3, 1000, torch.bfloat16, synth.normal(), seed=9, block=77)
    for a, b in zip(whole, blocked):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    idx = torch.tensor([0, 5, 999])
    single = synth.to_dtype(synth.rank_values(synth.normal(), 9, 2, idx), torch.bfloat16)
    assert torch.equal(single.view(torch.int16), whole[2][idx].view(torch.int16))


def test_ranks_and_seeds_differ():
    a = synth.make_inputs(2, 64, torch.float32, synth.normal(), seed=0)
    b = synth.make_inputs(2, 64, torch.float32, synth.normal(), seed=1)
    assert not torch.equal(a[0], a[1]) and not torch.equal(a[0], b[0])


def test_box_muller_single_value():
    # Element 0 of rank 0, seed 0, from the stated formula with Python floats.
    start = _splitmix_stream(0, 1)[0]
    d1, d2 = _splitmix_stream(start, 2)
    u1 = ((d1 >> 11) + 1) * 2.0**-53
    u2 = (d2 >> 11) * 2.0**-53
    z = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
    got = synth.rank_values(synth.normal(), 0, 0, torch.tensor([0])).item()
    assert abs(got - z) <= 1e-15 * max(1.0, abs(z))


def test_parse_dist():
    assert synth.parse_dist("int8") == synth.INT8
    assert synth.parse_dist("normal:0,0.02") == synth.normal(0.0, 0.02)
    assert synth.parse_dist("uniform:-1,1") == synth.uniform(-1.0, 1.0)
    assert np.isclose(synth.parse_dist("normal").b, 1.0)
