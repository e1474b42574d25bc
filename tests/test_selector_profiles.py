"""The selector tables against the sweeps they were measured from: every row
of profiles/selector_sweep.md and profiles/selector_sweep_fp8.md names the
kernel the table picks for that shape, and the library must pick the same
(vrar_kernel_name needs no device)."""

import os
import re

import pytest
import torch

import collective_all_reduce_virtual_b200 as vrar

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = {"oneshot": "k_oneshot", "write plain": "k_twostage_write", "write staged": "k_twostage_write_staged",
          "write async": "k_twostage_write_async", "write batched": "k_twostage_write_batched",
          "plain": "k_twostage_write", "staged": "k_twostage_write_staged", "async": "k_twostage_write_async",
          "batched": "k_twostage_write_batched"}


def rows(name, pick_col):
    out = []
    for line in open(os.path.join(ROOT, "profiles", name)):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) > pick_col and re.fullmatch(r"\d+", cells[0]) and re.fullmatch(r"\d+", cells[1]):
            out.append((int(cells[0]), int(cells[1]), cells[pick_col]))
    return out


@pytest.fixture(autouse=True)
def _no_overrides():
    if os.environ.get("VRAR_WRITE_KERNEL") or os.environ.get("VRAR_ALGO"):
        pytest.skip("an override is set in the environment")
    yield
    vrar.set_fp8_quant(False)


def test_selector_table_matches_its_sweep():
    rs = rows("selector_sweep.md", 9)
    assert len(rs) == 60
    for P, kib, pick in rs:
        n = kib * 512  # bf16 elements per rank
        assert vrar.kernel_name(P, n, torch.bfloat16, "auto") == KERNEL[pick], (P, kib, pick)


def test_fp8_write_kernel_table_matches_its_sweep():
    rs = rows("selector_sweep_fp8.md", 8)
    assert len(rs) == 60
    vrar.set_fp8_quant(True)
    for P, kib, pick in rs:
        assert vrar.kernel_name(P, kib * 512, torch.bfloat16, "twostage_write") == KERNEL[pick], (P, kib, pick)
