"""Host-thread model of the synchronisation protocol (tests/protocol/), on the CPU.

The model restates the kernels' protocol (device ticket, flag barriers,
sequence-numbered payload words reused round by round in two slot sets, bounded
waits) with one std::thread per CTA.
These tests run it over thousands of calls of changing shape, with a missing
rank, under ThreadSanitizer (the race check that stands in for device-side
sanitizers, which are closed here), and with planted protocol mistakes that it
must catch.
"""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "protocol", "protocol_model.cpp")

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="no C++ compiler")


def _build(tmp_path, name, *flags):
    exe = str(tmp_path / name)
    r = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pthread", *flags, SRC, "-o", exe],
                       capture_output=True, text=True, timeout=300)
    return exe if r.returncode == 0 else (None, r.stderr)


def _run(exe, calls):
    return subprocess.run([exe, str(calls)], capture_output=True, text=True, timeout=600)


def test_protocol_holds_over_many_calls_and_a_missing_rank(tmp_path):
    exe = _build(tmp_path, "model", "-O2")
    assert isinstance(exe, str), exe
    r = _run(exe, 3000)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr[-2000:]


def _tsan(tmp_path, name, *flags):
    exe = _build(tmp_path, name, "-O1", "-g", "-fsanitize=thread", *flags)
    if not isinstance(exe, str):
        pytest.skip("ThreadSanitizer is not available with this compiler")
    return exe


def test_protocol_has_no_data_race_under_thread_sanitizer(tmp_path):
    r = _run(_tsan(tmp_path, "model_tsan"), 300)
    assert "ThreadSanitizer" not in r.stderr, r.stderr[-4000:]
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr[-2000:]


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5])
def test_planted_protocol_mistakes_are_caught(tmp_path, mutant):
    """1: payload polls ignore the sequence number; 2: the ticket never returns
    its low half to 0, so calls share a flag; 3: barrier posts go to the wrong
    words, so a barrier no longer waits for its peers; 4: the rounds of a
    recursive doubling share one slot set, so a writer overwrites a word its
    reader has not read yet; 5: round tags carry no lap bit, so a reader takes
    the word left two rounds earlier for the current one."""
    exe = _build(tmp_path, f"model_m{mutant}", "-O2", f"-DMODEL_MUTANT={mutant}")
    assert isinstance(exe, str), exe
    r = _run(exe, 300)
    assert r.returncode != 0, f"mutant {mutant} passed: {r.stdout}"


def test_thread_sanitizer_sees_a_broken_barrier(tmp_path):
    """The race check itself works: with the barrier broken (mutant 3), the
    2-stage's plain reads are no longer ordered after the writes."""
    r = _run(_tsan(tmp_path, "model_tsan_m3", "-DMODEL_MUTANT=3"), 50)
    assert "data race" in r.stderr
