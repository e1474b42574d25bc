"""The fp8 wire's group scale amax / 448 on the device is a product by
RN(1/448) corrected once with fma (Markstein's correction step), not a
division. This checks that formula against the exactly rounded quotient for
every binary32 amax from 2^-120 up (below it the device divides), and that
the check catches the product left uncorrected. The formula is restated in
tests/c/div448_check.c with the same constant and operations (binary32
products and fused multiply-adds, rounded to nearest even)."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "c", "div448_check.c")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    exe = str(tmp_path_factory.mktemp("div448") / "div448_check")
    subprocess.run([gcc, "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-o", exe, SRC, "-lm"],
                   check=True)
    return exe


def test_scale_division_is_exactly_rounded_everywhere(checker):
    res = subprocess.run([checker], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert " 0 mismatches" in res.stdout


def test_the_check_catches_the_uncorrected_product(checker):
    res = subprocess.run([checker, "mutant"], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
