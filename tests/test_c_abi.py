"""The boundary from plain C: vrar.h compiles as strict C (and C++), and a C99
program that includes it and links libvrar.so and the CUDA runtime builds
here and, on a GPU, reproduces exact integer sums for every algorithm, the
reduce-scatter and the all-gather in all three element types (tests/c/)."""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "collective_all_reduce_virtual_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
EXAMPLE = os.path.join(ROOT, "tests", "c", "abi_example.c")

needs_cc = pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")


def _cc(*args, cwd=None):
    return subprocess.run(["gcc", *args], capture_output=True, text=True, cwd=cwd, timeout=120)


@needs_cc
@pytest.mark.parametrize("std", ["c89", "c99", "c11"])
def test_header_is_strict_c(tmp_path, std):
    src = tmp_path / "h.c"
    src.write_text('#include "vrar.h"\nint main(void) { return vrar_version() > 0 ? 0 : 1; }\n')
    r = _cc(f"-std={std}", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, "-c", str(src), "-o",
            str(tmp_path / "h.o"))
    assert r.returncode == 0, r.stderr


@pytest.mark.skipif(shutil.which("g++") is None, reason="no C++ compiler")
def test_header_is_strict_cxx(tmp_path):
    src = tmp_path / "h.cpp"
    src.write_text('#include "vrar.h"\nint main() { return vrar_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run(["g++", "-std=c++11", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, "-c",
                        str(src), "-o", str(tmp_path / "h.o")], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr


def build_example(out_dir) -> str:
    exe = os.path.join(str(out_dir), "abi_example")
    lib64 = os.path.join(CUDA, "lib64")
    r = _cc("-std=c99", "-Wall", "-Wextra", "-Werror", "-O2", "-I", INCLUDE, "-I", os.path.join(CUDA, "include"),
            EXAMPLE, "-L", PKG, "-lvrar", "-L", lib64, "-lcudart", f"-Wl,-rpath,{PKG}:{lib64}", "-o", exe)
    assert r.returncode == 0, r.stderr
    return exe


@needs_cc
def test_c_example_builds_and_links(tmp_path):
    if not os.path.exists(os.path.join(PKG, "libvrar.so")):
        pytest.skip("libvrar.so not built")
    assert os.path.exists(build_example(tmp_path))


@needs_cc
@pytest.mark.gpu
def test_c_example_runs_on_the_gpu(tmp_path):
    exe = build_example(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]
