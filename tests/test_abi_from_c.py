"""The C ABI used from plain C: tests/c/abi_host_checks.c includes
include/prism.h as C11 (-Wall -Werror), links libprism.so and runs host-side
checks that return before any CUDA work, so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from dynamic_block_sparse_stats_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_compiles_as_c_and_the_library_links(tmp_path):
    _lib.load()                                  # builds are checked elsewhere; the .so must exist
    exe = tmp_path / "abi_host_checks"
    pkg = os.path.dirname(_lib.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host_checks.c"), "-o", str(exe),
           "-L", pkg, "-l:libprism.so", "-Wl,-rpath," + pkg]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr
