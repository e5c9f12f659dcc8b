"""The product path has no CPU fallback: without libprism.so the binding
raises ImportError, and without a GPU the benchmark's library arm stops
with a clear message instead of computing anything on the host."""
import os
import subprocess
import sys

import pytest
import torch

from dynamic_block_sparse_stats_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_missing_library_raises_import_error(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libprism.so"))
    with pytest.raises(ImportError, match="libprism.so not found"):
        _lib.load()
    p = api.params(8, 16, 16, 1, 64, topk_abs=2)
    with pytest.raises(ImportError):
        api.alloc_plan(p, "cpu")


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the CPU-only behaviour")
def test_bench_library_arm_refuses_to_run_without_a_gpu():
    r = subprocess.run([sys.executable, "bench.py", "--steps", "1", "--warmup", "3", "--workload", "tiny"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "needs a CUDA device" in r.stderr
    assert not any(ln.startswith("{") for ln in r.stdout.splitlines())
