"""A CPU dry run of the benchmark's library arm (bench.run_prism).

The library calls are replaced by stand-ins that return the oracle's plan and
selection of the tiny grid in the library's layout, and CUDA events report a
fixed time.  What runs for real is the benchmark's own orchestration:
warm-up and timed steps with reused buffers, the pair count, the per-kernel
rooflines, the stored DRAM traffic, the oracle's CPU-baseline sample, the
selection report and the JSON line with every key of the contract."""
import argparse
import dataclasses
import json

import numpy as np
import pytest
import torch

import bench
from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS
from oracle import prism_oracle as O

_KERNEL_MS = {"zone_video_stats": 0.1, "block_mean": 0.2, "block_score": 0.05, "select_row": 0.3, "attn_fwd": 8.0,
              "attn_bwd_dkdv": 15.0, "attn_bwd_dq": 10.0, "a2v_norm": 0.05, "zone_a2v_stats": 0.01,
              "plan_finalize": 0.02, "perm": 0.01, "select_scan": 0.01, "csr_fill": 0.01, "csc_count": 0.01,
              "csc_scan": 0.01, "csc_fill": 0.01, "csc_sort": 0.01, "permute3": 0.05, "unit_block": 0.01,
              "tile_units": 0.01, "bwd_prep": 0.03, "project_v": 0.5,
              "range_fix": 0.01, "attn_bwd_fused": 0.0, "dq_convert": 0.0}


class _Lib:
    """The library's host entry points that run_prism calls directly."""

    def __init__(self):
        self.launches = 0

    def prism_attn_workspace_size(self, p, backward):
        return 4096

    def prism_kernel_timing(self, on):
        return 0

    def prism_kernel_launches(self):
        self.launches += 17
        return self.launches

    def prism_kernel_timing_read(self, i, n, ms, name):
        nm = list(_KERNEL_MS)[i]
        n._obj.value, ms._obj.value, name._obj.value = 2, 2 * _KERNEL_MS[nm], nm.encode()
        return 0

    def prism_last_error(self):
        return b""


class _Event:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 25.0


class _Stream:
    cuda_stream = 0


def _oracle_api(monkeypatch, w):
    """api.* stand-ins backed by the oracle (calls are counted)."""
    calls = []
    NB = w.N // 64
    state = {}

    def a2v_norm(hhat, out=None, stream=None):
        calls.append("a2v_norm")
        n = hhat.float().norm(dim=1)
        if out is None:
            return n
        out.copy_(n)
        return out

    def plan(p, V, a, out=None, stream=None):
        calls.append("plan")
        if out is not None:
            return out
        opl = O.plan(V.float().numpy(), a.numpy(), w.T, w.H, w.W)
        blocks = np.zeros((w.heads, NB, 4), np.int32)
        for h, hp in enumerate(opl.heads):
            b = hp.blocks
            blocks[h, :len(b)] = np.stack([b[:, 5], b[:, 4], (b[:, 0] * w.H + b[:, 1]) * w.W + b[:, 2], b[:, 3]], 1)
        state["opl"] = opl
        Z = len(opl.heads[0].shape)
        return api.Plan(p, torch.zeros((w.heads, Z), dtype=torch.uint8), torch.zeros((w.heads, Z, 3), dtype=torch.float64),
                        torch.zeros((w.heads, Z), dtype=torch.float64),
                        torch.tensor([hp.blocks.shape[0] for hp in opl.heads], dtype=torch.int32),
                        torch.tensor(blocks), torch.zeros((w.heads, w.N), dtype=torch.int32),
                        torch.zeros((w.heads, w.N), dtype=torch.int32), torch.zeros(256, dtype=torch.uint8))

    def select(p, pl, Q, K, out=None, cap=None, transpose=True, stream=None):
        calls.append("select")
        if out is not None:
            return out
        osel = O.select(Q.float().numpy(), K.float().numpy(), state["opl"], w.topk_frac, w.topk_abs, w.top_p)
        row_ptr, col = O.csr_from_selection(osel, NB)
        cap = max(cap or 0, col.size)
        colt = torch.zeros(cap, dtype=torch.int32)
        colt[:col.size] = torch.tensor(col)
        return api.Selection(p, torch.tensor(row_ptr, dtype=torch.int32), colt,
                             torch.zeros(row_ptr.size, dtype=torch.int32), torch.zeros(cap, dtype=torch.int32),
                             int(col.size), torch.zeros(256, dtype=torch.uint8))

    def attn_fwd(p, pl, sel, Q, K, V, O=None, lse=None, ws=None, O_res=None, residual=True, stream=None):
        calls.append("attn_fwd")
        return api.FwdResult(O if O is not None else torch.zeros_like(Q),
                             lse if lse is not None else torch.zeros((w.heads, w.N)),
                             ws if ws is not None else torch.zeros(256, dtype=torch.uint8),
                             O_res if O_res is not None else torch.zeros_like(Q))

    def attn_bwd(p, pl, sel, Q, K, V, O, dO, lse, grad_fp32=False, out=None, ws=None, O_res=None, stream=None,
                 deterministic=False):
        calls.append("attn_bwd")
        return out if out is not None else tuple(torch.zeros_like(Q) for _ in range(3))

    def project_v_plan(p, X, Wv, a, V=None, out=None, stream=None):
        calls.append("project_v_plan")
        Vx = (X.float() @ Wv.float().T).to(torch.bfloat16).view(w.N, w.heads, w.head_dim)
        return Vx, plan(p, Vx, a, out=out)

    for name, fn in (("a2v_norm", a2v_norm), ("plan", plan), ("select", select), ("attn_fwd", attn_fwd),
                     ("attn_bwd", attn_bwd), ("project_v_plan", project_v_plan)):
        monkeypatch.setattr(api, name, fn)
    return calls, state


def test_run_prism_orchestration_on_cpu(monkeypatch):
    w = dataclasses.replace(WORKLOADS["tiny"], backward=True)
    calls, state = _oracle_api(monkeypatch, w)
    lib = _Lib()
    monkeypatch.setattr(_lib, "load", lambda: lib)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(bench, "read_stream_gbs", lambda device: 7000.0)
    args = argparse.Namespace(steps=2, warmup=3, no_e2e=True, no_cpu_baseline=False, no_dense=True,
                              shard="layers", workload="tiny", backward=True, no_projection=False,
                              deterministic=True)
    line = bench.run_prism(args, w, rank=0, world=1, device=torch.device("cpu"))
    json.dumps(line)                                        # serialisable as one JSON line

    # 1 set-up pass (select twice) + 3 warm-up + 2 timed steps
    assert calls.count("attn_bwd") == 1 + 3 + 2 and calls.count("select") == 2 + 3 + 2
    P = line["config"]["pairs"]
    assert P > 0 and line["config"]["pair_density"] == P / (w.N * w.N * w.heads)
    assert line["ms_per_step"] == 25.0 / 2
    assert line["value"] == pytest.approx(14.0 * P * w.head_dim / 12.5e-3 / 1e12, rel=1e-12)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "clocks",
                "gpu_launches", "e2e"):
        assert key in line, key
    r = line["roofline"]
    assert r["kernel"] == "attn_bwd_dkdv" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(8.0 * P * w.head_dim / 15e-3 / 1e12, rel=1e-12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-12)
    assert r["traffic"] == bench.stored_traffic("attn_bwd_dkdv")
    assert line["gpu_launches"] == 17
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1 and "query blocks" in cb["sample"]
    sel = line["config"]["selection"]
    assert "error" not in sel and sel["rows"] == sum(hp.blocks.shape[0] for hp in state["opl"].heads)
    assert set(line["stage_ms"]) == {"plan", "select", "fwd", "bwd"}
    assert line["clocks"]["reasons"] == ["nvidia-smi unavailable"] or "sm_mhz" in line["clocks"]
    assert set(line["kernels"]) == set(_KERNEL_MS) | {"attn_bwd", "attn_fwd_bwd"}
    # every step plans through the fused projection (whose stand-in plans with the oracle)
    assert calls.count("project_v_plan") == 1 + 3 + 2 == calls.count("plan")
    pv = line["kernels"]["project_v"]                     # 2*N*C*h*D FLOP per launch, C = h*D here
    assert pv["achieved"] == pytest.approx(2.0 * w.N * (w.heads * w.head_dim) ** 2 / 0.5e-3 / 1e12)
    assert len(_KERNEL_MS) == _lib.KERNEL_TIMING_IDS
    bwd = line["kernels"]["attn_bwd"]                       # the backward on the 10*P*D convention
    assert bwd["achieved"] == pytest.approx(10.0 * P * w.head_dim / 25e-3 / 1e12, rel=1e-12)
    assert line["kernels"]["a2v_norm"]["frac_read_stream"] == pytest.approx(
        line["kernels"]["a2v_norm"]["achieved"] / 7000.0)
