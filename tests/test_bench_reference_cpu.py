"""The benchmark's oracle sampler and its reference arm, on the CPU.

The sampler times the oracle on a bounded sample of a layer and extrapolates;
with every query block of a one-head grid in the sample there is nothing to
extrapolate, so its pair count must equal the pairs of the oracle's full
selection, counted here from the oracle's output independently.  The
reference arm must print the benchmark's JSON contract for the oracle arm."""
import argparse
import dataclasses

import numpy as np

import bench
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs
from oracle import prism_oracle as O


def _pairs(hp, row_sets):
    return sum(int(hp.blocks[i, 4]) * int(hp.blocks[ids, 4].sum()) for (i, ids, _) in row_sets)


def test_sampler_with_every_row_counts_the_exact_pairs():
    w = dataclasses.replace(WORKLOADS["tiny"], backward=True)
    inp = make_inputs(w, "cpu", with_grad=True)
    layer_time, P, desc, threads, wall = bench.oracle_sample(w, inp, n_rows=2, n_sel=10 ** 6)
    V, Q, K = (inp[x].float().numpy() for x in ("V", "Q", "K"))
    pl = O.plan(V, inp["a"].numpy(), w.T, w.H, w.W)
    sel = O.select(Q, K, pl, w.topk_frac, w.topk_abs, w.top_p)
    assert P == _pairs(pl.heads[0], sel[0])
    nb = pl.heads[0].blocks.shape[0]
    assert f"selection of {nb} of its {nb} query blocks" in desc and "rows x1.0" in desc
    assert layer_time > 0 and wall > 0 and threads >= 1


def test_sampler_extrapolates_a_row_sample_by_its_fraction():
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cpu")
    _, P, desc, _, _ = bench.oracle_sample(w, inp, head=1, n_rows=1, n_sel=64, seed=3)
    V, Q, K = (inp[x][:, 1:2].float().numpy() for x in ("V", "Q", "K"))
    pl = O.plan(V, inp["a"].numpy(), w.T, w.H, w.W)
    nb = pl.heads[0].blocks.shape[0]
    rows = sorted(np.random.default_rng(3).choice(nb, size=64, replace=False).tolist())
    sel = O.select(Q, K, pl, w.topk_frac, w.topk_abs, w.top_p, rows=rows)
    want = _pairs(pl.heads[0], sel[0]) * (nb / 64) * w.heads
    assert abs(P - want) <= 1e-9 * want
    assert f"selection of 64 of its {nb} query blocks" in desc


def test_reference_arm_prints_the_contract():
    w = WORKLOADS["tiny"]
    args = argparse.Namespace(warmup=3, steps=2, no_projection=False)
    line = bench.run_reference(args, w, rank=0, world=1)
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "tiny" and line["metric"] == bench.METRIC
    assert bench.run_reference(args, w, rank=1, world=2) is None      # other ranks do no work


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    """The launch the driver uses for N > 1, on the CPU: every rank exits 0,
    rank 0 alone prints one JSON line, the other ranks do no work."""
    import json
    import os
    import socket
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
