#!/usr/bin/env python
"""Benchmark of the Prism dynamic block-sparse video self-attention layer.

One step = one pass of the whole path over one synthetic layer:
prism_a2v_norm (the A2V map from the previous layer's bridge output) ->
prism_plan -> prism_select -> prism_attn_fwd -> prism_attn_bwd, on the
native-2K training grid (T=56, H=96, W=160: 860,160 tokens, 24 heads,
head_dim 128, bf16, Top-k 4%, Top-p 0.9) unless --workload says otherwise.

    python bench.py [--gpus N --steps K --warmup W] [--impl prism|reference]

Prints one JSON line (rank 0).  `value` is the effective TFLOP/s of the whole
step over all ranks, counting only the computed blocks: (4 + 10) * P * D per
layer, P = number of computed (query, key) token pairs.  Multi-GPU runs are
weak scaling by default: every rank runs its own independent layer (seeded by
rank).  With --shard heads the ranks split one layer's heads instead (strong
scaling).  Either way the ranks exchange nothing on the path, only the timing
barrier and the max/sum of their measurements.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_stats_b200 import _lib, api  # noqa: E402
from dynamic_block_sparse_stats_b200.synth import (WORKLOADS, make_bridge_output, make_inputs,  # noqa: E402
                                                   make_projection)

METRIC = "Prism sparse-attn fwd+bwd ms/layer & effective TFLOP/s at ~860K tokens"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- ranks
def rank_seed(rank: int) -> int:
    """Each rank runs its own independent layer (weak scaling)."""
    return rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank time over all ranks (identity on one rank)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return world * units_per_rank / (ms_max * 1e-3)


def head_range(rank: int, world: int, heads: int) -> tuple[int, int]:
    """Contiguous, balanced share of a layer's heads for one rank (the path
    has no cross-head exchange: plan, selection and attention are per head,
    and the A2V map is per token, so each rank recomputes it)."""
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def sum_over_ranks(x: float, world: int, device=None) -> float:
    """Sum of a per-rank count over all ranks (measurement only)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------- flops
def computed_pairs(p, pl, sel):
    """P = sum over heads and query blocks i of B_i * sum_{j in S_i} B_j."""
    NB = p.T * p.H * p.W // 64
    row_ptr = sel.row_ptr.long()
    counts = row_ptr[1:] - row_ptr[:-1]
    Bsz = pl.blocks[:, :, 1].reshape(-1).long()            # [heads*NB] (garbage past n_blocks)
    rows = torch.arange(p.heads * NB, device=row_ptr.device)
    valid = (rows % NB) < pl.n_blocks.long().repeat_interleave(NB)
    Bq = torch.where(valid, Bsz, torch.zeros_like(Bsz))
    row_of = torch.repeat_interleave(rows, counts)
    head_of = row_of // NB
    col = sel.col[:sel.nnz].long()
    Bk = Bsz[head_of * NB + col]
    return int((Bq[row_of] * Bk).sum().item())


def selection_stats(p, pl, sel):
    """Realised density per query block over the live rows of all heads: the
    number of selected key blocks, and the share of the head's tokens the
    block's queries attend (sum of B_j over j in S_i, divided by N); each as
    mean, median and 99th percentile (linear interpolation)."""
    NB = p.T * p.H * p.W // 64
    N = p.T * p.H * p.W
    row_ptr = sel.row_ptr.long()
    counts = row_ptr[1:] - row_ptr[:-1]
    rows = torch.arange(p.heads * NB, device=row_ptr.device)
    valid = (rows % NB) < pl.n_blocks.long().repeat_interleave(NB)
    Bsz = pl.blocks[:, :, 1].reshape(-1).long()
    row_of = torch.repeat_interleave(rows, counts)
    col = sel.col[:sel.nnz].long()
    keys = torch.zeros(p.heads * NB, dtype=torch.float64, device=row_ptr.device)
    keys.index_add_(0, row_of, Bsz[(row_of // NB) * NB + col].double())
    q = torch.tensor([0.5, 0.99], dtype=torch.float64, device=row_ptr.device)

    def summary(x):
        qs = torch.quantile(x, q)
        return {"mean": float(x.mean()), "p50": float(qs[0]), "p99": float(qs[1])}

    return {"rows": int(valid.sum()), "blocks_per_row": summary(counts[valid].double()),
            "key_share_per_row": summary(keys[valid] / N)}


# ----------------------------------------------------------------------------- kernel rooflines
def read_kernel_times(lib):
    out = {}
    for i in range(_lib.KERNEL_TIMING_IDS):
        n, ms, name = _lib.C.c_int(0), _lib.C.c_double(0.0), _lib.C.c_char_p()
        _lib.check(lib.prism_kernel_timing_read(i, _lib.C.byref(n), _lib.C.byref(ms), _lib.C.byref(name)))
        out[name.value.decode()] = (n.value, ms.value)
    return out


def kernel_rooflines(ktimes, P, D, N, h, nb, peaks, peak_src, steps, nnz=0, sm_mhz=None, proj_c=None):
    """Per kernel: launches, ms per launch (CUDA events on the launching
    stream, timed region), algorithmic work per launch and its fraction of the
    measured peak: bf16 (sustained, for tensor kernels inside this long step;
    the burst figure is reported beside it) or the STREAM copy bandwidth for
    HBM-bound kernels.  `work` is per step; kernels launched several times per
    step (once per head, or in both the forward and the backward) share it
    evenly.  The backward's two kernels are also reported together as
    `attn_bwd` on the FlashAttention convention, 10*P*D FLOP per layer: dK/dV
    does 8*P*D of it (S^T, dP^T, dV, dK), dQ the remaining 2*P*D (dQ = dS K);
    dQ's recomputed S and dP (4*P*D more) are issued work, reported as
    `issued_TFLOPs`, not algorithmic work.  On the fused path (one kernel
    for dK, dV and dQ, then the accumulator's conversion) `attn_bwd` is
    10*P*D over those two kernels' time, issued and algorithmic alike."""
    sustained = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    burst = peaks.get("bf16_tflops", sustained)
    hbm = peaks["hbm_gbs"]
    fused = bool(ktimes.get("attn_bwd_fused", (0, 0.0))[0])  # the backward ran the fused kernel
    sum_nb2 = float((nb.double() ** 2).sum().item())
    sum_nb = float(nb.double().sum().item())
    Z = N // 512
    HBD, HN = float(N) * h * D, float(N) * h
    spec = {
        # name: (bound, algorithmic work per step, issued work per step or None, description)
        "attn_fwd": ("tensor", 4.0 * P * D, None, "4*P*D FLOP (QK^T and PV on the computed pairs)"),
        "attn_bwd_dkdv": ("tensor", 8.0 * P * D, None, "8*P*D FLOP (S^T, dP^T, dV, dK on the computed pairs)"),
        "attn_bwd_dq": ("tensor", 2.0 * P * D, 6.0 * P * D,
                        "2*P*D FLOP algorithmic (dQ = dS K); 6*P*D issued (S and dP recomputed)"),
        "attn_bwd_fused": ("tensor", 10.0 * P * D, None,
                           "10*P*D FLOP (S^T, dP^T, dV, dK, dQ^T on the computed pairs; dQ added by fp32 "
                           "reductions)"),
        "dq_convert": ("hbm", 6.0 * HBD + 4.0 * HN, None,
                       "fp32 dQ accumulator read, bf16 dQ written (6*N*h*D bytes) + perm (4*N*h)"),
        "zone_video_stats": ("hbm", 2.0 * HBD, None, "one read of V: 2*N*h*D bytes"),
        "zone_a2v_stats": ("hbm", 4.0 * N, None, "one read of the A2V map: 4*N bytes"),
        "plan_finalize": ("hbm", h * Z * 77.0 + 32.0 * Z + 16.0 * sum_nb, None,
                          "zone statistics in, plan tables out: h*Z*77 + 32*Z + 16*sum(N_b) bytes "
                          "(one CTA per head: latency-bound)"),
        "perm": ("hbm", 8.0 * HN + h * Z, None, "perm and inv_perm written: 8*N*h bytes"),
        "block_mean": ("hbm", 4.0 * HBD, None, "one read of Q and K: 4*N*h*D bytes"),
        "block_score": ("alu", 2.0 * D * sum_nb2, None, "2*D*sum_h Nb^2 fp32 FLOP (mul + add)"),
        "select_row": ("hbm", 4.0 * sum_nb2, None, "one read of the fp32 score rows: 4*sum_h Nb^2 bytes"),
        "select_scan": ("hbm", 8.0 * h * (N // 64), None, "row counts in, row offsets out: 8*h*NB bytes"),
        "csr_fill": ("hbm", 4.0 * sum_nb2 + 4.0 * nnz, None, "score rows read, column ids written: "
                                                          "4*sum_h Nb^2 + 4*nnz bytes"),
        "csc_count": ("hbm", 8.0 * nnz, None, "column ids read, column counts incremented: 8*nnz bytes"),
        "csc_scan": ("hbm", 8.0 * h * (N // 64), None, "column counts in, offsets out: 8*h*NB bytes"),
        "csc_fill": ("hbm", 12.0 * nnz, None, "CSR read, transpose written: 12*nnz bytes"),
        "csc_sort": ("hbm", 8.0 * nnz, None, "each transposed column read and written: 8*nnz bytes"),
        "permute3": ("hbm", 2 * (12.0 * HBD + 4.0 * HN), None,
                     "per launch three bf16 tensors read and written as fp16 (12*N*h*D bytes) + perm (4*N*h); "
                     "launched in the forward and the backward"),
        "unit_block": ("hbm", 2 * (16.0 * sum_nb + 4.0 * HN / 64), None,
                       "block table read, unit->block map written (forward and backward)"),
        "tile_units": ("hbm", 3 * 12.0 * nnz, None,
                       "per launch the selection's ids and the block sizes they index (about 12*nnz bytes; "
                       "one launch in the forward, two in the backward)"),
        "bwd_prep": ("hbm", (12.0 if fused else 8.0) * HBD + 16.0 * HN, None,
                     "dO, O, O_res read, fp16 dO written (8*N*h*D bytes) + LSE, Delta (16*N*h)"
                     + (" + the fused path's fp32 dQ accumulator zeroed (4*N*h*D)" if fused else "")),
        "a2v_norm": ("hbm", 2.0 * HBD + 4.0 * N, None,
                     "one read of the bridge output (2*N*h*D bytes) + the fp32 norms (4*N)"),
        "range_fix": ("hbm", None, None, "pre-scale fix-up of operands above the fp16 range: every block "
                                         "returns at once when no value is"),
        "project_v": ("tensor", 2.0 * N * proj_c * h * D if proj_c else None, None,
                      "2*N*C*h*D FLOP (V = X Wv^T; the zone statistics ride in its epilogue)"),
    }
    # nominal dense bf16 rate at the sampled SM clock: 148 SMs x 8192 FLOP per clock
    at_clock = 148 * 8192 * sm_mhz * 1e6 / 1e12 if sm_mhz else None
    out = {}
    for name, (n, ms) in ktimes.items():
        bound, work, issued, desc = spec[name]
        rec = {"launches": n, "total_ms": ms, "ms_per_launch": ms / n if n else None, "bound": bound,
               "algorithmic": desc, "unit": None, "achieved": None, "peak": None, "frac": None, "peak_source": None}
        if n and work is not None and ms > 0:
            per_launch = work * steps / n
            sec = (ms / n) * 1e-3
            if bound == "tensor":
                rec["unit"] = "TFLOP/s"
                rec["achieved"] = per_launch / sec / 1e12
                rec["peak"] = sustained
                rec["peak_source"] = f"{peak_src} bf16 sustained"
                rec["frac_burst"] = rec["achieved"] / burst
                if issued is not None:
                    rec["issued_TFLOPs"] = issued * steps / n / sec / 1e12
                if at_clock:
                    rec["frac_nominal_at_clock"] = (issued or work) * steps / n / sec / 1e12 / at_clock
            elif bound == "hbm":
                rec["unit"] = "GB/s"
                rec["achieved"] = per_launch / sec / 1e9
                rec["peak"] = hbm
                rec["peak_source"] = f"{peak_src} HBM copy"
            else:
                rec["unit"] = "TFLOP/s"
                rec["achieved"] = per_launch / sec / 1e12
                # FP32 SIMT: 148 SMs x 128 lanes x (1 op per lane per cycle) at the max SM clock
                rec["peak"] = 148 * 128 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
                rec["peak_source"] = "derived: 148 SMs x 128 fp32 lanes x max SM clock (one FMUL or FADD each)"
            rec["frac"] = rec["achieved"] / rec["peak"]
        out[name] = rec
    def launched(*names):
        recs = [out.get(n) for n in names]
        return recs if all(r and r["launches"] and r["total_ms"] > 0 for r in recs) else None

    two = launched("attn_bwd_dkdv", "attn_bwd_dq")
    one = launched("attn_bwd_fused", "dq_convert")
    if two or one:
        kd, kq = one or two
        ms_b = kd["ms_per_launch"] + kq["ms_per_launch"]
        t = 10.0 * P * D / (ms_b * 1e-3) / 1e12
        out["attn_bwd"] = {
            "launches": kd["launches"], "ms_per_launch": ms_b, "bound": "tensor", "unit": "TFLOP/s",
            "algorithmic": ("10*P*D FLOP (FlashAttention convention) over the fused kernel + dQ conversion time"
                            if one else "10*P*D FLOP (FlashAttention convention) over dK/dV + dQ time"),
            "path": "fused" if one else "two-kernel deterministic",
            "achieved": t, "peak": sustained, "frac": t / sustained, "frac_burst": t / burst,
            "peak_source": f"{peak_src} bf16 sustained",
            "issued_TFLOPs": (10.0 if one else 14.0) * P * D / (ms_b * 1e-3) / 1e12}
        kf = out.get("attn_fwd")
        if kf and kf["launches"]:
            ms_a = ms_b + kf["ms_per_launch"]
            t = 14.0 * P * D / (ms_a * 1e-3) / 1e12
            out["attn_fwd_bwd"] = {
                "launches": kd["launches"], "ms_per_launch": ms_a, "bound": "tensor", "unit": "TFLOP/s",
                "algorithmic": "14*P*D FLOP over forward + backward time",
                "achieved": t, "peak": sustained, "frac": t / sustained, "frac_burst": t / burst,
                "peak_source": f"{peak_src} bf16 sustained"}
    return out


# The source file of each timed kernel, under the package's csrc/, and the
# ncu kernel-name fragment that identifies its launches.
KERNEL_SOURCES = {"project_v": "project.cu", "zone_video_stats": "plan.cu", "zone_a2v_stats": "plan.cu", "plan_finalize": "plan.cu",
                  "perm": "plan.cu", "block_mean": "select.cu", "block_score": "select.cu",
                  "select_row": "select.cu", "select_scan": "select.cu", "csr_fill": "select.cu",
                  "csc_count": "select.cu", "csc_scan": "select.cu", "csc_fill": "select.cu",
                  "csc_sort": "select.cu", "attn_fwd": "attn_fwd.cu", "permute3": "attn_fwd.cu",
                  "unit_block": "attn_fwd.cu", "tile_units": "attn_fwd.cu", "attn_bwd_dkdv": "attn_bwd.cu",
                  "attn_bwd_dq": "attn_bwd.cu", "bwd_prep": "attn_bwd.cu", "a2v_norm": "a2v_norm.cu",
                  "attn_bwd_fused": "attn_bwd.cu", "dq_convert": "attn_bwd.cu",
                  "range_fix": "range.cu"}
NCU_KERNEL_NAMES = {"a2v_norm": "a2v_norm_kernel", "zone_video_stats": "zone_video_stats_kernel",
                    "block_mean": "block_mean_kernel", "attn_fwd": "attn_fwd_kernel",
                    "attn_bwd_dkdv": "dkdv_kernel", "attn_bwd_dq": "dq_kernel", "attn_bwd_fused": "dkdvq_kernel",
                    "project_v": "project_v_kernel"}


def strip_comments(text: str) -> str:
    """C/C++/CUDA source without its comments and formatting: // and /* */
    comments removed, runs of spaces and tabs outside string and character
    literals reduced to one space, lines trimmed and empty lines dropped (line
    breaks stay: preprocessor directives depend on them)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            if not out or out[-1] != " ":
                out.append(" ")
            i = n if j < 0 else j + 2
        elif c in " \t\r\f\v":
            if not out or out[-1] != " ":
                out.append(" ")
            i += 1
        else:
            out.append(c)
            i += 1
    lines = (ln.strip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln) + "\n"


def source_digest(source: str, csrc=None) -> str:
    """sha256 of a kernel's code: its source file under csrc/ and every local
    header it includes, transitively (quoted #include paths, resolved from the
    including file), each with its comments and blank space removed.  A
    comment edit leaves the digest unchanged; an edit of the code, or of a
    header the code includes, changes it."""
    import hashlib
    import re
    csrc = csrc or os.path.join(ROOT, "dynamic_block_sparse_stats_b200", "csrc")
    todo, seen = [os.path.normpath(os.path.join(csrc, source))], {}
    while todo:
        path = todo.pop()
        if path in seen:
            continue
        with open(path) as f:
            seen[path] = strip_comments(f.read())
        for inc in re.findall(r'^\s*#\s*include\s+"([^"]+)"', seen[path], flags=re.M):
            todo.append(os.path.normpath(os.path.join(os.path.dirname(path), inc)))
    h = hashlib.sha256()
    for path in sorted(seen):
        h.update(os.path.relpath(path, csrc).encode() + b"\0" + seen[path].encode() + b"\0")
    return h.hexdigest()


def stored_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when the summary is missing or the kernel's code (its source file or a
    header it includes) changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    try:
        if source_digest(d["source"]) != d["code_digest"]:
            return None
    except (OSError, KeyError):
        return None
    return d["bytes_per_launch"]


def write_traffic(csv_paths, out_path=None):
    """profiles/traffic.json from ncu captures of dram__bytes_read.sum and
    dram__bytes_write.sum (`ncu --csv --log-file`, one or more files): per
    timed kernel, the mean of read + write bytes over its captured launches,
    keyed to the digest of the kernel's code as it is now (run it on the code
    that was captured)."""
    if isinstance(csv_paths, str):
        csv_paths = [csv_paths]
    records = []
    for k, path in enumerate(csv_paths):
        rows, start = [], False
        with open(path) as f:
            for line in f:
                if line.startswith('"ID"'):
                    start = True
                if start:
                    rows.append(line)
        records += [dict(r, ID=f"{k}:{r['ID']}") for r in csv.DictReader(io.StringIO("".join(rows)))]
    per = {}
    for r in records:
        if r["Metric Name"] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        name = next((k for k, frag in NCU_KERNEL_NAMES.items() if frag in r["Kernel Name"]), None)
        if name is None:
            continue
        scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}[r["Metric Unit"]]
        launch = per.setdefault(name, {}).setdefault(r["ID"], 0.0)
        per[name][r["ID"]] = launch + float(r["Metric Value"].replace(",", "")) * scale
    out = {"_about": "DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch, mean over the "
                     "captured launches of each kernel (see traffic_2k_training_layer.md for the command). "
                     "Valid while the kernel's code digest (bench.source_digest: its source file and the "
                     "headers it includes, comments removed) equals code_digest."}
    for name in NCU_KERNEL_NAMES:
        if name in per:
            vals = list(per[name].values())
            out[name] = {"bytes_per_launch": sum(vals) / len(vals), "launches_captured": len(vals),
                         "source": KERNEL_SOURCES[name], "code_digest": source_digest(KERNEL_SOURCES[name])}
    with open(out_path or os.path.join(ROOT, "profiles", "traffic.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    return out


# ----------------------------------------------------------------------------- oracle sample
def oracle_sample(w, inp, head=0, n_rows=2, n_sel=512, seed=0):
    """Time the CPU oracle on a bounded sample of the same layer: the A2V norms
    of a row sample of a bridge output, the plan of one head over the full
    grid, the selection of `n_sel` seeded query blocks of that head, and
    forward+backward attention of `n_rows` of those blocks.  The layer time is
    extrapolated from the oracle's own numbers only:
      * norms x (N / rows normed);
      * plan x heads;
      * selection: its fixed part (the block means of the head, timed alone)
        plus its per-row part x (blocks of the head / rows selected), x heads;
      * attention x (computed pairs of the layer) / (pairs of the sampled
        blocks), where the layer's pairs are the sampled rows' pairs x
        (blocks / rows selected) x heads.
    Returns (layer time, layer computed pairs, description, threads, wall
    seconds)."""
    from threadpoolctl import threadpool_info

    from oracle import prism_oracle as O
    T, H, W = w.T, w.H, w.W
    Vh = inp["V"][:, head:head + 1].float().cpu().numpy()
    Qh = inp["Q"][:, head:head + 1].float().cpu().numpy()
    Kh = inp["K"][:, head:head + 1].float().cpu().numpy()
    a = inp["a"].cpu().numpy()
    dOh = inp["dO"][:, head:head + 1].float().cpu().numpy() if "dO" in inp else None
    n_norm = min(w.N, 16384)
    hs = make_bridge_output(inp["a"][:n_norm], w.heads * w.head_dim, seed=seed).float().cpu().numpy()
    tn = time.perf_counter()
    O.a2v_norm(hs)
    norm_time = (time.perf_counter() - tn) * (w.N / n_norm)
    del hs
    proj_time, proj_desc = 0.0, ""
    if "X" in inp and "Wv" in inp:    # the value projection of a row sample, all heads
        n_pr = min(w.N, 2048)
        Xs = inp["X"][:n_pr].float().cpu().numpy()
        Ws = inp["Wv"].float().cpu().numpy()
        tp = time.perf_counter()
        O.project_v(Xs, Ws)
        proj_time = (time.perf_counter() - tp) * (w.N / n_pr)
        proj_desc = f"value projection of {n_pr} token rows (x{w.N / n_pr:.0f}, {proj_time:.2f}s); "
        del Xs, Ws
    t0 = time.perf_counter()
    opl = O.plan(Vh, a, T, H, W)
    t1 = time.perf_counter()
    hp = opl.heads[0]
    nb = hp.blocks.shape[0]
    rng = np.random.default_rng(seed)
    sel_rows = sorted(rng.choice(nb, size=min(n_sel, nb), replace=False).tolist())
    O.select(Qh, Kh, opl, w.topk_frac, w.topk_abs, w.top_p, rows=[])      # the fixed part: block means
    t2 = time.perf_counter()
    osel = O.select(Qh, Kh, opl, w.topk_frac, w.topk_abs, w.top_p, rows=sel_rows)
    t3 = time.perf_counter()
    row_frac = nb / len(sel_rows)
    sel_time = (t2 - t1) + max(0.0, (t3 - t2) - (t2 - t1)) * row_frac
    picks = sorted(rng.choice(len(sel_rows), size=min(n_rows, len(sel_rows)), replace=False).tolist())
    sub = [[osel[0][r] for r in picks]]
    scale = float(np.float32(1.0 / math.sqrt(w.head_dim)))
    t4 = time.perf_counter()
    O.attention_fwd(Qh, Kh, Vh, opl, sub, scale)
    if dOh is not None:
        O.attention_bwd(Qh, Kh, Vh, dOh, opl, sub, scale)
    t5 = time.perf_counter()
    pairs_sample = sum(int(hp.blocks[i, 4]) * int(hp.blocks[ids, 4].sum()) for (i, ids, _) in sub[0])
    pairs_rows = sum(int(hp.blocks[i, 4]) * int(hp.blocks[ids, 4].sum()) for (i, ids, _) in osel[0])
    P_total = pairs_rows * row_frac * w.heads
    attn_time = (t5 - t4) * (P_total / max(pairs_sample, 1))
    layer_time = norm_time + proj_time + w.heads * ((t1 - t0) + sel_time) + attn_time
    threads = max([t.get("num_threads", 1) for t in threadpool_info()] + [1])
    desc = (f"oracle A2V norms of {n_norm} bridge-output rows (x{w.N / n_norm:.1f}, {norm_time:.2f}s); {proj_desc}"
            f"plan of head {head} over the full {T}x{H}x{W} grid ({t1 - t0:.2f}s, x{w.heads} heads); "
            f"selection of {len(sel_rows)} of its {nb} query blocks ({t3 - t2:.2f}s, of which block means "
            f"{t2 - t1:.2f}s; rows x{row_frac:.1f}, x{w.heads} heads); fwd{'+bwd' if dOh is not None else ''} "
            f"of {len(picks)} of those blocks ({t5 - t4:.2f}s, x{P_total / max(pairs_sample, 1):.0f} by computed "
            f"pairs, estimated from the selected rows); extrapolated layer time {layer_time:.1f}s")
    return layer_time, P_total, desc, threads, (t5 - t0)


# ----------------------------------------------------------------------------- main arms
def dense_sdpa(inp, w, backward, heads=1, iters=2):
    """Dense bf16 attention (torch scaled_dot_product_attention) over the same
    tokens on the same GPU, timed on `heads` of the layer's heads and scaled to
    all of them (heads are independent and equal in cost).  The fastest
    available backend is tried first; the one that ran is reported."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    import torch.nn.functional as F
    N, D = w.N, w.head_dim
    sub = [inp[k][:, :heads, :].permute(1, 0, 2).unsqueeze(0).contiguous() for k in ("Q", "K", "V")]
    dO = inp["dO"][:, :heads, :].permute(1, 0, 2).unsqueeze(0).contiguous() if backward else None
    stream = torch.cuda.current_stream()
    for be in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION):
        try:
            q, k, v = (t.detach().requires_grad_(backward) for t in sub)

            def run():
                with sdpa_kernel(be):
                    o = F.scaled_dot_product_attention(q, k, v)
                    if backward:
                        torch.autograd.grad(o, (q, k, v), dO)

            run()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(iters):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
            ms_heads = e0.elapsed_time(e1) / iters
            ms = ms_heads * w.heads / heads
            flops = (4.0 + (10.0 if backward else 0.0)) * float(N) * N * D * w.heads
            return {"backend": be.name, "ms_per_layer": ms, "TFLOPs": flops / (ms * 1e-3) / 1e12,
                    "pass": "fwd+bwd" if backward else "fwd",
                    "sample": f"{heads} of {w.heads} heads over all {N} tokens, x{w.heads // heads}",
                    "iters": iters}
        except RuntimeError as e:  # backend refuses the shape: try the next one
            last = f"{be.name}: {str(e).splitlines()[0][:160]}"
    return {"unavailable": last}


def read_stream_gbs(device, nbytes=4 << 30, iters=5):
    """Read-only HBM bandwidth on this GPU, for kernels that only read: a
    sum over a buffer larger than L2 (torch's reduction; a reference figure,
    not part of the path), timed with CUDA events."""
    x = torch.ones(nbytes // 8, dtype=torch.int64, device=device)
    x.sum()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        x.sum()
    e1.record()
    torch.cuda.synchronize(device)
    gbs = nbytes * iters / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del x
    return gbs


def pinned_like(t):
    """A page-locked host tensor of t's shape and dtype."""
    return torch.empty(tuple(t.shape), dtype=t.dtype, pin_memory=True)


def pinned_copy(t):
    """t copied into page-locked host memory directly (no pageable copy in
    between: each rank holds tens of GB of these at the 2K size)."""
    return pinned_like(t).copy_(t)


def run_e2e(args, primary, step, names, backward, total_flops, world, device):
    """The same metric end to end through the public API with host buffers:
    every step copies its inputs from pinned host memory and its results (O,
    and dQ, dK, dV) back.  When the device has room for a second set of those
    tensors, step k+1's inputs go up and step k's results come down on a copy
    stream while step k (k+1) computes; otherwise the copies run in line with
    the steps.  Timed with CUDA events from before the first copy to after the
    last, over ksteps steps."""
    hin = {k: pinned_copy(primary[k]) for k in names}
    outs_of = lambda b: [b["O"]] + (list(b["grads"]) if backward else [])  # noqa: E731
    hout = [pinned_like(t) for t in outs_of(primary)]
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = sum(t.numel() * t.element_size() for t in hout)
    free, _ = torch.cuda.mem_get_info(device)
    overlap = free > h2d + d2h + (4 << 30)
    sets = [primary]
    if overlap:
        second = dict(primary)
        for k in names:
            second[k] = torch.empty_like(primary[k])
        second["O"] = torch.empty_like(primary["O"])
        if backward:
            second["grads"] = tuple(torch.empty_like(t) for t in primary["grads"])
        sets.append(second)
    cs, xs = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ksteps = max(1, min(args.steps, 5))

    def run(k_total):
        ev_in = [torch.cuda.Event() for _ in sets]
        ev_done = [torch.cuda.Event() for _ in sets]
        ev_out = [torch.cuda.Event() for _ in sets]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def up(b):
            with torch.cuda.stream(xs):
                for k_, t in hin.items():
                    sets[b][k_].copy_(t, non_blocking=True)
                ev_in[b].record(xs)

        def down(b):
            xs.wait_event(ev_done[b])
            with torch.cuda.stream(xs):
                for src, dst in zip(outs_of(sets[b]), hout):
                    dst.copy_(src, non_blocking=True)
                ev_out[b].record(xs)

        e0.record(cs)
        xs.wait_event(e0)
        up(0)
        for k in range(k_total):
            b = k % len(sets)
            if len(sets) == 2 and k + 1 < k_total:   # next step's inputs into the other set
                if k >= 1:
                    xs.wait_event(ev_done[1 - b])
                up(1 - b)
            elif len(sets) == 1 and k >= 1:          # in line: after the previous step
                xs.wait_event(ev_done[b])
                up(b)
            cs.wait_event(ev_in[b])
            if k >= len(sets):
                cs.wait_event(ev_out[b])             # the results of step k - 2 (or k - 1) have left
            with torch.cuda.stream(cs):
                step(b=sets[b])
                ev_done[b].record(cs)
            down(b)
        cs.wait_event(ev_out[(k_total - 1) % len(sets)])
        e1.record(cs)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / k_total

    run(1)                                           # warm the copy path
    if world > 1:
        torch.distributed.barrier()
    ems = max_over_ranks(run(ksteps), world, device)
    del hin, hout, sets
    return {"value": total_flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ems,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ksteps,
            "copies": "overlapped with compute (two buffer sets, copy stream)" if overlap else "in line with compute"}


def run_prism(args, w, rank, world, device):
    lib = _lib.load()
    read_gbs = read_stream_gbs(device)
    heads_mode = args.shard == "heads" and world > 1
    if heads_mode and world > w.heads:
        raise SystemExit(f"--shard heads needs at most {w.heads} ranks")
    # layers: every rank its own layer (weak); heads: one layer, heads split over ranks (strong)
    inp = make_inputs(w, device, seed=0 if heads_mode else rank_seed(rank))
    N, h, D = w.N, w.heads, w.head_dim
    h0, h1 = head_range(rank, world, h) if heads_mode else (0, h)
    if heads_mode:
        for k in ("Q", "K", "V", "dO"):
            if k in inp:
                inp[k] = inp[k][:, h0:h1].contiguous()
        import dataclasses
        w = dataclasses.replace(w, heads=h1 - h0)
        h = h1 - h0
    p = api.params_for(w)
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    # the layer's value projection, with the plan's zone statistics in its
    # epilogue (the synthetic V becomes the projection's input features)
    proj = not args.no_projection
    if proj:
        X, Wv = make_projection(V, seed=0 if heads_mode else rank_seed(rank))
        inp["X"], inp["Wv"] = X, Wv
    # the previous layer's bridge output, whose row norms are this layer's A2V map
    hhat = make_bridge_output(inp["a"], (w.heads if not heads_mode else WORKLOADS[args.workload].heads) * D,
                              seed=0 if heads_mode else rank_seed(rank))
    inp["hhat"] = hhat
    dO = inp.get("dO")
    backward = dO is not None
    # buffers reused by every step
    a = api.a2v_norm(hhat)
    if proj:
        V, pl = api.project_v_plan(p, X, Wv, a)
    else:
        pl = api.plan(p, V, a)
    sel = api.select(p, pl, Q, K)
    sel = api.select(p, pl, Q, K, cap=int(sel.nnz * 1.1) + 1024)
    fw = api.attn_fwd(p, pl, sel, Q, K, V)
    O_, lse, O_res = fw.O, fw.lse, fw.O_res
    grads = None
    bws = None
    if backward:
        grads = api.attn_bwd(p, pl, sel, Q, K, V, O_, dO, lse, O_res=O_res, deterministic=args.deterministic)
        bws = torch.empty(lib.prism_attn_workspace_size(api.C.byref(p), 1), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    stages = ["plan", "select", "fwd", "bwd"] if backward else ["plan", "select", "fwd"]

    # the tensors a step reads from the host side (inputs) and hands back to it (results)
    primary = {"Q": Q, "K": K, "V": V, "X": inp.get("X"), "hhat": hhat, "dO": dO, "O": O_, "grads": grads}

    def step(ev=None, b=None):
        b = b or primary
        Qb, Kb, Vb, Ob = b["Q"], b["K"], b["V"], b["O"]
        if ev is not None:
            ev[0].record(stream)
        api.a2v_norm(b["hhat"], out=a)
        if proj:
            api.project_v_plan(p, b["X"], Wv, a, V=Vb, out=pl)
        else:
            api.plan(p, Vb, a, out=pl)
        if ev is not None:
            ev[1].record(stream)
        api.select(p, pl, Qb, Kb, out=sel)
        if ev is not None:
            ev[2].record(stream)
        api.attn_fwd(p, pl, sel, Qb, Kb, Vb, O=Ob, lse=lse, ws=fw.ws, O_res=O_res)
        if ev is not None:
            ev[3].record(stream)
        if backward:
            api.attn_bwd(p, pl, sel, Qb, Kb, Vb, Ob, b["dO"], lse, out=b["grads"], ws=bws, O_res=O_res,
                         deterministic=args.deterministic)
            if ev is not None:
                ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    P = computed_pairs(p, pl, sel)
    flops_fwd, flops_bwd = 4.0 * P * D, (10.0 * P * D if backward else 0.0)
    # whole-job work: the sum of every rank's computed pairs (own layer, or own heads)
    total_flops = sum_over_ranks(flops_fwd + flops_bwd, world, device)
    flops = flops_fwd + flops_bwd

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    lib.prism_kernel_timing(1)
    clk = ClockSampler(torch.cuda.current_device())
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk.start()
    l0 = lib.prism_kernel_launches()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = lib.prism_kernel_launches() - l0
    clocks = clk.stop()
    ktimes = read_kernel_times(lib)
    lib.prism_kernel_timing(0)
    ms = t_start.elapsed_time(t_end) / args.steps
    stage_ms = {s: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps))
                for i, s in enumerate(stages)}
    ms_max = max_over_ranks(ms, world, device)

    # end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, primary, step, names=["Q", "K", "X" if proj else "V", "hhat"] + (["dO"] if backward else []),
                      backward=backward, total_flops=total_flops, world=world, device=device)

    peaks, peak_src = load_peaks()
    nb = pl.n_blocks.long()
    kernels = kernel_rooflines(ktimes, P, D, N, h, nb, peaks, peak_src, args.steps, nnz=sel.nnz,
                               sm_mhz=clocks.get("sm_mhz"), proj_c=X.shape[1] if proj else None)
    for name in ("a2v_norm", "zone_video_stats", "zone_a2v_stats", "block_mean", "select_row"):
        rec = kernels.get(name)
        if rec and rec.get("achieved") is not None:   # read-dominated: also against a read-only stream
            rec["frac_read_stream"] = rec["achieved"] / read_gbs
    dom = max((k for k in kernels if kernels[k]["launches"] and "total_ms" in kernels[k]),
              key=lambda k: kernels[k]["total_ms"])
    kd = kernels[dom]
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"], "peak": kd["peak"],
                "unit": kd["unit"], "frac": kd["frac"], "peak_source": kd["peak_source"],
                "traffic": stored_traffic(dom), "algorithmic": kd["algorithmic"],
                "ms_per_launch": kd["ms_per_launch"]}
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    # the plan stage: a2v_norm reads the bridge output, and the plan reads V
    # (with the fused projection V is written instead, and X read)
    plan_bytes = N * h * D * 2 + N * 4
    plan_bytes += N * h * D * 2 + N * 4 if not proj else N * X.shape[1] * 2 + N * h * D * 2
    stage_roofline = {
        "plan_GBps": plan_bytes / (stage_ms["plan"] * 1e-3) / 1e9,
        "plan_frac_hbm": plan_bytes / (stage_ms["plan"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "fwd_call_TFLOPs": flops_fwd / (stage_ms["fwd"] * 1e-3) / 1e12,
        "fwd_call_frac_bf16": flops_fwd / (stage_ms["fwd"] * 1e-3) / 1e12 / peak,
    }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        layer_time, P_or, desc, threads, wall = oracle_sample(w, inp, n_rows=4, n_sel=2048)
        flops_or = (4.0 + (10.0 if backward else 0.0)) * P_or * D
        cpu = {"value": flops_or / layer_time / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc, "host_cpus": os.cpu_count(), "sample_wall_s": wall}

    dense = None
    if not args.no_dense and world == 1:
        dense = dense_sdpa(inp, w, backward)
        if "ms_per_layer" in dense:
            dense["speedup_of_prism_step"] = dense["ms_per_layer"] / ms

    density = P / (float(N) * N * h)
    try:    # a report of the selection's shape; the measurement above does not depend on it
        selection_report = selection_stats(p, pl, sel)
    except (RuntimeError, ValueError) as e:
        selection_report = {"error": str(e).splitlines()[0][:200]}
    line = {
        "metric": METRIC, "value": total_flops / (ms_max * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "strong" if heads_mode else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded generator; stands in for the pages' 2K-Bench latents)",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "W": w.W, "tokens": N,
                   "heads": WORKLOADS[args.workload].heads, "heads_per_rank": h, "head_dim": D,
                   "topk_frac": w.topk_frac, "top_p": w.top_p, "backward": backward,
                   "bwd_path": (None if not backward else
                                "two-kernel, deterministic" if args.deterministic or D != 128 else
                                "fused dK/dV/dQ, dQ summed by fp32 bulk reductions"),
                   "plan_from": ("prism_project_v_plan: V = X Wv^T (C = %d) with the zone statistics in the "
                                 "GEMM epilogue" % X.shape[1]) if proj else "prism_plan of a given V",
                   "parallelism": (f"heads split over {world} ranks (this rank {h0}-{h1 - 1}), no collectives on the path"
                                   if heads_mode else f"weak x{world} (independent layers, no collectives)"),
                   "l2": "inputs larger than L2 (each bf16 tensor %.2f GB)" % (N * h * D * 2 / 1e9),
                   "pairs": P, "pair_density": density, "nnz_blocks": sel.nnz,
                   "selection": selection_report},
        "stage_ms": stage_ms, "stage_roofline": stage_roofline, "kernels": kernels,
        "read_stream_gbs": read_gbs,
        "clocks": clocks, "e2e": e2e, "gpu_launches": launches, "roofline": roofline, "cpu_baseline": cpu,
        "dense_sdpa": dense,
    }
    return line


def run_reference(args, w, rank, world):
    """The CPU oracle as the reference arm: each step is a bounded sample of the
    same layer (the plan of one head, the selection of a seeded sample of its
    query blocks, fwd+bwd of two of them), extrapolated to the layer."""
    if rank != 0:
        return None
    # inputs are drawn by the seeded generator (on the GPU when there is one,
    # only for speed); every computation below is the CPU oracle's
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, dev, seed=0)  # oracle_sample moves one head at a time to the host
    if not args.no_projection:         # the same step as the library arm: plan from the value projection
        inp["X"], inp["Wv"] = make_projection(inp["V"], seed=0)
    times, rates, desc, threads = [], [], "", 1
    for k in range(args.warmup + args.steps):
        lt, P, desc, threads, _wall = oracle_sample(w, inp, head=k % w.heads, seed=k)
        if k >= args.warmup:
            times.append(lt)
            rates.append((4.0 + (10.0 if w.backward else 0.0)) * P * w.head_dim / lt)
    layer = statistics.mean(times)
    v = statistics.mean(rates) / 1e12
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": layer * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generator; stands in for the pages' 2K-Bench latents)",
            "config": {"workload": w.name, "T": w.T, "H": w.H, "W": w.W, "tokens": w.N, "heads": w.heads,
                       "head_dim": w.head_dim, "topk_frac": w.topk_frac, "top_p": w.top_p, "backward": w.backward,
                       "parallelism": "rank 0 only (CPU oracle)"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["prism", "reference"], default="prism")
    ap.add_argument("--workload", default="2k_train", choices=sorted(WORKLOADS))
    ap.add_argument("--backward", action="store_true", help="time the backward on any workload")
    ap.add_argument("--deterministic", action="store_true",
                    help="backward on the two-kernel, bitwise reproducible path (default: the fused kernel)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense SDPA comparison")
    ap.add_argument("--no-projection", action="store_true",
                    help="plan from a given V (prism_plan) instead of the fused value projection "
                         "(prism_project_v_plan) in the step")
    ap.add_argument("--write-traffic", metavar="NCU_CSV", nargs="+",
                    help="write profiles/traffic.json from an ncu DRAM-bytes capture and exit (no GPU needed)")
    ap.add_argument("--shard", choices=["layers", "heads"], default="layers",
                    help="N>1: every rank its own layer (weak scaling, default) or one layer's heads split "
                         "over the ranks (strong scaling); neither exchanges data on the path")
    args = ap.parse_args()
    if args.write_traffic:
        print(json.dumps(write_traffic(args.write_traffic), indent=1))
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.backward and not w.backward:
        import dataclasses
        w = dataclasses.replace(w, backward=True)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        # one process per GPU: N > 1 ranks come from the launcher (torchrun), never from this process
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N > 1 GPUs with "
                 f"`python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py --gpus {args.gpus} ...`")

    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the prism arm has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        line = run_prism(args, w, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
