"""The PRISM_DEBUG build (device-side bounds checks that record
PRISM_ERR_INVALID_ARG in the status word instead of accessing out of
bounds) computes the same bits as the release build on well-formed inputs,
and records no error.  Runs the debug library in a fresh process
(PRISM_LIB=debug selects it at load time)."""
import os
import subprocess
import sys

import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RUN = r"""
import sys, torch
sys.path.insert(0, ROOT)
from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs
assert _lib.LIB_PATH.endswith(LIBNAME), _lib.LIB_PATH
import dataclasses
w = dataclasses.replace(WORKLOADS["small"], backward=True)
inp = make_inputs(w, "cuda")
p = api.params_for(w)
pl = api.plan(p, inp["V"], inp["a"])
sel = api.select(p, pl, inp["Q"], inp["K"])
fw = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"])
nbw = _lib.load().prism_attn_workspace_size(api.C.byref(p), 1)
bws = [torch.empty(nbw, dtype=torch.uint8, device="cuda") for _ in range(2)]
g = api.attn_bwd(p, pl, sel, inp["Q"], inp["K"], inp["V"], fw.O, inp["dO"], fw.lse, grad_fp32=True, O_res=fw.O_res,
                 ws=bws[0], deterministic=True)
gf = api.attn_bwd(p, pl, sel, inp["Q"], inp["K"], inp["V"], fw.O, inp["dO"], fw.lse, grad_fp32=True, O_res=fw.O_res,
                  ws=bws[1], deterministic=False)
torch.cuda.synchronize()
st = [api.workspace_status(x) for x in (pl.ws, sel.ws, fw.ws, bws[0], bws[1])]
torch.save({"perm": pl.perm.cpu(), "col": sel.col[:sel.nnz].cpu(), "O": fw.O.cpu(), "lse": fw.lse.cpu(),
            "dQ": g[0].cpu(), "dK": g[1].cpu(), "dV": g[2].cpu(),
            "dQf": gf[0].cpu(), "dKf": gf[1].cpu(), "dVf": gf[2].cpu(), "status": st}, OUT)
"""


def _run(tmp_path, variant):
    out = str(tmp_path / f"{variant}.pt")
    env = dict(os.environ)
    env.pop("PRISM_LIB", None)
    if variant == "debug":
        env["PRISM_LIB"] = "debug"
    lib = "libprism_debug.so" if variant == "debug" else "libprism.so"
    code = f"ROOT = {ROOT!r}\nOUT = {out!r}\nLIBNAME = {lib!r}\n" + _RUN
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return torch.load(out)


def test_debug_build_matches_release_bits(tmp_path):
    rel = _run(tmp_path, "release")
    dbg = _run(tmp_path, "debug")
    assert dbg["status"] == [0] * 5 and rel["status"] == [0] * 5
    # every output of the deterministic backward, and dK, dV of the fused
    # one, bit for bit; the fused dQ is summed by fp32 reductions in no
    # fixed order
    for k in ("perm", "col", "O", "lse", "dQ", "dK", "dV", "dKf", "dVf"):
        assert torch.equal(rel[k], dbg[k]), k
    d = (rel["dQf"] - dbg["dQf"]).abs().max().item()
    assert d <= 1e-5 * rel["dQf"].abs().max().item(), d
