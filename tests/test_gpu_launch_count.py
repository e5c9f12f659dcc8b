"""prism_kernel_launches (the library's own launch counter, which bench.py
reports as gpu_launches) against an independent count: the CUDA kernels the
profiler (CUPTI, through torch.profiler) sees while the whole path runs once
on the tiny grid, both backward paths.  Kernels of the torch runtime (the
wrapper's output allocations) are told apart by name."""
import pytest
import torch

from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_bridge_output, make_inputs

pytestmark = pytest.mark.gpu


def _path(name, deterministic):
    w = WORKLOADS[name]
    inp = make_inputs(w, "cuda", with_grad=True)
    hhat = make_bridge_output(inp["a"], 256)
    p = api.params_for(w)

    def run():
        a = api.a2v_norm(hhat)
        pl = api.plan(p, inp["V"], a)
        sel = api.select(p, pl, inp["Q"], inp["K"])
        fw = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"])
        api.attn_bwd(p, pl, sel, inp["Q"], inp["K"], inp["V"], fw.O, inp["dO"], fw.lse, O_res=fw.O_res,
                     deterministic=deterministic)
        torch.cuda.synchronize()

    return run


def _ours(name):
    return "at::" not in name and "at_cuda_detail" not in name and "cub::" not in name


@pytest.mark.parametrize("name,deterministic", [("tiny", True), ("tiny_d128", False), ("tiny_d128", True)])
def test_launch_counter_matches_the_profiler(name, deterministic):
    run = _path(name, deterministic)
    run()                                            # first use: lazy set-up outside the window
    lib = _lib.load()
    with torch.profiler.profile(activities=[torch.profiler.ProfilerActivity.CUDA]) as prof:
        n0 = lib.prism_kernel_launches()
        run()
        n1 = lib.prism_kernel_launches()
    kernels = [e.name for e in prof.events()
               if e.device_type == torch.autograd.DeviceType.CUDA and "memset" not in e.name.lower()
               and "memcpy" not in e.name.lower()]
    ours = [k for k in kernels if _ours(k)]
    print(f"{name} det={deterministic}: counter {n1 - n0}, profiler {len(ours)} of {len(kernels)} kernels")
    assert n1 - n0 == len(ours), sorted(set(ours))
    assert len(ours) > 0
