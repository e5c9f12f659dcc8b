"""prism_plan_noalloc: planning without any device allocation by the caller.

Some callers cannot allocate device memory for a workspace: a plugin living
inside another program that owns every device allocation, or code that must
not pay cudaMalloc's implicit device synchronisation.  For them the library
offers prism_plan_noalloc, which keeps its scratch in a fixed device array of
the library.  These tests call it through the C ABI and check that two calls
in a row, on different grids, give exactly what prism_plan gives, and that a
grid whose scratch exceeds the array is refused with a clear error.

This file is collected last on purpose (see its name), so that a run that
stops at the first failure has already run every other test.
"""
import ctypes as C

import pytest
import torch

from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _noalloc(p, V, a, out):
    lib = _lib.load()
    cs = out.c_struct()
    rc = lib.prism_plan_noalloc(C.byref(p), C.c_void_p(V.data_ptr()),
                                C.c_void_p(a.data_ptr()) if a is not None else None, C.byref(cs),
                                torch.cuda.current_stream().cuda_stream)
    _lib.check(rc)
    return out


def _same_plan(got, ref, p):
    torch.cuda.synchronize()
    assert torch.equal(got.n_blocks, ref.n_blocks)
    assert torch.equal(got.zone_shape, ref.zone_shape)
    assert torch.equal(got.zone_g, ref.zone_g)
    assert torch.equal(got.zone_rho, ref.zone_rho)
    assert torch.equal(got.perm, ref.perm)
    assert torch.equal(got.inv_perm, ref.inv_perm)
    for h in range(p.heads):
        nb = int(ref.n_blocks[h])
        assert torch.equal(got.blocks[h, :nb], ref.blocks[h, :nb])


def test_noalloc_plan_matches_plan_on_two_calls_in_a_row():
    cases = []
    for name in ("small", "tiny"):
        w = WORKLOADS[name]
        inp = make_inputs(w, "cuda")
        p = api.params_for(w)
        ref = api.plan(p, inp["V"], inp["a"])                    # caller-workspace path
        cases.append((p, inp, ref))
    # two calls in a row on different grids, outputs into fresh buffers
    for p, inp, ref in cases:
        got = _noalloc(p, inp["V"], inp["a"], api.alloc_plan(p, "cuda"))
        _same_plan(got, ref, p)
    # and the first grid again, after the second one overwrote the scratch
    p, inp, ref = cases[0]
    _same_plan(_noalloc(p, inp["V"], inp["a"], api.alloc_plan(p, "cuda")), ref, p)


def test_noalloc_plan_first_layer_without_a2v_norms():
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cuda")
    p = api.params_for(w)
    ref = api.plan(p, inp["V"], None)
    _same_plan(_noalloc(p, inp["V"], None, api.alloc_plan(p, "cuda")), ref, p)


def test_noalloc_plan_refuses_grids_beyond_its_scratch():
    lib = _lib.load()
    p = api.params(128, 256, 256, 24, 128)          # 16,384 zones x 24 heads: ~17 MB of scratch
    dummy = _lib.PrismPlan(256, 256, 256, 256, 256, 256, 256)
    rc = lib.prism_plan_noalloc(C.byref(p), C.c_void_p(256), None, C.byref(dummy), None)
    assert rc == _lib.PRISM_ERR_CAPACITY
    msg = lib.prism_last_error().decode()
    assert "scratch" in msg and "prism_plan" in msg
