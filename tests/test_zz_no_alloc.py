"""prism_plan_noalloc: planning without any device allocation by the caller.

Some callers cannot allocate device memory for a workspace: a plugin living
inside another program that owns every device allocation, or code that must
not pay cudaMalloc's implicit device synchronisation.  For them the library
offers prism_plan_noalloc, which keeps its scratch in a fixed device array of
the library.  These tests call it through the C ABI and check that two calls
in a row, on different grids, give exactly what prism_plan gives (up to the
native-2K grid with 24 heads), that a second CUDA context on the same device
gets its own copy of the array, and that a grid whose scratch exceeds the
array is refused with a clear error.

This file is collected last on purpose (see its name), so that a run that
stops at the first failure has already run every other test.
"""
import ctypes as C
import os
import subprocess
import sys

import pytest
import torch

from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRATCH_BYTES = 4 << 20  # the entry point's fixed scratch


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


def test_noalloc_plan_native_2k_grid_fits_and_matches_plan():
    """The grid the fixed scratch is sized for: native 2K, 24 heads."""
    lib = _lib.load()
    w = WORKLOADS["2k"]
    p = api.params_for(w)
    assert lib.prism_plan_workspace_size(C.byref(p)) <= SCRATCH_BYTES
    inp = make_inputs(w, "cuda")
    ref = api.plan(p, inp["V"], inp["a"])
    for _ in range(2):
        _same_plan(_noalloc(p, inp["V"], inp["a"], api.alloc_plan(p, "cuda")), ref, p)


# Runs in a fresh process: plans on the small grid with prism_plan_noalloc in
# the primary context, then in a second context created on the same device
# (cuCtxCreate, buffers from cuMemAlloc, as a host that manages its own
# context would do), then in the primary context again.  Each context has its
# own copy of the library's device array, so each call must use the address
# of its own context's copy.
_SECOND_CONTEXT = r"""
import ctypes as C
import sys
import numpy as np
import torch
sys.path.insert(0, ROOT)
from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs

w = WORKLOADS["small"]
inp = make_inputs(w, "cuda")
p = api.params_for(w)
ref = api.plan(p, inp["V"], inp["a"])
torch.cuda.synchronize()
names = ("zone_shape", "zone_g", "zone_rho", "n_blocks", "blocks", "perm", "inv_perm")
want = {n: getattr(ref, n).cpu().numpy() for n in names}
V_h, a_h = inp["V"].view(torch.int16).cpu().numpy(), inp["a"].cpu().numpy()
lib = _lib.load()

def noalloc(ptrs, Vp, ap, stream):
    cs = _lib.PrismPlan(*[ptrs[n] for n in names])
    _lib.check(lib.prism_plan_noalloc(C.byref(p), C.c_void_p(Vp), C.c_void_p(ap), C.byref(cs), stream))

def same(got):
    for n in names:
        g, r = got[n], want[n]
        if n == "blocks":
            for h in range(p.heads):
                nb = int(want["n_blocks"][h])
                assert np.array_equal(g[h, :nb], r[h, :nb]), n
        else:
            assert np.array_equal(g, r), n

def primary_call():
    out = api.alloc_plan(p, "cuda")
    noalloc({n: getattr(out, n).data_ptr() for n in names}, inp["V"].data_ptr(), inp["a"].data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    same({n: getattr(out, n).cpu().numpy() for n in names})

primary_call()

cu = C.CDLL("libcuda.so.1")
dev = C.c_int()
assert cu.cuDeviceGet(C.byref(dev), torch.cuda.current_device()) == 0
ctx = C.c_void_p()
assert cu.cuCtxCreate_v2(C.byref(ctx), 0, dev) == 0
bufs = {}
try:
    def alloc(nbytes):
        d = C.c_uint64()
        assert cu.cuMemAlloc_v2(C.byref(d), C.c_size_t(max(nbytes, 256))) == 0
        bufs[len(bufs)] = d
        return d.value
    ptrs = {n: alloc(want[n].nbytes) for n in names}
    Vd, ad = alloc(V_h.nbytes), alloc(a_h.nbytes)
    assert cu.cuMemcpyHtoD_v2(C.c_uint64(Vd), V_h.ctypes.data_as(C.c_void_p), C.c_size_t(V_h.nbytes)) == 0
    assert cu.cuMemcpyHtoD_v2(C.c_uint64(ad), a_h.ctypes.data_as(C.c_void_p), C.c_size_t(a_h.nbytes)) == 0
    for _ in range(2):
        noalloc(ptrs, Vd, ad, None)
        assert cu.cuCtxSynchronize() == 0
        got = {}
        for n in names:
            h = np.empty_like(want[n])
            assert cu.cuMemcpyDtoH_v2(h.ctypes.data_as(C.c_void_p), C.c_uint64(ptrs[n]), C.c_size_t(h.nbytes)) == 0
            got[n] = h
        same(got)
finally:
    for d in bufs.values():
        cu.cuMemFree_v2(d)
    cu.cuCtxDestroy_v2(ctx)

primary_call()
print("second-context plans equal prism_plan")
"""


def test_noalloc_plan_in_a_second_context_on_the_same_device():
    code = "ROOT = %r\n" % ROOT + _SECOND_CONTEXT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "second-context plans equal prism_plan" in r.stdout
