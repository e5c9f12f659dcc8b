"""Failure detection without a GPU fault: every wait inside the library's
kernels is bounded, and a wait that runs out records PRISM_ERR_TIMEOUT in
the workspace status word instead of hanging.  prism_diag_wait_timeout runs
that path on an mbarrier nothing completes; the test checks the recorded
status and that the context is still usable afterwards."""
import ctypes as C

import pytest
import torch

from dynamic_block_sparse_stats_b200 import _lib, api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_records_timeout_and_context_survives():
    lib = _lib.load()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    _lib.check(lib.prism_diag_wait_timeout(C.c_void_p(ws.data_ptr()), 256, 2_000_000, stream))  # ~1 ms
    assert lib.prism_workspace_status(C.c_void_p(ws.data_ptr()), stream) == _lib.PRISM_ERR_TIMEOUT
    assert int(ws[4:8].view(torch.int32).item()) == 900          # the wait's site code
    # a zero limit gives up at once, the same way
    _lib.check(lib.prism_diag_wait_timeout(C.c_void_p(ws.data_ptr()), 256, 0, stream))
    assert lib.prism_workspace_status(C.c_void_p(ws.data_ptr()), stream) == _lib.PRISM_ERR_TIMEOUT
    # the context is intact: a full plan runs and agrees with itself
    w = WORKLOADS["tiny"]
    inp = make_inputs(w, "cuda")
    p = api.params_for(w)
    a = api.plan(p, inp["V"], inp["a"])
    b = api.plan(p, inp["V"], inp["a"])
    torch.cuda.synchronize()
    assert torch.equal(a.perm, b.perm) and api.workspace_status(a.ws) == _lib.PRISM_OK


def test_wait_timeout_argument_checks():
    lib = _lib.load()
    assert lib.prism_diag_wait_timeout(None, 256, 10, None) == _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_diag_wait_timeout(C.c_void_p(256), 255, 10, None) == _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_diag_wait_timeout(C.c_void_p(256), 256, 2_000_000_000, None) == _lib.PRISM_ERR_INVALID_ARG
