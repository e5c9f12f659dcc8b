"""The C-ABI library loads, exports every function include/prism.h declares,
and validates arguments on the host (no GPU needed: every check below
returns before any CUDA call)."""
import ctypes as C
import os
import re

import pytest

from dynamic_block_sparse_stats_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "prism.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(prism_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_what_the_binding_exports():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_library_loads_and_exports_every_symbol():
    lib = _lib.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.prism_version().decode().count(".") == 2


def test_struct_layouts_match_header():
    assert C.sizeof(_lib.PrismParams) == 15 * 4
    assert C.sizeof(_lib.PrismPlan) == 7 * 8
    assert C.sizeof(_lib.PrismSelect) == 6 * 8


@pytest.mark.parametrize("bad,code", [
    (dict(T=12), _lib.PRISM_ERR_UNSUPPORTED),
    (dict(head_dim=96), _lib.PRISM_ERR_UNSUPPORTED),
    (dict(heads=0), _lib.PRISM_ERR_INVALID_ARG),
    (dict(top_p=-0.5), _lib.PRISM_ERR_INVALID_ARG),
    (dict(tau128=0.1, tau256=0.2), _lib.PRISM_ERR_INVALID_ARG),
    (dict(map_exponent=-1.0), _lib.PRISM_ERR_INVALID_ARG),
    (dict(map_exponent=9.0), _lib.PRISM_ERR_INVALID_ARG),
    (dict(guidance=4), _lib.PRISM_ERR_INVALID_ARG),
    (dict(density=4), _lib.PRISM_ERR_INVALID_ARG),
    (dict(eps=0.0), _lib.PRISM_ERR_INVALID_ARG),
    (dict(topk_abs=-1), _lib.PRISM_ERR_INVALID_ARG),
    (dict(topk_frac=-0.1), _lib.PRISM_ERR_INVALID_ARG),
    (dict(sm_scale=-1.0), _lib.PRISM_ERR_INVALID_ARG),
    (dict(top_p=float("nan")), _lib.PRISM_ERR_INVALID_ARG),
    (dict(tau128=float("nan")), _lib.PRISM_ERR_INVALID_ARG),
    (dict(T=1024, H=1024, W=1024), _lib.PRISM_ERR_UNSUPPORTED),     # N = 2^30 tokens
    (dict(W=0), _lib.PRISM_ERR_INVALID_ARG),
])
def test_invalid_params_are_rejected_before_any_cuda_call(bad, code):
    lib = _lib.load()
    kw = dict(T=8, H=16, W=16, heads=1, head_dim=64, topk_abs=2, top_p=0.9)
    kw.update(bad)
    p = api.params(**kw)
    assert lib.prism_plan_workspace_size(C.byref(p)) == 0
    plan = _lib.PrismPlan(8, 8, 8, 8, 8, 8, 8)  # non-null dummies, never dereferenced
    rc = lib.prism_plan(C.byref(p), C.c_void_p(8), None, C.byref(plan), C.c_void_p(256), 1 << 20, None)
    assert rc == code
    assert lib.prism_last_error().decode()


def test_a2v_density_without_norms_is_rejected():
    lib = _lib.load()
    p = api.params(8, 16, 16, 1, 64, topk_abs=2, density=api.DENSITY_A2V)
    plan = _lib.PrismPlan(256, 256, 256, 256, 256, 256, 256)
    rc = lib.prism_plan(C.byref(p), C.c_void_p(256), None, C.byref(plan), C.c_void_p(256), 1 << 20, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG and "a2v_norm" in lib.prism_last_error().decode()
    assert lib.prism_plan_noalloc(C.byref(p), C.c_void_p(256), None, C.byref(plan), None) == _lib.PRISM_ERR_INVALID_ARG


def test_null_pointers_and_short_workspace_are_rejected():
    lib = _lib.load()
    p = api.params(8, 16, 16, 1, 64, topk_abs=2)
    plan = _lib.PrismPlan(256, 256, 256, 256, 256, 256, 256)
    assert lib.prism_plan(C.byref(p), None, None, C.byref(plan), C.c_void_p(256), 1 << 20, None) == \
        _lib.PRISM_ERR_INVALID_ARG
    need = lib.prism_plan_workspace_size(C.byref(p))
    assert need > 256
    rc = lib.prism_plan(C.byref(p), C.c_void_p(256), None, C.byref(plan), C.c_void_p(256), need - 1, None)
    assert rc == _lib.PRISM_ERR_CAPACITY and "need" in lib.prism_last_error().decode()
    rc = lib.prism_plan(C.byref(p), C.c_void_p(256), None, C.byref(plan), C.c_void_p(264), need, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG  # misaligned workspace
    sel = _lib.PrismSelect(256, 256, 10, 0, 256, None)  # col_ptr without row
    assert lib.prism_select(C.byref(p), C.byref(plan), C.c_void_p(256), C.c_void_p(256), C.byref(sel),
                            C.c_void_p(256), 1 << 30, None) == _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_attn_bwd(C.byref(p), C.byref(plan), C.byref(_lib.PrismSelect(256, 256, 10, 0, None, None)),
                              *([C.c_void_p(256)] * 10), 0, 0, C.c_void_p(256), 1 << 30, None) == _lib.PRISM_ERR_INVALID_ARG


def test_workspace_sizes_grow_with_the_grid():
    lib = _lib.load()
    small = api.params(8, 16, 16, 1, 64)
    big = api.params(56, 96, 160, 24, 128)
    for f in (lib.prism_plan_workspace_size, lib.prism_select_workspace_size):
        assert 0 < f(C.byref(small)) < f(C.byref(big))
    assert lib.prism_attn_workspace_size(C.byref(big), 0) >= 3 * 860160 * 24 * 128 * 2


def test_a2v_norm_argument_checks_need_no_gpu():
    lib = _lib.load()
    ok = C.c_void_p(256)
    assert lib.prism_a2v_norm(ok, 0, 3072, 3072, ok, None) == _lib.PRISM_OK        # n = 0: nothing to do
    assert lib.prism_a2v_norm(ok, -1, 3072, 3072, ok, None) == _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_a2v_norm(ok, 4, 12, 16, ok, None) == _lib.PRISM_ERR_INVALID_ARG   # width % 8
    assert lib.prism_a2v_norm(ok, 4, 64, 56, ok, None) == _lib.PRISM_ERR_INVALID_ARG   # ld < width
    assert lib.prism_a2v_norm(ok, 4, 64, 68, ok, None) == _lib.PRISM_ERR_INVALID_ARG   # ld % 8
    assert lib.prism_a2v_norm(C.c_void_p(264), 4, 64, 64, ok, None) == _lib.PRISM_ERR_INVALID_ARG  # alignment
    assert lib.prism_a2v_norm(None, 4, 64, 64, ok, None) == _lib.PRISM_ERR_INVALID_ARG
    assert "prism_a2v_norm" in lib.prism_last_error().decode()


def test_misaligned_tensor_pointers_are_rejected_before_any_cuda_call():
    """The kernels move rows in 16-byte vectors: a pointer off that grid is an
    argument error, reported before anything is launched."""
    lib = _lib.load()
    p = api.params(8, 16, 16, 1, 64, topk_abs=2)
    plan = _lib.PrismPlan(256, 256, 256, 256, 256, 256, 256)
    ws = C.c_void_p(256)
    rc = lib.prism_plan(C.byref(p), C.c_void_p(8), None, C.byref(plan), ws, 1 << 20, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG and "V" in lib.prism_last_error().decode()
    bad_plan = _lib.PrismPlan(256, 256, 256, 256, 264, 256, 256)     # blocks off by 8 bytes
    rc = lib.prism_plan(C.byref(p), C.c_void_p(256), None, C.byref(bad_plan), ws, 1 << 20, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG and "blocks" in lib.prism_last_error().decode()
    sel = _lib.PrismSelect(256, 256, 10, 0, 256, 256)
    rc = lib.prism_select(C.byref(p), C.byref(plan), C.c_void_p(256), C.c_void_p(258), C.byref(sel), ws, 1 << 30,
                          None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG and "K" in lib.prism_last_error().decode()
    a = [C.c_void_p(256)] * 5
    rc = lib.prism_attn_fwd(C.byref(p), C.byref(plan), C.byref(sel), a[0], a[1], C.c_void_p(264), a[3], a[4],
                            C.c_void_p(256), ws, 1 << 40, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG and "V" in lib.prism_last_error().decode()
    rc = lib.prism_attn_bwd(C.byref(p), C.byref(plan), C.byref(sel), *[C.c_void_p(256)] * 5, C.c_void_p(256),
                            C.c_void_p(256), C.c_void_p(256), C.c_void_p(260), C.c_void_p(256), 1, 0, ws, 1 << 40, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG and "dK" in lib.prism_last_error().decode()
    # the backward's path selector takes 0 (fused) or 1 (deterministic) only
    for det in (2, -1):
        rc = lib.prism_attn_bwd(C.byref(p), C.byref(plan), C.byref(sel), *[C.c_void_p(256)] * 10, 1, det, ws,
                                1 << 40, None)
        assert rc == _lib.PRISM_ERR_INVALID_ARG and "deterministic" in lib.prism_last_error().decode()


def test_backward_workspace_holds_the_fused_accumulator():
    """For head_dim 128 the backward's workspace includes the fused path's
    fp32 dQ accumulator (4 * N * heads * 128 bytes) on top of the two-kernel
    path's needs; head_dim 64 has no fused path and no accumulator."""
    lib = _lib.load()
    for D in (64, 128):
        p = api.params(56, 96, 160, 24, D)
        N = 56 * 96 * 160
        bwd, fwd = lib.prism_attn_workspace_size(C.byref(p), 1), lib.prism_attn_workspace_size(C.byref(p), 0)
        copies = 4 * N * 24 * D * 2      # Q, K, V, dO gathered as fp16
        acc = 4 * N * 24 * D if D == 128 else 0
        assert copies + acc <= bwd < copies + acc + (256 << 20), (D, bwd)  # + LSE, Delta, walk tables
        assert fwd < bwd


@pytest.mark.parametrize("C_", [0, 32, 100, 70000])
def test_project_v_plan_rejects_bad_channel_counts(C_):
    lib = _lib.load()
    p = api.params(8, 16, 16, 1, 64, topk_abs=2)
    dummy = _lib.PrismPlan(256, 256, 256, 256, 256, 256, 256)
    rc = lib.prism_project_v_plan(C.byref(p), C.c_void_p(256), C_, C.c_void_p(256), C.c_void_p(256), None,
                                  C.byref(dummy), C.c_void_p(256), 1 << 20, None)
    assert rc == _lib.PRISM_ERR_INVALID_ARG
    assert "multiple of 64" in lib.prism_last_error().decode()


def test_project_v_plan_rejects_null_and_misaligned_inputs():
    lib = _lib.load()
    p = api.params(8, 16, 16, 1, 64, topk_abs=2)
    dummy = _lib.PrismPlan(256, 256, 256, 256, 256, 256, 256)
    for X, Wv in ((None, 256), (256, None), (264, 256), (256, 260)):
        rc = lib.prism_project_v_plan(C.byref(p), C.c_void_p(X) if X else None, 64, C.c_void_p(Wv) if Wv else None,
                                      C.c_void_p(256), None, C.byref(dummy), C.c_void_p(256), 1 << 20, None)
        assert rc == _lib.PRISM_ERR_INVALID_ARG, (X, Wv)


def test_debug_build_exports_the_same_functions():
    """The PRISM_DEBUG build (device-side bounds checks) is the same ABI."""
    import subprocess
    import sys
    from dynamic_block_sparse_stats_b200 import build
    lib = build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True, check=True).stdout
    names = {ln.split()[-1] for ln in out.splitlines() if " T prism_" in ln}
    assert names == set(declared_functions())
    code = ("import os; os.environ['PRISM_LIB'] = 'debug'; import sys; sys.path.insert(0, %r); "
            "from dynamic_block_sparse_stats_b200 import _lib; l = _lib.load(); "
            "assert _lib.LIB_PATH.endswith('libprism_debug.so'); print(l.prism_version().decode())" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.count(".") == 2, r.stderr
