"""ctypes binding of libprism.so (the C ABI in include/prism.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Loading fails loudly when the library is missing; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# PRISM_LIB=debug selects the build with device-side bounds checks
LIB_PATH = os.path.join(_HERE, "libprism_debug.so" if os.environ.get("PRISM_LIB") == "debug" else "libprism.so")

PRISM_OK = 0
PRISM_ERR_INVALID_ARG = 1
PRISM_ERR_UNSUPPORTED = 2
PRISM_ERR_CAPACITY = 3
PRISM_ERR_CUDA = 4
PRISM_ERR_TIMEOUT = 5
PRISM_ERR_RANGE = 6
STATUS_NAMES = {0: "PRISM_OK", 1: "PRISM_ERR_INVALID_ARG", 2: "PRISM_ERR_UNSUPPORTED", 3: "PRISM_ERR_CAPACITY",
                4: "PRISM_ERR_CUDA", 5: "PRISM_ERR_TIMEOUT", 6: "PRISM_ERR_RANGE"}

# Every function the header declares, with its ctypes signature.
EXPORTS = (
    "prism_plan_workspace_size", "prism_plan", "prism_select_workspace_size", "prism_select",
    "prism_attn_workspace_size", "prism_attn_fwd", "prism_attn_bwd", "prism_workspace_status",
    "prism_last_error", "prism_version", "prism_kernel_launches", "prism_plan_noalloc",
    "prism_kernel_timing", "prism_kernel_timing_read", "prism_a2v_norm", "prism_diag_exp2",
    "prism_diag_wait_timeout", "prism_project_v_plan",
)
KERNEL_TIMING_IDS = 25  # PRISM_KERNEL_TIMING_IDS in include/prism.h


class PrismParams(C.Structure):
    _fields_ = [("T", C.c_int32), ("H", C.c_int32), ("W", C.c_int32), ("heads", C.c_int32),
                ("head_dim", C.c_int32), ("tau128", C.c_float), ("tau256", C.c_float), ("eps", C.c_float),
                ("topk_frac", C.c_float), ("topk_abs", C.c_int32), ("top_p", C.c_float), ("sm_scale", C.c_float),
                ("map_exponent", C.c_float), ("guidance", C.c_int32), ("density", C.c_int32)]


class PrismPlan(C.Structure):
    _fields_ = [("zone_shape", C.c_void_p), ("zone_g", C.c_void_p), ("zone_rho", C.c_void_p),
                ("n_blocks", C.c_void_p), ("blocks", C.c_void_p), ("perm", C.c_void_p), ("inv_perm", C.c_void_p)]


class PrismSelect(C.Structure):
    _fields_ = [("row_ptr", C.c_void_p), ("col", C.c_void_p), ("cap", C.c_int64), ("nnz", C.c_int64),
                ("col_ptr", C.c_void_p), ("row", C.c_void_p)]


class PrismError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def load() -> C.CDLL:
    """Load libprism.so from the package directory (raises if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}; build it with "
                          "`python -m dynamic_block_sparse_stats_b200.build`"
                          + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
    lib = C.CDLL(LIB_PATH)
    P = C.POINTER
    vp, sz, st = C.c_void_p, C.c_size_t, C.c_void_p
    sig = {
        "prism_plan_workspace_size": (sz, [P(PrismParams)]),
        "prism_plan": (C.c_int, [P(PrismParams), vp, vp, P(PrismPlan), vp, sz, st]),
        "prism_select_workspace_size": (sz, [P(PrismParams)]),
        "prism_select": (C.c_int, [P(PrismParams), P(PrismPlan), vp, vp, P(PrismSelect), vp, sz, st]),
        "prism_attn_workspace_size": (sz, [P(PrismParams), C.c_int]),
        "prism_attn_fwd": (C.c_int, [P(PrismParams), P(PrismPlan), P(PrismSelect), vp, vp, vp, vp, vp, vp, vp, sz,
                                     st]),
        "prism_attn_bwd": (C.c_int, [P(PrismParams), P(PrismPlan), P(PrismSelect), vp, vp, vp, vp, vp, vp, vp, vp,
                                     vp, vp, C.c_int, C.c_int, vp, sz, st]),
        "prism_workspace_status": (C.c_int, [vp, st]),
        "prism_last_error": (C.c_char_p, []),
        "prism_version": (C.c_char_p, []),
        "prism_kernel_launches": (C.c_uint64, []),
        "prism_plan_noalloc": (C.c_int, [P(PrismParams), vp, vp, P(PrismPlan), st]),
        "prism_kernel_timing": (C.c_int, [C.c_int]),
        "prism_kernel_timing_read": (C.c_int, [C.c_int, P(C.c_int), P(C.c_double), P(C.c_char_p)]),
        "prism_a2v_norm": (C.c_int, [vp, C.c_int64, C.c_int32, C.c_int64, vp, st]),
        "prism_diag_exp2": (C.c_int, [vp, vp, vp, C.c_int64, st]),
        "prism_diag_wait_timeout": (C.c_int, [vp, sz, C.c_int64, st]),
        "prism_project_v_plan": (C.c_int, [P(PrismParams), vp, C.c_int32, vp, vp, vp, P(PrismPlan), vp, sz, st]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def check(code: int) -> None:
    if code != PRISM_OK:
        raise PrismError(code, load().prism_last_error().decode(errors="replace"))
