"""Torch-facing wrapper of the Prism C ABI.

PyTorch provides device memory and the current stream; every computation runs
in libprism.so.  Tensors follow the layout of include/prism.h:
Q, K, V, O, dO bf16 [N, heads, head_dim] contiguous on one CUDA device, the
A2V norm map fp32 [N].
"""
from __future__ import annotations

import ctypes as C
import math
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import PrismParams, PrismPlan, PrismSelect, check


# guidance bits and density modes of the ablation variants (include/prism.h)
GUIDE_NO_VIDEO, GUIDE_NO_A2V = 1, 2
DENSITY_BOTH, DENSITY_SPATIAL, DENSITY_TEMPORAL, DENSITY_A2V = 0, 1, 2, 3


def params(T, H, W, heads, head_dim, topk_frac=0.0, topk_abs=0, top_p=0.9, tau128=0.5, tau256=0.25,
           eps=1e-6, sm_scale=0.0, map_exponent=0.0, guidance=0, density=0) -> PrismParams:
    """Layer parameters; map_exponent 0 means the Lagrange value 1/2, and
    guidance = density = 0 is the method as published."""
    return PrismParams(T, H, W, heads, head_dim, tau128, tau256, eps, topk_frac, topk_abs, top_p, sm_scale,
                       map_exponent, guidance, density)


def params_for(w, **over) -> PrismParams:
    """Parameters of a synthetic workload (dynamic_block_sparse_stats_b200.synth.Workload)."""
    kw = dict(topk_frac=w.topk_frac, topk_abs=w.topk_abs, top_p=w.top_p)
    kw.update(over)
    return params(w.T, w.H, w.W, w.heads, w.head_dim, **kw)


def _stream(stream, device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _check_tensor(t, name, dtype, shape):
    """Structure of one tensor argument: type, dtype, shape, contiguity.  The
    C ABI sees bare pointers, so buffer sizes can only be checked here."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_workspace(ws, name):
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 1-D uint8 tensor")


def _check_devices(named) -> torch.device:
    """Every (name, tensor) pair, None entries skipped, must live on one CUDA
    device; returns it.  Run after the structural checks, so that a wrong
    size is reported before a wrong device."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other arguments on {dev}")
    return dev


def _grid(p: PrismParams):
    return (p.T, p.H, p.W, p.heads, p.head_dim)


def _check_grid(p: PrismParams, q: PrismParams, what: str):
    if _grid(p) != _grid(q):
        raise ValueError(f"{what} was made for (T, H, W, heads, head_dim) = {_grid(q)}, "
                         f"the call is for {_grid(p)}")


def _sizes(p: PrismParams):
    N = p.T * p.H * p.W
    return N, (p.T // 8) * (p.H // 8) * (p.W // 8), N // 64


def _workspace(nbytes, device):
    # 256-byte alignment is guaranteed by the CUDA caching allocator
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def a2v_norm(hhat: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """prism_a2v_norm: ||h_hat||_2 of every row of the bf16 bridge output
    h_hat [N, width] (rows may be strided; width a multiple of 8) -> fp32 [N],
    the a2v_norm input of the next layer's plan."""
    if not isinstance(hhat, torch.Tensor) or hhat.dtype != torch.bfloat16 or hhat.dim() != 2:
        raise ValueError("hhat must be a 2-D bf16 tensor [N, width]")
    if hhat.stride(1) != 1:
        raise ValueError("hhat rows must be contiguous")
    n, width = hhat.shape
    if out is not None:
        _check_tensor(out, "a2v_norm", torch.float32, (n,))
    dev = _check_devices([("hhat", hhat), ("a2v_norm", out)])
    ld = hhat.stride(0) if n > 1 else width
    with torch.cuda.device(dev):
        out = out if out is not None else torch.empty((n,), dtype=torch.float32, device=dev)
        check(_lib.load().prism_a2v_norm(_ptr(hhat), n, width, ld, _ptr(out), _stream(stream, dev)))
    return out


@dataclass
class Plan:
    """Output of prism_plan (device tensors, Z zones, NB = N/64):
    zone_shape u8 [heads, Z] candidate id per zone; zone_g f64 [heads, Z, 3]
    (g_T, g_H, g_W); zone_rho f64 [heads, Z] normalised density; n_blocks
    i32 [heads]; blocks i32 [heads, NB, 4] {first permuted position, volume,
    natural index of the block's origin token, candidate id} (rows past
    n_blocks unspecified); perm / inv_perm i32 [heads, N]; ws the call's
    workspace."""
    p: PrismParams
    zone_shape: torch.Tensor
    zone_g: torch.Tensor
    zone_rho: torch.Tensor
    n_blocks: torch.Tensor
    blocks: torch.Tensor
    perm: torch.Tensor
    inv_perm: torch.Tensor
    ws: torch.Tensor

    def c_struct(self) -> PrismPlan:
        return PrismPlan(self.zone_shape.data_ptr(), self.zone_g.data_ptr(), self.zone_rho.data_ptr(),
                         self.n_blocks.data_ptr(), self.blocks.data_ptr(), self.perm.data_ptr(),
                         self.inv_perm.data_ptr())


def alloc_plan(p: PrismParams, device) -> Plan:
    N, Z, NB = _sizes(p)
    lib = _lib.load()
    ws = _workspace(lib.prism_plan_workspace_size(C.byref(p)), device)
    return Plan(p, torch.empty((p.heads, Z), dtype=torch.uint8, device=device),
                torch.empty((p.heads, Z, 3), dtype=torch.float64, device=device),
                torch.empty((p.heads, Z), dtype=torch.float64, device=device),
                torch.empty((p.heads,), dtype=torch.int32, device=device),
                torch.empty((p.heads, NB, 4), dtype=torch.int32, device=device),
                torch.empty((p.heads, N), dtype=torch.int32, device=device),
                torch.empty((p.heads, N), dtype=torch.int32, device=device), ws)


def _check_plan(p: PrismParams, pl: Plan):
    """Structural checks of a plan against the call's grid; returns its
    named tensors for the device check."""
    if not isinstance(pl, Plan):
        raise TypeError(f"plan must be an api.Plan, got {type(pl).__name__}")
    _check_grid(p, pl.p, "the plan")
    N, Z, NB = _sizes(p)
    h = p.heads
    named = []
    for name, dtype, shape in (("zone_shape", torch.uint8, (h, Z)), ("zone_g", torch.float64, (h, Z, 3)),
                               ("zone_rho", torch.float64, (h, Z)), ("n_blocks", torch.int32, (h,)),
                               ("blocks", torch.int32, (h, NB, 4)), ("perm", torch.int32, (h, N)),
                               ("inv_perm", torch.int32, (h, N))):
        _check_tensor(getattr(pl, name), "plan." + name, dtype, shape)
        named.append(("plan." + name, getattr(pl, name)))
    _check_workspace(pl.ws, "plan.ws")
    return named + [("plan.ws", pl.ws)]


def plan(p: PrismParams, V: torch.Tensor, a: torch.Tensor | None = None, out: Plan | None = None,
         stream=None) -> Plan:
    """prism_plan: zone statistics -> volumes, shapes, block table, permutation."""
    N = p.T * p.H * p.W
    _check_tensor(V, "V", torch.bfloat16, (N, p.heads, p.head_dim))
    if a is not None:
        _check_tensor(a, "a2v_norm", torch.float32, (N,))
    named = [("V", V), ("a2v_norm", a)] + (_check_plan(p, out) if out is not None else [])
    dev = _check_devices(named)
    with torch.cuda.device(dev):
        out = out if out is not None else alloc_plan(p, dev)
        cs = out.c_struct()
        check(_lib.load().prism_plan(C.byref(p), _ptr(V), _ptr(a), C.byref(cs), _ptr(out.ws), out.ws.numel(),
                                     _stream(stream, dev)))
    return out


def project_v_plan(p: PrismParams, X: torch.Tensor, Wv: torch.Tensor, a: torch.Tensor | None = None,
                   V: torch.Tensor | None = None, out: Plan | None = None, stream=None):
    """prism_project_v_plan: V = X Wv^T (bf16 [N, heads, head_dim]) with the
    plan computed from the zone statistics of the projection's own tiles.
    X bf16 [N, C], Wv bf16 [heads*head_dim, C].  Returns (V, plan)."""
    N = p.T * p.H * p.W
    if not isinstance(X, torch.Tensor) or X.dim() != 2:
        raise ValueError("X must be a 2-D tensor [N, C]")
    Cin = X.shape[1]
    _check_tensor(X, "X", torch.bfloat16, (N, Cin))
    _check_tensor(Wv, "Wv", torch.bfloat16, (p.heads * p.head_dim, Cin))
    if V is not None:
        _check_tensor(V, "V", torch.bfloat16, (N, p.heads, p.head_dim))
    if a is not None:
        _check_tensor(a, "a2v_norm", torch.float32, (N,))
    named = [("X", X), ("Wv", Wv), ("V", V), ("a2v_norm", a)] + (_check_plan(p, out) if out is not None else [])
    dev = _check_devices(named)
    with torch.cuda.device(dev):
        V = V if V is not None else torch.empty((N, p.heads, p.head_dim), dtype=torch.bfloat16, device=dev)
        out = out if out is not None else alloc_plan(p, dev)
        cs = out.c_struct()
        check(_lib.load().prism_project_v_plan(C.byref(p), _ptr(X), Cin, _ptr(Wv), _ptr(V), _ptr(a), C.byref(cs),
                                               _ptr(out.ws), out.ws.numel(), _stream(stream, dev)))
    return V, out


@dataclass
class Selection:
    """Output of prism_select (device tensors): a CSR over rows h*NB + i
    (head h, query block i) with row_ptr i32 [heads*NB + 1] and col i32
    [capacity] (selected key blocks, ascending; the first nnz entries are
    valid), and optionally its transpose col_ptr / row (needed by the
    backward); ws the call's workspace."""
    p: PrismParams
    row_ptr: torch.Tensor
    col: torch.Tensor
    col_ptr: torch.Tensor | None
    row: torch.Tensor | None
    nnz: int
    ws: torch.Tensor

    def c_struct(self) -> PrismSelect:
        return PrismSelect(self.row_ptr.data_ptr(), self.col.data_ptr(), self.col.numel(), self.nnz,
                           self.col_ptr.data_ptr() if self.col_ptr is not None else None,
                           self.row.data_ptr() if self.row is not None else None)


def alloc_select(p: PrismParams, device, cap: int, transpose: bool = True) -> Selection:
    _, _, NB = _sizes(p)
    lib = _lib.load()
    ws = _workspace(lib.prism_select_workspace_size(C.byref(p)), device)
    rows = p.heads * NB + 1
    return Selection(p, torch.empty((rows,), dtype=torch.int32, device=device),
                     torch.empty((max(cap, 1),), dtype=torch.int32, device=device),
                     torch.empty((rows,), dtype=torch.int32, device=device) if transpose else None,
                     torch.empty((max(cap, 1),), dtype=torch.int32, device=device) if transpose else None,
                     0, ws)


def _check_selection(p: PrismParams, sel: Selection, transpose: bool):
    """Structural checks of a selection against the call's grid; returns its
    named tensors for the device check."""
    if not isinstance(sel, Selection):
        raise TypeError(f"selection must be an api.Selection, got {type(sel).__name__}")
    _check_grid(p, sel.p, "the selection")
    _, _, NB = _sizes(p)
    rows = p.heads * NB + 1
    if not isinstance(sel.col, torch.Tensor) or sel.col.dim() != 1:
        raise ValueError("selection.col must be a 1-D tensor")
    cap = sel.col.numel()
    _check_tensor(sel.row_ptr, "selection.row_ptr", torch.int32, (rows,))
    _check_tensor(sel.col, "selection.col", torch.int32, (cap,))
    if (sel.col_ptr is None) != (sel.row is None):
        raise ValueError("selection.col_ptr and selection.row must both be set or both be None")
    if sel.col_ptr is not None:
        _check_tensor(sel.col_ptr, "selection.col_ptr", torch.int32, (rows,))
        _check_tensor(sel.row, "selection.row", torch.int32, (cap,))
    elif transpose:
        raise ValueError("the backward needs the selection's transpose (select(..., transpose=True))")
    if not 0 <= sel.nnz <= cap:
        raise ValueError(f"selection.nnz = {sel.nnz} exceeds its capacity {cap}")
    _check_workspace(sel.ws, "selection.ws")
    return [("selection.row_ptr", sel.row_ptr), ("selection.col", sel.col), ("selection.col_ptr", sel.col_ptr),
            ("selection.row", sel.row), ("selection.ws", sel.ws)]


def default_capacity(p: PrismParams) -> int:
    _, _, NB = _sizes(p)
    k = p.topk_abs if p.topk_abs > 0 else max(1, math.ceil(p.topk_frac * NB))
    return p.heads * NB * min(NB, 2 * k + 64)


def select(p: PrismParams, pl: Plan, Q: torch.Tensor, K: torch.Tensor, out: Selection | None = None,
           cap: int | None = None, transpose: bool = True, stream=None) -> Selection:
    """prism_select: block means, block scores, hybrid Top-k U Top-p (CSR and
    optionally its transpose).  Grows the output once if its capacity is short."""
    N = p.T * p.H * p.W
    _check_tensor(Q, "Q", torch.bfloat16, (N, p.heads, p.head_dim))
    _check_tensor(K, "K", torch.bfloat16, (N, p.heads, p.head_dim))
    named = [("Q", Q), ("K", K)] + _check_plan(p, pl)
    if out is not None:
        named += _check_selection(p, out, False)
    dev = _check_devices(named)
    lib = _lib.load()
    with torch.cuda.device(dev):
        if out is None:
            out = alloc_select(p, dev, cap if cap is not None else default_capacity(p), transpose)
        cpl = pl.c_struct()
        for attempt in range(2):
            cs = out.c_struct()
            rc = lib.prism_select(C.byref(p), C.byref(cpl), _ptr(Q), _ptr(K), C.byref(cs), _ptr(out.ws),
                                  out.ws.numel(), _stream(stream, dev))
            if rc == _lib.PRISM_ERR_CAPACITY and attempt == 0 and out.col.numel() < cs.nnz <= 0x7fffffff:
                need = int(cs.nnz)
                out.col = torch.empty((need,), dtype=torch.int32, device=dev)
                if out.row is not None:
                    out.row = torch.empty((need,), dtype=torch.int32, device=dev)
                continue
            check(rc)
            out.nnz = int(cs.nnz)
            return out
    raise AssertionError("unreachable")


@dataclass
class FwdResult:
    """Output of prism_attn_fwd: O bf16 [N, heads, D] (natural order), lse
    f32 [heads, N] (natural log), ws the call's workspace (its status word
    says whether a kernel recorded an error), O_res the bf16 rounding
    residual of O, or None."""
    O: torch.Tensor
    lse: torch.Tensor
    ws: torch.Tensor
    O_res: torch.Tensor | None = None


def attn_fwd(p: PrismParams, pl: Plan, sel: Selection, Q, K, V, O=None, lse=None, ws=None, O_res=None,
             residual: bool = True, stream=None) -> FwdResult:
    """prism_attn_fwd: attention over the selected blocks; O natural order,
    lse [heads, N]; with `residual`, also O's bf16 rounding residual for the
    backward's Delta."""
    N = p.T * p.H * p.W
    shape = (N, p.heads, p.head_dim)
    for name, t in (("Q", Q), ("K", K), ("V", V)):
        _check_tensor(t, name, torch.bfloat16, shape)
    if O is not None:
        _check_tensor(O, "O", torch.bfloat16, shape)
    if residual and O_res is not None:
        _check_tensor(O_res, "O_res", torch.bfloat16, shape)
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32, (p.heads, N))
    if ws is not None:
        _check_workspace(ws, "ws")
    named = [("Q", Q), ("K", K), ("V", V), ("O", O), ("O_res", O_res if residual else None), ("lse", lse),
             ("ws", ws)] + _check_plan(p, pl) + _check_selection(p, sel, False)
    dev = _check_devices(named)
    lib = _lib.load()
    with torch.cuda.device(dev):
        O = O if O is not None else torch.empty_like(Q)
        if residual and O_res is None:
            O_res = torch.empty_like(Q)
        lse = lse if lse is not None else torch.empty((p.heads, N), dtype=torch.float32, device=dev)
        ws = ws if ws is not None else _workspace(lib.prism_attn_workspace_size(C.byref(p), 0), dev)
        cpl, cs = pl.c_struct(), sel.c_struct()
        check(lib.prism_attn_fwd(C.byref(p), C.byref(cpl), C.byref(cs), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                 _ptr(O_res) if residual else None, _ptr(lse), _ptr(ws), ws.numel(),
                                 _stream(stream, dev)))
    return FwdResult(O, lse, ws, O_res if residual else None)


def attn_bwd(p: PrismParams, pl: Plan, sel: Selection, Q, K, V, O, dO, lse, grad_fp32=False, out=None, ws=None,
             O_res=None, stream=None, deterministic=False):
    """prism_attn_bwd: dQ, dK, dV through the selected blocks (natural order).
    Pass the forward's O_res for an fp32-accurate Delta.  deterministic=False
    (head_dim 128) takes the fused kernel, whose dQ is summed by fp32
    reductions in no fixed order; True takes the two-kernel path, bitwise
    reproducible."""
    N = p.T * p.H * p.W
    shape = (N, p.heads, p.head_dim)
    for name, t in (("Q", Q), ("K", K), ("V", V), ("O", O), ("dO", dO)):
        _check_tensor(t, name, torch.bfloat16, shape)
    if O_res is not None:
        _check_tensor(O_res, "O_res", torch.bfloat16, shape)
    _check_tensor(lse, "lse", torch.float32, (p.heads, N))
    dt = torch.float32 if grad_fp32 else torch.bfloat16
    if out is not None:
        if len(out) != 3:
            raise ValueError("out must hold the three gradients (dQ, dK, dV)")
        for name, t in zip(("dQ", "dK", "dV"), out):
            _check_tensor(t, name, dt, shape)
    if ws is not None:
        _check_workspace(ws, "ws")
    named = [("Q", Q), ("K", K), ("V", V), ("O", O), ("dO", dO), ("O_res", O_res), ("lse", lse), ("ws", ws)]
    if out is not None:
        named += list(zip(("dQ", "dK", "dV"), out))
    named += _check_plan(p, pl) + _check_selection(p, sel, True)
    dev = _check_devices(named)
    lib = _lib.load()
    with torch.cuda.device(dev):
        if out is None:
            out = tuple(torch.empty(shape, dtype=dt, device=dev) for _ in range(3))
        ws = ws if ws is not None else _workspace(lib.prism_attn_workspace_size(C.byref(p), 1), dev)
        cpl, cs = pl.c_struct(), sel.c_struct()
        dQ, dK, dV = out
        check(lib.prism_attn_bwd(C.byref(p), C.byref(cpl), C.byref(cs), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                 _ptr(O_res), _ptr(dO), _ptr(lse), _ptr(dQ), _ptr(dK), _ptr(dV),
                                 int(bool(grad_fp32)), int(bool(deterministic)), _ptr(ws), ws.numel(),
                                 _stream(stream, dev)))
    return dQ, dK, dV


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    """The status word a call left in its workspace (PRISM_OK, or the error a
    kernel recorded, e.g. PRISM_ERR_TIMEOUT or PRISM_ERR_RANGE)."""
    _check_workspace(ws, "ws")
    dev = _check_devices([("ws", ws)])
    with torch.cuda.device(dev):
        return _lib.load().prism_workspace_status(_ptr(ws), _stream(stream, dev))
