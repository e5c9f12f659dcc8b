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


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _check_tensor(t, name, dtype, shape):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes, device):
    # 256-byte alignment is guaranteed by the CUDA caching allocator
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def a2v_norm(hhat: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """prism_a2v_norm: ||h_hat||_2 of every row of the bf16 bridge output
    h_hat [N, width] (rows may be strided; width a multiple of 8) -> fp32 [N],
    the a2v_norm input of the next layer's plan."""
    if not hhat.is_cuda or hhat.dtype != torch.bfloat16 or hhat.dim() != 2:
        raise ValueError("hhat must be a 2-D bf16 CUDA tensor [N, width]")
    if hhat.stride(1) != 1:
        raise ValueError("hhat rows must be contiguous")
    n, width = hhat.shape
    out = out if out is not None else torch.empty((n,), dtype=torch.float32, device=hhat.device)
    _check_tensor(out, "a2v_norm", torch.float32, (n,))
    ld = hhat.stride(0) if n > 1 else width
    check(_lib.load().prism_a2v_norm(_ptr(hhat), n, width, ld, _ptr(out), _stream(stream)))
    return out


@dataclass
class Plan:
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
    N = p.T * p.H * p.W
    Z = (p.T // 8) * (p.H // 8) * (p.W // 8)
    NB = N // 64
    lib = _lib.load()
    ws = _workspace(lib.prism_plan_workspace_size(C.byref(p)), device)
    return Plan(p, torch.empty((p.heads, Z), dtype=torch.uint8, device=device),
                torch.empty((p.heads, Z, 3), dtype=torch.float64, device=device),
                torch.empty((p.heads, Z), dtype=torch.float64, device=device),
                torch.empty((p.heads,), dtype=torch.int32, device=device),
                torch.empty((p.heads, NB, 4), dtype=torch.int32, device=device),
                torch.empty((p.heads, N), dtype=torch.int32, device=device),
                torch.empty((p.heads, N), dtype=torch.int32, device=device), ws)


def plan(p: PrismParams, V: torch.Tensor, a: torch.Tensor | None = None, out: Plan | None = None,
         stream=None) -> Plan:
    """prism_plan: zone statistics -> volumes, shapes, block table, permutation."""
    N = p.T * p.H * p.W
    _check_tensor(V, "V", torch.bfloat16, (N, p.heads, p.head_dim))
    if a is not None:
        _check_tensor(a, "a2v_norm", torch.float32, (N,))
    out = out or alloc_plan(p, V.device)
    cs = out.c_struct()
    check(_lib.load().prism_plan(C.byref(p), _ptr(V), _ptr(a), C.byref(cs), _ptr(out.ws), out.ws.numel(),
                                 _stream(stream)))
    return out


@dataclass
class Selection:
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
    NB = p.T * p.H * p.W // 64
    lib = _lib.load()
    ws = _workspace(lib.prism_select_workspace_size(C.byref(p)), device)
    rows = p.heads * NB + 1
    return Selection(p, torch.empty((rows,), dtype=torch.int32, device=device),
                     torch.empty((max(cap, 1),), dtype=torch.int32, device=device),
                     torch.empty((rows,), dtype=torch.int32, device=device) if transpose else None,
                     torch.empty((max(cap, 1),), dtype=torch.int32, device=device) if transpose else None,
                     0, ws)


def default_capacity(p: PrismParams) -> int:
    NB = p.T * p.H * p.W // 64
    k = p.topk_abs if p.topk_abs > 0 else max(1, math.ceil(p.topk_frac * NB))
    return p.heads * NB * min(NB, 2 * k + 64)


def select(p: PrismParams, pl: Plan, Q: torch.Tensor, K: torch.Tensor, out: Selection | None = None,
           cap: int | None = None, transpose: bool = True, stream=None) -> Selection:
    """prism_select: block means, block scores, hybrid Top-k U Top-p (CSR and
    optionally its transpose).  Grows the output once if its capacity is short."""
    N = p.T * p.H * p.W
    _check_tensor(Q, "Q", torch.bfloat16, (N, p.heads, p.head_dim))
    _check_tensor(K, "K", torch.bfloat16, (N, p.heads, p.head_dim))
    lib = _lib.load()
    if out is None:
        out = alloc_select(p, Q.device, cap if cap is not None else default_capacity(p), transpose)
    cpl = pl.c_struct()
    for attempt in range(2):
        cs = out.c_struct()
        rc = lib.prism_select(C.byref(p), C.byref(cpl), _ptr(Q), _ptr(K), C.byref(cs), _ptr(out.ws),
                              out.ws.numel(), _stream(stream))
        if rc == _lib.PRISM_ERR_CAPACITY and attempt == 0 and cs.nnz > out.col.numel():
            need = int(cs.nnz)
            out.col = torch.empty((need,), dtype=torch.int32, device=Q.device)
            if out.row is not None:
                out.row = torch.empty((need,), dtype=torch.int32, device=Q.device)
            continue
        check(rc)
        out.nnz = int(cs.nnz)
        return out
    raise AssertionError("unreachable")


@dataclass
class FwdResult:
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
    for name, t in (("Q", Q), ("K", K), ("V", V)):
        _check_tensor(t, name, torch.bfloat16, (N, p.heads, p.head_dim))
    lib = _lib.load()
    O = O if O is not None else torch.empty_like(Q)
    if residual and O_res is None:
        O_res = torch.empty_like(Q)
    lse = lse if lse is not None else torch.empty((p.heads, N), dtype=torch.float32, device=Q.device)
    ws = ws if ws is not None else _workspace(lib.prism_attn_workspace_size(C.byref(p), 0), Q.device)
    cpl, cs = pl.c_struct(), sel.c_struct()
    check(lib.prism_attn_fwd(C.byref(p), C.byref(cpl), C.byref(cs), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                             _ptr(O_res) if residual else None, _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return FwdResult(O, lse, ws, O_res if residual else None)


def attn_bwd(p: PrismParams, pl: Plan, sel: Selection, Q, K, V, O, dO, lse, grad_fp32=False, out=None, ws=None,
             O_res=None, stream=None):
    """prism_attn_bwd: dQ, dK, dV through the selected blocks (natural order).
    Pass the forward's O_res for an fp32-accurate Delta."""
    N = p.T * p.H * p.W
    lib = _lib.load()
    dt = torch.float32 if grad_fp32 else torch.bfloat16
    if out is None:
        out = tuple(torch.empty((N, p.heads, p.head_dim), dtype=dt, device=Q.device) for _ in range(3))
    ws = ws if ws is not None else _workspace(lib.prism_attn_workspace_size(C.byref(p), 1), Q.device)
    cpl, cs = pl.c_struct(), sel.c_struct()
    dQ, dK, dV = out
    check(lib.prism_attn_bwd(C.byref(p), C.byref(cpl), C.byref(cs), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                             _ptr(O_res), _ptr(dO), _ptr(lse), _ptr(dQ), _ptr(dK), _ptr(dV), int(bool(grad_fp32)),
                             _ptr(ws), ws.numel(), _stream(stream)))
    return dQ, dK, dV


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    return _lib.load().prism_workspace_status(_ptr(ws), _stream(stream))
