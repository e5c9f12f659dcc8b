"""Shared helpers for the parity tests: run the library on a workload and
build the oracle's view of the same plan and selection (stage-wise)."""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import prism_oracle as O

TIE = 1e-6  # decision margins at or below this are logged and excluded


def cuda_ok() -> bool:
    return torch.cuda.is_available()


def oracle_plan_from_shapes(T, H, W, shapes):
    """Oracle HeadPlans built from per-head zone shapes (used to check the
    selection and attention stages on the library's own plan)."""
    pl = O.Plan(T, H, W)
    cands = O.candidate_shapes()
    for sid in shapes:
        sid = np.asarray(sid, dtype=np.int64)
        B = np.array([int(np.prod(cands[s])) for s in sid])
        blocks = O.head_blocks(T, H, W, sid)
        pl.heads.append(O.HeadPlan(B, sid, None, None, None, None, blocks, O.permutation(T, H, W, blocks)))
    return pl


def scale_of(head_dim):
    return float(np.float32(1.0 / math.sqrt(head_dim)))


def to_np(t):
    return t.detach().cpu().numpy()


def csr_rows(row_ptr, col, NB, h, i):
    r = h * NB + i
    return col[row_ptr[r]:row_ptr[r + 1]]
