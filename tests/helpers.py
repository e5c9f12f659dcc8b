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


def check_ties(excluded, total, what):
    """Exclusions at logged ties must stay rare: at most 0.1% of the
    decisions checked (and never more than 2 on grids too small for that
    share to reach 1)."""
    print(f"{what}: {excluded} of {total} excluded at ties")
    assert excluded <= max(2.0, 1e-3 * total), f"{what}: {excluded} of {total} decisions excluded at ties"


def compare_plan(w, pl, ref, heads):
    """Library plan vs oracle plan (heads[k] of the library = ref.heads[k]).
    Statistic values within fp32-partial-sum rounding; shapes, block table
    and permutation bit-exact except at decisions whose oracle margin is
    <= TIE.  A zone excluded at a tie changes only its own blocks: every zone
    owns the permuted positions [512m, 512m + 512), so the block-table rows
    and permutation entries of all other zones are still compared.  Returns
    (zone decisions excluded at ties, zones checked)."""
    shapes, g, rho = to_np(pl.zone_shape), to_np(pl.zone_g), to_np(pl.zone_rho)
    nblk, blocks, perm, inv = to_np(pl.n_blocks), to_np(pl.blocks), to_np(pl.perm), to_np(pl.inv_perm)
    excluded = total = 0
    for k, h in enumerate(heads):
        hp = ref.heads[k]
        np.testing.assert_allclose(rho[h], hp.rho, rtol=1e-6, atol=1e-12)
        np.testing.assert_allclose(g[h], hp.g, rtol=1e-6, atol=1e-12)
        diff = shapes[h] != hp.shape
        tie = (hp.vol_margin <= TIE) | (hp.shape_margin <= TIE)
        assert not (diff & ~tie).any(), f"head {h}: shape differs outside ties at zones {np.nonzero(diff & ~tie)}"
        excluded += int((diff & tie).sum())
        total += diff.size
        keep = ~diff                                             # zones whose decisions agree
        nb = hp.blocks.shape[0]
        if not diff.any():
            assert nblk[h] == nb
        got = blocks[h, :nblk[h]]
        got = got[keep[got[:, 0] // 512]]
        want = hp.blocks[keep[hp.blocks[:, 5] // 512]]
        np.testing.assert_array_equal(got[:, 0], want[:, 5])    # p0
        np.testing.assert_array_equal(got[:, 1], want[:, 4])    # B
        np.testing.assert_array_equal(got[:, 2], (want[:, 0] * w.H + want[:, 1]) * w.W + want[:, 2])
        np.testing.assert_array_equal(got[:, 3], want[:, 3])    # shape id
        pos = np.repeat(keep, 512)
        np.testing.assert_array_equal(perm[h][pos], hp.perm[pos])
        np.testing.assert_array_equal(inv[h][perm[h]], np.arange(w.N))
    return excluded, total
