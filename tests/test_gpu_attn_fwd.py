"""GPU parity of prism_attn_fwd (tcgen05 kernel) against the float64 oracle
on the library's own plan and selection: O within max-abs 2e-2 and mean-abs
2e-3, LSE within 2e-2; and equality with dense attention (PyTorch SDPA on
the GPU) when every block is selected."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs
from oracle import prism_oracle as O
from tests.helpers import oracle_plan_from_shapes, scale_of, to_np

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 2e-2


def _selection_lists(sel, NB, heads, nb_per_head):
    row_ptr = to_np(sel.row_ptr).astype(np.int64)
    col = to_np(sel.col)[:sel.nnz]
    out = []
    for h in heads:
        out.append([(i, col[row_ptr[h * NB + i]:row_ptr[h * NB + i + 1]], {}) for i in range(nb_per_head[h])])
    return out


def _check(name, heads=None, rows_per_head=None, seed=0):
    w = WORKLOADS[name]
    inp = make_inputs(w, "cuda")
    p = api.params_for(w)
    pl = api.plan(p, inp["V"], inp["a"])
    sel = api.select(p, pl, inp["Q"], inp["K"])
    res = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"])
    torch.cuda.synchronize()
    assert api.workspace_status(res.ws) == 0
    NB = w.N // 64
    heads = list(range(w.heads)) if heads is None else heads
    shapes = to_np(pl.zone_shape)
    nb = to_np(pl.n_blocks)
    ref_plan = oracle_plan_from_shapes(w.T, w.H, w.W, [shapes[h] for h in range(w.heads)])
    lists = _selection_lists(sel, NB, range(w.heads), nb)
    rng = np.random.default_rng(seed)
    Q, K, V = (inp[x].float().cpu().numpy() for x in ("Q", "K", "V"))
    Og = inp["Q"].new_empty(0)
    Og = to_np(res.O.float())
    Lg = to_np(res.lse)
    errs, n = [], 0
    for h in heads:
        hp = ref_plan.heads[h]
        rows = range(nb[h]) if rows_per_head is None else rng.choice(nb[h], size=min(rows_per_head, nb[h]),
                                                                        replace=False)
        for i in rows:
            qi, o, lse = O.attention_fwd_block(Q[:, h], K[:, h], V[:, h], hp, int(i), lists[h][int(i)][1],
                                               scale_of(w.head_dim))
            d = np.abs(Og[qi, h] - o)
            errs.append(d.reshape(-1))
            assert np.abs(Lg[h, qi] - lse).max() < LSE_ABS, (h, i)
    e = np.concatenate(errs)
    print(f"{name}: O max-abs {e.max():.3e} mean-abs {e.mean():.3e} over {e.size} values")
    assert np.isfinite(Og).all()
    assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS


def test_fwd_tiny():
    _check("tiny")


def test_fwd_small_d128():
    _check("small")


def test_fwd_small_d64_multihead():
    _check("small_d64")


def test_fwd_720p_sampled_rows():
    _check("720p", heads=[0, 7, 23], rows_per_head=48)


def test_fwd_1080p_sampled_rows():
    _check("1080p", heads=[0, 23], rows_per_head=16, seed=1)


def test_fwd_select_all_equals_dense_sdpa():
    """Every block selected: the sparse kernel must equal dense attention."""
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cuda")
    NB = w.N // 64
    p = api.params_for(w, topk_abs=NB, top_p=0.5)
    pl = api.plan(p, inp["V"], inp["a"])
    sel = api.select(p, pl, inp["Q"], inp["K"])
    res = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"])
    q, k, v = (inp[x].permute(1, 0, 2).unsqueeze(0) for x in ("Q", "K", "V"))
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float(),
                                                           scale=scale_of(w.head_dim))
    ref = ref.squeeze(0).permute(1, 0, 2)
    d = (res.O.float() - ref).abs()
    print(f"select-all vs dense: max {d.max().item():.3e} mean {d.mean().item():.3e}")
    assert d.max().item() <= MAX_ABS and d.mean().item() <= MEAN_ABS
    s = torch.einsum("qhd,khd->hqk", inp["Q"].float(), inp["K"].float()) * scale_of(w.head_dim)
    lse_ref = torch.logsumexp(s, dim=-1)
    assert (res.lse - lse_ref).abs().max().item() < LSE_ABS


def test_non_finite_input_is_reported():
    """An infinite input has no fp16 pre-scale: the call records
    PRISM_ERR_RANGE in its workspace; the next call on finite inputs is
    clean."""
    w = WORKLOADS["tiny"]
    inp = make_inputs(w, "cuda")
    p = api.params_for(w)
    pl = api.plan(p, inp["V"], inp["a"])
    sel = api.select(p, pl, inp["Q"], inp["K"])
    K = inp["K"].clone()
    K[5, 0, 3] = float("inf")
    res = api.attn_fwd(p, pl, sel, inp["Q"], K, inp["V"])
    assert api.workspace_status(res.ws) == api._lib.PRISM_ERR_RANGE
    ok = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"], ws=res.ws)
    assert api.workspace_status(ok.ws) == 0
