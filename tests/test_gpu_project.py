"""GPU parity of prism_project_v_plan (the value projection with the zone
statistics in its epilogue) through the C ABI.

  * V = X Wv^T against the oracle's float64 product: within the bf16
    rounding of the output (half an ulp: at most 2^-8 of the value, bf16
    having 8 significant bits) plus the fp32 accumulation error
    (C * 2^-24 * sum_c |x_c w_c|, taken four times);
  * the plan from the epilogue's statistics is bit-identical to prism_plan's
    plan of the V just written (both run the same statistics arithmetic);
  * stage-wise, that plan equals the oracle's plan of the same V except at
    logged ties;
  * two calls in a row give the same bits, and the first layer (no A2V map)
    works too."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs, make_projection
from oracle import prism_oracle as O
from tests.helpers import check_ties, compare_plan, to_np

pytestmark = pytest.mark.gpu

PLAN_FIELDS = ("zone_shape", "zone_g", "zone_rho", "n_blocks", "perm", "inv_perm")


def _same_plan(a, b, heads):
    for name in PLAN_FIELDS:
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    for h in range(heads):
        nb = int(b.n_blocks[h])
        assert torch.equal(a.blocks[h, :nb], b.blocks[h, :nb])


def _check_v(X, Wv, V, rows):
    """V rows against the oracle product, within bf16 output rounding plus
    the fp32 accumulation bound (taken four times: the tensor core's
    accumulation order and rounding are its own)."""
    idx = torch.as_tensor(rows, device=X.device)
    Xh = X[idx].float().cpu().numpy()
    Wh = Wv.float().cpu().numpy()
    ref = O.project_v(Xh, Wh)
    mag = np.abs(Xh) @ np.abs(Wh).T
    got = V.reshape(V.shape[0], -1)[idx].float().cpu().numpy()
    bound = 2.0 ** -8 * np.abs(ref) + 4.0 * Xh.shape[1] * 2.0 ** -24 * mag + 1e-30
    err = np.abs(got - ref)
    print(f"V: max |err| / bound = {(err / bound).max():.3f} over {err.size} values")
    assert (err <= bound).all()


@pytest.mark.parametrize("name", ["small", "small_d64", "720p"])
def test_project_v_plan_matches_oracle_and_plan(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, "cuda")
    X, Wv = make_projection(inp["V"])
    p = api.params_for(w)
    V, pl = api.project_v_plan(p, X, Wv, inp["a"])
    torch.cuda.synchronize()
    assert api.workspace_status(pl.ws) == 0
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(w.N, size=min(w.N, 4096), replace=False))
    _check_v(X, Wv, V, rows)
    # the same plan as prism_plan of this V
    ref = api.plan(p, V, inp["a"])
    _same_plan(pl, ref, w.heads)
    # and, stage-wise, the oracle's plan of this V
    heads = list(range(w.heads)) if w.heads <= 3 else [0, 11, 23]
    oref = O.plan(V[:, heads].float().cpu().numpy(), inp["a"].cpu().numpy(), w.T, w.H, w.W)
    excluded, total = compare_plan(w, pl, oref, heads)
    check_ties(excluded, total, f"{name} projected plan zones")


def test_project_v_plan_twice_and_first_layer():
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cuda")
    X, Wv = make_projection(inp["V"])
    p = api.params_for(w)
    V1, pl1 = api.project_v_plan(p, X, Wv, inp["a"])
    V2, pl2 = api.project_v_plan(p, X, Wv, inp["a"])
    torch.cuda.synchronize()
    assert torch.equal(V1, V2)
    _same_plan(pl1, pl2, w.heads)
    V3, pl3 = api.project_v_plan(p, X, Wv, None)
    ref = api.plan(p, V3, None)
    torch.cuda.synchronize()
    assert torch.equal(V3, V1)
    _same_plan(pl3, ref, w.heads)


def test_project_v_plan_general_weight_and_width():
    """A dense random weight and an input width that is not heads * D."""
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    Cin = 192
    X = torch.randn((w.N, Cin), generator=g, device="cuda").to(torch.bfloat16)
    Wv = (torch.randn((w.heads * w.head_dim, Cin), generator=g, device="cuda") / Cin ** 0.5).to(torch.bfloat16)
    p = api.params_for(w)
    V, pl = api.project_v_plan(p, X, Wv, inp["a"])
    torch.cuda.synchronize()
    assert api.workspace_status(pl.ws) == 0
    rng = np.random.default_rng(6)
    _check_v(X, Wv, V, np.sort(rng.choice(w.N, size=2048, replace=False)))
    _same_plan(pl, api.plan(p, V, inp["a"]), w.heads)
