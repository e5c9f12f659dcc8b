"""Parity at the full native-2K training size (56 x 96 x 160 = 860,160 tokens,
24 heads, D = 128), in the launch configuration the benchmark times:
a2v_norm -> plan -> select -> fwd -> bwd through the C ABI on one layer.

The oracle cannot redo the whole layer in test time, so it checks samples
it can compute one by one, stage-wise on the library's own plan and
selection (as everywhere else):
  * plan: every head in full (shapes, block table, permutation bit-exact,
    statistic values within rounding);
  * selection: 32 sampled query blocks on every head, bit-exact except at
    logged ties;
  * forward: O and LSE of 8 sampled query blocks on each of two heads;
  * backward: dQ of 3 sampled query blocks per head, and dK, dV of three key
    blocks per head: one drawn at random, and the ones whose columns (the
    query blocks that selected them) have the head's median and 90th
    percentile length (a key block's gradients need the full rows of all
    its users, which the oracle computes block by block).
Tolerances are the ones of the smaller grids: indices bit-exact, outputs
within max-abs 2e-2 and mean-abs 2e-3 (fp32 gradients)."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_bridge_output, make_inputs
from oracle import prism_oracle as O
from tests.helpers import TIE, check_ties, compare_plan, oracle_plan_from_shapes, scale_of, to_np

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 2e-2
HEADS = (0, 23)
_S = {}


def _layer():
    if _S:
        return _S
    w = WORKLOADS["2k_train"]
    inp = make_inputs(w, "cuda")
    hhat = make_bridge_output(inp["a"], w.heads * w.head_dim)
    p = api.params_for(w)
    a = api.a2v_norm(hhat)
    pl = api.plan(p, inp["V"], a)
    sel = api.select(p, pl, inp["Q"], inp["K"])
    fw = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"])
    g = api.attn_bwd(p, pl, sel, inp["Q"], inp["K"], inp["V"], fw.O, inp["dO"], fw.lse, grad_fp32=True,
                     O_res=fw.O_res)
    torch.cuda.synchronize()
    assert api.workspace_status(pl.ws) == 0 and api.workspace_status(fw.ws) == 0
    del hhat
    NB = w.N // 64
    host = {}
    for h in HEADS:
        host[h] = {x: inp[x][:, h].float().cpu().numpy() for x in ("Q", "K", "V", "dO")}
    _S.update(w=w, inp=inp, p=p, a=a.cpu().numpy(), pl=pl, sel=sel, fw=fw, g=g, host=host, NB=NB,
              nb=to_np(pl.n_blocks), shapes=to_np(pl.zone_shape), row_ptr=to_np(sel.row_ptr).astype(np.int64),
              col=to_np(sel.col)[:sel.nnz], col_ptr=to_np(sel.col_ptr).astype(np.int64),
              rows=to_np(sel.row)[:sel.nnz])
    return _S


def _csr(S, h, i):
    r = h * S["NB"] + i
    return S["col"][S["row_ptr"][r]:S["row_ptr"][r + 1]]


def _csc(S, h, j):
    c = h * S["NB"] + j
    return S["rows"][S["col_ptr"][c]:S["col_ptr"][c + 1]]


def _head(S, h, names):
    """Host copies (fp32) of one head's tensors, [N, 1, D] for the oracle."""
    return [S["inp"][x][:, h:h + 1].float().cpu().numpy() for x in names]


def test_2k_plan_every_head_in_full():
    S = _layer()
    w = S["w"]
    excluded = total = 0
    for h in range(w.heads):
        (V,) = _head(S, h, ("V",))
        ref = O.plan(V, S["a"], w.T, w.H, w.W)
        e, t = compare_plan(w, S["pl"], ref, [h])
        excluded, total = excluded + e, total + t
    check_ties(excluded, total, f"2K plan, {w.heads} heads in full, zone decisions")


def test_2k_selection_sampled_rows_on_every_head():
    S = _layer()
    w = S["w"]
    rng = np.random.default_rng(1)
    excluded = checked = 0
    for h in range(w.heads):
        ref_plan = oracle_plan_from_shapes(w.T, w.H, w.W, [S["shapes"][h]])
        rows = sorted(rng.choice(S["nb"][h], size=32, replace=False).tolist())
        Q, K = _head(S, h, ("Q", "K"))
        ref = O.select(Q, K, ref_plan, w.topk_frac, w.topk_abs, w.top_p, scale_of(w.head_dim), rows=rows)
        for (i, ids, info) in ref[0]:
            checked += 1
            got = _csr(S, h, i)
            if got.size == ids.size and (got == ids).all():
                continue
            if info["p_margin"] <= TIE or info["score_gap"] <= TIE * max(1.0, abs(info["score_gap"])):
                excluded += 1
                continue
            raise AssertionError(f"head {h} row {i}: got {got.size} ids, want {ids.size}; info {info}")
    check_ties(excluded, checked, f"2K selection, rows over {w.heads} heads")


def test_2k_forward_sampled_blocks():
    S = _layer()
    w = S["w"]
    Og, Lg = to_np(S["fw"].O[:, list(HEADS)].float()), to_np(S["fw"].lse)
    rng = np.random.default_rng(2)
    errs = []
    for k, h in enumerate(HEADS):
        hp = oracle_plan_from_shapes(w.T, w.H, w.W, [S["shapes"][h]]).heads[0]
        H_ = S["host"][h]
        for i in rng.choice(S["nb"][h], size=8, replace=False):
            qi, o, lse = O.attention_fwd_block(H_["Q"], H_["K"], H_["V"], hp, int(i), _csr(S, h, int(i)),
                                               scale_of(w.head_dim))
            errs.append(np.abs(Og[qi, k] - o).reshape(-1))
            assert np.abs(Lg[h, qi] - lse).max() < LSE_ABS
    e = np.concatenate(errs)
    print(f"2K O: max-abs {e.max():.3e} mean-abs {e.mean():.3e} over {e.size}")
    assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS


def test_2k_backward_sampled_blocks():
    S = _layer()
    w = S["w"]
    dQ, dK, dV = (to_np(t[:, list(HEADS)]) for t in S["g"])
    scale = scale_of(w.head_dim)
    rng = np.random.default_rng(3)
    errs = {"dQ": [], "dK": [], "dV": []}
    lengths = []
    for k, h in enumerate(HEADS):
        hp = oracle_plan_from_shapes(w.T, w.H, w.W, [S["shapes"][h]]).heads[0]
        sub = O.Plan(w.T, w.H, w.W, [hp])
        H_ = S["host"][h]
        X = [H_[x][:, None] for x in ("Q", "K", "V", "dO")]
        for i in rng.choice(S["nb"][h], size=3, replace=False):
            rQ, _, _ = O.attention_bwd(*X, sub, [[(int(i), _csr(S, h, int(i)), {})]], scale)
            toks = hp.perm[hp.blocks[i, 5]:hp.blocks[i, 5] + hp.blocks[i, 4]]
            errs["dQ"].append(np.abs(dQ[toks, k] - rQ[toks, 0]).reshape(-1))
        # key blocks: one drawn at random, and those whose column (number of
        # query blocks that selected them) has the head's median and 90th
        # percentile length, where dK/dV spends its time
        nbh = int(S["nb"][h])
        cl = np.array([_csc(S, h, j).size for j in range(nbh)])
        order = np.argsort(cl, kind="stable")
        live = order[cl[order] > 0]
        picks = [int(rng.choice(live)), int(live[len(live) // 2]), int(live[(9 * len(live)) // 10])]
        for j in picks:
            users = [(int(i), _csr(S, h, int(i))) for i in _csc(S, h, j)]
            kj, rK, rV = O.attention_bwd_key_block(H_["Q"], H_["K"], H_["V"], H_["dO"], hp, j, users, scale)
            errs["dK"].append(np.abs(dK[kj, k] - rK).reshape(-1))
            errs["dV"].append(np.abs(dV[kj, k] - rV).reshape(-1))
            lengths.append(len(users))
    print(f"2K dK/dV columns checked (users per key block): {lengths}")
    for nm, e in errs.items():
        e = np.concatenate(e)
        print(f"2K {nm}: max-abs {e.max():.3e} mean-abs {e.mean():.3e} over {e.size}")
        assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, nm


def test_2k_gradient_column_sums():
    """Properties that hold at any size, checked on every key of two heads.
    sum_k dV_k = sum_q dO_q, because each query's weights sum to 1; the
    GPU's weights are fp16-rounded (relative 2^-11 each) on top of an fp32
    LSE, so the two sums may differ by (2^-11 + 1e-6) sum_q |dO_q| per
    channel, taken twice.  sum_k dK_k = 0, because each query's dS row sums
    to 0; with P and dS rounded to fp16 a row sum is at most 2^-10 of
    sum_k |dS_qk| <= 2 |dO_q| max_k |v_k|, so per channel c the sum is at most
    2^-10 * scale * sum_q 2 |dO_q| max|v| |q_qc|."""
    S = _layer()
    w = S["w"]
    scale = scale_of(w.head_dim)
    dK, dV = S["g"][1], S["g"][2]
    for h in HEADS:
        dO = S["inp"]["dO"][:, h].double()
        sv = dV[:, h].double().sum(0)
        assert ((sv - dO.sum(0)).abs() <= 2.0 ** -10 * dO.abs().sum(0)).all()
        q = S["inp"]["Q"][:, h].double()
        vmax = S["inp"]["V"][:, h].double().norm(dim=1).max()
        bound = 2.0 ** -10 * scale * (2.0 * dO.norm(dim=1, keepdim=True) * vmax * q.abs()).sum(0)
        sk = dK[:, h].double().sum(0)
        assert (sk.abs() <= bound).all()
