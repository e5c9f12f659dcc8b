"""Attention operands beyond the fp16 range (|x| > 65504, valid bf16).

The tensor-core operands are fp16; a (tensor, head) holding a larger value is
converted with a power-of-two pre-scale that the kernels fold back exactly.
Power-of-two scalings commute with every rounding on the path except where
a value crosses fp16's subnormal boundary (2^-14), so the inputs here have
no magnitudes in (0, 2^-12), and scaling an input by 2^17 must scale the
outputs exactly:
  * K x 2^17 (all heads) with the attention scale x 2^-17: the same
    scores, hence the same selection, O, LSE, dQ and dV bit for bit, and
    dK x 2^-17;
  * V x 2^17: O x 2^17 and the same LSE, dV unchanged; dQ and dK x 2^17
    within the parity tolerance (the unscaled run keeps dS entries below
    2^-14 as fp16 subnormals, the scaled run as normal numbers);
  * dO x 2^17: dV x 2^17 exactly, dQ and dK x 2^17 within the tolerance.
Against the unscaled run of the same layer (itself checked against the oracle
by the other attention tests), on a grid with two heads where only head 1 is
scaled, so head 0 also checks that an in-range head is untouched."""
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs
from tests.helpers import scale_of

pytestmark = pytest.mark.gpu

S17 = 2.0 ** 17
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _no_tiny(x):
    """x with magnitudes below 2^-12 set to zero (exactly representable)."""
    return torch.where(x.float().abs() < 2.0 ** -12, torch.zeros_like(x), x)


def _close(got, want):
    d = (got.double() - want.double()).abs()
    assert d.max().item() <= MAX_ABS and d.mean().item() <= MEAN_ABS, (d.max().item(), d.mean().item())


def _layer(w, Q, K, V, dO, a, sm_scale=0.0, deterministic=True):
    """The bit-for-bit comparisons below use the deterministic backward (the
    fused one sums dQ in no fixed order); the fused path is checked against
    it on the same out-of-range inputs at the end."""
    p = api.params_for(w, sm_scale=sm_scale)
    pl = api.plan(p, V, a)
    sel = api.select(p, pl, Q, K)
    fw = api.attn_fwd(p, pl, sel, Q, K, V)
    g = api.attn_bwd(p, pl, sel, Q, K, V, fw.O, dO, fw.lse, grad_fp32=True, O_res=fw.O_res,
                     deterministic=deterministic)
    torch.cuda.synchronize()
    assert api.workspace_status(fw.ws) == 0
    return sel, fw, g


def _scaled(x, head, f):
    y = x.clone()
    y[:, head] = (y[:, head].float() * f).to(x.dtype)  # exact: a power of two
    return y


@pytest.fixture(scope="module")
def base():
    import dataclasses
    w = dataclasses.replace(WORKLOADS["small"], backward=True)
    inp = make_inputs(w, "cuda")
    for k in ("Q", "K", "V", "dO"):
        inp[k] = _no_tiny(inp[k])
    return w, inp, _layer(w, inp["Q"], inp["K"], inp["V"], inp["dO"], inp["a"])


def test_large_keys_with_a_compensating_scale(base):
    w, inp, (sel0, fw0, g0) = base
    # the attention scale is one parameter for all heads, so every head's K
    # is scaled here
    K = _scaled(_scaled(inp["K"], 0, S17), 1, S17)
    assert K.float().abs().max().item() > 65504
    sel, fw, g = _layer(w, inp["Q"], K, inp["V"], inp["dO"], inp["a"], sm_scale=scale_of(w.head_dim) / S17)
    assert sel.nnz == sel0.nnz and torch.equal(sel.col[:sel.nnz], sel0.col[:sel0.nnz])
    assert torch.equal(fw.O, fw0.O) and torch.equal(fw.lse, fw0.lse)
    assert torch.equal(g[0], g0[0]) and torch.equal(g[2], g0[2])
    assert torch.equal(g[1] * S17, g0[1])


def test_large_values(base):
    w, inp, (sel0, fw0, g0) = base
    V = _scaled(inp["V"], 1, S17)
    assert V.float().abs().max().item() > 65504
    # the plan is scale invariant (a power-of-two scaling of V leaves it bit-identical)
    sel, fw, g = _layer(w, inp["Q"], inp["K"], V, inp["dO"], inp["a"])
    assert torch.equal(fw.O[:, 0], fw0.O[:, 0]) and torch.equal(fw.lse, fw0.lse)
    assert torch.equal(fw.O[:, 1].float(), fw0.O[:, 1].float() * S17)
    assert torch.equal(g[2], g0[2])
    for k in (0, 1):
        assert torch.equal(g[k][:, 0], g0[k][:, 0])
        _close(g[k][:, 1] / S17, g0[k][:, 1])


def test_large_upstream_gradient(base):
    w, inp, (sel0, fw0, g0) = base
    dO = _scaled(inp["dO"], 1, S17)
    assert dO.float().abs().max().item() > 65504
    sel, fw, g = _layer(w, inp["Q"], inp["K"], inp["V"], dO, inp["a"])
    for k in range(3):
        assert torch.equal(g[k][:, 0], g0[k][:, 0])
    assert torch.equal(g[2][:, 1], g0[2][:, 1] * S17)
    for k in (0, 1):
        _close(g[k][:, 1] / S17, g0[k][:, 1])


@pytest.mark.parametrize("which", ["K", "V", "dO"])
def test_fused_backward_with_out_of_range_heads(base, which):
    """The fused backward folds the same pre-scales back (dK, dV in its
    stores, dQ in the conversion pass): on each out-of-range input it gives
    the deterministic path's dK and dV bit for bit and its dQ within a few
    fp32 roundings."""
    w, inp, _ = base
    x = dict(Q=inp["Q"], K=inp["K"], V=inp["V"], dO=inp["dO"])
    sm = 0.0
    if which == "K":
        x["K"] = _scaled(_scaled(inp["K"], 0, S17), 1, S17)
        sm = scale_of(w.head_dim) / S17
    else:
        x[which] = _scaled(inp[which], 1, S17)
    assert x[which].float().abs().max().item() > 65504
    _, _, gd = _layer(w, x["Q"], x["K"], x["V"], x["dO"], inp["a"], sm_scale=sm, deterministic=True)
    _, _, gf = _layer(w, x["Q"], x["K"], x["V"], x["dO"], inp["a"], sm_scale=sm, deterministic=False)
    assert torch.equal(gf[1], gd[1]) and torch.equal(gf[2], gd[2])
    d = (gf[0] - gd[0]).abs().max().item()
    assert d <= 1e-5 * gd[0].abs().max().item(), d
