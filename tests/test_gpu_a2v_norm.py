"""GPU parity of prism_a2v_norm (the A2V guidance signal a = ||h_hat||_2 per
video token) against the oracle, through the C ABI.

Tolerance, from the arithmetic: squares of bf16 values are exact in fp32;
each of a lane's eight partial sums adds at most width/256 terms, then a
3-level and a 5-level tree follow, so the fp32 sum of squares is within
(width/256 + 8) * 2^-24 relative of the exact sum (all terms are >= 0), and
the square root halves that and adds at most one more unit of 2^-24 (taken
whole here).  For width 3072 that is 6.6e-7, the rtol of these tests."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_bridge_output, make_inputs
from oracle import prism_oracle as O

pytestmark = pytest.mark.gpu


def _rtol(width):
    return 0.5 * (-(-width // 256) + 8) * 2.0 ** -24 + 2.0 ** -24


def _randn_bf16(n, width, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    mag = torch.exp(torch.randn((n, 1), generator=g, device="cuda") * 3.0)  # magnitudes over ~e^+-9
    return (torch.randn((n, width), generator=g, device="cuda") * mag).to(torch.bfloat16)


@pytest.mark.parametrize("n,width", [(1, 8), (37, 136), (1000, 3072), (4099, 1024), (300, 8200)])
def test_a2v_norm_matches_oracle(n, width):
    h = _randn_bf16(n, width, seed=n + width)
    a = api.a2v_norm(h)
    torch.cuda.synchronize()
    want = O.a2v_norm(h.float().cpu().numpy())
    np.testing.assert_allclose(a.cpu().numpy(), want, rtol=_rtol(width), atol=0)


def test_a2v_norm_strided_rows_and_special_rows():
    big = _randn_bf16(513, 4096, seed=5)
    big[3] = 0                                             # all-zero row -> exactly 0
    big[4, :] = 0
    big[4, 9], big[4, 100] = 3.0, -4.0                     # -> exactly 5
    view = big[:, 8:8 + 3000]                              # ld 4096, 16-byte aligned start
    a = api.a2v_norm(view)
    torch.cuda.synchronize()
    got = a.cpu().numpy()
    want = O.a2v_norm(view.float().cpu().numpy())
    np.testing.assert_allclose(got, want, rtol=_rtol(3000), atol=0)
    assert got[3] == 0.0
    assert got[4] == 5.0                                   # columns 9 and 100 are inside the view


def test_a2v_norm_is_deterministic_and_recovers_the_workload_map():
    w = WORKLOADS["720p"]
    inp = make_inputs(w, "cuda")
    h = make_bridge_output(inp["a"], w.heads * w.head_dim)
    a1 = api.a2v_norm(h)
    a2 = api.a2v_norm(h)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2)
    # chi spread of a 3072-wide Gaussian row (~1.3% rms) plus bf16 rounding
    rel = ((a1 - inp["a"]) / inp["a"]).abs()
    assert rel.mean().item() < 0.02 and rel.max().item() < 0.1
    idx = torch.randperm(w.N, generator=torch.Generator().manual_seed(0))[:2048]
    want = O.a2v_norm(h[idx.cuda()].float().cpu().numpy())
    np.testing.assert_allclose(a1[idx.cuda()].cpu().numpy(), want, rtol=_rtol(3072), atol=0)


def test_a2v_norm_full_2k_size_sampled():
    """The 2K grid's bridge output (860,160 x 3072 bf16, 5.3 GB) in the launch
    configuration the benchmark uses; sampled rows against the oracle."""
    w = WORKLOADS["2k"]
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    a0 = torch.rand((w.N,), generator=g, device="cuda") + 0.05
    h = make_bridge_output(a0, w.heads * w.head_dim, seed=3)
    a = api.a2v_norm(h)
    torch.cuda.synchronize()
    idx = torch.cat([torch.arange(64), torch.arange(w.N - 64, w.N),
                     torch.randperm(w.N, generator=torch.Generator().manual_seed(1))[:4096]]).cuda()
    want = O.a2v_norm(h[idx].float().cpu().numpy())
    np.testing.assert_allclose(a[idx].cpu().numpy(), want, rtol=_rtol(3072), atol=0)
    assert torch.isfinite(a).all() and (a > 0).all()


def test_plan_from_gpu_norms_matches_oracle_plan_from_oracle_norms():
    """The step as a layer runs it: the bridge output's norms feed the plan.
    Stage-wise: the norms are checked against the oracle's, and the oracle
    plans from the library's norms, so a rounding-level difference in a
    cannot move a plan decision."""
    from tests.helpers import compare_plan
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cuda")
    h = make_bridge_output(inp["a"], w.heads * w.head_dim, seed=4)
    a = api.a2v_norm(h)
    p = api.params_for(w)
    pl = api.plan(p, inp["V"], a)
    torch.cuda.synchronize()
    a_got = a.cpu().numpy()
    np.testing.assert_allclose(a_got, O.a2v_norm(h.float().cpu().numpy()), rtol=_rtol(h.shape[1]), atol=0)
    ref = O.plan(inp["V"].float().cpu().numpy(), a_got, w.T, w.H, w.W)
    excluded = compare_plan(w, pl, ref, range(w.heads))
    print(f"plan from bridge-output norms: excluded at ties {excluded}")
