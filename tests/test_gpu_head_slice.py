"""Head sharding on the CUDA path: the library run on a slice of a layer's
heads gives, bit for bit, the same plan, selection, forward and backward
outputs as the same heads of the full-layer call.  The path has no
cross-head step (plan, selection and attention are per head; the A2V map is
per token and shared), which is what `bench.py --shard heads` relies on when
it splits one layer's heads over ranks.  The fused backward sums dQ in no
fixed order, so for it dK and dV are compared bit for bit and dQ within a
few fp32 roundings; the deterministic backward is compared bit for bit."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs
from tests.helpers import to_np

pytestmark = pytest.mark.gpu


def _run(w, inp):
    p = api.params_for(w)
    pl = api.plan(p, inp["V"], inp["a"])
    sel = api.select(p, pl, inp["Q"], inp["K"])
    fw = api.attn_fwd(p, pl, sel, inp["Q"], inp["K"], inp["V"])
    g = [api.attn_bwd(p, pl, sel, inp["Q"], inp["K"], inp["V"], fw.O, inp["dO"], fw.lse, O_res=fw.O_res,
                      grad_fp32=True, deterministic=det) for det in (True, False)]
    torch.cuda.synchronize()
    assert api.workspace_status(fw.ws) == 0
    return pl, sel, fw, g


def _rows(sel, h, NB):
    rp = to_np(sel.row_ptr).astype(np.int64)
    col = to_np(sel.col)[:sel.nnz]
    return [col[rp[h * NB + i]:rp[h * NB + i + 1]] for i in range(NB)]


@pytest.mark.parametrize("h0,h1", [(12, 24), (5, 6)])
def test_head_slice_equals_full_layer(h0, h1):
    import dataclasses
    w = dataclasses.replace(WORKLOADS["720p"], backward=True)
    inp = make_inputs(w, "cuda")
    full = _run(w, inp)
    ws = dataclasses.replace(w, heads=h1 - h0)
    sub_inp = {k: (v[:, h0:h1].contiguous() if k in ("Q", "K", "V", "dO") else v) for k, v in inp.items()}
    part = _run(ws, sub_inp)
    NB = w.N // 64
    pl_f, sel_f, fw_f, g_f = full
    pl_p, sel_p, fw_p, g_p = part
    for name in ("zone_shape", "zone_g", "zone_rho", "n_blocks", "perm", "inv_perm"):
        assert torch.equal(getattr(pl_f, name)[h0:h1], getattr(pl_p, name)), name
    for k, h in enumerate(range(h0, h1)):
        nb = int(pl_p.n_blocks[k])
        assert torch.equal(pl_f.blocks[h, :nb], pl_p.blocks[k, :nb])
        rf, rp = _rows(sel_f, h, NB), _rows(sel_p, k, NB)
        assert all(np.array_equal(a, b) for a, b in zip(rf, rp)), f"selection of head {h}"
    assert torch.equal(fw_f.O[:, h0:h1], fw_p.O)
    assert torch.equal(fw_f.O_res[:, h0:h1], fw_p.O_res)
    assert torch.equal(fw_f.lse[h0:h1], fw_p.lse)
    for a, b in zip(g_f[0], g_p[0]):       # deterministic backward
        assert torch.equal(a[:, h0:h1], b)
    for a, b in zip(g_f[1][1:], g_p[1][1:]):  # fused: dK, dV
        assert torch.equal(a[:, h0:h1], b)
    d = (g_f[1][0][:, h0:h1] - g_p[1][0]).abs().max().item()
    assert d <= 1e-5 * g_p[1][0].abs().max().item(), d
