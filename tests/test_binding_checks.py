"""Host-side argument checks of the Python binding (no GPU needed).

The C ABI receives bare device pointers, so it cannot see a buffer's size or
device; the binding checks dtype, shape, contiguity, device and the grid a
plan or selection was made for before any call reaches the library.  Every
case below fails one of those checks before anything touches CUDA."""
import pytest
import torch

from dynamic_block_sparse_stats_b200 import api

T, H, W, HEADS, D = 8, 16, 16, 2, 64
N = T * H * W
P = api.params(T, H, W, HEADS, D, topk_abs=2, top_p=0.9)
CPU = torch.device("cpu")


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_attn_fwd_rejects_wrong_dtype_shape_and_host_memory():
    pl, sel = api.alloc_plan(P, CPU), api.alloc_select(P, CPU, 64)
    good = _bf16(N, HEADS, D)
    with pytest.raises(ValueError, match="Q must be torch.bfloat16"):
        api.attn_fwd(P, pl, sel, good.float(), good, good)
    with pytest.raises(ValueError, match=r"K must have shape \(2048, 2, 64\)"):
        api.attn_fwd(P, pl, sel, good, _bf16(N, HEADS, 128), good)
    with pytest.raises(ValueError, match="V must be contiguous"):
        api.attn_fwd(P, pl, sel, good, good, _bf16(N, D, HEADS).transpose(1, 2))
    with pytest.raises(ValueError, match="Q must be a CUDA tensor"):
        api.attn_fwd(P, pl, sel, good, good, good)


def test_attn_bwd_checks_every_tensor_before_the_device():
    pl, sel = api.alloc_plan(P, CPU), api.alloc_select(P, CPU, 64)
    x = _bf16(N, HEADS, D)
    lse = torch.zeros((HEADS, N), dtype=torch.float32)
    with pytest.raises(ValueError, match="dO must have shape"):
        api.attn_bwd(P, pl, sel, x, x, x, x, _bf16(N, HEADS, D - 8), lse)
    with pytest.raises(ValueError, match="O must be torch.bfloat16"):
        api.attn_bwd(P, pl, sel, x, x, x, x.float(), x, lse)
    with pytest.raises(ValueError, match="O_res must have shape"):
        api.attn_bwd(P, pl, sel, x, x, x, x, x, lse, O_res=_bf16(N, HEADS))
    with pytest.raises(ValueError, match=r"lse must have shape \(2, 2048\)"):
        api.attn_bwd(P, pl, sel, x, x, x, x, x, lse.t().contiguous())


def test_select_and_plan_check_their_inputs():
    pl = api.alloc_plan(P, CPU)
    x = _bf16(N, HEADS, D)
    with pytest.raises(ValueError, match="K must be torch.bfloat16"):
        api.select(P, pl, x, x.half())
    with pytest.raises(ValueError, match="V must have shape"):
        api.plan(P, _bf16(N - 64, HEADS, D))
    with pytest.raises(ValueError, match="V must be a CUDA tensor"):
        api.plan(P, x)


def test_plan_made_for_another_grid_is_refused():
    other = api.params(T, H, W + 8, HEADS, D)
    pl = api.alloc_plan(other, CPU)
    with pytest.raises(ValueError, match="the plan was made for"):
        api._check_plan(P, pl)
    with pytest.raises(TypeError):
        api._check_plan(P, object())


def test_plan_buffers_of_the_wrong_size_are_refused():
    pl = api.alloc_plan(P, CPU)
    pl.perm = torch.zeros((HEADS, N - 1), dtype=torch.int32)
    with pytest.raises(ValueError, match=r"plan.perm must have shape \(2, 2048\)"):
        api._check_plan(P, pl)
    pl = api.alloc_plan(P, CPU)
    pl.blocks = pl.blocks.long()
    with pytest.raises(ValueError, match="plan.blocks must be torch.int32"):
        api._check_plan(P, pl)
    pl = api.alloc_plan(P, CPU)
    with pytest.raises(ValueError, match="plan.zone_shape must be a CUDA tensor"):
        api._check_devices(api._check_plan(P, pl))      # right sizes: only the device is wrong


def test_selection_checks():
    sel = api.alloc_select(P, CPU, 64, transpose=False)
    with pytest.raises(ValueError, match="needs the selection's transpose"):
        api._check_selection(P, sel, True)
    sel = api.alloc_select(P, CPU, 64)
    sel.nnz = 65
    with pytest.raises(ValueError, match="exceeds its capacity 64"):
        api._check_selection(P, sel, False)
    sel = api.alloc_select(P, CPU, 64)
    sel.row = None
    with pytest.raises(ValueError, match="both be set or both be None"):
        api._check_selection(P, sel, False)
    sel = api.alloc_select(P, CPU, 64)
    sel.row_ptr = sel.row_ptr[:-1]
    with pytest.raises(ValueError, match="selection.row_ptr must have shape"):
        api._check_selection(P, sel, False)
    sel = api.alloc_select(api.params(T, H, W, HEADS + 1, D), CPU, 64)
    with pytest.raises(ValueError, match="the selection was made for"):
        api._check_selection(P, sel, False)


def test_device_check_reports_the_first_host_tensor():
    x = _bf16(4)
    with pytest.raises(ValueError, match="b must be a CUDA tensor"):
        api._check_devices([("a", None), ("b", x)])
    assert api._check_devices([("a", None)]) is None


def test_a2v_norm_checks():
    with pytest.raises(ValueError, match="2-D bf16"):
        api.a2v_norm(torch.zeros((4, 64), dtype=torch.float32))
    with pytest.raises(ValueError, match="rows must be contiguous"):
        api.a2v_norm(_bf16(64, 4).t())
    with pytest.raises(ValueError, match="a2v_norm must have shape"):
        api.a2v_norm(_bf16(4, 64), out=torch.zeros(5))
    with pytest.raises(ValueError, match="hhat must be a CUDA tensor"):
        api.a2v_norm(_bf16(4, 64))


def test_workspace_checks():
    with pytest.raises(ValueError, match="1-D uint8"):
        api._check_workspace(torch.zeros(256, dtype=torch.int32), "ws")
    with pytest.raises(ValueError, match="1-D uint8"):
        api.workspace_status(torch.zeros((2, 128), dtype=torch.uint8))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        api.workspace_status(torch.zeros(256, dtype=torch.uint8))


class _FakeLib:
    """Stands in for libprism.so: records every call's arguments, returns
    PRISM_OK, and makes the first selection report a short capacity."""

    def __init__(self):
        self.calls = []
        self.selects = 0

    def __getattr__(self, name):
        def f(*args):
            self.calls.append((name, args))
            if name.endswith("workspace_size"):
                return 4096
            if name == "prism_last_error":
                return b"fake"
            if name == "prism_select":
                sel = args[4]._obj
                self.selects += 1
                first = self.selects == 1
                sel.nnz = sel.cap + 5 if first else sel.cap
                return 3 if first else 0
            return 0
        return f


class _Stream:
    cuda_stream = 1234


def test_marshalling_through_a_fake_library(monkeypatch):
    """The whole Python path (a2v_norm -> plan -> select -> fwd -> bwd) on host
    tensors against a fake library: every entry point gets the data pointers
    of the right tensors, the byte sizes of its workspaces and the caller's
    stream, and a short selection capacity is grown once."""
    import contextlib

    from dynamic_block_sparse_stats_b200 import _lib
    fake = _FakeLib()
    monkeypatch.setattr(_lib, "load", lambda: fake)
    monkeypatch.setattr(api, "_check_devices", lambda named: CPU)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: _Stream())
    x = {k: _bf16(N, HEADS, D) for k in ("Q", "K", "V", "dO")}
    hhat = _bf16(N, 3 * 64)

    a = api.a2v_norm(hhat)
    name, args = fake.calls[-1]
    assert name == "prism_a2v_norm" and args[0].value == hhat.data_ptr() and args[1:4] == (N, 192, 192)
    assert args[4].value == a.data_ptr() and args[5] == 1234 and a.shape == (N,)

    pl = api.plan(P, x["V"], a)
    name, args = fake.calls[-1]
    assert name == "prism_plan" and args[1].value == x["V"].data_ptr() and args[2].value == a.data_ptr()
    cs = args[3]._obj
    assert cs.perm == pl.perm.data_ptr() and cs.blocks == pl.blocks.data_ptr()
    assert args[4].value == pl.ws.data_ptr() and args[5] == pl.ws.numel() == 4096

    sel = api.select(P, pl, x["Q"], x["K"], cap=10)
    sels = [c for c in fake.calls if c[0] == "prism_select"]
    assert len(sels) == 2 and sel.col.numel() == 15 and sel.row.numel() == 15 and sel.nnz == 15
    args = sels[-1][1]
    assert args[2].value == x["Q"].data_ptr() and args[3].value == x["K"].data_ptr()
    assert args[4]._obj.col == sel.col.data_ptr() and args[4]._obj.row == sel.row.data_ptr()

    fw = api.attn_fwd(P, pl, sel, x["Q"], x["K"], x["V"])
    name, args = fake.calls[-1]
    assert name == "prism_attn_fwd"
    assert [t.value for t in args[3:9]] == [t.data_ptr() for t in (x["Q"], x["K"], x["V"], fw.O, fw.O_res, fw.lse)]
    assert args[9].value == fw.ws.data_ptr() and args[10] == 4096 and args[11] == 1234
    assert fw.lse.shape == (HEADS, N) and fw.lse.dtype == torch.float32

    dQ, dK, dV = api.attn_bwd(P, pl, sel, x["Q"], x["K"], x["V"], fw.O, x["dO"], fw.lse, grad_fp32=True,
                              O_res=fw.O_res)
    name, args = fake.calls[-1]
    assert name == "prism_attn_bwd"
    want = (x["Q"], x["K"], x["V"], fw.O, fw.O_res, x["dO"], fw.lse, dQ, dK, dV)
    assert [t.value for t in args[3:13]] == [t.data_ptr() for t in want]
    assert args[13] == 1 and args[14] == 0 and args[16] == 4096 and dQ.dtype == torch.float32 and dQ.shape == (N, HEADS, D)

    api.attn_bwd(P, pl, sel, x["Q"], x["K"], x["V"], fw.O, x["dO"], fw.lse, grad_fp32=True, deterministic=True)
    assert fake.calls[-1][1][14] == 1                # the path selector reaches the library
    with pytest.raises(ValueError, match="dQ must be torch.bfloat16"):
        api.attn_bwd(P, pl, sel, x["Q"], x["K"], x["V"], fw.O, x["dO"], fw.lse, out=(dQ, dK, dV))
    assert api.workspace_status(fw.ws) == 0


def test_buffer_reuse_as_the_benchmark_step_does(monkeypatch):
    """The benchmark allocates every output once, then passes the same buffers
    to each call of its timed step; the binding must accept them and hand the
    library the same pointers every time."""
    import contextlib

    from dynamic_block_sparse_stats_b200 import _lib
    fake = _FakeLib()
    monkeypatch.setattr(_lib, "load", lambda: fake)
    monkeypatch.setattr(api, "_check_devices", lambda named: CPU)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: _Stream())
    x = {k: _bf16(N, HEADS, D) for k in ("Q", "K", "V", "dO")}
    hhat = _bf16(N, 128)
    a = api.a2v_norm(hhat)
    pl = api.plan(P, x["V"], a)
    sel = api.select(P, pl, x["Q"], x["K"])               # the fake grows it once
    sel = api.select(P, pl, x["Q"], x["K"], cap=sel.nnz + 8)
    fw = api.attn_fwd(P, pl, sel, x["Q"], x["K"], x["V"])
    grads = api.attn_bwd(P, pl, sel, x["Q"], x["K"], x["V"], fw.O, x["dO"], fw.lse, O_res=fw.O_res)
    bws = torch.empty(4096, dtype=torch.uint8)
    fake.calls.clear()
    for _ in range(2):                                   # the timed step, twice
        assert api.a2v_norm(hhat, out=a) is a
        assert api.plan(P, x["V"], a, out=pl) is pl
        assert api.select(P, pl, x["Q"], x["K"], out=sel) is sel
        f2 = api.attn_fwd(P, pl, sel, x["Q"], x["K"], x["V"], O=fw.O, lse=fw.lse, ws=fw.ws, O_res=fw.O_res)
        assert f2.O is fw.O and f2.lse is fw.lse and f2.ws is fw.ws and f2.O_res is fw.O_res
        g2 = api.attn_bwd(P, pl, sel, x["Q"], x["K"], x["V"], fw.O, x["dO"], fw.lse, out=grads, ws=bws,
                          O_res=fw.O_res)
        assert all(u is v for u, v in zip(g2, grads))
    names = [c[0] for c in fake.calls]
    assert names == ["prism_a2v_norm", "prism_plan", "prism_select", "prism_attn_fwd", "prism_attn_bwd"] * 2
    bwd = [c[1] for c in fake.calls if c[0] == "prism_attn_bwd"]
    assert bwd[0][15].value == bws.data_ptr() and bwd[0][16] == 4096
    assert [t.value for t in bwd[0][10:13]] == [t.data_ptr() for t in grads]


def test_explicit_stream_and_no_residual(monkeypatch):
    """A stream passed by the caller reaches the library (not the current
    one), and residual=False passes a NULL O_res."""
    import contextlib

    from dynamic_block_sparse_stats_b200 import _lib
    fake = _FakeLib()
    monkeypatch.setattr(_lib, "load", lambda: fake)
    monkeypatch.setattr(api, "_check_devices", lambda named: CPU)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: _Stream())

    class Mine:
        cuda_stream = 777

    x = {k: _bf16(N, HEADS, D) for k in ("Q", "K", "V")}
    a = api.a2v_norm(_bf16(N, 64), stream=Mine())
    assert fake.calls[-1][1][5] == 777
    pl = api.plan(P, x["V"], a, stream=Mine())
    assert fake.calls[-1][1][6] == 777
    sel = api.select(P, pl, x["Q"], x["K"], cap=10 ** 4, stream=Mine())
    assert fake.calls[-1][1][7] == 777
    fw = api.attn_fwd(P, pl, sel, x["Q"], x["K"], x["V"], residual=False, stream=Mine())
    name, args = fake.calls[-1]
    assert name == "prism_attn_fwd" and args[7] is None and args[11] == 777 and fw.O_res is None
    # a residual buffer handed over with residual=False is not written
    fw = api.attn_fwd(P, pl, sel, x["Q"], x["K"], x["V"], O_res=_bf16(N, HEADS, D), residual=False)
    assert fake.calls[-1][1][7] is None and fw.O_res is None
