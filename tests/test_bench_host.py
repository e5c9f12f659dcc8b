"""Host arithmetic of the benchmark (no GPU).

* The computed-pair count P behind every FLOP figure: bench.computed_pairs
  reads the library's block table and CSR; here it gets the oracle's plan and
  selection in that layout and must equal a brute-force count of the
  (query token, key token) pairs of the dense attention mask.
* The per-kernel roofline arithmetic (work per launch, achieved rate,
  fraction of the peak) on hand-computed numbers.
* The parsing of the nvidia-smi samples taken during the timed region, and
  the rule that a stored DRAM traffic figure is dropped once its kernel's
  source has changed."""
import json
import types

import numpy as np
import pytest
import torch

import bench
from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs
from oracle import prism_oracle as O


def _library_layout(w, opl, osel):
    """The oracle's plan and selection in the library's layout: blocks
    [h][N/64][4] = {p0, B, n0, shape} (rows past n_blocks hold garbage), and a
    CSR over rows h*(N/64) + i."""
    NB = w.N // 64
    heads = len(opl.heads)
    blocks = torch.full((heads, NB, 4), -7, dtype=torch.int32)
    n_blocks = torch.zeros(heads, dtype=torch.int32)
    counts, cols = np.zeros(heads * NB, np.int64), []
    for h, hp in enumerate(opl.heads):
        n_blocks[h] = hp.blocks.shape[0]
        for b, (t0, y0, x0, sid, B, p0) in enumerate(hp.blocks):
            blocks[h, b] = torch.tensor([int(p0), int(B), int((t0 * w.H + y0) * w.W + x0), int(sid)])
        rows = {int(i): np.asarray(ids) for (i, ids, _) in osel[h]}
        for i in range(NB):
            ids = rows.get(i, np.zeros(0, np.int64))
            counts[h * NB + i] = ids.size
            cols.append(ids)
    row_ptr = np.concatenate([[0], np.cumsum(counts)])
    col = np.concatenate(cols)
    pl = types.SimpleNamespace(blocks=blocks, n_blocks=n_blocks)
    sel = types.SimpleNamespace(row_ptr=torch.tensor(row_ptr, dtype=torch.int32),
                                col=torch.tensor(np.concatenate([col, [-1, -1]]), dtype=torch.int32),
                                nnz=int(col.size))
    return pl, sel


def _dense_mask_pairs(w, opl, osel):
    """Pairs of the token-level mask: query token q may attend key token k
    iff k's block is in the selection of q's block."""
    total = 0
    for h, hp in enumerate(opl.heads):
        nb = hp.blocks.shape[0]
        blk = np.empty(w.N, np.int64)
        for b in range(nb):
            p0, B = int(hp.blocks[b, 5]), int(hp.blocks[b, 4])
            blk[hp.perm[p0:p0 + B]] = b
        allowed = np.zeros((nb, nb), bool)
        for (i, ids, _) in osel[h]:
            allowed[i, ids] = True
        total += int(allowed[blk[:, None], blk[None, :]].sum())
    return total


@pytest.mark.parametrize("name", ["tiny", "small_d64"])
def test_computed_pairs_equals_the_dense_mask_count(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, "cpu")
    V, Q, K = (inp[x].float().numpy() for x in ("V", "Q", "K"))
    opl = O.plan(V, inp["a"].numpy(), w.T, w.H, w.W)
    osel = O.select(Q, K, opl, w.topk_frac, w.topk_abs, w.top_p)
    pl, sel = _library_layout(w, opl, osel)
    p = types.SimpleNamespace(T=w.T, H=w.H, W=w.W, heads=w.heads)
    got = bench.computed_pairs(p, pl, sel)
    assert got == _dense_mask_pairs(w, opl, osel)
    assert 0 < got <= w.N * w.N * w.heads


def test_computed_pairs_with_a_different_block_table_per_head():
    """Two heads with different plans (all-256 blocks vs all-64 blocks) and
    random selections: each key's size must come from its own head's table."""
    T, H, W = 8, 16, 16
    w = types.SimpleNamespace(T=T, H=H, W=W, N=T * H * W, heads=2)
    rng = np.random.default_rng(4)
    opl = O.Plan(T, H, W)
    osel = []
    for sid in (13, 0):                      # (4,8,8) volume 256, then (2,4,8) volume 64
        shapes = np.full(4, sid)
        blocks = O.head_blocks(T, H, W, shapes)
        opl.heads.append(O.HeadPlan(None, shapes, None, None, None, None, blocks,
                                    O.permutation(T, H, W, blocks)))
        nb = blocks.shape[0]
        osel.append([(i, np.sort(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False)), {})
                     for i in range(nb)])
    pl, sel = _library_layout(w, opl, osel)
    got = bench.computed_pairs(types.SimpleNamespace(T=T, H=H, W=W, heads=2), pl, sel)
    assert got == _dense_mask_pairs(w, opl, osel)


def test_kernel_roofline_arithmetic_on_the_fused_backward():
    """With the fused kernel (and its dQ conversion) the combined backward
    is 10PD over those two kernels, issued and algorithmic alike, and
    bwd_prep's bytes include the accumulator's zeroing."""
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1000.0, "bf16_tflops": 1200.0}
    P, D, N, h, steps = 1.0e12, 128, 860160, 24, 2
    nb = torch.tensor([100, 200])
    kt = {"attn_fwd": (2, 1000.0), "attn_bwd_fused": (2, 2396.0), "dq_convert": (2, 4.0), "bwd_prep": (2, 10.0),
          "attn_bwd_dkdv": (0, 0.0), "attn_bwd_dq": (0, 0.0)}
    out = bench.kernel_rooflines(kt, P, D, N, h, nb, peaks, "measured", steps)
    assert out["attn_bwd_fused"]["achieved"] == pytest.approx(10 * P * D / 1.198 / 1e12)
    bwd = out["attn_bwd"]
    assert bwd["path"] == "fused" and bwd["ms_per_launch"] == pytest.approx(1200.0)
    assert bwd["achieved"] == pytest.approx(10 * P * D / 1.2 / 1e12)
    assert bwd["issued_TFLOPs"] == pytest.approx(bwd["achieved"])
    assert out["attn_fwd_bwd"]["achieved"] == pytest.approx(14 * P * D / 1.7 / 1e12)
    assert out["dq_convert"]["achieved"] == pytest.approx((6 * N * h * D + 4 * N * h) / 2e-3 / 1e9)
    assert out["bwd_prep"]["achieved"] == pytest.approx((12 * N * h * D + 16 * N * h) / 5e-3 / 1e9)
    # the two-kernel path's bwd_prep has no accumulator to zero
    kt2 = {"attn_bwd_dkdv": (2, 1600.0), "attn_bwd_dq": (2, 1200.0), "bwd_prep": (2, 10.0)}
    out2 = bench.kernel_rooflines(kt2, P, D, N, h, nb, peaks, "measured", steps)
    assert out2["bwd_prep"]["achieved"] == pytest.approx((8 * N * h * D + 16 * N * h) / 5e-3 / 1e9)
    assert out2["attn_bwd"]["path"] == "two-kernel deterministic"


def test_kernel_roofline_arithmetic():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1000.0, "bf16_tflops": 1200.0, "sm_max_mhz": 2000.0}
    P, D, N, h, steps = 1.0e12, 128, 860160, 24, 2
    nb = torch.tensor([100, 200])
    kt = {"attn_fwd": (2, 1000.0), "attn_bwd_dkdv": (2, 1600.0), "attn_bwd_dq": (2, 1200.0),
          "block_mean": (2, 4.0), "block_score": (48, 24.0), "select_row": (48, 10.0)}
    out = bench.kernel_rooflines(kt, P, D, N, h, nb, peaks, "measured", steps, nnz=1000, sm_mhz=1500.0)
    fwd = out["attn_fwd"]                        # one launch per step, 500 ms each
    assert fwd["ms_per_launch"] == 500.0
    assert fwd["achieved"] == pytest.approx(4 * P * D / 0.5 / 1e12)
    assert fwd["peak"] == 1000.0 and fwd["frac"] == pytest.approx(fwd["achieved"] / 1000.0)
    assert fwd["frac_burst"] == pytest.approx(fwd["achieved"] / 1200.0)
    assert fwd["frac_nominal_at_clock"] == pytest.approx(fwd["achieved"] / (148 * 8192 * 1500e6 / 1e12))
    dq = out["attn_bwd_dq"]                      # algorithmic 2PD (dQ = dS K); 6PD issued
    assert dq["achieved"] == pytest.approx(2 * P * D / 0.6 / 1e12)
    assert dq["issued_TFLOPs"] == pytest.approx(6 * P * D / 0.6 / 1e12)
    assert out["attn_bwd_dkdv"]["achieved"] == pytest.approx(8 * P * D / 0.8 / 1e12)
    bwd = out["attn_bwd"]                        # the convention: 10PD over dK/dV + dQ
    assert bwd["ms_per_launch"] == pytest.approx(1400.0)
    assert bwd["achieved"] == pytest.approx(10 * P * D / 1.4 / 1e12)
    assert bwd["frac"] == pytest.approx(bwd["achieved"] / 1000.0)
    assert bwd["frac_burst"] == pytest.approx(bwd["achieved"] / 1200.0)
    assert bwd["issued_TFLOPs"] == pytest.approx(14 * P * D / 1.4 / 1e12)
    both = out["attn_fwd_bwd"]
    assert both["achieved"] == pytest.approx(14 * P * D / 1.9 / 1e12)
    bm = out["block_mean"]                       # one read of Q and K per launch, 2 ms
    assert bm["achieved"] == pytest.approx(4 * N * h * D / 2e-3 / 1e9) and bm["peak"] == 6000.0
    bs = out["block_score"]                      # 24 launches per step share 2*D*sum(nb^2)
    per_launch = 2 * D * (100 ** 2 + 200 ** 2) * steps / 48
    assert bs["achieved"] == pytest.approx(per_launch / 0.5e-3 / 1e12)
    assert bs["peak"] == pytest.approx(148 * 128 * 2000e6 / 1e12)
    sr = out["select_row"]                       # one read of the score rows
    assert sr["achieved"] == pytest.approx(4 * (100 ** 2 + 200 ** 2) * steps / 48 / (10.0 / 48 * 1e-3) / 1e9)
    assert sr["frac"] == pytest.approx(sr["achieved"] / 6000.0)


class _FakeProc:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, None


def test_clock_samples_are_parsed():
    c = bench.ClockSampler(0)
    c.proc = _FakeProc("0, 1600, 1965, 700.5, 0x4, Not Active, Not Active, Not Active, Active\n"
                       "0, 1700, 1965, 710.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                       "0, 1000, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                       "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                       "garbage line\n")
    r = c.stop()        # the median of three samples (the mean would be 1433)
    assert r == {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c = bench.ClockSampler(0)
    c.proc = _FakeProc("0, 1200, 1965, 900, 0x40, Not Active, Active, Not Active, Not Active\n")
    assert c.stop()["reasons"] == ["hw_thermal_slowdown"]
    assert bench.ClockSampler(0).stop()["reasons"] == ["nvidia-smi unavailable"]


def test_strip_comments_keeps_code_and_literals():
    src = ('#include "a.h"  // trailing\n'
           '/* block\n   comment */ int x = 1; /* inline */ int y = 2;\n'
           '\n'
           '\tconst  char *s = "not // a comment /* either */";\n'
           "char c = '\\''; char d = '/'; // it's a comment\n")
    assert bench.strip_comments(src) == ('#include "a.h"\n'
                                         'int x = 1; int y = 2;\n'
                                         'const char *s = "not // a comment /* either */";\n'
                                         "char c = '\\''; char d = '/';\n")


def _tree(tmp_path, kernel, header, shared):
    csrc = tmp_path / "dynamic_block_sparse_stats_b200" / "csrc"
    inc = tmp_path / "include"
    csrc.mkdir(parents=True, exist_ok=True)
    inc.mkdir(exist_ok=True)
    (csrc / "k.cu").write_text('#include "k.cuh"\n' + kernel)
    (csrc / "k.cuh").write_text('#include "../../include/api.h"\n' + header)
    (inc / "api.h").write_text(shared)
    return str(csrc)


def test_code_digest_ignores_comments_and_follows_includes(tmp_path):
    csrc = _tree(tmp_path, "int k() { return 1; }\n", "int h();\n", "int api();\n")
    d0 = bench.source_digest("k.cu", csrc)
    _tree(tmp_path, "// new comment\nint k() {  return 1; }  /* more */\n", "int h();  // note\n",
          "/* doc */ int api();\n")
    assert bench.source_digest("k.cu", csrc) == d0
    _tree(tmp_path, "int k() { return 2; }\n", "int h();\n", "int api();\n")
    assert bench.source_digest("k.cu", csrc) != d0          # the kernel's own code
    _tree(tmp_path, "int k() { return 1; }\n", "int h(int);\n", "int api();\n")
    assert bench.source_digest("k.cu", csrc) != d0          # an included header
    _tree(tmp_path, "int k() { return 1; }\n", "int h();\n", "long api();\n")
    assert bench.source_digest("k.cu", csrc) != d0          # a header included by a header


_NCU_CSV = """==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","prism::fwd::attn_fwd_kernel<128>(Params)","1","7","(384, 1, 1)","(148, 1, 1)","0","10.0","m","dram__bytes_read.sum","Gbyte","2,000.5"
"0","1","python","h","prism::fwd::attn_fwd_kernel<128>(Params)","1","7","(384, 1, 1)","(148, 1, 1)","0","10.0","m","dram__bytes_write.sum","Mbyte","500"
"0","1","python","h","prism::fwd::attn_fwd_kernel<128>(Params)","1","7","(384, 1, 1)","(148, 1, 1)","0","10.0","m","gpu__time_duration.sum","msecond","800"
"1","1","python","h","prism::fwd::attn_fwd_kernel<128>(Params)","1","7","(384, 1, 1)","(148, 1, 1)","0","10.0","m","dram__bytes_read.sum","Gbyte","1,000.5"
"1","1","python","h","prism::fwd::attn_fwd_kernel<128>(Params)","1","7","(384, 1, 1)","(148, 1, 1)","0","10.0","m","dram__bytes_write.sum","Mbyte","500"
"2","1","python","h","void at::native::elementwise_kernel<128>(int)","1","7","(128, 1, 1)","(1, 1, 1)","0","10.0","m","dram__bytes_read.sum","byte","64"
"""


def test_write_traffic_and_stored_traffic(tmp_path, monkeypatch):
    _tree(tmp_path, "int k() { return 1; }\n", "int h();\n", "int api();\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "ncu.csv").write_text(_NCU_CSV)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "attn_fwd", "k.cu")
    out = bench.write_traffic(str(tmp_path / "ncu.csv"))
    assert set(out) == {"_about", "attn_fwd"}          # torch kernels are not ours
    assert out["attn_fwd"]["bytes_per_launch"] == pytest.approx((2000.5e9 + 0.5e9 + 1000.5e9 + 0.5e9) / 2)
    assert out["attn_fwd"]["launches_captured"] == 2
    assert bench.stored_traffic("attn_fwd") == out["attn_fwd"]["bytes_per_launch"]
    assert bench.stored_traffic("attn_bwd_dq") is None
    (tmp_path / "dynamic_block_sparse_stats_b200" / "csrc" / "k.cu").write_text(
        '#include "k.cuh"\n// only a comment changed\nint k() { return 1; }\n')
    assert bench.stored_traffic("attn_fwd") is not None
    (tmp_path / "dynamic_block_sparse_stats_b200" / "csrc" / "k.cuh").write_text(
        '#include "../../include/api.h"\nint h(int);\n')
    assert bench.stored_traffic("attn_fwd") is None


def test_committed_traffic_figures_cover_the_measured_kernels():
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    assert set(bench.NCU_KERNEL_NAMES) <= set(d)
    for name in bench.NCU_KERNEL_NAMES:
        assert d[name]["source"] == bench.KERNEL_SOURCES[name] and d[name]["bytes_per_launch"] > 0


@pytest.mark.parametrize("name", ["tiny", "small_d64"])
def test_selection_stats_match_the_oracle_rows(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, "cpu")
    V, Q, K = (inp[x].float().numpy() for x in ("V", "Q", "K"))
    opl = O.plan(V, inp["a"].numpy(), w.T, w.H, w.W)
    osel = O.select(Q, K, opl, w.topk_frac, w.topk_abs, w.top_p)
    pl, sel = _library_layout(w, opl, osel)
    p = types.SimpleNamespace(T=w.T, H=w.H, W=w.W, heads=w.heads)
    got = bench.selection_stats(p, pl, sel)
    nblk = np.array([len(ids) for h in range(w.heads) for (_, ids, _) in osel[h]], float)
    share = np.array([opl.heads[h].blocks[ids, 4].sum() / w.N for h in range(w.heads) for (_, ids, _) in osel[h]])
    assert got["rows"] == nblk.size == sum(hp.blocks.shape[0] for hp in opl.heads)
    for key, x in (("blocks_per_row", nblk), ("key_share_per_row", share)):
        assert got[key]["mean"] == pytest.approx(x.mean(), rel=1e-12)
        assert got[key]["p50"] == pytest.approx(np.percentile(x, 50), rel=1e-12)
        assert got[key]["p99"] == pytest.approx(np.percentile(x, 99), rel=1e-12)
    # the mean key share, weighted by block size, is the pair density
    Bq = np.array([opl.heads[h].blocks[i, 4] for h in range(w.heads) for (i, _, _) in osel[h]])
    assert (share * Bq).sum() * w.N == pytest.approx(bench.computed_pairs(p, pl, sel), rel=1e-12)


def test_every_timed_kernel_has_a_roofline_spec_and_a_source():
    """The kernel names come from the library (no CUDA call while nothing was
    recorded); the bench must know each one, or its line would fail."""
    import ctypes as C
    from dynamic_block_sparse_stats_b200 import _lib
    lib = _lib.load()
    names = []
    for i in range(_lib.KERNEL_TIMING_IDS):
        n, ms, name = C.c_int(-1), C.c_double(-1.0), C.c_char_p()
        assert lib.prism_kernel_timing_read(i, C.byref(n), C.byref(ms), C.byref(name)) == _lib.PRISM_OK
        assert n.value == 0 and ms.value == 0.0
        names.append(name.value.decode())
    assert lib.prism_kernel_timing_read(_lib.KERNEL_TIMING_IDS, C.byref(n), C.byref(ms),
                                        C.byref(name)) == _lib.PRISM_ERR_INVALID_ARG
    assert len(set(names)) == len(names)
    kt = {nm: (0, 0.0) for nm in names}
    out = bench.kernel_rooflines(kt, 1e12, 128, 860160, 24, torch.tensor([100]), {"hbm_gbs": 1.0}, "measured", 1)
    assert set(out) == set(names)                 # no launches: no combined backward entries
    assert set(names) == set(bench.KERNEL_SOURCES)
    assert set(bench.NCU_KERNEL_NAMES) <= set(names)
