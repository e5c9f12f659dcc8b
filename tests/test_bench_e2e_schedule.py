"""The end-to-end leg's copy/compute schedule (bench.run_e2e) on fake CUDA
streams and events, on the CPU.  Every operation the schedule enqueues is
logged with the buffers it reads and writes; the happens-before relation is
the order within a stream plus the event edges (a wait on an event orders
everything enqueued after it behind the operation recorded into it).  Any
two operations on the same buffer, one of them a write, must be ordered,
and each step must read the inputs uploaded for it and have its results
downloaded after it ran.  Checked with the second buffer set (overlapped
copies) and without it (copies in line)."""
import argparse
import contextlib

import pytest
import torch

import bench


class _Buf:
    """A device or host tensor stand-in: identity only."""
    count = 0

    def __init__(self, name):
        _Buf.count += 1
        self.name = f"{name}#{_Buf.count}"

    def cpu(self):
        return _Buf("host")

    def pin_memory(self):
        return self

    def numel(self):
        return 1 << 20

    def element_size(self):
        return 2

    def copy_(self, src, non_blocking=False):
        assert non_blocking
        _Sim.op("copy", reads=[src], writes=[self])
        return self


class _Event:
    def __init__(self, enable_timing=False):
        self.op = None

    def record(self, stream):
        self.op = _Sim.op("record", stream=stream)

    def elapsed_time(self, other):
        return 10.0


class _Stream:
    def __init__(self, device=None):
        self.last = None
        self.pending = []   # ops this stream waits for before its next op

    def wait_event(self, ev):
        assert ev.op is not None, "wait on an event that was never recorded"
        self.pending.append(ev.op)


class _Sim:
    ops = []
    current = None

    @classmethod
    def op(cls, kind, reads=(), writes=(), stream=None):
        s = stream or cls.current
        assert s is not None, f"{kind} outside a stream context"
        node = {"kind": kind, "reads": list(reads), "writes": list(writes), "deps": list(s.pending),
                "id": len(cls.ops), "step": getattr(cls, "step_no", None)}
        if s.last is not None:
            node["deps"].append(s.last)
        s.pending = []
        s.last = node
        cls.ops.append(node)
        return node


def _before(a, b):
    """a happens before b."""
    seen, todo = set(), [b]
    while todo:
        n = todo.pop()
        for d in n["deps"]:
            if d is a:
                return True
            if d["id"] not in seen:
                seen.add(d["id"])
                todo.append(d)
    return False


@pytest.mark.parametrize("free_gb", [1 << 10, 0])
@pytest.mark.parametrize("backward", [True, False])
def test_e2e_schedule_orders_every_copy(monkeypatch, free_gb, backward):
    _Sim.ops, _Sim.current = [], None
    default = _Stream()

    @contextlib.contextmanager
    def stream_ctx(s):
        prev = _Sim.current
        _Sim.current = s
        try:
            yield
        finally:
            _Sim.current = prev

    monkeypatch.setattr(torch.cuda, "Stream", _Stream)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "stream", stream_ctx)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "mem_get_info", lambda *a: (free_gb << 30, 180 << 30))
    monkeypatch.setattr(torch, "empty_like", lambda t, **kw: _Buf("empty"))
    monkeypatch.setattr(bench, "pinned_copy", lambda t: _Buf("host"))
    monkeypatch.setattr(bench, "pinned_like", lambda t: _Buf("host"))
    _Sim.current = default

    names = ["Q", "K", "X", "hhat"] + (["dO"] if backward else [])
    primary = {k: _Buf(k) for k in names + ["V", "O"]}
    primary["grads"] = tuple(_Buf(g) for g in ("dQ", "dK", "dV")) if backward else None
    runs = []

    def step(b):
        runs.append(b)
        _Sim.step_no = len(runs)
        ins = [b[k] for k in names]
        outs = [b["O"]] + (list(b["grads"]) if backward else [])
        _Sim.op("step", reads=ins, writes=outs + [b["V"]])

    args = argparse.Namespace(steps=5)
    e2e = bench.run_e2e(args, primary, step, names, backward, total_flops=1e12, world=1, device=None)
    assert e2e["steps"] == 5 and runs and e2e["h2d_bytes_per_step"] == len(names) * (1 << 21)
    assert ("overlapped" in e2e["copies"]) == (free_gb > 0)
    if free_gb > 0:
        assert len({id(b["Q"]) for b in runs}) == 2     # the two sets alternate
    ops = _Sim.ops
    # 1. every pair of operations on one buffer with a write among them is ordered
    touching = {}
    for n in ops:
        for t in n["reads"]:
            touching.setdefault(t.name, []).append((n, False))
        for t in n["writes"]:
            touching.setdefault(t.name, []).append((n, True))
    for name, acc in touching.items():
        for i in range(len(acc)):
            for j in range(i + 1, len(acc)):
                (a, wa), (b, wb) = acc[i], acc[j]
                if (wa or wb) and a is not b:
                    assert _before(a, b) or _before(b, a), f"unordered access to {name}: {a['kind']} / {b['kind']}"
    # 2. each step reads inputs written after the previous step that used them
    steps = [n for n in ops if n["kind"] == "step"]
    for n in steps:
        for t in n["reads"]:
            ups = [u for u in ops if u["kind"] == "copy" and t in u["writes"] and _before(u, n)]
            assert ups, f"step {n['step']} reads {t.name} before any upload"
    # 3. every step's results are downloaded after it
    for n in steps:
        for t in n["writes"]:
            if t.name.split("#")[0] in ("V",):
                continue
            assert any(d["kind"] == "copy" and t in d["reads"] and _before(n, d) for d in ops), t.name
