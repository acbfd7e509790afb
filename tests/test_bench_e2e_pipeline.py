"""Host logic of the benchmark's end-to-end leg (no GPU): `bench.run_e2e` runs against fake
streams, events and tensors that record every copy, launch, record and wait, and the
resulting happens-before graph is checked.

* No race: two operations on the same device buffer, one of them a write, are always
  ordered (two buffer sets alternate between steps).
* Right data: every launch reads the inputs uploaded in its own step, and every download
  reads the results of its own step.
* Overlap is possible: the upload of step s + 1 and the download of step s - 1 are not
  ordered against the compute of step s.
* The timed region opens before the first upload and closes after the last download, and
  the byte counts are those of the tensors copied.
"""
import contextlib
import math
import os
import sys
from types import SimpleNamespace

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class Sim:
    def __init__(self):
        self.ops = []          # dicts: kind, stream, reads, writes, preds
        self.streams = []
        self.current = None
        self.timing_events = []
        self.last_sync = None   # work issued after a host-blocking call comes after it

    def add(self, stream, kind, reads=(), writes=(), deps=()):
        preds = [p for p in [stream.last, *deps] if p is not None]
        self.ops.append(dict(kind=kind, stream=stream.name, reads=list(reads),
                             writes=list(writes), preds=preds))
        stream.last = len(self.ops) - 1
        return stream.last

    def synchronize(self):
        preds = [s.last for s in self.streams if s.last is not None]
        self.ops.append(dict(kind="sync", stream="*", reads=[], writes=[], preds=preds))
        self.last_sync = len(self.ops) - 1
        for s in self.streams:
            s.last = self.last_sync

    def closure(self):
        """anc[i]: bitset of the operations that happen before operation i."""
        anc = []
        for op in self.ops:
            a = 0
            for p in op["preds"]:
                a |= anc[p] | (1 << p)
            anc.append(a)
        return anc


class FakeStream:
    def __init__(self, sim, name):
        self.sim, self.name, self.last = sim, name, sim.last_sync
        sim.streams.append(self)

    def wait_event(self, ev):
        assert ev.op is not None, "wait on an event that was never recorded"
        self.sim.add(self, "wait", deps=[ev.op])


class FakeEvent:
    def __init__(self, sim, enable_timing=False):
        self.sim, self.op = sim, None
        if enable_timing:
            sim.timing_events.append(self)

    def record(self, stream=None):
        self.op = self.sim.add(stream or self.sim.current, "record")

    def elapsed_time(self, other):
        return 1.0


class FakeTensor:
    count = 0

    def __init__(self, sim, shape, dtype, host):
        FakeTensor.count += 1
        self.sim, self.shape, self.dtype, self.host = sim, tuple(shape), dtype, host
        self.key = ("host" if host else "dev", FakeTensor.count)

    def numel(self):
        return math.prod(self.shape)

    def element_size(self):
        return torch.tensor([], dtype=self.dtype).element_size()

    def copy_(self, src, non_blocking=False):
        kind = "h2d" if src.host and not self.host else ("d2h" if self.host else "d2d")
        self.sim.add(self.sim.current, kind, reads=[src.key], writes=[self.key])
        if not non_blocking:        # a blocking copy returns once it is done
            self.sim.synchronize()
        return self


class FakeRA:
    def __init__(self, sim):
        self.sim = sim

    def race_forward_ex(self, q, k, v, W, out, a, stream):
        self.sim.add(stream, "fwd", reads=[q.key, k.key, v.key, W.key], writes=[out.key])

    def race_backward_ex(self, q, k, v, W, out, dout, dq, dk, dv, dW, a, stream):
        self.sim.add(stream, "bwd", reads=[q.key, k.key, v.key, W.key, out.key, dout.key],
                     writes=[dq.key, dk.key, dv.key, dW.key])


def _run(monkeypatch, backward, steps):
    sim = Sim()
    main = FakeStream(sim, "main")
    sim.current = main

    @contextlib.contextmanager
    def use_stream(st):
        prev, sim.current = sim.current, st
        try:
            yield
        finally:
            sim.current = prev

    monkeypatch.setattr(torch.cuda, "Stream", lambda dev=None: FakeStream(sim, "s%d" % len(sim.streams)))
    monkeypatch.setattr(torch.cuda, "Event", lambda enable_timing=False: FakeEvent(sim, enable_timing))
    monkeypatch.setattr(torch.cuda, "stream", use_stream)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda dev=None: sim.synchronize())
    monkeypatch.setattr(torch, "empty", lambda shape, dtype=None, pin_memory=False:
                        FakeTensor(sim, shape, dtype, host=True))
    monkeypatch.setattr(torch, "empty_like", lambda t: FakeTensor(sim, t.shape, t.dtype, host=False))

    H, N, d = 2, 8, 4
    bf = torch.bfloat16
    x = {n: FakeTensor(sim, (H, N, d), bf, host=False) for n in ["q", "k", "v", "dout"]}
    x["W"] = FakeTensor(sim, (3, d, 2), torch.float32, host=False)
    outs = {"out": FakeTensor(sim, (H, N, d), bf, host=False)}
    if backward:
        outs.update({n: FakeTensor(sim, (H, N, d), bf, host=False) for n in ["dq", "dk", "dv"]})
        outs["dW"] = FakeTensor(sim, (3, d, 2), torch.float32, host=False)
    args = SimpleNamespace(steps=steps, e2e_steps=0)
    wl = SimpleNamespace(batch=1, N=N)
    res = bench.run_e2e(args, wl, x, outs, None, FakeRA(sim), None, main, 1, backward)
    assert "error" not in res, res
    return sim, res, x, outs


def _conflict(a, b):
    dev = lambda keys: {k for k in keys if k[0] == "dev"}  # noqa: E731
    ra, wa, rb, wb = dev(a["reads"]), dev(a["writes"]), dev(b["reads"]), dev(b["writes"])
    return bool(wa & (rb | wb) or wb & ra)


@pytest.mark.parametrize("backward", [True, False])
def test_e2e_pipeline_orders_every_conflicting_access_and_overlaps_the_rest(monkeypatch,
                                                                            backward):
    steps = 4
    sim, res, x, outs = _run(monkeypatch, backward, steps)
    ops, anc = sim.ops, sim.closure()
    hb = lambda i, j: bool(anc[j] >> i & 1)  # noqa: E731
    work = [i for i, op in enumerate(ops) if op["kind"] in ("h2d", "d2h", "fwd", "bwd")]

    # no race on device memory
    for ia, i in enumerate(work):
        for j in work[ia + 1:]:
            if _conflict(ops[i], ops[j]):
                assert hb(i, j), (ops[i], ops[j])

    # each launch reads what its own step uploaded; each download reads its own step's result
    for j in work:
        for key in ops[j]["reads"]:
            if key[0] != "dev" or key == x["W"].key:
                continue
            writers = [i for i in work if i < j and key in ops[i]["writes"]]
            if writers:
                assert hb(writers[-1], j), (ops[writers[-1]], ops[j])

    # the steps: two warm-up steps, then `steps` timed ones
    fwd = [i for i in work if ops[i]["kind"] == "fwd"]
    assert len(fwd) == 2 + steps
    step_of = {}
    s = -1
    for i in work:
        if ops[i]["kind"] == "h2d" and (s < 0 or ops[work[work.index(i) - 1]]["kind"] != "h2d"):
            s += 1
        step_of[i] = s
    up = lambda t: [i for i in work if step_of[i] == t and ops[i]["kind"] == "h2d"]  # noqa: E731
    down = lambda t: [i for i in work if step_of[i] == t and ops[i]["kind"] == "d2h"]  # noqa: E731
    comp = lambda t: [i for i in work if step_of[i] == t and ops[i]["kind"] in ("fwd", "bwd")]  # noqa: E731
    last_timed = 2 + steps - 1
    for t in range(3, last_timed):
        # the next step's upload and the previous step's downloads may run beside this
        # step's compute
        for c in comp(t):
            assert not any(hb(c, u) for u in up(t + 1)), t
            assert not any(hb(dl, c) for dl in down(t - 1)), t

    # the timed region: opened before the first timed upload, closed after the last download
    e0, e1 = sim.timing_events[-2:]
    for i in work:
        if step_of[i] >= 2:
            assert hb(e0.op, i) and hb(i, e1.op), ops[i]

    names = ["q", "k", "v"] + (["dout"] if backward else [])
    assert res["h2d_bytes_per_step"] == sum(x[n].numel() * x[n].element_size() for n in names)
    assert res["d2h_bytes_per_step"] == sum(t.numel() * t.element_size() for t in outs.values())
    assert res["steps"] == steps and res["buffer_sets"] == 2
    # every timed step uploads every input and downloads every result once
    for t in range(2, 2 + steps):
        assert len(up(t)) == len(names)
        assert len(down(t)) == len(outs)
