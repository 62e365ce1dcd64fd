"""Host logic of bench.py's pipelined end-to-end measurement, on the CPU.

Streams, events and the layer call are replaced by CPU fakes that record the order of stream
operations, so the test checks (1) the output check against the serial step, and (2) the
dependencies that make the double buffers safe: a slot's inputs are overwritten only after the
compute that read them, its output only after the copy that read it, and every copy of the
timed steps waits for the start event.
"""
import contextlib
import itertools
import sys
import types
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from hstu_sequential_transducer_jagged_b200 import binding as Bd  # noqa: E402


class Log:
    def __init__(self):
        self.ops = []  # (stream name, op, detail)
        self.current = "compute"


def install_fakes(monkeypatch, log):
    names = itertools.cycle(["h2d", "d2h"])

    class FakeStream:
        cuda_stream = 0

        def __init__(self, *a, name=None, **k):
            self.name = name or next(names)

        def wait_event(self, e):
            log.ops.append((self.name, "wait", e.tag))

    class FakeEvent:
        count = 0

        def __init__(self, *a, **k):
            FakeEvent.count += 1
            self.tag = f"e{FakeEvent.count}"

        def record(self, s=None):
            log.ops.append((s.name if s is not None else log.current, "record", self.tag))

        def elapsed_time(self, other):
            return 10.0

    @contextlib.contextmanager
    def stream_ctx(s):
        prev, log.current = log.current, s.name
        try:
            yield
        finally:
            log.current = prev

    real_copy = torch.Tensor.copy_

    def tracked_copy(self, src, non_blocking=False):
        log.ops.append((log.current, "copy", None))
        return real_copy(self, src)

    def fake_layer(cur, w1, w2, off, maxlen, ts, rp, rt, *, out, ws, stream, **kw):
        log.ops.append((stream.name, "layer", None))
        real_copy(out, cur + w1)
        return out

    monkeypatch.setattr(torch.cuda, "Stream", FakeStream)
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "stream", stream_ctx)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(torch.Tensor, "copy_", tracked_copy)
    monkeypatch.setattr(Bd, "layer_forward", fake_layer)
    return FakeStream(name="compute")


def make_inputs(L=4, T=32):
    x = torch.randn(T, 8)
    layers = [dict(w1=torch.full((T, 8), float(l + 1)), w2=None, rp=None, rt=None)
              for l in range(L)]
    wl = types.SimpleNamespace(max_seq_len=T, num_heads=1, d_qk=8, d_v=8, max_pos_dist=0,
                               num_time_buckets=1, alpha=1.0, mask=0, num_candidates=0)
    off = torch.tensor([0, T], dtype=torch.int32)
    ts = torch.arange(T)
    y = x.clone()
    for ly in layers:
        y = y + ly["w1"]
    return x, layers, wl, off, ts, y


def test_pipelined_output_check(monkeypatch):
    log = Log()
    compute = install_fakes(monkeypatch, log)
    x, layers, wl, off, ts, y = make_inputs()
    ms, check = bench.run_e2e_pipelined(6, 4, layers, wl, x, off, ts, y, x, off, ts, compute,
                                        None, 1, "cpu")
    assert ms == 10.0 and check == "output identical to the serial step"
    ms, check = bench.run_e2e_pipelined(6, 4, layers, wl, x, off, ts, y + 1, x, off, ts, compute,
                                        None, 1, "cpu")
    assert check == "output differs: not used"
    assert bench.run_e2e_pipelined(1, 4, layers, wl, x, off, ts, y, x, off, ts, compute, None, 1,
                                   "cpu") is None


def test_pipelined_dependencies(monkeypatch):
    log = Log()
    compute = install_fakes(monkeypatch, log)
    x, layers, wl, off, ts, y = make_inputs()
    K = 5
    bench.run_e2e_pipelined(K, 4, layers, wl, x, off, ts, y, x, off, ts, compute, None, 1, "cpu")
    ops = log.ops
    # the timed region starts where the start event is recorded on the compute stream and both
    # copy streams wait for it
    rec = [i for i, o in enumerate(ops) if o[0] == "compute" and o[1] == "record"]
    start = next(i for i in range(len(ops))
                 if ops[i][1] == "record" and ops[i][0] == "compute"
                 and ops[i + 1][:2] == ("h2d", "wait") and ops[i + 2][:2] == ("d2h", "wait"))
    timed = ops[start:]
    assert rec  # sanity
    # per stream, program order of the timed steps
    h2d = [o for o in timed if o[0] == "h2d"]
    d2h = [o for o in timed if o[0] == "d2h"]
    comp = [o for o in timed if o[0] == "compute"]
    # each step copies 3 inputs in and 1 output out
    assert sum(1 for o in h2d if o[1] == "copy") == 3 * K
    assert sum(1 for o in d2h if o[1] == "copy") == K
    assert sum(1 for o in comp if o[1] == "layer") == 4 * K
    # compute events recorded after each step's last layer, in order: the tags of "comp_done"
    comp_done = []
    seen_layers = 0
    for o in comp:
        if o[1] == "layer":
            seen_layers += 1
        elif o[1] == "record" and seen_layers and seen_layers % 4 == 0 and \
                len(comp_done) < seen_layers // 4:
            comp_done.append(o[2])
    assert len(comp_done) == K
    # step i >= 2 of the input copy stream waits for the compute of step i-2 before copying
    waits_h2d = [o[2] for o in h2d if o[1] == "wait"][1:]  # first wait: the start event
    assert waits_h2d == comp_done[:K - 2]
    # the output copy of step i waits for the compute of step i
    waits_d2h = [o[2] for o in d2h if o[1] == "wait"][1:]
    assert waits_d2h == comp_done
    # the compute of step i waits for step i's input copy and, from step 2 on, for the output
    # copy of step i-2 (same output slot); then the 4 layers; then its completion event
    h2d_recs = [o[2] for o in h2d if o[1] == "record"]
    d2h_recs = [o[2] for o in d2h if o[1] == "record"]
    assert len(h2d_recs) == K and len(d2h_recs) == K
    expected = [("compute", "record", comp[0][2])]
    for i in range(K):
        expected.append(("compute", "wait", h2d_recs[i]))
        if i >= 2:
            expected.append(("compute", "wait", d2h_recs[i - 2]))
        expected += [("compute", "layer", None)] * 4
        expected.append(("compute", "record", comp_done[i]))
    assert comp[:len(expected)] == expected
    # the compute stream's last operations wait for every output copy before the end event
    tail = comp[-3:]
    assert [o[1] for o in tail] == ["wait", "wait", "record"]
    assert {tail[0][2], tail[1][2]} == set(d2h_recs[-2:])
