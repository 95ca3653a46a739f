"""The ordering of bench.py's pipelined end-to-end steps, checked on the host
with fake streams and events and a small discrete-event simulation: every
step's inputs are in place before it computes, a buffer is reused only after
its previous reader is done, results leave before they are overwritten, and
copies do overlap compute."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class FakeEvent:
    def __init__(self):
        self.records = 0        # how many records have been enqueued
        self.done = {}          # record number -> completion time

    def record(self, stream):
        self.records += 1
        stream.ops.append(("record", self, self.records))


class FakeStream:
    def __init__(self, name):
        self.name, self.ops = name, []

    def wait_event(self, ev):
        stream_ops = self.ops
        stream_ops.append(("wait", ev, ev.records))   # waits for the latest record enqueued so far


DUR = {"in": 1.0, "replay": 3.0, "out": 1.0}


def simulate(streams):
    """Run every stream's ops in order, streams concurrently; returns
    {(kind, step): (start, end)}.  Fails on a deadlock."""
    ready = {s.name: 0.0 for s in streams}
    pos = {s.name: 0 for s in streams}
    log = {}
    progress = True
    while progress:
        progress = False
        for s in streams:
            while pos[s.name] < len(s.ops):
                op = s.ops[pos[s.name]]
                if op[0] == "wait":
                    ev, n = op[1], op[2]
                    if n == 0:
                        pass
                    elif n in ev.done:
                        ready[s.name] = max(ready[s.name], ev.done[n])
                    else:
                        break
                elif op[0] == "record":
                    op[1].done[op[2]] = ready[s.name]
                else:
                    kind, i = op[1], op[2]
                    start = ready[s.name]
                    ready[s.name] = start + DUR[kind]
                    log[(kind, i)] = (start, ready[s.name])
                pos[s.name] += 1
                progress = True
    assert all(pos[s.name] == len(s.ops) for s in streams), "deadlock"
    return log


@pytest.mark.parametrize("n", [1, 2, 3, 7])
def test_pipeline_orders_and_overlaps(n):
    h2d, comp, d2h = FakeStream("h2d"), FakeStream("compute"), FakeStream("d2h")
    buf_of = {}

    def work(kind):
        def f(i, b, s):
            buf_of[(kind, i)] = b
            s.ops.append(("work", kind, i))
        return f

    start = FakeEvent()
    comp.ops.append(("work", "replay", -1))   # something already on the compute stream
    start.record(comp)
    pipe = bench.E2EPipeline(2, h2d, comp, d2h, FakeEvent, work("in"), work("replay"), work("out"))
    pipe.run(n, start_event=start)
    log = simulate([h2d, comp, d2h])
    t0 = log[("replay", -1)][1]
    for i in range(n):
        assert log[("in", i)][0] >= t0 and log[("out", i)][0] >= t0
        assert log[("replay", i)][0] >= log[("in", i)][1]            # inputs in place
        assert log[("out", i)][0] >= log[("replay", i)][1]           # result computed
        assert buf_of[("in", i)] == buf_of[("replay", i)] == buf_of[("out", i)] == i % 2
        if i >= 2:
            assert log[("in", i)][0] >= log[("replay", i - 2)][1]    # buffer's previous reader done
            assert log[("replay", i)][0] >= log[("out", i - 2)][1]   # previous result has left
    # the compute stream ends after the last copy-out
    comp_end = max(e for (k, i), (s0, e) in log.items() if k == "replay")
    assert log[("out", n - 1)][1] >= comp_end
    if n >= 3:   # copies overlap compute: shorter than running everything back to back
        serial = n * (DUR["in"] + DUR["replay"] + DUR["out"])
        assert log[("out", n - 1)][1] - t0 < serial
