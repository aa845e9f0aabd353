"""Stream ordering of the benchmark's end-to-end timing, checked on CPU.

The timing helpers are driven with fake streams, events and buffers that
record every operation. The recorded program is then read the way a GPU
runs it: each stream runs its operations in order, and a wait on an event
orders everything recorded before that event's latest record ahead of the
waiting stream's later operations. The tests check, for every step, that its
inputs are copied in before it runs, that its results are copied out after it
runs, that a buffer set is not overwritten while a step still needs it, and
that the timed region covers every copy."""
import contextlib

import pytest

import bench


class FakeStream:
    def __init__(self, name):
        self.name, self.ops = name, []

    def wait_event(self, ev):
        self.ops.append(("wait", ev.last))


class FakeEvent:
    def __init__(self, enable_timing=False):
        self.last = None  # (stream, op index) of the latest record

    def record(self, stream):
        stream.ops.append(("record", self))
        self.last = (stream, len(stream.ops) - 1)

    def elapsed_time(self, other):
        return 1.0


class FakeCuda:
    def __init__(self, compute):
        self.current = compute
        self.Event = FakeEvent
        self.synced = 0

    @contextlib.contextmanager
    def stream(self, s):
        prev, self.current = self.current, s
        try:
            yield
        finally:
            self.current = prev

    def synchronize(self):
        self.synced += 1


class FakeBuf:
    def __init__(self, cuda, name):
        self.cuda, self.name = cuda, name

    def copy_(self, src, non_blocking=False):
        assert non_blocking
        self.cuda.current.ops.append(("copy", self.name, src.name))


def _happens_before(streams):
    """Reachability over (stream, index) nodes: program order within a
    stream plus an edge from an event's record to every wait on it."""
    nodes = [(s, i) for s in streams for i in range(len(s.ops))]
    preds = {n: set() for n in nodes}
    for s in streams:
        for i, op in enumerate(s.ops):
            if i > 0:
                preds[(s, i)].add((s, i - 1))
            if op[0] == "wait" and op[1] is not None:
                preds[(s, i)].add(op[1])
    memo = {}

    def ancestors(n):
        if n not in memo:
            acc = set()
            stack = list(preds[n])
            while stack:
                m = stack.pop()
                if m not in acc:
                    acc.add(m)
                    stack.extend(preds[m])
            memo[n] = acc
        return memo[n]

    return lambda a, b: a in ancestors(b)


def _find(streams, pred):
    return [(s, i) for s in streams for i, op in enumerate(s.ops) if pred(op)]


def _program(k, overlapped):
    compute, s_in, s_out = FakeStream("compute"), FakeStream("in"), FakeStream("out")
    cuda = FakeCuda(compute)
    host_ins = [FakeBuf(cuda, f"host_{n}") for n in ("Q", "K", "V")]
    nsets = 2 if overlapped else 1
    sets = [([FakeBuf(cuda, f"{n}{b}") for n in ("Q", "K", "V")], [FakeBuf(cuda, f"O{b}")]) for b in range(nsets)]
    hosts = [[FakeBuf(cuda, f"host_O{b}")] for b in range(nsets)]
    step_no = [0]

    def step(io=None):
        b = next(i for i, s in enumerate(sets) if s is io)
        cuda.current.ops.append(("step", step_no[0], b))
        step_no[0] += 1

    if overlapped:
        ms = bench.e2e_overlapped_ms(k, step, sets, host_ins, hosts, compute, s_in, s_out, cuda=cuda)
    else:
        ms = bench.e2e_serial_ms(k, step, sets[0], host_ins, hosts[0], compute, cuda=cuda)
    assert ms == pytest.approx(1.0 / k) and cuda.synced == 1
    return [compute, s_in, s_out], compute


def _check(streams, compute, k, nsets):
    hb = _happens_before(streams)
    steps = _find(streams, lambda op: op[0] == "step")
    assert len(steps) == k and all(s is compute for s, _ in steps)
    assert [compute.ops[i][1] for _, i in steps] == list(range(k))
    # The copies of step i, in issue order per stream (each step copies 3 in, 1 out).
    ins = _find(streams, lambda op: op[0] == "copy" and op[2].startswith("host_"))
    outs = _find(streams, lambda op: op[0] == "copy" and op[1].startswith("host_"))
    assert len(ins) == 3 * k and len(outs) == k
    ins = sorted(ins, key=lambda n: (n[0].name, n[1]))
    outs = sorted(outs, key=lambda n: (n[0].name, n[1]))
    for i in range(k):
        b = i % nsets
        st = steps[i]
        assert compute.ops[st[1]][2] == b
        for c in ins[3 * i:3 * i + 3]:
            assert c[0].ops[c[1]][1].endswith(str(b))  # into set b
            assert hb(c, st), f"step {i} may run before its inputs arrive"
        o = outs[i]
        assert o[0].ops[o[1]][2] == f"O{b}" and hb(st, o), f"step {i}'s results may be read before it ran"
        if i + nsets < k:
            nxt = steps[i + nsets]
            for c in ins[3 * (i + nsets):3 * (i + nsets) + 3]:
                assert hb(st, c), f"step {i + nsets}'s copy-in may overwrite inputs step {i} still reads"
            assert hb(o, nxt), f"step {i + nsets} may overwrite results before step {i}'s copy-out"
    # The timed region: first record on the compute stream, last record on it.
    recs = [i for i, op in enumerate(compute.ops) if op[0] == "record"]
    e0, e1 = (compute, recs[0]), (compute, recs[-1])
    for c in ins + outs + steps:
        assert hb(e0, c) and hb(c, e1), "an operation falls outside the timed region"


@pytest.mark.parametrize("k", [1, 2, 3, 6])
def test_overlapped_copies_respect_every_dependency(k):
    streams, compute = _program(k, overlapped=True)
    _check(streams, compute, k, nsets=2)


@pytest.mark.parametrize("k", [1, 4])
def test_serial_copies_are_in_stream_order(k):
    streams, compute = _program(k, overlapped=False)
    assert not streams[1].ops and not streams[2].ops
    _check(streams, compute, k, nsets=1)


def test_overlap_actually_overlaps():
    """Step i + 1's copy-in is not ordered after step i (it may run beside it),
    and step i's copy-out is not ordered before step i + 1."""
    k = 4
    streams, compute = _program(k, overlapped=True)
    hb = _happens_before(streams)
    steps = _find(streams, lambda op: op[0] == "step")
    s_in, s_out = streams[1], streams[2]
    ins = [(s_in, i) for i, op in enumerate(s_in.ops) if op[0] == "copy"]
    outs = [(s_out, i) for i, op in enumerate(s_out.ops) if op[0] == "copy"]
    for i in range(k - 1):
        assert not hb(steps[i], ins[3 * (i + 1)])
        assert not hb(outs[i], steps[i + 1])


def test_a_dropped_wait_is_caught(monkeypatch):
    """The checker itself: removing the wait that protects set reuse fails it."""
    real = FakeStream.wait_event

    def lossy(self, ev):
        if self.name == "in" and ev.last is not None and ev.last[0].name == "compute" and len(self.ops) > 2:
            self.ops.append(("wait", None))  # the copy-in no longer waits for the step two back
        else:
            real(self, ev)

    monkeypatch.setattr(FakeStream, "wait_event", lossy)
    streams, compute = _program(4, overlapped=True)
    with pytest.raises(AssertionError, match="copy-in may overwrite"):
        _check(streams, compute, 4, nsets=2)
