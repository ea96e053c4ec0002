"""Host test of the end-to-end pipeline's ordering (no GPU): a fake CUDA
runtime records every copy, call, event record and stream wait as a node of a
happens-before graph (stream order plus waits on recorded events), and each
step's operations must be ordered as the pipeline promises."""
import contextlib

import pytest

import bench


class _Graph:
    def __init__(self):
        self.nodes, self.edges, self.current = [], {}, None

    def add(self, stream, label):
        n = len(self.nodes)
        self.nodes.append(label)
        self.edges[n] = set()
        if stream.last is not None:
            self.edges[n].add(stream.last)       # stream order
        for e in stream.pending:                  # waits issued on this stream since its last op
            self.edges[n].add(e)
        stream.pending = []
        stream.last = n
        return n

    def before(self, a, b):
        """a happens before b (b reachable backwards to a)."""
        seen, todo = set(), [b]
        while todo:
            x = todo.pop()
            if x == a:
                return True
            if x in seen:
                continue
            seen.add(x)
            todo.extend(self.edges[x])
        return False


class _Stream:
    def __init__(self, g, name):
        self.g, self.name, self.last, self.pending = g, name, None, []

    def wait_event(self, ev):
        assert ev.node is not None, "a stream waits on an event that was never recorded"
        self.pending.append(ev.node)


class _Event:
    def __init__(self, g, enable_timing=False):
        self.g, self.node = g, None

    def record(self, stream):
        self.node = self.g.add(stream, ("record", stream.name))

    def elapsed_time(self, other):
        return 1.0


class _Tensor:
    def __init__(self, g, name):
        self.g, self.name = g, name

    def copy_(self, src, non_blocking=False):
        self.g.add(self.g.current, ("copy", src.name, self.name))


class _FakeTorch:
    def __init__(self):
        self.g = _Graph()
        g = self.g
        self.default = _Stream(g, "default")
        g.current = self.default
        names = iter(["in", "cmp", "out"])

        class cuda:
            @staticmethod
            def Stream():
                return _Stream(g, next(names))

            @staticmethod
            def Event(enable_timing=False):
                return _Event(g, enable_timing)

            @staticmethod
            @contextlib.contextmanager
            def stream(s):
                prev, g.current = g.current, s
                try:
                    yield
                finally:
                    g.current = prev

            @staticmethod
            def synchronize():
                pass

        self.cuda = cuda


def _run(steps, warmup):
    torch = _FakeTorch()
    g = torch.g
    ops = {}
    host_in = [_Tensor(g, f"h{k}") for k in range(3)]
    sets = [[_Tensor(g, f"s{j}.{k}") for k in range(4)] for j in range(2)]
    host_out = [_Tensor(g, f"ho{j}") for j in range(2)]
    calls = []

    def launch(dev, stream):
        i = len(calls)
        calls.append(i)
        ops[("cmp", i)] = g.add(stream, ("call", dev[0].name))

    P = dict(host_in=host_in, host_out=host_out, dev_sets=sets, launch=launch, result_dev=None)
    ms, last = bench.pipelined_e2e(P, steps, warmup, torch)
    # map copies to steps: per step, three input copies then one output copy
    ins = [n for n, lab in enumerate(g.nodes) if lab[0] == "copy" and lab[1].startswith("h")]
    outs = [n for n, lab in enumerate(g.nodes) if lab[0] == "copy" and lab[2].startswith("ho")]
    n = steps + warmup
    assert len(ins) == 3 * n and len(outs) == n and len(calls) == n
    for i in range(n):
        for k in range(3):
            ops[("in", i, k)] = ins[3 * i + k]
        ops[("out", i)] = outs[i]
    return g, ops, n, last, host_out


@pytest.mark.parametrize("steps,warmup", [(1, 0), (5, 2), (8, 3)])
def test_every_step_is_ordered(steps, warmup):
    g, ops, n, last, host_out = _run(steps, warmup)
    for i in range(n):
        for k in range(3):
            assert g.before(ops[("in", i, k)], ops[("cmp", i)])      # inputs before the call
        assert g.before(ops[("cmp", i)], ops[("out", i)])            # the call before its copy-out
        if i >= 2:
            # a set's inputs are refilled only after the call that read them
            for k in range(3):
                assert g.before(ops[("cmp", i - 2)], ops[("in", i, k)])
            # its output is overwritten only after it was copied out
            assert g.before(ops[("out", i - 2)], ops[("cmp", i)])
    assert last is host_out[(n - 1) % 2]


def test_steps_overlap_across_streams():
    """The pipeline does not serialise: step i+1's input copy does not wait for
    step i's call, and step i's call does not wait for step i-1's copy-out."""
    g, ops, n, _, _ = _run(6, 0)
    for i in range(1, n - 1):
        assert not g.before(ops[("cmp", i)], ops[("in", i + 1, 0)])
        assert not g.before(ops[("out", i - 1)], ops[("cmp", i)])


def test_timed_region_brackets_the_timed_steps():
    g, ops, n, _, _ = _run(4, 2)
    rec = [k for k, lab in enumerate(g.nodes) if lab == ("record", "in")]
    t1 = [k for k, lab in enumerate(g.nodes) if lab == ("record", "out")][-1]
    # t0 is the record on the copy-in stream placed just before the first timed step's copies
    t0 = max(k for k in rec if k < ops[("in", 2, 0)])
    for i in range(2, n):
        assert g.before(t0, ops[("in", i, 0)])
        assert g.before(ops[("out", i)], t1)
        assert g.before(ops[("cmp", i)], t1)
