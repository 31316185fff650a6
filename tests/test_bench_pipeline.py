"""The end-to-end serving loop of bench.py (e2e_pipelined_step) on a model of
CUDA streams and events, on the CPU.

A stream runs its work in order; an event recorded on a stream captures all
the work submitted to it so far; a stream that waits on an event runs its
next work only after everything the event captured (an event never recorded
imposes nothing).  The test builds the happens-before graph of twelve steps
and checks that every buffer hazard of the two slots is ordered, and that the
overlap the loop exists for is allowed: step i+1's input copy need not wait
for step i's kernels, and step i+1's kernels need not wait for step i's
result copy.
"""
import itertools

import bench


class Node:
    def __init__(self, kind, step, slot, deps):
        self.kind, self.step, self.slot, self.deps = kind, step, slot, deps


class FakeStream:
    def __init__(self):
        self.frontier = []  # what the next piece of work on this stream depends on

    def add(self, node):
        self.frontier = [node]

    def wait_event(self, ev):
        if ev.marker is not None:
            self.frontier = self.frontier + [ev.marker]


class FakeEvent:
    def __init__(self):
        self.marker = None

    def record(self, stream):
        self.marker = Node("record", None, None, list(stream.frontier))


def build_graph(n_steps):
    ops = {}
    slots = [bench.E2ESlot(FakeEvent, slot_id=0), bench.E2ESlot(FakeEvent, slot_id=1)]
    compute, h2d, d2h = FakeStream(), FakeStream(), FakeStream()
    step = {"i": 0}

    def issue(kind, sl, st):
        node = Node(kind, step["i"], sl.slot_id, list(st.frontier))
        st.add(node)
        ops[(kind, step["i"])] = node

    for i in range(n_steps):
        step["i"] = i
        bench.e2e_pipelined_step(i, slots, compute, h2d, d2h, issue)
    # the end of the timed region: the compute stream waits for both slots' results
    for sl in slots:
        compute.wait_event(sl.results_home)
    end = Node("end", None, None, list(compute.frontier))
    return ops, end


def happens_before(a, b):
    """a is an ancestor of b in the dependency graph."""
    seen, todo = set(), [b]
    while todo:
        n = todo.pop()
        for d in n.deps:
            if d is a:
                return True
            if id(d) not in seen:
                seen.add(id(d))
                todo.append(d)
    return False


N = 12


def test_each_step_copies_in_computes_then_copies_out():
    ops, _ = build_graph(N)
    for i in range(N):
        assert happens_before(ops[("h2d", i)], ops[("compute", i)])
        assert happens_before(ops[("compute", i)], ops[("d2h", i)])
        assert ops[("h2d", i)].slot == ops[("compute", i)].slot == ops[("d2h", i)].slot == i % 2


def test_a_slot_is_reused_only_after_its_previous_step_let_go():
    ops, _ = build_graph(N)
    for i in range(N - 2):
        # the inputs of step i are not overwritten while its kernels may still read them
        assert happens_before(ops[("compute", i)], ops[("h2d", i + 2)])
        # the outputs of step i are not overwritten before they reach the host
        assert happens_before(ops[("d2h", i)], ops[("compute", i + 2)])


def test_neighbouring_steps_may_overlap():
    ops, _ = build_graph(N)
    for i in range(N - 1):
        assert not happens_before(ops[("compute", i)], ops[("h2d", i + 1)])
        assert not happens_before(ops[("d2h", i)], ops[("compute", i + 1)])


def test_the_region_ends_after_every_result_reached_the_host():
    ops, end = build_graph(N)
    for kind, i in itertools.product(("h2d", "compute", "d2h"), range(N)):
        assert happens_before(ops[(kind, i)], end)


def test_kernels_run_in_step_order():
    ops, _ = build_graph(N)
    for i in range(N - 1):
        assert happens_before(ops[("compute", i)], ops[("compute", i + 1)])
