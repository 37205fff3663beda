"""A model of fa_fwd_host's stream ordering, run under random execution orders on the CPU.

fa_fwd_host enqueues, for each call, in this order (streams: the caller's S, the library's
input stream I and output stream O; events start, in_done, chunk_done, out_done, each
re-recorded every time):
  record(start, S); wait(I, start); wait(O, start)
  per chunk c: copy-in(c) on I; record(in_done, I); wait(S, in_done); kernel(c) on S;
               record(chunk_done, S); wait(O, chunk_done); copy-out(c) on O
  record(in_done, I); wait(S, in_done); record(out_done, O); wait(S, out_done)
CUDA semantics modelled: operations of one stream run in order; a wait captures the
latest record of the event enqueued before it (later re-records do not affect it) and
blocks its stream until that record has run.  Any ready operation may run next.

Checked for several calls in a row on the same device buffers: a chunk's kernel runs
after its copy-in; a chunk's copy-out after its kernel; a copy-in of call k+1 only after
every kernel of call k that reads that chunk's inputs; a kernel of call k+1 only after
call k's copy-out of that chunk (the kernel overwrites the device outputs); and the host
sees every copy-out of a call once it has synchronised the caller's stream (here: once
all of S has run)."""
import random

import pytest


class Sim:
    def __init__(self):
        self.streams = {"S": [], "I": [], "O": []}
        self.latest = {}            # event -> the record op most recently enqueued
        self.done = set()
        self.log = []               # executed ops in order
        self.count = 0

    def enqueue(self, stream, op, needs=None):
        self.streams[stream].append((op, needs))

    def record(self, event, stream):
        self.count += 1
        op = ("record", event, self.count, stream)
        self.latest[event] = op
        self.enqueue(stream, op)

    def wait(self, stream, event):
        self.count += 1
        self.enqueue(stream, ("wait", event, self.count), self.latest.get(event))

    def run(self, rng):
        while any(self.streams.values()):
            ready = [k for k, q in self.streams.items()
                     if q and (q[0][1] is None or q[0][1] in self.done)]
            assert ready, "deadlock"
            k = rng.choice(ready)
            op, _ = self.streams[k].pop(0)
            self.done.add(op)
            self.log.append(op)


def enqueue_call(sim, call, chunks):
    sim.record("start", "S")
    sim.wait("I", "start")
    sim.wait("O", "start")
    for c in range(chunks):
        sim.enqueue("I", ("copy_in", call, c))
        sim.record("in_done", "I")
        sim.wait("S", "in_done")
        sim.enqueue("S", ("kernel", call, c))
        sim.record("chunk_done", "S")
        sim.wait("O", "chunk_done")
        sim.enqueue("O", ("copy_out", call, c))
    sim.record("in_done", "I")
    sim.wait("S", "in_done")
    sim.record("out_done", "O")
    sim.wait("S", "out_done")


@pytest.mark.parametrize("chunk_list", [[1], [3], [1, 4, 2], [5, 5, 5], [2, 7, 1, 3]])
def test_host_pipeline_orders_copies_kernels_and_calls(chunk_list):
    for seed in range(200):
        sim = Sim()
        for call, n in enumerate(chunk_list):
            enqueue_call(sim, call, n)
        sim.run(random.Random(seed))
        pos = {op: i for i, op in enumerate(sim.log) if op[0] in ("copy_in", "kernel",
                                                                   "copy_out")}
        for call, n in enumerate(chunk_list):
            for c in range(n):
                assert pos[("copy_in", call, c)] < pos[("kernel", call, c)]
                assert pos[("kernel", call, c)] < pos[("copy_out", call, c)]
                if call > 0 and c < chunk_list[call - 1]:
                    # the previous call's chunk c used the same device bytes only if the
                    # chunking matches; require the stronger, chunk-independent order:
                    # every kernel and copy-out of the previous call comes first
                    prev = call - 1
                    last = max(pos[(k, prev, cc)] for k in ("kernel", "copy_out")
                               for cc in range(chunk_list[prev]))
                    assert last < pos[("copy_in", call, c)]
        # the caller's stream ends after every copy: its last operation (the final wait on
        # out_done) runs after the last copy-in and copy-out of every call
        assert len(pos) == 3 * sum(chunk_list)
        last_s = max(i for i, op in enumerate(sim.log)
                     if op[0] == "wait" and op[1] == "out_done")    # only S waits on it
        assert all(i < last_s for op, i in pos.items() if op[0] in ("copy_in", "copy_out"))


def test_model_catches_a_missing_start_wait():
    """Drop the input stream's wait on `start` in the second call: its first copy-in can
    then overtake the first call's kernels, which still read the same device buffers.
    The model finds such schedules."""
    caught = 0
    for seed in range(200):
        sim = Sim()
        for call, n in enumerate([3, 3]):
            sim.record("start", "S")
            if call == 0:
                sim.wait("I", "start")
            sim.wait("O", "start")
            for c in range(n):
                sim.enqueue("I", ("copy_in", call, c))
                sim.record("in_done", "I")
                sim.wait("S", "in_done")
                sim.enqueue("S", ("kernel", call, c))
                sim.record("chunk_done", "S")
                sim.wait("O", "chunk_done")
                sim.enqueue("O", ("copy_out", call, c))
            sim.record("in_done", "I")
            sim.wait("S", "in_done")
            sim.record("out_done", "O")
            sim.wait("S", "out_done")
        sim.run(random.Random(seed))
        pos = {op: i for i, op in enumerate(sim.log)}
        last_prev = max(pos[("kernel", 0, c)] for c in range(3))
        if pos[("copy_in", 1, 0)] < last_prev:
            caught += 1
    assert caught > 0
