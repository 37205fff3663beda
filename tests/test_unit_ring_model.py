"""A model of the kernels' work distribution, run under random interleavings on the CPU.

The forward and backward kernels hand work units to their warps the same way: each
CTA's TMA lane takes unit blockIdx.x first, then claims units from a counter shared by
the launch (atomicAdd) and publishes each one in a ring of UNIT_RING shared-memory slots.
The handshake uses one mbarrier pair per slot: `full` (1 arrival, the producer) and
`empty` (one arrival per consumer warp).  The producer waits on `empty` with parity
((n / R) & 1) ^ 1 before its n-th publication, and consumers wait on `full` with parity
(n / R) & 1 before their n-th read.  The first value >= num_units ends the list.
Variable-length units that are empty are never published.

The model implements mbarrier phases (an arrival count that completes a phase, and a
parity wait that succeeds once the phase of that parity has completed) and the same
index and parity arithmetic.  Random schedules of several CTAs must end with every
non-empty unit processed exactly once, every consumer warp of a CTA seeing the same
sequence, and no state in which no agent can move (deadlock)."""
import random

import pytest

UNIT_RING = 4


class MBarrier:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase ^= 1
            self.pending = self.count

    def try_wait(self, parity):
        # true once the phase with this parity has completed, i.e. the current phase
        # has moved past it
        return self.phase != parity


class CTA:
    def __init__(self, block, grid, num_units, counter, consumers, empty_units):
        self.full = [MBarrier(1) for _ in range(UNIT_RING)]
        self.empty = [MBarrier(consumers) for _ in range(UNIT_RING)]
        self.ring = [None] * UNIT_RING
        self.block, self.grid, self.num_units = block, grid, num_units
        self.counter, self.empty_units = counter, empty_units
        self.consumers = consumers
        # producer state
        self.u = block
        self.published = 0
        self.producer_done = False
        # consumer state
        self.taken = [0] * consumers
        self.done = [False] * consumers
        self.seen = [[] for _ in range(consumers)]

    def claim(self):
        v = self.counter[0]
        self.counter[0] += 1
        return self.grid + v

    def producer_step(self):
        """One attempt of the producer; returns True if it moved."""
        if self.producer_done:
            return False
        if self.u < self.num_units and self.u in self.empty_units:
            self.u = self.claim()           # empty unit: skipped, never published
            return True
        s = self.published % UNIT_RING
        if not self.empty[s].try_wait(((self.published // UNIT_RING) & 1) ^ 1):
            return False
        self.ring[s] = self.u
        self.full[s].arrive()
        self.published += 1
        if self.u >= self.num_units:
            self.producer_done = True
        else:
            self.u = self.claim()           # (loads for the unit would be issued first)
        return True

    def consumer_step(self, c):
        if self.done[c]:
            return False
        s = self.taken[c] % UNIT_RING
        if not self.full[s].try_wait((self.taken[c] // UNIT_RING) & 1):
            return False
        u = self.ring[s]
        self.empty[s].arrive()
        self.taken[c] += 1
        if u >= self.num_units:
            self.done[c] = True
        else:
            self.seen[c].append(u)
        return True

    def finished(self):
        return self.producer_done and all(self.done)


def run(num_units, grid, consumers, empty_units, seed):
    rng = random.Random(seed)
    counter = [0]
    ctas = [CTA(b, grid, num_units, counter, consumers, empty_units) for b in range(grid)]
    agents = [(k, -1) for k in range(grid)] + [(k, c) for k in range(grid)
                                               for c in range(consumers)]
    steps = 0
    while not all(t.finished() for t in ctas):
        rng.shuffle(agents)
        moved = False
        for k, c in agents:
            t = ctas[k]
            if (t.producer_step() if c < 0 else t.consumer_step(c)):
                moved = True
                break
        assert moved, "deadlock: no agent can move"
        steps += 1
        assert steps < 10_000_000
    return ctas


@pytest.mark.parametrize("num_units,grid,consumers,empty_frac", [
    (1, 1, 10, 0.0), (7, 3, 10, 0.0), (50, 4, 10, 0.0), (200, 7, 13, 0.0),
    (200, 7, 5, 0.3), (33, 33, 10, 0.5), (64, 5, 13, 0.9), (9, 12, 10, 0.0),
])
def test_unit_ring_delivers_every_unit_once_in_order(num_units, grid, consumers, empty_frac):
    for seed in range(20):
        rng = random.Random(1000 + seed)
        empty = {u for u in range(num_units) if rng.random() < empty_frac}
        grid_eff = min(grid, num_units)     # the host launches min(units, SMs) CTAs
        ctas = run(num_units, grid_eff, consumers, empty, seed)
        processed = []
        for t in ctas:
            # every consumer warp of a CTA saw the same units, in the same order
            assert all(seq == t.seen[0] for seq in t.seen)
            processed += t.seen[0]
        expected = sorted(set(range(num_units)) - empty)
        assert sorted(processed) == expected, (num_units, grid, seed)


def test_model_detects_a_wrong_parity():
    """The model is sharp enough to see a plausible mistake: a producer that waits on
    `empty` with the consumers' parity (no ^ 1) cannot publish its first unit."""
    t = CTA(0, 1, 3, [0], 2, set())
    s = 0
    assert not t.empty[s].try_wait(0)      # the wrong parity blocks on a fresh barrier
    assert t.empty[s].try_wait(1)          # the kernel's parity passes


def test_model_detects_a_short_empty_count(monkeypatch):
    """An `empty` barrier that expects one arrival fewer than there are consumer warps
    lets the producer overwrite a slot that a warp has not read yet: the model sees it
    (warps disagree on the sequence, units go missing, or a wait never completes)."""
    orig = CTA.__init__

    def short_count(self, *a, **k):
        orig(self, *a, **k)
        self.empty = [MBarrier(self.consumers - 1) for _ in range(UNIT_RING)]

    monkeypatch.setattr(CTA, "__init__", short_count)
    caught = 0
    for seed in range(10):
        try:
            ctas = run(200, 7, 10, set(), seed)
            same = all(all(seq == t.seen[0] for seq in t.seen) for t in ctas)
            complete = sorted(u for t in ctas for u in t.seen[0]) == list(range(200))
            caught += not (same and complete)
        except AssertionError:
            caught += 1
    assert caught == 10
