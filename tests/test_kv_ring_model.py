"""A model of the forward kernel's K/V ring and Q handshake, run under random
interleavings on the CPU.

The TMA lane loads, per unit, the Q tiles (q_full / q_empty) and then K_j, V_j for the
n1 key tiles that Q tile 1 visits, one ring slot each (slot = load index mod NSLOT; it
waits on slot_empty with parity ((index / NSLOT) & 1) ^ 1).  Each of the two MMA warps
(Q tile x visits n_x key tiles, n0 <= n1) waits on slot_full with parity
(index / NSLOT) & 1, issues its products, and releases a slot with a tcgen05 commit, an
arrival that happens when the tensor core has finished the products, not at issue.
slot_empty expects one arrival per Q tile.  On key tiles that only tile 1 visits
(causal), tile 1's warp also makes tile 0's arrival, as an immediate arrive after its
own wait on the slot.  Issue order per warp: S(0) .. S(NBUF-1), then for every j: wait
V_j, P.V(j), release V_j, S(j+NBUF) (wait K, issue, release K).

The model keeps the same counts, parities and order.  A tensor-core agent runs each
warp's operations in issue order and checks, at execution, that the slot still holds the
K or V tile the operation reads.  So a slot overwritten before both tiles' products have
finished with it is caught, and so is a deadlock."""
import random

import pytest


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
        return self.phase != parity


class Model:
    def __init__(self, units, nslot, nbuf, seed, tile0_arrive=True, release_at_issue=False,
                 nt=2):
        self.units, self.nslot, self.nbuf, self.nt = units, nslot, nbuf, nt
        self.rng = random.Random(seed)
        self.slot_full = [MBarrier(1) for _ in range(nslot)]
        self.slot_empty = [MBarrier(nt) for _ in range(nslot)]   # one arrival per Q tile
        self.q_full, self.q_empty = MBarrier(1), MBarrier(nt)
        self.content = [None] * nslot
        self.q_content = None
        self.tile0_arrive = tile0_arrive
        self.release_at_issue = release_at_issue
        self.loader = self._loader()
        self.mma = [self._mma(x) for x in range(nt)]
        self.tc = [[], []]              # per warp: issued operations, retired in order
        self.done = [False, nt < 2, False]     # a missing tile 1 counts as done

    # ---- agents are generators that yield a predicate to wait on, or None to move on
    def _loader(self):
        issued = 0
        for u, (n0, n1) in enumerate(self.units):
            yield lambda q=u: self.q_empty.try_wait((q & 1) ^ 1)
            self.q_content = u
            self.q_full.arrive()
            for j in range(n1):
                for t in "KV":
                    s, ph = issued % self.nslot, (issued // self.nslot) & 1
                    yield lambda s=s, ph=ph: self.slot_empty[s].try_wait(ph ^ 1)
                    self.content[s] = (u, j, t)
                    self.slot_full[s].arrive()
                    issued += 1
        self.done[2] = True

    def _mma(self, x):
        kv_base = 0
        for u, (n0, n1) in enumerate(self.units):
            nx = n1 if x else n0
            yield lambda q=u: self.q_full.try_wait(q & 1)

            def wait_slot(idx):
                return lambda: self.slot_full[idx % self.nslot].try_wait(
                    (idx // self.nslot) & 1)

            def issue(idx, j, t, last_s):
                s = idx % self.nslot
                ops = [("check", s, (u, j, t))]
                if self.release_at_issue:
                    self.slot_empty[s].arrive()         # wrong: before the product ran
                else:
                    ops.append(("arrive", self.slot_empty[s]))
                if last_s:
                    ops.append(("check_q", u))
                    ops.append(("arrive", self.q_empty))
                self.tc[x].extend(ops)
                if x == 1 and j >= n0 and self.tile0_arrive:
                    self.slot_empty[s].arrive()       # immediate, for tile 0

            for j in range(min(self.nbuf, nx)):
                idx = kv_base + 2 * j
                yield wait_slot(idx)
                issue(idx, j, "K", j == nx - 1)
            for j in range(nx):
                vi = kv_base + 2 * j + 1
                yield wait_slot(vi)
                issue(vi, j, "V", False)
                if j + self.nbuf < nx:
                    ki = kv_base + 2 * (j + self.nbuf)
                    yield wait_slot(ki)
                    issue(ki, j + self.nbuf, "K", j + self.nbuf == nx - 1)
            kv_base += 2 * n1
        self.done[x] = True

    def _retire(self, x):
        kind, *rest = self.tc[x].pop(0)
        if kind == "check":
            s, expect = rest
            assert self.content[s] == expect, ("slot overwritten", s, self.content[s], expect)
        elif kind == "check_q":
            assert self.q_content == rest[0], "Q overwritten"
        else:
            rest[0].arrive()

    def run(self):
        gens = {"load": self.loader, "mma0": self.mma[0]}
        if self.nt == 2:
            gens["mma1"] = self.mma[1]
        waiting = {k: None for k in gens}
        while not (all(self.done) and not self.tc[0] and not self.tc[1]):
            moves = []
            for k, g in gens.items():
                if self.done[{"mma0": 0, "mma1": 1, "load": 2}[k]]:
                    continue
                if waiting[k] is None or waiting[k]():
                    moves.append(("agent", k))
            for x in (0, 1):
                if self.tc[x]:
                    moves.append(("tc", x))
            assert moves, "deadlock"
            kind, k = self.rng.choice(moves)
            if kind == "tc":
                self._retire(k)
            else:
                try:
                    waiting[k] = next(gens[k])
                except StopIteration:
                    waiting[k] = None


def unit_mix(rng, n, causal):
    out = []
    for _ in range(n):
        n0 = rng.randint(1, 9)
        out.append((n0, n0 + (rng.randint(0, 2) if causal else 0)))
    return out


@pytest.mark.parametrize("nslot,nbuf", [(4, 2), (8, 2), (16, 3), (8, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_kv_ring_never_overwrites_a_slot_in_use(nslot, nbuf, causal):
    for seed in range(40):
        rng = random.Random(seed)
        Model(unit_mix(rng, rng.randint(1, 6), causal), nslot, nbuf, seed).run()


def test_model_catches_a_missing_tile0_arrival():
    """Without tile 1's arrival for tile 0 on the key tiles tile 0 skips, the slots of
    those tiles never empty: the loader stalls and the model reports the deadlock."""
    caught = 0
    for seed in range(20):
        units = [(2, 4), (3, 5), (1, 3)]
        try:
            Model(units, 4, 2, seed, tile0_arrive=False).run()
        except AssertionError:
            caught += 1
    assert caught == 20


def test_model_catches_a_release_before_the_product_ran():
    """A slot released at issue time (a plain arrive instead of a commit) can be refilled
    while the product that reads it is still queued: the model sees the overwrite."""
    caught = 0
    for seed in range(40):
        rng = random.Random(seed)
        try:
            Model(unit_mix(rng, rng.randint(2, 6), True), 4, 2, seed,
                  release_at_issue=True).run()
        except AssertionError:
            caught += 1
    assert caught >= 30


@pytest.mark.parametrize("nslot", [2, 4])
def test_kv_ring_with_one_q_tile_per_unit(nslot):
    """Head dim 256: one Q tile per unit (n0 = n1), one arrival per slot and per Q tile."""
    for seed in range(40):
        rng = random.Random(seed)
        units = [(n, n) for n in (rng.randint(1, 9) for _ in range(rng.randint(1, 6)))]
        Model(units, nslot, 2, seed, nt=1).run()
