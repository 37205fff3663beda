"""A model of the backward kernel's pipeline, run under random interleavings on the CPU.

Roles and handshakes, as in the kernel (g = global step, b = g & 1, st = g % 3):
- loader: per unit, wait kv_empty, load K and V (kv_full); per step, wait q_empty(st),
  load Q, dO and the per-row vectors into stage st (q_full(st)).
- MMA warp (its products run on the tensor core in issue order; a commit arrives when
  the products before it have finished): per unit, wait kv_full, start steps g and g+1;
  start(g) = wait q_full(st), S^T(g) into score columns b; wait dq_empty(b); dP^T(g) into
  the dP columns of b; commit sdp_full(b).  Then per step: wait ds_full(b); dQ^T(g) (reads
  dS from shared memory, writes the dP columns of b); commit dq_full(b); at the unit's
  first step wait acc_empty; dV += P^T dO, dK += dS^T Q (read P / dS^T from the score
  columns of b and stage st); commit q_empty(st); at the last step commit acc_full and
  kv_empty; start(g+2).
- softmax warps: per step wait sdp_full(b), read S^T(g) and dP^T(g) and the vectors of
  stage st, write P and dS^T over the score columns of b; if g > 0 wait dq_full of step
  g-1 (its dQ^T has read the shared dS tile), write dS to shared memory, arrive ds_full(b);
  per unit wait acc_full, read dV and dK, arrive acc_empty.
- dQ drain warps: per step wait dq_full(b), read dQ^T(g), arrive dq_empty(b).

Every buffer holds a tag of what was last written there; every read checks the tag it
needs, at the moment it happens (for products: when the tensor core runs them).  Random
schedules must finish without a stale or overwritten read and without deadlock."""
import random

import pytest

QSTAGES = 3


class MBarrier:
    def __init__(self, count=1):
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
    def __init__(self, units, seed, mutant=None):
        self.units = units              # steps per unit
        self.rng = random.Random(seed)
        self.mutant = mutant
        B = MBarrier
        self.kv_full, self.kv_empty = B(), B()
        self.q_full = [B() for _ in range(QSTAGES)]
        self.q_empty = [B() for _ in range(QSTAGES)]
        self.sdp_full, self.ds_full = [B(), B()], [B(), B()]
        self.dq_full, self.dq_empty = [B(), B()], [B(), B()]
        self.acc_full, self.acc_empty = B(), B()
        self.buf = {"kv": None, "q": [None] * QSTAGES, "ts": [None, None],
                    "tdp": [None, None], "sds": None, "acc": None}
        self.tc = []                    # products and commits, in issue order
        self.agents = {"load": self._loader(), "mma": self._mma(), "soft": self._softmax(),
                       "drain": self._drain()}
        self.waiting = {k: None for k in self.agents}
        self.finished = set()

    def need(self, got, want, what):
        assert got == want, (what, got, want)

    # ------------------------------------------------------------------ roles
    def _loader(self):
        issued = 0
        g = 0
        for u, steps in enumerate(self.units):
            yield lambda u=u: self.kv_empty.try_wait((u & 1) ^ 1)
            self.buf["kv"] = u
            self.kv_full.arrive()
            for s in range(steps):
                st, use = issued % QSTAGES, issued // QSTAGES
                yield lambda st=st, use=use: self.q_empty[st].try_wait((use & 1) ^ 1)
                self.buf["q"][st] = g
                self.q_full[st].arrive()
                issued += 1
                g += 1

    def _mma(self):
        gm = 0
        for u, steps in enumerate(self.units):
            yield lambda u=u: self.kv_full.try_wait(u & 1)

            def start(g):
                b, st = g & 1, g % QSTAGES
                yield lambda: self.q_full[st].try_wait((g // QSTAGES) & 1)
                self.tc.append(("S", g, u))
                if self.mutant != "no_dq_empty_wait":
                    yield lambda: self.dq_empty[b].try_wait(((g >> 1) & 1) ^ 1)
                self.tc.append(("dP", g, u))
                self.tc.append(("commit", self.sdp_full[b]))

            for s in range(min(2, steps)):
                yield from start(gm + s)
            for s in range(steps):
                g = gm + s
                b, st = g & 1, g % QSTAGES
                yield lambda: self.ds_full[b].try_wait((g >> 1) & 1)
                self.tc.append(("dQ", g, u))
                self.tc.append(("commit", self.dq_full[b]))
                if s == 0:
                    yield lambda: self.acc_empty.try_wait((u & 1) ^ 1)
                if self.mutant == "early_q_release":
                    self.tc.append(("commit", self.q_empty[st]))
                self.tc.append(("acc", g, u, s))
                if self.mutant != "early_q_release":
                    self.tc.append(("commit", self.q_empty[st]))
                if s == steps - 1:
                    self.tc.append(("commit", self.acc_full))
                    self.tc.append(("commit", self.kv_empty))
                if s + 2 < steps:
                    yield from start(g + 2)
            gm += steps

    def _softmax(self):
        gs = 0
        for u, steps in enumerate(self.units):
            for s in range(steps):
                g = gs + s
                b, st = g & 1, g % QSTAGES
                yield lambda: self.sdp_full[b].try_wait((g >> 1) & 1)
                self.need(self.buf["ts"][b], ("S", g), "softmax reads S^T")
                self.need(self.buf["tdp"][b], ("dP", g), "softmax reads dP^T")
                self.need(self.buf["q"][st], g, "softmax reads the row vectors")
                self.buf["ts"][b] = ("P", g)
                if g > 0 and self.mutant != "no_dq_full_wait":
                    yield lambda: self.dq_full[(g - 1) & 1].try_wait(((g - 1) >> 1) & 1)
                self.buf["sds"] = g
                self.ds_full[b].arrive()
            yield lambda u=u: self.acc_full.try_wait(u & 1)
            self.need(self.buf["acc"], (u, steps), "epilogue reads dV, dK")
            self.acc_empty.arrive()
            gs += steps

    def _drain(self):
        g = 0
        for steps in self.units:
            for _ in range(steps):
                b = g & 1
                yield lambda g=g, b=b: self.dq_full[b].try_wait((g >> 1) & 1)
                self.need(self.buf["tdp"][b], ("dQ", g), "drain reads dQ^T")
                self.dq_empty[b].arrive()
                g += 1

    # ------------------------------------------------------------------ tensor core
    def _run_product(self):
        op = self.tc.pop(0)
        kind = op[0]
        if kind == "commit":
            op[1].arrive()
            return
        g, u = op[1], op[2]
        b, st = g & 1, g % QSTAGES
        self.need(self.buf["kv"], u, "product reads K/V")
        if kind in ("S", "dP"):
            self.need(self.buf["q"][st], g, "S^T/dP^T read Q/dO")
            self.buf["ts" if kind == "S" else "tdp"][b] = (kind, g)
        elif kind == "dQ":
            self.need(self.buf["sds"], g, "dQ^T reads the shared dS tile")
            self.buf["tdp"][b] = ("dQ", g)
        else:                                   # dV, dK accumulation
            s = op[3]
            self.need(self.buf["ts"][b], ("P", g), "dV/dK read P/dS^T")
            self.need(self.buf["q"][st], g, "dV/dK read dO/Q")
            prev = (u, s) if s > 0 else None
            if s == 0:
                assert self.buf["acc"] is None or self.buf["acc"][0] == u - 1, "acc reused"
            else:
                self.need(self.buf["acc"], prev, "accumulation order")
            self.buf["acc"] = (u, s + 1)

    def run(self):
        while len(self.finished) < len(self.agents) or self.tc:
            moves = [("tc", None)] if self.tc else []
            for k in self.agents:
                if k not in self.finished and (self.waiting[k] is None or self.waiting[k]()):
                    moves.append(("agent", k))
            assert moves, "deadlock"
            kind, k = self.rng.choice(moves)
            if kind == "tc":
                self._run_product()
                continue
            try:
                self.waiting[k] = next(self.agents[k])
            except StopIteration:
                self.finished.add(k)
                self.waiting[k] = None


def mix(rng):
    return [rng.randint(1, 7) for _ in range(rng.randint(1, 5))]


def test_backward_pipeline_has_no_stale_read_or_deadlock():
    for seed in range(300):
        Model(mix(random.Random(seed)), seed).run()


@pytest.mark.parametrize("mutant", ["no_dq_full_wait", "no_dq_empty_wait", "early_q_release"])
def test_model_catches_a_missing_wait_or_an_early_release(mutant):
    caught = 0
    for seed in range(100):
        try:
            Model(mix(random.Random(seed)), seed, mutant).run()
        except AssertionError:
            caught += 1
    assert caught > 0, mutant
