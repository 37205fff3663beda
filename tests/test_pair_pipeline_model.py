"""A model of the CTA-pair forward kernel's handshakes (fa_fwd_pair.cuh), run under random
interleavings on the CPU.

One CTA's view of the pair (the partner CTA's warps only add arrivals to the same
barriers).  Agents:
- producer: per unit K_0, K_1, then per block j K_(j+2) and V_j into an NSLOT ring
  (slot_empty waited with the preceding phase's parity, slot_full arrived when the copy
  lands);
- MMA warp: a loop of non-blocking probes that issues S(k) into score buffer k & 1 once the
  buffer has been read (s_free), K_k has landed and k <= next_pv + 2, or P(j) V once P(j)
  is written (and, for j = 0, the previous unit's epilogue has read O).  Its commits:
  s_full and the K slot's slot_empty after S, pv_done(j & 1) and the V slot's slot_empty
  after P V, o_full after the unit's last P V.  The tensor core runs products and commits
  in issue order;
- two softmax streams h = 0, 1 (blocks j = h, h + 2, ...): wait s_full(h), read S(j),
  arrive s_free(h); take block j-1's maximum from the other stream (hand barrier), publish
  block j's; sometimes rescale O, which first waits pv_done((j-1) & 1) for P(j-1) V with
  the parity of that barrier's product count; before writing P(j) into numerator buffer h,
  wait pv_done(h) for P(j-2) V; arrive p_full(h).  Epilogue per unit: the last block's
  maximum if the other stream had it, wait o_full, exchange the row sums (xchg barrier,
  two arrivals), arrive o_empty (two arrivals).

Every read checks what it needs when it happens: S(j) in its buffer, K_k / V_j in their
slots, P(j) not overwritten before P(j-2) V read it, the maximum handed over being block
j-1's, O holding exactly the products before j when it is rescaled, the epilogue seeing all
n products and the partner's sum of the same unit, and P(0) V of a unit overwriting O only
after the previous unit's epilogue read it.  Random schedules must finish without a failed
check or a deadlock; each planted mistake must be caught by some schedule."""
import random

import pytest


class MBarrier:
    def __init__(self, count=1):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase ^= 1
            self.pending = self.count

    def done(self, parity):  # the phase with this parity has completed
        return self.phase != parity


def k_pos(k, alias):
    return k if k < 2 else (2 * k - 1 if alias else 2 * k - 2)


def v_pos(j, n, alias):
    return (2 if n > 1 else 1) + j + min(j if alias else j + 1, max(n - 2, 0))


class PairModel:
    def __init__(self, units, seed, nslot=8, rescale_p=0.3, mutant=None, alias=False):
        # alias: the head-dim-256 layout, where P(b) lies over the first columns of S(b), the
        # producer loads V_j before K_(j+2), and S(k) waits until P(k-2) V has been issued
        self.units, self.nslot, self.mutant, self.alias = units, nslot, mutant, alias
        self.rng = random.Random(seed)
        self.rescale_p = rescale_p
        self.slot_full = [MBarrier() for _ in range(nslot)]
        self.slot_empty = [MBarrier() for _ in range(nslot)]
        self.s_full = [MBarrier(), MBarrier()]
        self.s_free = [MBarrier(), MBarrier()]
        self.p_full = [MBarrier(), MBarrier()]
        self.pv_done = [MBarrier(), MBarrier()]
        self.hand = [MBarrier(), MBarrier()]
        self.o_full, self.o_empty, self.xchg = MBarrier(), MBarrier(2), MBarrier(2)
        self.slot = [None] * nslot
        self.sbuf = [None, None]
        self.pbuf = [None, None]           # (u, j, read by its P V yet)
        self.o = None                      # (unit, products accumulated)
        self.o_reads = {}                  # unit -> epilogue reads of O
        self.mh = [None, None]             # (unit, block) of the maximum last published
        self.xl = [None, None]             # unit of the row sum last written
        self.tc = []
        self.agents = {"load": self._producer(), "mma": self._mma(),
                       "s0": self._softmax(0), "s1": self._softmax(1)}
        self.waiting = {k: None for k in self.agents}
        self.finished = set()

    # ---------------------------------------------------------------- producer
    def _producer(self):
        issued = 0
        for u, n in enumerate(self.units):
            order = [("K", 0)] + ([("K", 1)] if n > 1 else [])
            for j in range(n):
                if self.alias:
                    order.append(("V", j))
                if j + 2 < n:
                    order.append(("K", j + 2))
                if not self.alias:
                    order.append(("V", j))
            for kind, idx in order:
                s = issued % self.nslot
                yield lambda s=s, ph=((issued // self.nslot) & 1) ^ 1: self.slot_empty[s].done(ph)
                self.slot[s] = (kind, u, idx)
                self.slot_full[s].arrive()
                issued += 1

    # ---------------------------------------------------------------- MMA warp
    def _can_scores(self, m):
        n = self.units[m["u"]]
        if not (m["next_s"] < n and m["next_s"] <= m["next_pv"] + m["lead"]):
            return False
        k, b = m["next_s"], m["next_s"] & 1
        buf_free = not (m["s_issued"] >> b) & 1 or self.s_free[b].done((m["sfph"] >> b) & 1)
        ki = m["kv_base"] + k_pos(k, self.alias)
        return buf_free and self.slot_full[ki % self.nslot].done((ki // self.nslot) & 1)

    def _can_values(self, m):
        n = self.units[m["u"]]
        if not m["next_pv"] < m["next_s"]:
            return False
        j, b = m["next_pv"], m["next_pv"] & 1
        vi = m["kv_base"] + v_pos(j, n, self.alias)
        o_ok = j > 0 or self.mutant == "no_o_empty_wait" or self.o_empty.done((m["unit_it"] & 1) ^ 1)
        return (self.p_full[b].done((m["pph"] >> b) & 1) and o_ok and
                self.slot_full[vi % self.nslot].done((vi // self.nslot) & 1))

    def _mma(self):
        lead = 1 if self.alias else 2
        if self.mutant == "scores_four_ahead":
            lead = 3
        elif self.mutant == "alias_scores_three_ahead":
            lead = 2
        m = dict(kv_base=0, pph=0, sfph=0, unit_it=0, u=0, next_s=0, next_pv=0, s_issued=0,
                 lead=lead)
        for u, n in enumerate(self.units):
            m.update(u=u, next_s=0, next_pv=0)  # s_issued persists across units
            if self.mutant == "buffers_free_at_unit_start":
                m["s_issued"] = 0
            while m["next_pv"] < n:
                progressed = False
                if self._can_scores(m):
                    k, b = m["next_s"], m["next_s"] & 1
                    ki = m["kv_base"] + k_pos(k, self.alias)
                    if (m["s_issued"] >> b) & 1:
                        m["sfph"] ^= 1 << b
                    self.tc += [("S", u, k, ki % self.nslot),
                                ("commit", [self.s_full[b], self.slot_empty[ki % self.nslot]])]
                    m["s_issued"] |= 1 << b
                    m["next_s"] += 1
                    progressed = True
                if self._can_values(m):
                    j, b = m["next_pv"], m["next_pv"] & 1
                    vi = m["kv_base"] + v_pos(j, n, self.alias)
                    m["pph"] ^= 1 << b
                    bars = [self.pv_done[b], self.slot_empty[vi % self.nslot]]
                    if j == n - 1:
                        bars.append(self.o_full)
                    self.tc += [("PV", u, j, vi % self.nslot), ("commit", bars)]
                    m["next_pv"] += 1
                    progressed = True
                if not progressed:
                    yield lambda: self._can_scores(m) or self._can_values(m)
            m["kv_base"] += 2 * n
            m["unit_it"] += 1

    # ---------------------------------------------------------------- softmax streams
    def _softmax(self, h):
        sph = hph = xph = 0
        pvc = [0, 0]
        for u, n in enumerate(self.units):
            for j in range(h, n, 2):
                yield lambda ph=sph: self.s_full[h].done(ph)
                sph ^= 1
                assert self.sbuf[h] == ("S", u, j), ("softmax reads S", self.sbuf[h], u, j)
                self.s_free[h].arrive()
                if j > 0:
                    if self.mutant != "hand_without_wait":
                        yield lambda ph=hph: self.hand[h ^ 1].done(ph)
                    hph ^= 1
                    assert self.mh[h ^ 1] == (u, j - 1), ("maximum handed over", self.mh[h ^ 1], u, j)
                self.mh[h] = (u, j)
                self.hand[h].arrive()
                if j > 0 and self.rng.random() < self.rescale_p:
                    b1 = (j - 1) & 1
                    nn = pvc[b1] + (j - 1) // 2
                    yield lambda b1=b1, p=nn & 1: self.pv_done[b1].done(p)
                    assert self.o == (u, j), ("rescale finds O", self.o, u, j)
                    assert not any(op[0] == "PV" for op in self.tc), "a product in flight"
                if j >= 2 and self.mutant != "numerators_without_wait":
                    nn = pvc[h] + (j - 2) // 2
                    yield lambda p=nn & 1: self.pv_done[h].done(p)
                prev = self.pbuf[h]
                assert prev is None or prev[2], ("P overwritten before its P V read it", prev, u, j)
                if self.alias:  # P(j) goes over the columns S(j) came from
                    assert self.sbuf[h] == ("S", u, j), ("P written over other scores", self.sbuf[h], u, j)
                self.pbuf[h] = (u, j, False)
                self.p_full[h].arrive()
            # epilogue
            if ((n - 1) & 1) != h:
                yield lambda ph=hph: self.hand[h ^ 1].done(ph)
                hph ^= 1
                assert self.mh[h ^ 1] == (u, n - 1), ("last maximum", self.mh[h ^ 1], u, n)
            if self.mutant != "sum_before_o_full":
                yield lambda ph=u & 1: self.o_full.done(ph)
            self.xl[h] = u
            if self.mutant == "sum_before_o_full":
                yield lambda ph=u & 1: self.o_full.done(ph)
            assert self.o == (u, n), ("epilogue reads O", self.o, u, n)
            self.xchg.arrive()
            yield lambda ph=xph: self.xchg.done(ph)
            xph ^= 1
            assert self.xl[h ^ 1] == u, ("partner's row sum", self.xl[h ^ 1], u)
            self.o_reads[u] = self.o_reads.get(u, 0) + 1
            self.o_empty.arrive()
            pvc[0] += (n + 1) // 2
            pvc[1] += n // 2

    # ---------------------------------------------------------------- tensor core
    def _run(self):
        op = self.tc.pop(0)
        if op[0] == "commit":
            for bar in op[1]:
                bar.arrive()
            return
        kind, u, j, s = op
        if kind == "S":
            assert self.slot[s] == ("K", u, j), ("S reads K", self.slot[s], u, j)
            if self.alias:
                pb = self.pbuf[j & 1]
                assert pb is None or pb[2], ("S overwrites P before its P V read it", pb, u, j)
            self.sbuf[j & 1] = ("S", u, j)
        else:
            assert self.slot[s] == ("V", u, j), ("P V reads V", self.slot[s], u, j)
            pb = self.pbuf[j & 1]
            assert pb is not None and pb[:2] == (u, j), ("P V reads P", pb, u, j)
            self.pbuf[j & 1] = (u, j, True)
            if j == 0:
                assert self.o_reads.get(u - 1, 0) == 2 or u == 0, "O overwritten before the epilogue read it"
                self.o = (u, 1)
            else:
                assert self.o == (u, j), ("accumulation order", self.o, u, j)
                self.o = (u, j + 1)

    def run(self):
        steps = 0
        while len(self.finished) < len(self.agents) or self.tc:
            moves = [("tc", None)] if self.tc else []
            for k in self.agents:
                if k not in self.finished and (self.waiting[k] is None or self.waiting[k]()):
                    moves.append(("agent", k))
            assert moves, "deadlock"
            steps += 1
            assert steps < 200000, "livelock"
            kind, k = self.rng.choice(moves)
            if kind == "tc":
                self._run()
                continue
            try:
                self.waiting[k] = next(self.agents[k])
            except StopIteration:
                self.finished.add(k)
                self.waiting[k] = None


def unit_mix(rng):
    return [rng.randint(1, 9) for _ in range(rng.randint(1, 5))]


@pytest.mark.parametrize("alias,nslot", [(False, 8), (False, 4), (True, 4), (True, 2)])
def test_pair_handshakes_are_race_free(alias, nslot):
    """Head dim 128 (separate numerator buffers, 8 slots) and 256 (P over S, 4 slots), and
    smaller rings."""
    for seed in range(250):
        PairModel(unit_mix(random.Random(seed)), seed, nslot=nslot, rescale_p=0.5,
                  alias=alias).run()


@pytest.mark.parametrize("mutant", ["scores_four_ahead", "numerators_without_wait",
                                    "hand_without_wait", "no_o_empty_wait",
                                    "sum_before_o_full", "buffers_free_at_unit_start"])
def test_model_catches_a_planted_mistake(mutant):
    caught = 0
    for seed in range(150):
        try:
            PairModel(unit_mix(random.Random(seed)), seed, rescale_p=0.5, mutant=mutant).run()
        except AssertionError:
            caught += 1
    assert caught > 0, mutant


def test_model_catches_scores_over_unread_numerators():
    """With P over S, S(k) issued before P(k-2) V (the head-dim-128 lead of two) overwrites
    numerators the tensor core has not read yet."""
    caught = 0
    for seed in range(150):
        try:
            PairModel(unit_mix(random.Random(seed)), seed, nslot=4, rescale_p=0.5, alias=True,
                      mutant="alias_scores_three_ahead").run()
        except AssertionError:
            caught += 1
    assert caught > 0
