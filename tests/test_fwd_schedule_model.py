"""A model of the forward kernel's barrier protocol (csrc/attention.cu), checked
on CPU over randomised interleavings.

Agents, as in the kernel: the producer (Q into two buffers; K and V into a ring
in the order K0, K1, K2, V0, K3, V1, ... with B = 3 score buffers, K0 .. K3, V0,
K4, V1, ... with B = 4), the S issuer (S_g into TMEM buffer g mod B once
P_g-B V_g-B has completed), the P V issuer, and two softmax warps
per lane quadrant that take alternate blocks, publish each block's outcome for
the partner, may redo a block and rescale O, and share the epilogue through the
row-sum exchange.  MMAs of one issuer execute in its issue order; the two
issuers' streams interleave freely; a commit arrives once the issuing thread's
earlier MMAs executed; TMA loads land in any order.  A wait on parity p
succeeds once the phase with parity p has completed, which includes the phase
before the current one: a waiter two phases ahead passes at once, as with
try_wait.parity.

Every read checks that it sees the version it wants (the S or P of its block in
its quadrant's rows, O accumulated up to the right block, the right stage, Q
buffer, outcome slot and row-sum slot).

The kernel enforces two orderings that an earlier version of it lacked, and the
model shows what each one prevents:
  * "O overwritten": the first P V of an item (accumulate = 0) must come after
    the epilogue reads of O by every softmax warp.  Ordering it only after the
    warp that publishes the item's next block leaves the partner warp of that
    lane quadrant unprotected.  The kernel has an O-free barrier: every softmax
    thread arrives after its epilogue reads, and the P V issuer waits for it
    before an item's first product (modelled per warp, since a warp's threads
    read O together).
  * "V stage read": the P V issuer must wait for P_g before V_g.  Waiting for
    V_1 (ring load 5, stage 1 with four stages) first lets that parity wait
    pass at once if K_1 (ring load 1, same stage) has not landed yet, and P V_1
    could then read the stage before V_1 is in it.  P_g implies S_g ran, so K_g
    (and every earlier load on V_g's stage) has landed.
"""
import random

import pytest

O_OVERWRITE = "O overwritten"
V_STAGE = "V stage read"


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


class Forward:
    def __init__(self, items, seed, quads=2, stages=4, o_free=False, p_before_v=False, mutation=None,
                 p_redo=0.25, early_waits=False, sbufs=3, p_tma=None):
        self.rng = random.Random(seed)
        self.items, self.quads, self.stages, self.B = items, quads, stages, sbufs
        self.o_free, self.p_before_v, self.mutation, self.p_redo = o_free, p_before_v, mutation, p_redo
        self.early_waits = early_waits
        # p_tma: when set, a step completes a pending TMA load with this probability (else
        # another unit moves), so that loads can stay in flight for long stretches
        self.p_tma = p_tma
        self.blocks = [(k, j) for k, n in enumerate(items) for j in range(n)]
        self.G = len(self.blocks)
        self.bars = {"OFull": Bar(1), "OFree": Bar(2 * quads)}
        for i in range(2):
            self.bars[f"QFull{i}"], self.bars[f"QEmpty{i}"] = Bar(1), Bar(1)
        for s in range(stages):
            self.bars[f"KvFull{s}"], self.bars[f"KvEmpty{s}"] = Bar(1), Bar(1)
        for b in range(sbufs):
            self.bars[f"SFull{b}"], self.bars[f"PFull{b}"], self.bars[f"PvDone{b}"] = Bar(1), Bar(quads), Bar(1)
        for q in range(quads):
            self.bars[f"Out{q}"], self.bars[f"Lx{q}"] = Bar(1), Bar(2)
        self.qbuf = [None, None]
        self.stage = [None] * stages                 # ("K", g) or ("V", g)
        self.sbuf = [None] * sbufs                   # (block, quadrants whose rows already hold P)
        self.O = None                                # (item, last block accumulated)
        self.outslot = {q: [None, None] for q in range(quads)}
        self.outcome_read = set()                    # (block, quadrant) outcome read by the partner
        self.lx = {q: [[None, None], [None, None]] for q in range(quads)}
        self.s_read = set()                          # (block, quadrant) softmax done with S
        self.epilogue_read = set()                   # (item, quadrant, warp) done reading O
        self.queues = {"S": [], "PV": []}
        self.issued = {"S": 0, "PV": 0}
        self.done_n = {"S": 0, "PV": 0}
        self.commits = {"S": [], "PV": []}
        self.executed = set()
        self.tma = []

    def seq_k(self, g):
        return g + max(0, g - (self.B - 1))

    def seq_v(self, g):
        return min(self.G + g, 2 * g + self.B)

    # ------------------------------------------------------------ asynchronous units
    def issue(self, who, g):
        self.queues[who].append(g)
        self.issued[who] += 1

    def commit(self, who, bar):
        self.commits[who].append((self.issued[who], bar))

    def execute(self, who):
        g = self.queues[who].pop(0)
        k, j = self.blocks[g]
        b = g % self.B
        if who == "S":
            assert self.qbuf[k % 2] == k, f"S_{g} reads the Q of item {self.qbuf[k % 2]}"
            assert self.stage[self.seq_k(g) % self.stages] == ("K", g), f"S_{g} reads a stage without K_{g}"
            if self.sbuf[b] is not None:
                old = self.sbuf[b][0]
                assert ("PV", old) in self.executed, f"S_{g} overwrites P_{old} before its product"
                assert all((old, q) in self.s_read for q in range(self.quads)), f"S_{g} overwrites S_{old} in use"
            self.sbuf[b] = (g, set())
        else:
            assert self.stage[self.seq_v(g) % self.stages] == ("V", g), f"{V_STAGE}: P V_{g} reads a stage without V_{g}"
            assert self.sbuf[b][0] == g and len(self.sbuf[b][1]) == self.quads, f"P V_{g} before P_{g} is complete"
            if j == 0:
                for q in range(self.quads):
                    for h in (0, 1):
                        assert k == 0 or (k - 1, q, h) in self.epilogue_read, \
                            f"{O_OVERWRITE}: P V_{g} starts item {k} before warp ({q},{h}) read item {k - 1}"
            else:
                assert self.O == (k, g - 1), f"P V_{g} accumulates onto {self.O}"
            self.O = (k, g)
        self.executed.add(("S" if who == "S" else "PV", g))
        self.done_n[who] += 1
        keep = []
        for n, bar in self.commits[who]:
            if n <= self.done_n[who]:
                self.bars[bar].arrive()
            else:
                keep.append((n, bar))
        self.commits[who] = keep

    # ------------------------------------------------------------ agents (yield wait predicates)
    def wait(self, bar, parity):
        b = self.bars[bar]
        return lambda: b.done(parity)

    def producer(self):
        order = [("K", g) for g in range(min(self.B, self.G))]
        for g in range(self.G):
            order.append(("V", g))
            if g + self.B < self.G:
                order.append(("K", g + self.B))
        for n, (what, g) in enumerate(order):
            k, j = self.blocks[g]
            if what == "K" and j == 0:
                yield self.wait(f"QEmpty{k % 2}", ((k // 2) & 1) ^ 1)
                assert k < 2 or all(("S", gg) in self.executed for gg, (kk, _) in enumerate(self.blocks) if kk == k - 2), \
                    f"the Q of item {k} overwrites item {k - 2}'s in use"
                self.tma.append(("Q", k, f"QFull{k % 2}"))
            st = n % self.stages
            assert n == (self.seq_k(g) if what == "K" else self.seq_v(g)), "ring order differs from its closed form"
            yield self.wait(f"KvEmpty{st}", ((n // self.stages) & 1) ^ 1)
            old = self.stage[st]
            assert old is None or (("S" if old[0] == "K" else "PV"), old[1]) in self.executed, f"stage {st} reloaded in use"
            self.tma.append(("KV", (what, g, st), f"KvFull{st}"))

    def s_issuer(self):
        for g, (k, j) in enumerate(self.blocks):
            b, seq = g % self.B, self.seq_k(g)
            k_wait = self.wait(f"KvFull{seq % self.stages}", (seq // self.stages) & 1)
            if self.early_waits:       # K (and Q) before the buffer: they are off the chain
                yield k_wait
                if j == 0:
                    yield self.wait(f"QFull{k % 2}", (k // 2) & 1)
            if g >= self.B and self.mutation != "no_pvdone_wait":
                yield self.wait(f"PvDone{b}", ((g // self.B) & 1) ^ 1)
            if not self.early_waits:
                if j == 0:
                    yield self.wait(f"QFull{k % 2}", (k // 2) & 1)
                yield k_wait
            self.issue("S", g)
            self.commit("S", f"KvEmpty{seq % self.stages}")
            if j + 1 == self.items[k]:
                self.commit("S", f"QEmpty{k % 2}")
            self.commit("S", f"SFull{b}")

    def pv_issuer(self):
        for g, (k, j) in enumerate(self.blocks):
            b, seq = g % self.B, self.seq_v(g)
            v_wait = self.wait(f"KvFull{seq % self.stages}", (seq // self.stages) & 1)
            p_wait = self.wait(f"PFull{b}", (g // self.B) & 1)
            # V first is safe where the load before V_g on its stage is one this thread
            # waited for itself (V_g-stages/2, an even number of stages) or one that P_g-1
            # implies (an earlier K): from g = 2 with three score buffers (four or eight
            # stages), from g = 3 with four (six stages)
            v_from = 2 if self.B == 3 else self.stages // 2
            if self.mutation == "v_first_early":
                v_from = 2
            v_first = not self.p_before_v or (self.early_waits and g >= v_from and seq == 2 * g + self.B)
            for w in ((v_wait, p_wait) if v_first else (p_wait, v_wait)):
                yield w
            if self.o_free and j == 0 and k > 0:
                yield self.wait("OFree", (k - 1) & 1)
            self.issue("PV", g)
            self.commit("PV", f"KvEmpty{seq % self.stages}")
            self.commit("PV", f"PvDone{b}")
            if j + 1 == self.items[k]:
                self.commit("PV", "OFull")

    def softmax(self, q, h):
        consumed, have_m = -1, False

        def read_outcome(gg):
            nonlocal consumed
            yield self.wait(f"Out{q}", gg & 1)
            assert self.outslot[q][gg & 1] == gg, f"warp ({q},{h}) reads outcome {gg} from a reused slot"
            consumed = gg
            self.outcome_read.add((gg, q))

        for g, (k, j) in enumerate(self.blocks):
            b = g % self.B
            if j == 0:
                have_m = False
            if (g & 1) == h:
                yield self.wait(f"SFull{b}", (g // self.B) & 1)
                mine = lambda: self.sbuf[b][0] == g and q not in self.sbuf[b][1]   # noqa: E731
                assert mine(), f"warp ({q},{h}) reads S_{g} from a buffer holding {self.sbuf[b]}"
                if j > 0 and not have_m:
                    yield from read_outcome(g - 1)
                have_m = True
                if g > 0 and consumed != g - 1 and self.mutation != "no_outcome_read":
                    yield from read_outcome(g - 1)
                if j > 0 and self.rng.random() < self.p_redo:        # redo with the exact max: rescale O
                    yield self.wait(f"PvDone{(g - 1) % self.B}", ((g - 1) // self.B) & 1)
                    assert self.O == (k, g - 1), f"the rescale in block {g} sees O {self.O}"
                    yield lambda: True
                    assert self.O == (k, g - 1), f"O changed under the rescale in block {g}"
                assert mine(), f"S_{g} of quadrant {q} changed under the softmax"
                self.s_read.add((g, q))
                assert g < 2 or (g - 2, q) in self.outcome_read, f"publishing {g} overwrites outcome {g - 2} unread"
                self.outslot[q][g & 1] = g
                self.bars[f"Out{q}"].arrive()
                self.sbuf[b][1].add(q)
                self.bars[f"PFull{b}"].arrive()
                yield lambda: True
            if j + 1 == self.items[k]:
                if consumed != g and (g & 1) != h:
                    yield from read_outcome(g)
                yield self.wait("OFull", k & 1)
                self.lx[q][k & 1][h] = k
                self.bars[f"Lx{q}"].arrive()
                yield self.wait(f"Lx{q}", k & 1)
                assert self.lx[q][k & 1][h ^ 1] == k, f"the row sums of item {k} were overwritten"
                for _ in range(2):                                     # two 32-column loads of O
                    assert self.O == (k, g), f"{O_OVERWRITE}: warp ({q},{h}) reads O {self.O} for item {k}"
                    yield lambda: True
                self.epilogue_read.add((k, q, h))
                if self.o_free:
                    self.bars["OFree"].arrive()

    def run(self, max_steps=400_000):
        agents = [self.producer(), self.s_issuer(), self.pv_issuer()]
        agents += [self.softmax(q, h) for q in range(self.quads) for h in (0, 1)]
        waits, done = [None] * len(agents), [False] * len(agents)
        for _ in range(max_steps):
            choices = [("agent", i) for i in range(len(agents)) if not done[i] and (waits[i] is None or waits[i]())]
            choices += [("mma", who) for who in ("S", "PV") if self.queues[who]]
            tmas = [("tma", i) for i in range(len(self.tma))]
            if not choices and not tmas:
                assert all(done), "deadlock"
                assert not any(self.commits.values())
                return
            if self.p_tma is None:
                what, x = self.rng.choice(choices + tmas)
            elif tmas and (not choices or self.rng.random() < self.p_tma):
                what, x = self.rng.choice(tmas)
            else:
                what, x = self.rng.choice(choices)
            if what == "agent":
                try:
                    waits[x] = next(agents[x])
                except StopIteration:
                    done[x] = True
            elif what == "mma":
                self.execute(x)
            else:
                kind, val, bar = self.tma.pop(x)
                if kind == "Q":
                    self.qbuf[val % 2] = val
                else:
                    self.stage[val[2]] = (val[0], val[1])
                self.bars[bar].arrive()
        raise AssertionError("step limit")


def _failures(n, seed, stages=(4, 8), **kw):
    rng = random.Random(seed)
    out = []
    for t in range(n):
        items = [rng.randint(1, 5) for _ in range(rng.randint(1, 5))]
        try:
            Forward(items, seed=t, quads=rng.choice([1, 2]), stages=rng.choice(stages), **kw).run()
        except AssertionError as e:
            out.append(str(e))
    return out


def test_kernel_order_has_no_deadlock_and_no_stale_read():
    # the order of csrc/attention.cu: O-free barrier, P_g before V_g except where V_g's stage
    # last held V_g-2, and the S issuer's K and Q waits before its buffer wait
    assert _failures(3000, 1, o_free=True, p_before_v=True, early_waits=True) == []
    assert _failures(1000, 6, o_free=True, p_before_v=True) == []
    # loads that stay in flight for long stretches (the early-pass hazards need them)
    assert _failures(1500, 11, p_tma=0.05, o_free=True, p_before_v=True, early_waits=True) == []


def test_four_buffers_need_v_first_only_past_half_the_ring():
    # A variant with four score buffers of 96 keys and a six-stage ring (measured, not
    # adopted): there V_2's stage last held K_2, which P V_1 does not imply, so waiting
    # for V_2 before P_2 lets the parity wait pass early while K_2 is in flight; from
    # g = 3 (half the ring) V first is safe.
    kw = dict(stages=(6,), o_free=True, p_before_v=True, early_waits=True, sbufs=4, p_tma=0.05)
    assert _failures(1500, 7, **kw) == []
    fails = _failures(1500, 8, mutation="v_first_early", **kw)
    assert fails and all(f.startswith(V_STAGE) for f in fails), fails[:3]


def test_without_the_two_orderings_the_model_finds_both_hazards():
    # the earlier order (V_g before P_g, no O-free barrier) has exactly these two
    fails = _failures(6000, 2)
    kinds = {f.split(":")[0] for f in fails}
    assert kinds == {O_OVERWRITE, V_STAGE}, kinds
    # the O-free barrier alone leaves only the (rarer) stage hazard
    assert all(f.startswith(V_STAGE) for f in _failures(1500, 3, o_free=True))
    # P before V alone leaves only the O hazard
    assert all(f.startswith(O_OVERWRITE) for f in _failures(1500, 5, p_before_v=True))


@pytest.mark.parametrize("mutation", ["no_pvdone_wait", "no_outcome_read"])
def test_model_catches_planted_ordering_mistakes(mutation):
    fails = _failures(400, 4, o_free=True, p_before_v=True, early_waits=True, mutation=mutation)
    assert len(fails) >= 40, f"{mutation}: caught in only {len(fails)} schedules"
