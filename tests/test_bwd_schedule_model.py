"""A model of the backward kernels' barrier protocol (csrc/backward.cu), checked
on CPU for deadlock and stale reads over randomised interleavings.

The agents are the ones in the kernel: the producer warp (TMA loads of an item's
fixed operands and of the streamed blocks into a two-stage ring), the MMA-issuing
thread, and eight elementwise warps (phase A loads S, releases the S columns and
turns S into P; phase B turns dP into dS and stores it, with P^T for dK and dV,
over the dP columns; an epilogue per item).  The issuer tests some barriers early,
without waiting (a snapshot taken in the middle of an earlier MMA group), and skips
the wait at the point of use when the test succeeded.
Two asynchronous units complete work late and in their own order: TMA loads
complete in any order, and MMAs execute in issue order.  A commit arrives once
every MMA issued before it has executed.  An mbarrier wait on parity p succeeds
once the phase with parity p has completed, as try_wait.parity does.

Every MMA and every warp checks, at the moment it reads, that the buffer holds
the version it wants: the S or dP of its block in TMEM, the fixed operands of its
item, the block's stage, P^T or dS written by all eight warps.  A write checks
that every reader of the previous version is done.  Planted ordering mistakes
show that the checks catch what they should.
"""
import random

import pytest

KIND_DQ, KIND_DKDV = "dq", "dkdv"
NW = 8


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


class Model:
    def __init__(self, kind, items, seed, mutation=None):
        self.rng = random.Random(seed)
        self.kind = kind
        self.items = items                       # kv_len of each item of one CTA
        self.mutation = mutation
        self.bars = {n: Bar(c) for n, c in [
            ("FixFull", 1), ("FixEmpty", 1), ("KvFull0", 1), ("KvFull1", 1), ("KvEmpty0", 1), ("KvEmpty1", 1),
            ("SFull", 1), ("DFull", 1), ("SFree", NW), ("PFull", NW), ("OFull", 1), ("Drain", 1)]}
        self.blocks = [(k, j) for k, n in enumerate(items) for j in range(n)]
        self.fix = None                          # item whose fixed operands are in shared memory
        self.stage = [None, None]                # block held by each stage
        self.tS = self.tD = None                 # block whose S / dP the TMEM columns hold
        self.read_S, self.read_D, self.wrote_P, self.wrote_dS, self.read_stage = ({} for _ in range(5))
        self.epilogue_done = set()
        self.executed = set()
        self.mma_queue, self.commits, self.tma_queue = [], [], []
        self.n_issued = self.n_executed = 0

    # ------------------------------------------------------------ asynchronous units
    def issue(self, op, b):
        self.mma_queue.append((op, b))
        self.n_issued += 1

    def commit(self, bar):
        self.commits.append((self.n_issued, bar))

    def all_warps(self, table, b):
        return table.get(b, set()) == set(range(NW))

    def execute_mma(self):
        op, b = self.mma_queue.pop(0)
        k, _ = self.blocks[b]
        assert self.stage[b & 1] == b, f"{op} of block {b} reads a stage holding {self.stage[b & 1]}"
        if op in ("S", "dP"):
            assert self.fix == k, f"{op} of block {b} reads the fixed operands of item {self.fix}"
        if op == "S":
            if self.tS is not None:
                assert self.all_warps(self.read_S, self.tS), f"S of {b} overwrites S of {self.tS} before phase A"
            self.tS = b
        elif op == "dP":
            if self.tD is not None:
                assert self.all_warps(self.read_D, self.tD), f"dP of {b} overwrites dP of {self.tD} before phase B"
                assert ("acc", self.tD) in self.executed, f"dP of {b} overwrites dS of {self.tD} before its use"
                if self.kind == KIND_DKDV:
                    assert ("dV", self.tD) in self.executed, f"dP of {b} overwrites P^T of {self.tD} before dV"
            self.tD = b
        elif op == "dV":
            assert self.tD == b and self.all_warps(self.wrote_P, b), f"dV of {b} before P^T is complete"
            self.check_first_accumulation(b)
        elif op == "acc":
            assert self.tD == b and self.all_warps(self.wrote_dS, b), f"accumulation of {b} before dS is complete"
            self.check_first_accumulation(b)
        self.executed.add((op, b))
        self.n_executed += 1
        keep = []
        for n, bar in self.commits:
            if n <= self.n_executed:
                self.bars[bar].arrive()
            else:
                keep.append((n, bar))
        self.commits = keep

    def check_first_accumulation(self, b):
        k, j = self.blocks[b]
        if j == 0 and k > 0:
            assert all((k - 1, w) in self.epilogue_done for w in range(NW)), \
                f"item {k} overwrites the accumulators before item {k - 1}'s epilogue"

    def complete_tma(self, i):
        what, x, bar = self.tma_queue.pop(i)
        if what == "fix":
            self.fix = x
        else:
            self.stage[x & 1] = x
        self.bars[bar].arrive()

    # ------------------------------------------------------------ agents (yield wait predicates)
    def wait(self, bar, parity):
        b = self.bars[bar]
        return lambda: b.done(parity)

    def producer(self):
        seq = nfix = 0
        for k, n in enumerate(self.items):
            yield self.wait("FixEmpty", (nfix & 1) ^ 1)
            if k > 0:
                for b, (kk, _) in enumerate(self.blocks):
                    if kk == k - 1:
                        assert ("S", b) in self.executed and ("dP", b) in self.executed, \
                            f"item {k}'s fixed operands overwrite item {k - 1}'s while in use"
            nfix += 1
            self.tma_queue.append(("fix", k, "FixFull"))
            for _ in range(n):
                st = seq & 1
                yield self.wait(f"KvEmpty{st}", ((seq >> 1) & 1) ^ 1)
                if seq >= 2:
                    old = seq - 2
                    for op in ("S", "dP", "acc") + (("dV",) if self.kind == KIND_DKDV else ()):
                        assert (op, old) in self.executed, f"block {seq} overwrites stage of {old} before {op}"
                    if self.kind == KIND_DKDV:
                        assert self.all_warps(self.read_stage, old), f"block {seq} overwrites lse, D of {old}"
                self.tma_queue.append(("stage", seq, f"KvFull{st}"))
                seq += 1

    def test(self, bar, parity):
        """mbarrier.test_wait: a snapshot, no waiting."""
        return self.bars[bar].done(parity)

    def issuer(self):
        items, m = self.items, self.mutation
        k = j = seq = 0
        n = items[0]
        yield self.wait("FixFull", 0)
        yield self.wait("KvFull0", 0)
        nfix = 1
        self.issue("S", 0); self.commit("SFull")
        self.issue("dP", 0)
        s_free_ok = self.test("SFree", 0)
        kv_ok = n > 1 and self.test("KvFull1", 0)
        self.commit("DFull")
        if n == 1:
            self.commit("FixEmpty")
        while True:
            new_item = j + 1 == n
            n_next = (items[k + 1] if k + 1 < len(items) else 0) if new_item else n
            has_next = n_next > 0
            next_is_last = n_next == 1 if new_item else j + 2 == n
            if not s_free_ok and m != "no_sfree_wait":
                yield self.wait("SFree", seq & 1)
            p_ok = False
            if has_next and not new_item:
                if not kv_ok:
                    yield self.wait(f"KvFull{(seq + 1) & 1}", ((seq + 1) >> 1) & 1)
                self.issue("S", seq + 1)
                p_ok = self.test("PFull", seq & 1)
                self.commit("SFull")
            if not p_ok:
                yield self.wait("PFull", seq & 1)
            if m == "dp_before_acc" and has_next and not new_item:
                self.issue("dP", seq + 1); self.commit("DFull")
            if self.kind == KIND_DKDV:
                self.issue("dV", seq)
            self.issue("acc", seq)
            self.commit(f"KvEmpty{seq & 1}")
            if new_item:
                self.commit("OFull")
            if not has_next:
                break
            if new_item:
                yield self.wait("FixFull", nfix & 1)
                yield self.wait(f"KvFull{(seq + 1) & 1}", ((seq + 1) >> 1) & 1)
                nfix += 1
                self.issue("S", seq + 1); self.commit("SFull")
            if m == "early_fix_empty" and next_is_last:
                self.commit("FixEmpty")
            if not (m == "dp_before_acc" and not new_item):
                self.issue("dP", seq + 1)
            s_free_ok = self.test("SFree", (seq + 1) & 1)
            kv_ok = not next_is_last and self.test(f"KvFull{(seq + 2) & 1}", ((seq + 2) >> 1) & 1)
            if not (m == "dp_before_acc" and not new_item):
                self.commit("DFull")
            if m != "early_fix_empty" and next_is_last:
                self.commit("FixEmpty")
            seq += 1
            if new_item:
                k, j, n = k + 1, 0, n_next
            else:
                j += 1
        self.commit("Drain")
        yield self.wait("Drain", 0)

    def warp(self, w):
        seq = 0
        for k, n in enumerate(self.items):
            for _ in range(n):
                b = seq
                yield self.wait("SFull", seq & 1)
                if self.kind == KIND_DKDV:
                    yield self.wait(f"KvFull{seq & 1}", (seq >> 1) & 1)
                    assert self.stage[seq & 1] == b, f"warp {w} reads lse of block {self.stage[seq & 1]}"
                assert self.tS == b, f"warp {w} phase A of block {b} reads S of {self.tS}"
                self.read_S.setdefault(b, set()).add(w)
                self.bars["SFree"].arrive()
                yield lambda: True
                yield self.wait("DFull", seq & 1)
                assert self.tD == b, f"warp {w} phase B of block {b} reads dP of {self.tD}"
                if self.kind == KIND_DKDV:
                    assert self.stage[seq & 1] == b
                    self.read_stage.setdefault(b, set()).add(w)
                self.read_D.setdefault(b, set()).add(w)
                self.wrote_dS.setdefault(b, set()).add(w)
                if self.kind == KIND_DKDV:
                    self.wrote_P.setdefault(b, set()).add(w)
                self.bars["PFull"].arrive()
                seq += 1
            yield self.wait("OFull", k & 1)
            assert ("acc", seq - 1) in self.executed, f"warp {w} reads item {k}'s accumulators early"
            self.epilogue_done.add((k, w))

    def run(self, max_steps=200_000):
        agents = [self.producer(), self.issuer()] + [self.warp(w) for w in range(NW)]
        waits = [None] * len(agents)
        done = [False] * len(agents)
        for _ in range(max_steps):
            choices = [("agent", i) for i in range(len(agents))
                       if not done[i] and (waits[i] is None or waits[i]())]
            if self.mma_queue:
                choices.append(("mma", 0))
            choices += [("tma", t) for t in range(len(self.tma_queue))]
            if not choices:
                assert all(done), "deadlock"
                assert not self.commits and not self.mma_queue
                return
            what, i = self.rng.choice(choices)
            if what == "agent":
                try:
                    waits[i] = next(agents[i])
                except StopIteration:
                    done[i] = True
            elif what == "mma":
                self.execute_mma()
            else:
                self.complete_tma(i)
        raise AssertionError("step limit")


def _cases(n, seed):
    rng = random.Random(seed)
    for trial in range(n):
        kind = rng.choice([KIND_DQ, KIND_DKDV])
        items = [rng.randint(1, 5) for _ in range(rng.randint(1, 5))]
        yield kind, items, trial


def test_schedule_has_no_deadlock_and_no_stale_read():
    for kind, items, trial in _cases(2000, 1):
        Model(kind, items, seed=trial).run()


@pytest.mark.parametrize("mutation", ["no_sfree_wait", "dp_before_acc", "early_fix_empty"])
def test_model_catches_planted_ordering_mistakes(mutation):
    caught = 0
    for kind, items, trial in _cases(200, 2):
        try:
            Model(kind, items, seed=trial, mutation=mutation).run()
        except AssertionError:
            caught += 1
    assert caught >= 20, f"{mutation}: caught in only {caught} schedules"
