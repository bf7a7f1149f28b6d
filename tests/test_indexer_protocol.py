"""Model check of the FP8 indexer kernel's barrier protocol (CPU).

`index_scores_tc_kernel` (indexed_sparse_attention_fp8_b200/csrc/indexer_tc.cu) runs a TMA
producer warp, an MMA-issuing warp and 8 epilogue warps per CTA, coordinated by mbarriers: a
ring of key-tile stages (a_full / a_empty; 6 for query blocks of 4, 4 for the one-query decode
shape, which runs two CTAs per SM), two query-block buffers with their head weights
(b_full / b_empty) and two TMEM accumulators (acc_full / acc_empty).  This model restates each
role's waits, arrivals, expect-tx and asynchronous completions (TMA loads in any order, the
tensor pipe in issue order) and runs them under random schedules over many work-item patterns,
checking that no schedule deadlocks and that no stage, query block or accumulator is
overwritten before its readers are done or read at the wrong version.  Planted protocol
mistakes must each be caught.
"""
import random
import sys

import pytest

NA = 6          # key-tile stages (the tests below also run the decode shape's 4)
E = 8           # epilogue warps (4 TMEM lane quadrants x 2 column halves)


class Deadlock(Exception):
    pass


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.phase, self.pending, self.tx = name, count, 0, count, 0

    def _check(self):
        if self.pending < 0:
            raise AssertionError(f"over-arrival on {self.name} phase {self.phase}")
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._check()

    def expect_tx(self, n):
        self.tx += n
        self.pending -= 1
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def ready(self, parity):
        return (self.phase & 1) != parity


class Buf:
    def __init__(self, name):
        self.name, self.ver, self.left = name, None, 0

    def write(self, ver, readers):
        if self.left:
            raise AssertionError(f"{self.name}: {ver} written while {self.left} readers of {self.ver} remain")
        self.ver, self.left = ver, readers

    def read(self, ver):
        if self.ver != ver or self.left <= 0:
            raise AssertionError(f"{self.name}: read of {ver}, holds {self.ver} ({self.left} reads left)")
        self.left -= 1


class Cta:
    """One persistent CTA serving `items` (key tiles per item; 0 = nothing visible)."""

    def __init__(self, items, seed, mistakes=(), abort_at=None, async_p=None):
        self.rng = random.Random(seed)
        # async_p: when roles and asynchronous completions are both ready, the chance that a
        # completion goes next (None: uniform); small values keep copies and MMAs in flight longer
        self.async_p = async_p
        self.items, self.mk = items, set(mistakes)
        # abort_at: the scheduling step at which some bounded wait gives up (None: never); from
        # then on every wait returns "failed" and each role takes its exit path
        self.abort_at, self.aborted = abort_at, False
        self.q = {"tma": [], "tc": []}
        acc_empty = E - 1 if "acc_empty_count" in self.mk else E
        b_empty = E if "b_empty_without_mma" in self.mk else E + 1
        self.bar = {}
        for s in range(NA):
            self.bar[f"a_full{s}"] = Bar(f"a_full{s}", 1)
            self.bar[f"a_empty{s}"] = Bar(f"a_empty{s}", 1)
        for s in range(2):
            self.bar[f"b_full{s}"] = Bar(f"b_full{s}", 1)
            self.bar[f"b_empty{s}"] = Bar(f"b_empty{s}", b_empty)
            self.bar[f"acc_full{s}"] = Bar(f"acc_full{s}", 1)
            self.bar[f"acc_empty{s}"] = Bar(f"acc_empty{s}", acc_empty)
        self.bar["mma_drain"] = Bar("mma_drain", 1)
        self.buf = {n: Buf(n) for n in [f"A{s}" for s in range(NA)] + ["B0", "B1", "acc0", "acc1"]}

    def work(self):
        return [(i, n) for i, n in enumerate(self.items) if n > 0]

    def bpar(self, cnt):
        return cnt & 1 if "b_parity" in self.mk else (cnt >> 1) & 1

    def producer(self):
        B, R = self.bar, self.buf
        a_cnt = b_cnt = 0
        ok = True
        for it, nt in self.work():
            bs = b_cnt & 1
            ok = yield ("wait", B[f"b_empty{bs}"], self.bpar(b_cnt) ^ 1)
            if not ok:
                break
            B[f"b_full{bs}"].expect_tx(2)                     # the query block and its head weights

            def load_b(bs=bs, it=it, nt=nt):
                R[f"B{bs}"].write(it, nt + E)                 # read by nt MMAs and every epilogue warp
                B[f"b_full{bs}"].complete_tx(2)
            yield ("async", "tma", load_b)
            b_cnt += 1
            for _ in range(nt):
                s = a_cnt % NA
                if "no_a_empty_wait" not in self.mk:
                    ok = yield ("wait", B[f"a_empty{s}"], ((a_cnt // NA) & 1) ^ 1)
                    if not ok:
                        break
                B[f"a_full{s}"].expect_tx(1)

                def load_a(s=s, v=a_cnt):
                    R[f"A{s}"].write(v, 1)
                    B[f"a_full{s}"].complete_tx(1)
                yield ("async", "tma", load_a)
                a_cnt += 1
            if not ok:
                break
        if "no_tma_drain" not in self.mk:
            # drain, whether this warp gave up or not: the copies it issued land before it
            # leaves (bounded waits; after a normal run they have landed long ago)
            for i in range(max(0, a_cnt - NA), a_cnt):
                yield ("drain", B[f"a_full{i % NA}"], (i // NA) & 1)
            for i in range(max(0, b_cnt - 2), b_cnt):
                yield ("drain", B[f"b_full{i & 1}"], self.bpar(i))
        yield ("done",)

    def mma(self):
        B, R = self.bar, self.buf
        a_cnt = b_cnt = acc_cnt = 0
        ok = True
        for it, nt in self.work():
            bs = b_cnt & 1
            ok = yield ("wait", B[f"b_full{bs}"], self.bpar(b_cnt))
            if not ok:
                break
            for _ in range(nt):
                s, ab = a_cnt % NA, acc_cnt & 1
                ok = yield ("wait", B[f"a_full{s}"], (a_cnt // NA) & 1)
                if ok and "no_acc_empty_wait" not in self.mk:
                    ok = yield ("wait", B[f"acc_empty{ab}"], ((acc_cnt >> 1) & 1) ^ 1)
                if not ok:
                    break

                def run(s=s, ab=ab, va=a_cnt, vacc=acc_cnt, bs=bs, it=it):
                    R[f"A{s}"].read(va)
                    R[f"B{bs}"].read(it)
                    R[f"acc{ab}"].write(vacc, E)
                    B[f"a_empty{s}"].arrive()
                    B[f"acc_full{ab}"].arrive()
                yield ("async", "tc", run)
                a_cnt += 1
                acc_cnt += 1
            if not ok:
                break
            yield ("async", "tc", lambda bs=bs: B[f"b_empty{bs}"].arrive() if "b_empty_without_mma" not in self.mk
                   else None)
            b_cnt += 1
        if "no_mma_drain" not in self.mk:
            # drain, whether this warp gave up or not: a commit completes once every MMA issued
            # before it has finished (another role may have given up and left MMAs unconsumed)
            yield ("async", "tc", lambda: B["mma_drain"].arrive())
            yield ("drain", B["mma_drain"], 0)
        yield ("done",)

    def epilogue(self, w):
        B, R = self.bar, self.buf
        b_cnt = acc_cnt = 0
        for it, nt in self.work():
            bs = b_cnt & 1
            if not (yield ("wait", B[f"b_full{bs}"], self.bpar(b_cnt))):
                break
            R[f"B{bs}"].read(it)                               # head weights into registers
            ok = True
            for _ in range(nt):
                ab = acc_cnt & 1
                if "no_acc_full_wait" not in self.mk:
                    ok = yield ("wait", B[f"acc_full{ab}"], (acc_cnt >> 1) & 1)
                    if not ok:
                        break
                R[f"acc{ab}"].read(acc_cnt)
                yield ("step",)                                # loads complete, then the hand-back
                B[f"acc_empty{ab}"].arrive()
                acc_cnt += 1
            if not ok:
                break
            if "no_b_empty_arrive" not in self.mk:
                B[f"b_empty{bs}"].arrive()
            b_cnt += 1
        yield ("done",)

    def run(self, max_steps=500_000):
        actors = [[self.producer(), None], [self.mma(), None]] + [[self.epilogue(w), None] for w in range(E)]
        for a in actors:
            a[1] = next(a[0])
        self.steps = 0
        for step in range(max_steps):
            self.steps = step
            if self.abort_at is not None and step == self.abort_at:
                self.aborted = True                            # a bounded wait somewhere gave up
            # a wait is ready once its phase completed, or (after an abort) at once, failing; a
            # drain is a bounded wait: it may only succeed, the model requires it to complete
            ready = [("actor", i) for i, (_, op) in enumerate(actors)
                     if op[0] != "done" and not (op[0] == "wait" and not (self.aborted or op[1].ready(op[2])))
                     and not (op[0] == "drain" and not op[1].ready(op[2]))]
            if self.q["tc"]:
                ready.append(("async", "tc", 0))               # the tensor pipe runs in issue order
            ready += [("async", "tma", n) for n in range(len(self.q["tma"]))]
            if not ready:
                if all(op[0] == "done" for _, op in actors):
                    return
                raise Deadlock(str([(op[0], getattr(op[1], "name", "")) for _, op in actors if op[0] != "done"]))
            if all(op[0] == "done" for _, op in actors) and self.aborted:
                # every role has left after an abort: the CTA frees TMEM and exits now, so no
                # copy into shared memory and no MMA may still be in flight
                if self.q["tc"] or self.q["tma"]:
                    raise AssertionError(f"exit with {len(self.q['tc'])} MMA and {len(self.q['tma'])} copies in flight")
                return
            acts = [r for r in ready if r[0] == "actor"]
            if self.async_p is not None and acts and len(acts) < len(ready) and self.rng.random() >= self.async_p:
                ch = self.rng.choice(acts)
            else:
                ch = self.rng.choice(ready)
            if ch[0] == "async":
                self.q[ch[1]].pop(ch[2])()
                continue
            a = actors[ch[1]]
            op = a[1]
            if op[0] == "async":
                self.q[op[1]].append(op[2])
            res = None
            if op[0] == "wait":
                res = op[1].ready(op[2]) and not self.aborted
            elif op[0] == "drain":
                res = True
            a[1] = a[0].send(res)
        raise Deadlock("step limit")


PATTERNS = [[1], [2], [7], [13], [3, 3], [1, 0, 2, 0, 5], [0, 0, 4], [6, 6, 6, 6], [1, 1, 1, 1, 1], [9, 1, 8, 2],
            [0]]


def _run_all(mistakes=(), seeds=15):
    for items in PATTERNS:
        for s in range(seeds):
            Cta(items, seed=100 * len(items) + s, mistakes=mistakes).run()


@pytest.mark.parametrize("stages", [6, 4])
def test_protocol_completes_without_races(stages, monkeypatch):
    monkeypatch.setattr(sys.modules[__name__], "NA", stages, raising=True)
    _run_all(seeds=30)


# (Dropping the MMA's own arrival on b_empty would not be a mistake: the epilogue warps arrive
# only after reading the item's last accumulator, which the tensor pipe completes after every
# earlier MMA of the item has read the query block.  The model confirms that it stays safe.)
def test_b_empty_commit_is_redundant_but_harmless():
    _run_all(mistakes=("b_empty_without_mma",), seeds=5)


def _run_aborts(mistakes=(), seeds=10):
    for items in PATTERNS:
        for s in range(seeds):
            full = Cta(items, seed=100 * len(items) + s)
            full.run()                                 # how long the run takes without a timeout
            rng = random.Random(7 * s + len(items))
            Cta(items, seed=100 * len(items) + s, mistakes=mistakes,
                abort_at=rng.randrange(0, max(1, full.steps)), async_p=0.05).run()


@pytest.mark.parametrize("stages", [6, 4])
def test_abort_path_drains_every_copy_and_mma_before_exit(stages, monkeypatch):
    """A bounded wait gives up at a random point: every role leaves through its exit path, the
    producer's in-flight copies and the MMA warp's in-flight MMAs complete (bounded drain
    waits), and nothing is still writing shared memory or TMEM when the CTA frees TMEM."""
    monkeypatch.setattr(sys.modules[__name__], "NA", stages, raising=True)
    _run_aborts(seeds=60)


@pytest.mark.parametrize("mistake", ["no_mma_drain", "no_tma_drain"])
def test_abort_path_without_a_drain_is_caught(mistake):
    with pytest.raises(AssertionError):
        _run_aborts(mistakes=(mistake,), seeds=25)


@pytest.mark.parametrize("mistake", ["acc_empty_count", "b_parity", "no_a_empty_wait",
                                     "no_acc_empty_wait", "no_acc_full_wait", "no_b_empty_arrive"])
def test_planted_protocol_mistake_is_caught(mistake):
    with pytest.raises((AssertionError, Deadlock)):
        _run_all(mistakes=(mistake,))
