"""Model check of the MLA attention kernel's barrier protocol (CPU).

`sparse_mla_tc_kernel` (indexed_sparse_attention_fp8_b200/csrc/attn_tc.cu) coordinates, in
each CTA of a pair, the gather warps, the MMA-issuing warp, the 4 softmax warps (32 heads each,
with their own exchange barriers), the tensor pipe and the bulk copies into the partner CTA
through mbarriers only.  This model restates
that protocol operation by operation -- every wait (barrier and parity), arrival, expect-tx,
asynchronous completion (tensor-pipe FIFO, cp.async landings, bulk copies) -- and runs it
under random schedules.  It checks that
  * every role finishes (no deadlock) for many work-item patterns, including items without
    tiles, single-tile items and several items per CTA pair;
  * every buffer is read at the version its reader expects and is not overwritten before all
    readers of the previous version have read it: the key stages and their id slots, the S,
    P, O and q regions of TMEM, the staging and receive buffers of the score exchange.
Planted protocol mistakes (a wrong arrival count, a missing wait, an early remote arrival,
no re-arm of the exchange barrier) must each be caught.  The model checks the protocol, not
the kernel's arithmetic; the GPU parity tests check that.
"""
import random

import pytest

NS = 4           # key-tile stages
W = 4            # softmax warps


class Deadlock(Exception):
    pass


class Bar:
    """An mbarrier: arrival count per phase, transaction bytes, phase parity waits."""

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

    def ready(self, parity):        # try_wait.parity: the phase of that parity has completed
        return (self.phase & 1) != parity


class Buf:
    """A buffer version and the readers of that version still to come."""

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


class Pair:
    """One CTA pair serving `items` (key tiles per item) with cluster stride `grid`."""

    def __init__(self, items, grid, blk, seed, mistakes=(), abort_at=None, async_p=None):
        self.rng = random.Random(seed)
        # async_p: when roles and asynchronous completions are both ready, the chance that a
        # completion goes next (None: uniform over everything ready); small values keep copies
        # and MMAs in flight for longer, which is what an exit path must cope with
        self.async_p = async_p
        self.items, self.grid, self.blk, self.mk = items, grid, blk, set(mistakes)
        # abort_at: the scheduling step at which some bounded wait gives up (None: never); from
        # then on every wait fails and each role leaves through its exit path
        self.abort_at, self.aborted = abort_at, False
        self.asyncq = {}
        self.bulk_inflight = {}
        self.cta = [self._state(c) for c in range(2)]

    def _state(self, c):
        s_empty = 3 if "s_empty_count" in self.mk else W
        b = {"s_full": Bar(f"c{c}.s_full", 1), "s_empty": Bar(f"c{c}.s_empty", s_empty),
             "p_full": Bar(f"c{c}.p_full", W), "pv_done": Bar(f"c{c}.pv_done", 1),
             "q_ready": Bar(f"c{c}.q_ready", W), "mma_drain": Bar(f"c{c}.mma_drain", 1)}
        for st in range(NS):
            for n in ("kv_full", "kv_empty", "ids_ready"):
                b[f"{n}{st}"] = Bar(f"c{c}.{n}{st}", 1)   # kv_full: all gather threads' landings as one
        for w in range(W):
            b[f"x_full{w}"] = Bar(f"c{c}.x_full{w}", 1)
            b[f"x_free{w}"] = Bar(f"c{c}.x_free{w}", 1)
        r = {n: Buf(f"c{c}.{n}") for n in ["S"] + [f"kv{st}" for st in range(NS)] + [f"ids{st}" for st in range(NS)]
             + [f"{p}{w}" for p in ("P", "Q", "XS", "X") for w in range(W)]}
        return {"bar": b, "buf": r, "O": [dict(item=None, n=0, read=True) for _ in range(W)]}

    def mine(self):
        return list(range(self.blk, len(self.items), self.grid))

    # ------------------------------------------------------------------ roles
    def gather(self, c):
        B, R = self.cta[c]["bar"], self.cta[c]["buf"]
        g = 0
        ok = True
        for it in self.mine():
            for _ in range(self.items[it]):
                st = g % NS
                if "no_kv_empty_wait" not in self.mk:
                    ok = yield ("wait", B[f"kv_empty{st}"], ((g // NS) & 1) ^ 1)
                    if not ok:
                        break
                R[f"ids{st}"].write(g, W)
                B[f"ids_ready{st}"].arrive()

                def land(st=st, gg=g):
                    R[f"kv{st}"].write(gg, 2)              # read by S_g and by P_g.V_g
                    B[f"kv_full{st}"].arrive()
                yield ("async", f"cp{c}", land)
                g += 1
            if not ok:
                break
        if "no_cp_drain" not in self.mk:
            yield ("queue_empty", f"cp{c}")                # cp.async.wait_group 0: every copy landed
        yield ("done",)

    def mma(self, c):
        B, R, O = self.cta[c]["bar"], self.cta[c]["buf"], self.cta[c]["O"]

        def s_run(gg, item):
            st = gg % NS

            def run():
                R[f"kv{st}"].read(gg)
                for w in range(W):
                    R[f"Q{w}"].read(item)
                R["S"].write(gg, W)
                B["s_full"].arrive()
            return run

        def issue_s(gg, item):
            st = gg % NS
            if not (yield ("wait", B[f"kv_full{st}"], (gg // NS) & 1)):
                return False
            if not (yield ("wait", B["s_empty"], (gg & 1) ^ 1)):
                return False
            yield ("async", f"tc{c}", s_run(gg, item))
            return True

        def pv_run(gg, item, j):
            st = gg % NS

            def run():
                R[f"kv{st}"].read(gg)
                for w in range(W):
                    R[f"P{w}"].read(gg)
                    o = O[w]
                    if j == 0:
                        if not o["read"]:
                            raise AssertionError(f"c{c}.O{w}: item {item} accumulates before item {o['item']} was read")
                        o.update(item=item, n=1, read=False)
                    elif (o["item"], o["n"]) != (item, j):
                        raise AssertionError(f"c{c}.O{w}: P.V {j} of item {item} on {o}")
                    else:
                        o["n"] += 1
                B[f"kv_empty{st}"].arrive()
                B["pv_done"].arrive()
            return run

        def issue_pv(gg, item, j):
            if not (yield ("wait", B["p_full"], gg & 1)):
                return False
            yield ("async", f"tc{c}", pv_run(gg, item, j))
            return True

        g = nq = 0
        ok = True
        for it in self.mine():
            nt = self.items[it]
            if nt == 0:
                continue
            if "no_q_wait" not in self.mk:
                if not (yield ("wait", B["q_ready"], nq & 1)):
                    ok = False
                    break
            nq += 1
            ok = yield from issue_s(g, it)
            if ok and nt > 1:
                ok = yield from issue_s(g + 1, it)
            for j in range(nt):                        # S_{j+2} ahead of P_j.V_j
                if ok and j + 2 < nt:
                    ok = yield from issue_s(g + j + 2, it)
                if not ok:
                    break
                ok = yield from issue_pv(g + j, it, j)
            if not ok:
                break
            g += nt
        if "no_mma_drain" not in self.mk:
            # every MMA issued has finished before the TMEM is freed, whoever gave up
            yield ("async", f"tc{c}", lambda: B["mma_drain"].arrive())
            yield ("drain", B["mma_drain"], 0)
        yield ("done",)

    def softmax(self, c, w):
        B, R, O = self.cta[c]["bar"], self.cta[c]["buf"], self.cta[c]["O"]
        peer = self.cta[c ^ 1]

        def load_send(jj):
            if not (yield ("wait", B["s_full"], jj & 1)):
                return False
            R["S"].read(jj)
            B["s_empty"].arrive()
            if jj >= 1 and "no_stage_read_wait" not in self.mk:
                yield ("bulk_read", (c, w))
            R[f"XS{w}"].write(jj, 1)
            if "no_x_free_wait" not in self.mk:
                if not (yield ("wait", B[f"x_free{w}"], (jj & 1) ^ 1)):
                    return False
            self.bulk_inflight[(c, w)] = self.bulk_inflight.get((c, w), 0) + 1

            def copy():
                R[f"XS{w}"].read(jj)
                self.bulk_inflight[(c, w)] -= 1
                peer["buf"][f"X{w}"].write(jj, 1)
                peer["bar"][f"x_full{w}"].complete_tx(1)
            yield ("async", f"bulk{c}", copy)
            return True

        def part1(jj):
            st = jj % NS
            if not (yield ("wait", B[f"x_full{w}"], jj & 1)):
                return False
            if "early_x_free" in self.mk:
                peer["bar"][f"x_free{w}"].arrive()
                yield ("step",)
            R[f"X{w}"].read(jj)
            if "no_rearm" not in self.mk:
                B[f"x_full{w}"].expect_tx(1)
            if not (yield ("wait", B[f"ids_ready{st}"], (jj // NS) & 1)):
                return False
            R[f"ids{st}"].read(jj)
            if "early_x_free" not in self.mk:
                peer["bar"][f"x_free{w}"].arrive()
            return True

        def part2(jj, item, j):
            if jj >= 1 and "no_pv_wait" not in self.mk:
                if not (yield ("wait", B["pv_done"], (jj - 1) & 1)):
                    return False
            if j >= 1 and self.rng.random() < 0.3:     # the lazy O rescale: a TMEM read and write
                for _ in range(2):
                    o = O[w]
                    if (o["item"], o["n"]) != (item, j):
                        raise AssertionError(f"c{c}.O{w}: rescale at {item}/{j} on {o}")
                    yield ("step",)
            R[f"P{w}"].write(jj, 1)
            B["p_full"].arrive()
            return True

        def epilogue(item, nt, g_last, ok):
            if nt > 0 and ok:
                if "no_epilogue_wait" not in self.mk:
                    if not (yield ("wait", B["pv_done"], g_last & 1)):
                        return False
                o = O[w]
                if (o["item"], o["n"]) != (item, nt):
                    raise AssertionError(f"c{c}.O{w}: epilogue of {item} on {o}")
                o["read"] = True
            return ok

        B[f"x_full{w}"].expect_tx(1)                   # armed before the cluster sync
        yield ("cluster_sync",)
        g, prev = 0, None
        ok = True
        for it in self.mine() + [None]:
            real = it is not None and ok
            nt = self.items[it] if real else 0
            if nt > 0:                                 # the next query's q into TMEM first
                R[f"Q{w}"].write(it, nt)               # read by every S of the item
                B["q_ready"].arrive()
            if prev is not None:
                ok = yield from epilogue(prev[0], prev[1], g - 1, ok)
            if not real or not ok:
                break
            if nt > 0:
                g0 = g
                ok = yield from load_send(g0)
                j = 0
                while j < nt and ok:
                    if not (ok := (yield from part1(g0 + j))):
                        break
                    if j + 1 < nt and not (ok := (yield from load_send(g0 + j + 1))):
                        break
                    if not (ok := (yield from part2(g0 + j, it, j))):
                        break
                    if j + 1 >= nt:
                        break
                    if not (ok := (yield from part1(g0 + j + 1))):
                        break
                    if j + 2 < nt and not (ok := (yield from load_send(g0 + j + 2))):
                        break
                    if not (ok := (yield from part2(g0 + j + 1, it, j + 1))):
                        break
                    j += 2
                g += nt
            prev = (it, nt)
        if "no_bulk_drain" not in self.mk:
            yield ("bulk_all", (c, w))                 # cp.async.bulk.wait_group 0: own copies done
        yield ("done",)

    # ------------------------------------------------------------------ scheduler
    def run(self, max_steps=500_000):
        actors = []
        for c in range(2):
            actors += [[self.gather(c), None], [self.mma(c), None]] + [[self.softmax(c, w), None] for w in range(W)]
        for a in actors:
            a[1] = next(a[0])
        synced = False
        self.steps = 0
        for step in range(max_steps):
            self.steps = step
            if self.abort_at is not None and step == self.abort_at:
                self.aborted = True                    # a bounded wait somewhere gave up
            if not synced and sum(a[1][0] == "cluster_sync" for a in actors) == 2 * W:
                synced = True
            if self.aborted and all(op[0] == "done" for _, op in actors):
                # every role of both CTAs has left: the pair frees TMEM and exits now, so nothing
                # may still be landing in shared memory or running on the tensor pipe
                busy = {q: len(l) for q, l in self.asyncq.items() if l}
                if busy:
                    raise AssertionError(f"exit with work in flight: {busy}")
                return
            ready = []
            for i, (_, op) in enumerate(actors):
                k = op[0]
                if k == "done" or (k == "wait" and not (self.aborted or op[1].ready(op[2]))) \
                        or (k == "drain" and not op[1].ready(op[2])) or (k == "cluster_sync" and not synced) \
                        or (k in ("bulk_read", "bulk_all") and self.bulk_inflight.get(op[1], 0) > 0) \
                        or (k == "queue_empty" and self.asyncq.get(op[1])):
                    continue
                ready.append(("actor", i))
            for q, lst in self.asyncq.items():
                if q.startswith("tc"):
                    ready += [("async", q, 0)] if lst else []          # the tensor pipe runs in issue order
                else:
                    ready += [("async", q, n) for n in range(len(lst))]
            if not ready:
                if all(op[0] == "done" for _, op in actors):
                    return
                raise Deadlock(str([(op[0], getattr(op[1], "name", "")) for _, op in actors if op[0] != "done"]))
            acts = [r for r in ready if r[0] == "actor"]
            if self.async_p is not None and acts and len(acts) < len(ready) and self.rng.random() >= self.async_p:
                ch = self.rng.choice(acts)
            else:
                ch = self.rng.choice(ready)
            if ch[0] == "async":
                self.asyncq[ch[1]].pop(ch[2])()
                continue
            a = actors[ch[1]]
            op = a[1]
            if op[0] == "async":
                self.asyncq.setdefault(op[1], []).append(op[2])
            res = None
            if op[0] == "wait":
                res = op[1].ready(op[2]) and not self.aborted
            elif op[0] == "drain":
                res = True
            a[1] = a[0].send(res)
        raise Deadlock("step limit")


PATTERNS = [([1], 1), ([2], 1), ([3], 1), ([5], 1), ([16], 1), ([2, 3], 1), ([0, 2, 0, 1, 4], 1), ([1, 1, 1, 1], 1),
            ([0, 0, 3], 1), ([4, 4, 4, 4], 2), ([7, 0, 6, 1, 2, 9], 3), ([8, 8, 8], 1), ([0], 1)]


def _run_all(mistakes=(), seeds=12):
    for items, grid in PATTERNS:
        for s in range(seeds):
            Pair(items, grid, s % grid, seed=1000 * len(items) + s, mistakes=mistakes).run()


def test_protocol_completes_without_races():
    _run_all(seeds=25)


def _run_aborts(mistakes=(), seeds=8):
    for items, grid in PATTERNS:
        for s in range(seeds):
            seed = 1000 * len(items) + s
            full = Pair(items, grid, s % grid, seed=seed)
            full.run()                                 # how long the run takes without a timeout
            rng = random.Random(13 * s + len(items))
            Pair(items, grid, s % grid, seed=seed, mistakes=mistakes,
                 abort_at=rng.randrange(0, max(1, full.steps)), async_p=0.05).run()


def test_abort_path_drains_before_exit():
    """A bounded wait gives up at a random point: every role of both CTAs leaves through its exit
    path, and the gathers' copies, the MMAs and the bulk copies into the partner have all
    completed when the pair frees TMEM and exits."""
    _run_aborts(seeds=12)


@pytest.mark.parametrize("mistake", ["no_mma_drain", "no_cp_drain", "no_bulk_drain"])
def test_abort_path_without_a_drain_is_caught(mistake):
    with pytest.raises((AssertionError, Deadlock)):
        _run_aborts(mistakes=(mistake,), seeds=12)


@pytest.mark.parametrize("mistake", ["s_empty_count", "no_kv_empty_wait", "no_q_wait", "no_stage_read_wait",
                                     "no_x_free_wait", "early_x_free", "no_rearm", "no_pv_wait",
                                     "no_epilogue_wait"])
def test_planted_protocol_mistake_is_caught(mistake):
    with pytest.raises((AssertionError, Deadlock)):
        _run_all(mistakes=(mistake,))
