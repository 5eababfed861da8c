"""A CPU model of the attention kernel's synchronisation (one CTA of csrc/attn_tc.cu).

This checks the kernel's ordering argument by execution rather than by reading.
The model follows the kernel's roles, waits, breaks and drains as written there,
and is kept in step with it by hand:

* the load warp publishes lists into three slots, loads Q per item into one of
  two Q stages, and per step K into one of two K stages and then the previous
  step's V into one of two V stages (V runs one step behind K); it skips items
  whose list is empty (they never reach the consumers); on its way out it loads
  the last V and waits for the last copy into every stage;
* the MMA issuer computes S(n) = Q K(n)^T into TMEM buffer n % 2, then, for the
  previous step, O_g += P_g V for each of the two softmax groups once that
  group has written its weights, with commits to kempty, s_full, q_empty,
  pv_done, vempty and o_full; an item's last PV products are issued before
  the next item's first S product; the first product of an item waits until
  the epilogue of the item before has read O (o_empty); on its way out it
  commits once more and waits for that commit, so every product has completed;
* eight softmax warps, two groups of four (one warp per TMEM lane quadrant in
  each group): each reads its group's columns of S(n), sometimes rescales its
  group's O (a raised maximum; it first waits for its group's product of the
  previous step), and overwrites the first half of its columns with P.  At the
  end of an item every warp waits for o_full, writes its row maxima and sums to
  shared memory, meets the others at a barrier, reads the other group's values
  and reads both groups' O in its quadrant.

mbarriers wait on the parity of a phase, as the hardware does.  A wait for phase
k passes when the barrier's completed-phase count differs in parity from k.  It
is flagged when that answer differs from "phase k has completed": either k + 1
phases have already passed (the waiter would block), or it passes one phase
early.  Asynchronous work is also modelled.  Tensor copies complete in any
order.  Tensor-core products complete in issue order, and a commit arrives once
every earlier product has completed.

Every shared-memory stage, TMEM region and exchange slot carries a tag for what
it holds.  A product checks its operands' tags when it completes.  A thread
access or a copy into a region that an operation in flight reads or writes is a
hazard.  So is the CTA's exit (TMEM freed, shared memory released) with a copy
or product still in flight.  The abort path is modelled too.  A bounded wait
that runs out sets the CTA's abort flag and returns false.  A role whose wait is
not yet satisfied returns false once the flag is set.  The drains ignore the
flag.  Random schedules, with and without a timeout injected at a random wait,
must finish without a deadlock or a hazard, and mistakes planted in the model
must be caught.
"""
import random

import pytest

SLOTS = 3
GROUPS = 2
QUADS = 4
N_SOFT = GROUPS * QUADS
LIST_CONSUMERS = 1 + N_SOFT  # the MMA warp and the softmax warps release a slot
QS = KS = VS = 2             # Q, K and V stages


class Hazard(AssertionError):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.done = 0       # completed phases
        self.arrived = 0    # arrivals in the current phase
        self.pending_tx = 0

    def arrive(self):
        self.arrived += 1
        if self.arrived > self.count:
            raise Hazard(f"{self.name}: more arrivals than its count")
        self._maybe_complete()

    def expect_tx(self, n):
        self.pending_tx += n
        self.arrive()

    def tx_done(self, n):
        self.pending_tx -= n
        self._maybe_complete()

    def _maybe_complete(self):
        if self.arrived == self.count and self.pending_tx == 0:
            self.arrived = 0
            self.done += 1

    def ready(self, phase):
        intended = self.done >= phase + 1
        by_parity = (self.done & 1) != (phase & 1)
        if by_parity != intended:
            raise Hazard(f"{self.name}: the parity wait for phase {phase} "
                         f"{'passes' if by_parity else 'blocks'} after {self.done} phases")
        return intended


def s_regions(buf, g, w):
    # the columns of group g in lane quadrant w of S buffer `buf`: the half its
    # P is written over, and the rest
    return (f"SP{buf}{g}{w}", f"SR{buf}{g}{w}")


def all_s(buf):
    return [r for g in range(GROUPS) for w in range(QUADS) for r in s_regions(buf, g, w)]


class Cta:
    def __init__(self, items, rng, faults=(), timeout_at=None, raise_p=0.3, async_p=0.5):
        """items: steps per item in take order (0 = an empty list, never published).
        timeout_at: (actor, n): the actor's n-th bounded wait runs out.
        raise_p: chance that a softmax warp raises its maximum at a step > 0.
        async_p: chance that a copy or product progresses rather than a role
        (low values keep several copies in flight at once)."""
        self.items, self.rng, self.faults = list(items), rng, set(faults)
        self.timeout_at, self.raise_p, self.async_p = timeout_at, raise_p, async_p
        self.abort = False
        b = {}

        def bar(name, count=1):
            b[name] = Barrier(name, count)

        for s in range(SLOTS):
            bar(f"list_full{s}")
            bar(f"list_empty{s}", LIST_CONSUMERS)
        for s in range(QS):
            bar(f"q_full{s}"), bar(f"q_empty{s}")
        for s in range(KS):
            bar(f"kfull{s}"), bar(f"kempty{s}")
        for s in range(VS):
            bar(f"vfull{s}"), bar(f"vempty{s}")
        for buf in range(2):
            bar(f"s_full{buf}")
            for g in range(GROUPS):
                bar(f"p_ready{g}{buf}", QUADS)
                bar(f"pv_done{g}{buf}")
        bar("o_full"), bar("o_empty", N_SOFT), bar("xch", N_SOFT), bar("done")
        self.b = b
        self.slots = [None] * SLOTS
        self.holders = [set() for _ in range(SLOTS)]
        self.tag = {}
        for s in range(QS):
            self.tag[f"Q{s}"] = None
        for s in range(KS):
            self.tag[f"K{s}"] = None
        for s in range(VS):
            self.tag[f"V{s}"] = None
        for buf in range(2):
            for r in all_s(buf):
                self.tag[r] = None
        for g in range(GROUPS):
            for w in range(QUADS):
                self.tag[f"O{g}{w}"] = ("free",)
                self.tag[f"X{g}{w}"] = None
        self.o_readers = {}       # O region -> warps that read the item's result
        self.x_read = {}          # exchange slot -> whether its partner read it
        self.copies = []   # (region, tag, barrier)
        self.mma = []      # issue order: ("op", regions, on_complete) | ("commit", barrier)
        self.consumed = []
        self.raises = 0

    # ------------------------------------------------------------- memory
    def _touched_in_flight(self, region):
        return any(c[0] == region for c in self.copies) or any(
            op[0] == "op" and region in op[1] for op in self.mma)

    def thread_access(self, region, expect):
        if self._touched_in_flight(region):
            raise Hazard(f"thread access to {region} with an operation on it in flight")
        if expect is not None and self.tag[region] != expect:
            raise Hazard(f"{region} holds {self.tag[region]}, expected {expect}")

    def issue_copy(self, region, tag, bar):
        if self._touched_in_flight(region):
            raise Hazard(f"copy into {region} while an operation on it is in flight")
        self.tag[region] = ("writing",)
        bar.expect_tx(1)
        self.copies.append((region, tag, bar))

    def issue_mma(self, regions, on_complete):
        if any(c[0] in regions for c in self.copies):
            raise Hazard(f"product issued over a copy in flight into {regions}")
        self.mma.append(("op", tuple(regions), on_complete))

    def commit(self, bar):
        self.mma.append(("commit", bar))

    def check(self, region, expect):
        if self.tag[region] != expect:
            raise Hazard(f"product read {region} holding {self.tag[region]}, expected {expect}")

    def step_async(self):
        kinds = (["copy"] if self.copies else []) + (["mma"] if self.mma else [])
        if self.rng.choice(kinds) == "copy":
            region, tag, bar = self.copies.pop(self.rng.randrange(len(self.copies)))
            self.tag[region] = tag
            bar.tx_done(1)
        else:
            op = self.mma.pop(0)
            if op[0] == "commit":
                op[1].arrive()
            else:
                op[2]()

    # -------------------------------------------------------------- slots
    def hold(self, who, slot):
        self.holders[slot].add(who)

    def release(self, who, slot):
        self.holders[slot].discard(who)
        self.b[f"list_empty{slot}"].arrive()

    # -------------------------------------------------------------- roles
    # A role yields ("wait", barrier, phase) for a bounded wait and receives
    # True (passed) or False (gave up); ("drain", barrier, phase) for a wait
    # that ignores the abort flag; ("yield",) to let others run.
    def load_warp(self):
        b = self.b
        st = {"built": 0, "taken": 0, "ended": False}

        def publish():
            slot = st["built"] % SLOTS
            if st["built"] >= SLOTS and "no_list_empty_wait" not in self.faults:
                if not (yield ("wait", b[f"list_empty{slot}"], st["built"] // SLOTS - 1)):
                    return False
            if self.holders[slot]:
                raise Hazard(f"slot {slot} rewritten while {sorted(self.holders[slot])} read it")
            while st["taken"] < len(self.items) and self.items[st["taken"]] == 0:
                st["taken"] += 1   # an empty list: its output is written directly
            if st["taken"] < len(self.items):
                self.slots[slot] = (st["taken"], self.items[st["taken"]])
                st["taken"] += 1
            else:
                self.slots[slot] = None
                st["ended"] = True
            b[f"list_full{slot}"].arrive()
            st["built"] += 1
            return True

        cnt = {"q": 0, "k": 0, "v": 0, "v_pend": False}

        def load_v():
            if not cnt["v_pend"]:
                return True
            nv = cnt["v"]
            vs = nv % VS
            if nv >= VS and "no_vempty_wait" not in self.faults:
                if not (yield ("wait", b[f"vempty{vs}"], nv // VS - 1)):
                    return False
            self.issue_copy(f"V{vs}", ("V", nv), b[f"vfull{vs}"])
            cnt["v"] += 1
            cnt["v_pend"] = False
            return True

        ok = yield from publish()
        k = 0
        while ok:
            slot = k % SLOTS
            if self.slots[slot] is None:
                break
            self.hold("load", slot)
            item, n_steps = self.slots[slot]
            nq = cnt["q"]
            qs = nq % QS
            if nq >= QS and "no_q_empty_wait" not in self.faults:
                ok = yield ("wait", b[f"q_empty{qs}"], nq // QS - 1)
                if not ok:
                    break
            self.issue_copy(f"Q{qs}", ("Q", item), b[f"q_full{qs}"])
            cnt["q"] += 1
            for j in range(n_steps):
                nk = cnt["k"]
                ks = nk % KS
                if nk >= KS and "no_kempty_wait" not in self.faults:
                    ok = yield ("wait", b[f"kempty{ks}"], nk // KS - 1)
                    if not ok:
                        break
                self.issue_copy(f"K{ks}", ("K", nk), b[f"kfull{ks}"])
                cnt["k"] += 1
                yield ("yield",)
                ok = yield from load_v()
                if not ok:
                    break
                cnt["v_pend"] = True
                if j == 0 and not st["ended"]:
                    ok = yield from publish()
                    if not ok:
                        break
            self.holders[slot].discard("load")
            k += 1
        if ok:
            ok = yield from load_v()
        # the last copy into every stage lands before the CTA exits
        for name, n_copies, stages in (("kfull", cnt["k"], KS), ("vfull", cnt["v"], VS),
                                       ("q_full", cnt["q"], QS)):
            if "drain_last_only" in self.faults:
                if n_copies > 0:
                    c = n_copies - 1
                    yield ("drain", b[f"{name}{c % stages}"], c // stages)
                continue
            for s in range(stages):
                last = [c for c in range(n_copies) if c % stages == s]
                if last:
                    yield ("drain", b[f"{name}{s}"], last[-1] // stages)

    def mma_warp(self):
        b, n, t, k = self.b, 0, 0, 0
        ok = True
        pend = None   # (step, item, j, first, last) whose PV products are due

        def issue_pv(m, item, j, first, last):
            vs = m % VS
            ok = yield ("wait", b[f"vfull{vs}"], m // VS)
            if not ok:
                return False
            if first and item_index[item] > 0 and "no_o_empty_wait" not in self.faults:
                ok = yield ("wait", b["o_empty"], item_index[item] - 1)
                if not ok:
                    return False
            buf = m % 2
            for g in range(GROUPS):
                ok = yield ("wait", b[f"p_ready{g}{buf}"], m // 2)
                if not ok:
                    return False
                regions = [f"V{vs}"] + [s_regions(buf, g, w)[0] for w in range(QUADS)] + [
                    f"O{g}{w}" for w in range(QUADS)]
                self.issue_mma(regions, self._pv(g, m, item, j, first))
                self.commit(b[f"pv_done{g}{buf}"])
            self.commit(b[f"vempty{vs}"])
            if last:
                self.commit(b["o_full"])
            return True

        item_index = {}
        while ok:
            slot = k % SLOTS
            ok = yield ("wait", b[f"list_full{slot}"], k // SLOTS)
            if not ok:
                break
            hdr = self.slots[slot]
            self.release("mma", slot)   # the header is all this warp reads
            if hdr is None:
                break
            item, n_steps = hdr
            item_index[item] = t
            qs = t % QS
            ok = yield ("wait", b[f"q_full{qs}"], t // QS)
            if not ok:
                break
            for j in range(n_steps):
                ks = n % KS
                ok = yield ("wait", b[f"kfull{ks}"], n // KS)
                if not ok:
                    break
                buf = 0 if "single_s_buffer" in self.faults else n % 2
                self.issue_mma([f"Q{qs}", f"K{ks}"] + all_s(buf), self._s_product(item, n, qs, ks,
                                                                                  buf))
                self.commit(b[f"kempty{ks}"])
                self.commit(b[f"s_full{n % 2}"])
                if j == n_steps - 1:
                    self.commit(b[f"q_empty{qs}"])
                n += 1
                if pend is not None:
                    ok = yield from issue_pv(*pend)
                    if not ok:
                        break
                pend = (n - 1, item, j, j == 0, j == n_steps - 1)
                yield ("yield",)
            t += 1
            k += 1
            # the item's last products go out before the next item's first S
            if ok and pend is not None and "last_pv_deferred" not in self.faults:
                ok = yield from issue_pv(*pend)
                pend = None
        if ok and pend is not None:
            ok = yield from issue_pv(*pend)
        # every product issued completes before TMEM is released
        if "no_final_commit" not in self.faults:
            self.commit(b["done"])
            yield ("drain", b["done"], 0)

    def _s_product(self, item, n, qs, ks, buf):
        def done():
            self.check(f"Q{qs}", ("Q", item))
            self.check(f"K{ks}", ("K", n))
            for r in all_s(buf):
                self.tag[r] = ("S", n)
        return done

    def _pv(self, g, m, item, j, first):
        def done():
            self.check(f"V{m % VS}", ("V", m))
            for w in range(QUADS):
                self.check(s_regions(m % 2, g, w)[0], ("P", m))
                o = f"O{g}{w}"
                self.check(o, ("free",) if first else ("O", item, j - 1))
                self.tag[o] = ("O", item, j)
        return done

    def softmax_warp(self, g, w):
        b, n, k = self.b, 0, 0
        me = f"soft{g}{w}"
        o_own, x_own, x_oth = f"O{g}{w}", f"X{g}{w}", f"X{1 - g}{w}"
        xuses = 0
        while True:
            slot = k % SLOTS
            ok = yield ("wait", b[f"list_full{slot}"], k // SLOTS)
            if not ok or self.slots[slot] is None:
                break
            self.hold(me, slot)
            item, n_steps = self.slots[slot]
            for j in range(n_steps):
                buf = n % 2
                ok = yield ("wait", b[f"s_full{buf}"], n // 2)
                if not ok:
                    break
                sp, sr = s_regions(buf, g, w)
                for r in (sp, sr):
                    self.thread_access(r, ("S", n))
                yield ("yield",)
                if j > 0 and self.rng.random() < self.raise_p:
                    # a raised maximum: this group's product of step n - 1
                    # completes, then O is rescaled in place
                    self.raises += 1
                    if "no_pv_done_wait" not in self.faults:
                        pm = n if "pv_done_wrong_parity" in self.faults else n - 1
                        ok = yield ("wait", b[f"pv_done{g}{pm % 2}"], pm // 2)
                        if not ok:
                            break
                    self.thread_access(o_own, ("O", item, j - 1))
                    yield ("yield",)
                if "p_ready_early" in self.faults:
                    b[f"p_ready{g}{buf}"].arrive()
                    yield ("yield",)
                self.thread_access(sp, None)
                self.tag[sp] = ("P", n)
                if "p_ready_early" not in self.faults:
                    b[f"p_ready{g}{buf}"].arrive()
                n += 1
            if not ok:
                break
            # epilogue: both groups' products of the item have completed
            if "no_o_full_wait" not in self.faults:
                ok = yield ("wait", b["o_full"], k)
                if not ok:
                    break
            if self.tag[x_own] is not None and not self.x_read.get(x_own, False):
                raise Hazard(f"{x_own} rewritten before the other group read it")
            self.tag[x_own] = ("X", item)
            self.x_read[x_own] = False
            if "no_xch_sync" not in self.faults:
                b["xch"].arrive()
                ok = yield ("wait", b["xch"], xuses)
                xuses += 1
                if not ok:
                    break
            else:
                yield ("yield",)
            if self.tag[x_oth] != ("X", item):
                raise Hazard(f"{x_oth} holds {self.tag[x_oth]}, expected {('X', item)}")
            self.x_read[x_oth] = True
            for gg in range(GROUPS):
                o = f"O{gg}{w}"
                self.thread_access(o, ("O", item, n_steps - 1))
                yield ("yield",)
                readers = self.o_readers.setdefault(o, set())
                readers.add(me)
                if len(readers) == GROUPS:   # both groups' warps of this quadrant
                    self.tag[o] = ("free",)
                    readers.clear()
            b["o_empty"].arrive()
            if g == 0 and w == 0:
                self.consumed.append(item)
            self.release(me, slot)
            k += 1

    # ----------------------------------------------------------- schedule
    def actors(self):
        return [self.load_warp(), self.mma_warp()] + [
            self.softmax_warp(g, w) for g in range(GROUPS) for w in range(QUADS)]

    def run(self, max_events=800000):
        actors = self.actors()
        n = len(actors)
        req, live, waits = [None] * n, [True] * n, [0] * n

        def resume(i, value):
            try:
                req[i] = actors[i].send(value) if req[i] is not None else next(actors[i])
            except StopIteration:
                live[i] = False
                # the load warp's drain, not the other roles' pace, is what makes
                # its copies land before the CTA exits
                if i == 0 and self.copies:
                    raise Hazard("the load warp leaves with a copy in flight")

        for i in range(n):
            resume(i, None)
        for _ in range(max_events):
            moves = []
            for i in range(n):
                if not live[i]:
                    continue
                kind = req[i][0]
                if kind == "yield":
                    moves.append((i, None))
                elif kind == "drain":
                    if req[i][1].ready(req[i][2]):
                        moves.append((i, True))
                elif self.timeout_at == (i, waits[i]):
                    moves.append((i, "timeout"))
                elif req[i][1].ready(req[i][2]):
                    moves.append((i, True))
                elif self.abort:
                    moves.append((i, False))
            pending = bool(self.copies or self.mma)
            if not any(live):
                if pending:
                    raise Hazard("the CTA exits with a copy or product in flight")
                return
            if not moves and not pending:
                raise AssertionError("deadlock: " + ", ".join(
                    f"actor {i} on {req[i][1].name} phase {req[i][2]}"
                    for i in range(n) if live[i]))
            if moves and (not pending or self.rng.random() >= self.async_p):
                i, value = self.rng.choice(moves)
                if req[i][0] == "wait":
                    waits[i] += 1
                if value == "timeout":
                    self.abort, value = True, False
                resume(i, value)
            else:
                self.step_async()
        raise AssertionError("did not finish")


N_ACTORS = 2 + N_SOFT


def random_items(rng):
    return [rng.choice([0, 1, 1, 2, 3, 5, 8]) for _ in range(rng.randint(0, 10))]


@pytest.mark.parametrize("seed", range(60))
def test_protocol_finishes_without_hazard(seed):
    rng = random.Random(seed)
    items = random_items(rng)
    cta = Cta(items, rng)
    cta.run()
    kept = [i for i, s in enumerate(items) if s > 0]
    assert cta.consumed == kept
    steps = sum(items)
    per_stage = lambda stages, s: len([x for x in range(steps) if x % stages == s])
    for s in range(KS):
        assert cta.b[f"kfull{s}"].done == cta.b[f"kempty{s}"].done == per_stage(KS, s)
        assert cta.b[f"vfull{s}"].done == cta.b[f"vempty{s}"].done == per_stage(VS, s)
    for buf in range(2):
        assert cta.b[f"s_full{buf}"].done == per_stage(2, buf)
        for g in range(GROUPS):
            assert cta.b[f"p_ready{g}{buf}"].done == per_stage(2, buf)
            assert cta.b[f"pv_done{g}{buf}"].done == per_stage(2, buf)
    assert sum(cta.b[f"q_full{s}"].done for s in range(QS)) == len(kept)
    for name in ("o_full", "o_empty", "xch"):
        assert cta.b[name].done == len(kept), name
    assert all(cta.tag[f"O{g}{w}"] == ("free",) for g in range(GROUPS) for w in range(QUADS))


def test_raises_are_exercised():
    rng = random.Random(5)
    cta = Cta([8, 5, 3, 8], rng, raise_p=0.5)
    cta.run()
    assert cta.raises > 10


def test_no_items_and_only_empty_items():
    for items in ([], [0], [0, 0, 0, 0, 0]):
        cta = Cta(items, random.Random(0))
        cta.run()
        assert cta.consumed == []


@pytest.mark.parametrize("seed", range(200))
def test_a_timeout_anywhere_ends_every_role_with_nothing_in_flight(seed):
    """One bounded wait of one role runs out: every role leaves, the drains wait
    for what was issued, and the CTA exits with no copy or product in flight."""
    rng = random.Random(10_000 + seed)
    items = [rng.choice([1, 2, 3, 5]) for _ in range(rng.randint(1, 6))]
    cta = Cta(items, rng, timeout_at=(rng.randrange(N_ACTORS), rng.randrange(12)),
              async_p=0.5 if seed % 2 else 0.1)
    cta.run()


@pytest.mark.parametrize("fault", ["no_kempty_wait", "no_vempty_wait", "no_q_empty_wait",
                                   "no_list_empty_wait", "no_o_empty_wait", "no_pv_done_wait",
                                   "pv_done_wrong_parity", "p_ready_early", "no_o_full_wait",
                                   "no_xch_sync", "single_s_buffer", "no_final_commit",
                                   "drain_last_only"])
def test_planted_mistakes_are_caught(fault):
    """Each fault drops one wait, moves one arrival, waits on the wrong barrier,
    shares one S buffer between consecutive steps, or shortens a drain (the last
    one waits only for the very last copy, not the last into each stage); some
    schedule, with or without a timeout, must expose it."""
    caught = False
    for seed in range(600):
        rng = random.Random(seed)
        items = [rng.choice([1, 2, 3, 4]) for _ in range(6)]
        timeout = (rng.randrange(N_ACTORS), rng.randrange(12)) if seed % 2 else None
        cta = Cta(items, rng, faults={fault}, timeout_at=timeout,
                  async_p=0.5 if seed % 4 < 2 else 0.1)
        try:
            cta.run()
        except AssertionError:   # a hazard, an aliased phase or a deadlock
            caught = True
            break
    assert caught, fault
