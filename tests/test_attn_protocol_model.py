"""A CPU model of the attention kernel's synchronisation (one CTA of csrc/attn_tc.cu).

This checks the kernel's ordering argument by execution rather than by reading.
The model follows the kernel's roles, waits, breaks and drains as written there,
and is kept in step with it by hand:

* the load warp publishes lists into three slots, loads Q per item and one K and
  one V stage per step, and skips items whose list is empty (they never reach
  the consumers); on its way out it waits for its last K, V and Q copies;
* the MMA issuer computes S = Q K^T into TMEM, then O += P V in two halves (keys
  0..63 once every softmax warp has written their weights, then keys 64..127),
  with commits to kempty, s_full, q_empty, vempty and o_full; on its way out it
  commits once more and waits for that commit, so every product has completed;
* four softmax warps read S, may rescale O (lazy maximum), and overwrite the
  first 64 columns of S with the packed bf16 weights P: the low half, then the
  high half.  At the end of an item they read O for the epilogue.

mbarriers wait on the parity of a phase, as the hardware does.  A wait for phase
k passes when the barrier's completed-phase count differs in parity from k.  It
is flagged when that answer differs from "phase k has completed": either k + 1
phases have already passed (the waiter would block), or it passes one phase
early.  Asynchronous work is also modelled.  Tensor copies complete in any
order.  Tensor-core products complete in issue order, and a commit arrives once
every earlier product has completed.

Every shared-memory stage and TMEM region carries a tag for what it holds.  A
product checks its operands' tags when it completes.  A thread access or a copy
into a region that an operation in flight reads or writes is a hazard.  So is
the CTA's exit (TMEM freed, shared memory released) with a copy or product
still in flight.  The abort path is modelled too.  A bounded wait that runs out
sets the CTA's abort flag and returns false.  A role whose wait is not yet
satisfied returns false once the flag is set.  The drains ignore the flag.
Random schedules, with and without a timeout injected at a random wait, must
finish without a deadlock or a hazard, and mistakes planted in the model must
be caught.
"""
import random

import pytest

SLOTS = 3
N_SOFT = 4
LIST_CONSUMERS = 1 + N_SOFT  # the MMA warp and the softmax warps release a slot


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


def s_regions(w):
    # S's columns in quadrant w: P's low half, P's high half, the rest of S
    return (f"Slo{w}", f"Shi{w}", f"Srest{w}")


class Cta:
    def __init__(self, items, rng, faults=(), timeout_at=None):
        """items: steps per item in take order (0 = an empty list, never published).
        timeout_at: (actor, n): the actor's n-th bounded wait runs out."""
        self.items, self.rng, self.faults = list(items), rng, set(faults)
        self.timeout_at = timeout_at
        self.abort = False
        b = {}
        for s in range(SLOTS):
            b[f"list_full{s}"] = Barrier(f"list_full{s}", 1)
            b[f"list_empty{s}"] = Barrier(f"list_empty{s}", LIST_CONSUMERS)
        for name in ("q_full", "q_empty", "kfull", "kempty", "vfull", "vempty", "s_full",
                     "o_full", "done"):
            b[name] = Barrier(name, 1)
        b["p_half"] = Barrier("p_half", N_SOFT)
        b["p_full"] = Barrier("p_full", N_SOFT)
        self.b = b
        self.slots = [None] * SLOTS
        self.holders = [set() for _ in range(SLOTS)]
        self.tag = {"Q": None, "K": None, "V": None}
        for w in range(N_SOFT):
            for r in s_regions(w):
                self.tag[r] = None
            self.tag[f"O{w}"] = ("free",)
        self.copies = []   # (region, tag, barrier)
        self.mma = []      # issue order: ("op", regions, on_complete) | ("commit", barrier)
        self.consumed = []

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

        ok = yield from publish()
        g = nq = gk = gv = 0   # steps, Q copies, K copies, V copies issued
        k = 0
        while ok:
            slot = k % SLOTS
            if self.slots[slot] is None:
                break
            self.hold("load", slot)
            item, n_steps = self.slots[slot]
            if nq > 0 and "no_q_empty_wait" not in self.faults:
                ok = yield ("wait", b["q_empty"], nq - 1)
                if not ok:
                    break
            self.issue_copy("Q", ("Q", item), b["q_full"])
            nq += 1
            for j in range(n_steps):
                if g > 0:
                    ok = yield ("wait", b["kempty"], g - 1)
                    if not ok:
                        break
                self.issue_copy("K", ("K", g), b["kfull"])
                gk = g + 1
                yield ("yield",)
                if j == 0 and not st["ended"]:
                    ok = yield from publish()
                    if not ok:
                        break
                if g > 0 and "no_vempty_wait" not in self.faults:
                    ok = yield ("wait", b["vempty"], g - 1)
                    if not ok:
                        break
                self.issue_copy("V", ("V", g), b["vfull"])
                gv = g + 1
                g += 1
            self.holders[slot].discard("load")
            k += 1
        # every copy issued lands before the CTA exits
        if "drain_by_steps" in self.faults:
            gk = gv = g
        if gk > 0:
            yield ("drain", b["kfull"], gk - 1)
        if gv > 0:
            yield ("drain", b["vfull"], gv - 1)
        if nq > 0:
            yield ("drain", b["q_full"], nq - 1)

    def mma_warp(self):
        b, n, k = self.b, 0, 0
        ok = True
        while ok:
            slot = k % SLOTS
            ok = yield ("wait", b[f"list_full{slot}"], k // SLOTS)
            if not ok or self.slots[slot] is None:
                break
            self.hold("mma", slot)
            item, n_steps = self.slots[slot]
            ok = yield ("wait", b["q_full"], k)
            if not ok:
                break
            for j in range(n_steps):
                last = j == n_steps - 1
                ok = yield ("wait", b["kfull"], n)
                if not ok:
                    break
                self.issue_mma(["Q", "K"] + [r for w in range(N_SOFT) for r in s_regions(w)],
                               self._s_product(item, n))
                self.commit(b["kempty"])
                self.commit(b["s_full"])
                if last:
                    self.commit(b["q_empty"])
                if "pv_before_p_half" not in self.faults:
                    ok = yield ("wait", b["p_half"], n)
                    if not ok:
                        break
                ok = yield ("wait", b["vfull"], n)
                if not ok:
                    break
                self.issue_mma(["V"] + [f"Slo{w}" for w in range(N_SOFT)] +
                               [f"O{w}" for w in range(N_SOFT)], self._pv(item, j, n, "lo"))
                if "no_p_full_wait" not in self.faults:
                    ok = yield ("wait", b["p_full"], n)
                    if not ok:
                        break
                self.issue_mma(["V"] + [f"Shi{w}" for w in range(N_SOFT)] +
                               [f"O{w}" for w in range(N_SOFT)], self._pv(item, j, n, "hi"))
                self.commit(b["vempty"])
                if last:
                    self.commit(b["o_full"])
                n += 1
                yield ("yield",)
            self.release("mma", slot)
            k += 1
        # every product issued completes before TMEM is released
        if "no_final_commit" not in self.faults:
            self.commit(b["done"])
            yield ("drain", b["done"], 0)

    def _s_product(self, item, n):
        def done():
            self.check("Q", ("Q", item))
            self.check("K", ("K", n))
            for w in range(N_SOFT):
                for r in s_regions(w):
                    self.tag[r] = ("S", n)
        return done

    def _pv(self, item, j, n, half):
        def done():
            self.check("V", ("V", n))
            for w in range(N_SOFT):
                self.check(f"S{half}{w}", ("P", n))
                if half == "hi":
                    prev = ("O", item, j, "lo")
                else:
                    prev = ("O", item, j - 1, "hi") if j > 0 else ("free",)
                self.check(f"O{w}", prev)
                self.tag[f"O{w}"] = ("O", item, j, half)
        return done

    def softmax_warp(self, w):
        b, n, k = self.b, 0, 0
        slo, shi, srest = s_regions(w)
        while True:
            slot = k % SLOTS
            ok = yield ("wait", b[f"list_full{slot}"], k // SLOTS)
            if not ok or self.slots[slot] is None:
                break
            self.hold(f"soft{w}", slot)
            item, n_steps = self.slots[slot]
            for j in range(n_steps):
                ok = yield ("wait", b["s_full"], n)
                if not ok:
                    break
                for r in (slo, shi, srest):
                    self.thread_access(r, ("S", n))
                yield ("yield",)
                if j > 0:   # a raised maximum rescales O
                    self.thread_access(f"O{w}", ("O", item, j - 1, "hi"))
                yield ("yield",)
                if "p_half_early" in self.faults:
                    b["p_half"].arrive()
                    yield ("yield",)
                self.thread_access(slo, None)
                self.tag[slo] = ("P", n)
                if "p_half_early" not in self.faults:
                    b["p_half"].arrive()
                yield ("yield",)
                self.thread_access(shi, None)
                self.tag[shi] = ("P", n)
                b["p_full"].arrive()
                n += 1
            if not ok:
                break
            if "no_o_full_wait" not in self.faults:
                ok = yield ("wait", b["o_full"], k)
                if not ok:
                    break
            self.thread_access(f"O{w}", ("O", item, n_steps - 1, "hi"))
            self.tag[f"O{w}"] = ("free",)
            if w == 0:
                self.consumed.append(item)
            self.release(f"soft{w}", slot)
            k += 1

    # ----------------------------------------------------------- schedule
    def run(self, max_events=500000):
        actors = [self.load_warp(), self.mma_warp()] + [self.softmax_warp(w) for w in range(N_SOFT)]
        n = len(actors)
        req, live, waits = [None] * n, [True] * n, [0] * n

        def resume(i, value):
            try:
                req[i] = actors[i].send(value) if req[i] is not None else next(actors[i])
            except StopIteration:
                live[i] = False

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
            if moves and (not pending or self.rng.random() < 0.5):
                i, value = self.rng.choice(moves)
                if req[i][0] == "wait":
                    waits[i] += 1
                if value == "timeout":
                    self.abort, value = True, False
                resume(i, value)
            else:
                self.step_async()
        raise AssertionError("did not finish")


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
    for name in ("kfull", "kempty", "vfull", "vempty", "s_full", "p_half", "p_full"):
        assert cta.b[name].done == steps, name
    for name in ("q_full", "q_empty", "o_full"):
        assert cta.b[name].done == len(kept), name
    assert all(cta.tag[f"O{w}"] == ("free",) for w in range(N_SOFT))


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
    cta = Cta(items, rng, timeout_at=(rng.randrange(2 + N_SOFT), rng.randrange(12)))
    cta.run()


@pytest.mark.parametrize("fault", ["no_vempty_wait", "no_q_empty_wait", "no_list_empty_wait",
                                   "pv_before_p_half", "no_p_full_wait", "p_half_early",
                                   "no_o_full_wait", "no_final_commit", "drain_by_steps"])
def test_planted_mistakes_are_caught(fault):
    """Each fault drops one wait, moves one arrival or shortens a drain (the last
    one counts the load warp's copies by completed steps); some schedule, with
    or without a timeout, must expose it."""
    caught = False
    for seed in range(600):
        rng = random.Random(seed)
        items = [rng.choice([1, 2, 3, 4]) for _ in range(6)]
        timeout = (rng.randrange(2 + N_SOFT), rng.randrange(12)) if seed % 2 else None
        cta = Cta(items, rng, faults={fault}, timeout_at=timeout)
        try:
            cta.run()
        except AssertionError:   # a hazard, an aliased phase or a deadlock
            caught = True
            break
    assert caught, fault
