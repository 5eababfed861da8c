"""A CPU model of the attention kernel's synchronisation (one CTA of csrc/attn_tc.cu).

This checks the kernel's ordering argument by execution rather than by reading.
The model follows the kernel's roles and waits as written there, and is kept in
step with it by hand:

* the load warp publishes lists into three slots, loads Q per item and one K and
  one V stage per step, and skips items whose list is empty (they never reach
  the consumers);
* the MMA issuer computes S = Q K^T into TMEM, then O += P V in two halves (keys
  0..63 once every softmax warp has written their weights, then keys 64..127),
  with commits to kempty, s_full, q_empty, vempty and o_full;
* four softmax warps read S, may rescale O (lazy maximum), and overwrite the
  first 64 columns of S with the packed bf16 weights P: the low half, then the
  high half.  At the end of an item they read O for the epilogue.

mbarriers are modelled with their phase parity: a wait for phase k passes once
phase k has completed.  Waiting on a barrier that has already completed phase
k + 1 is flagged, because the parity would then alias.  Asynchronous work is
also modelled.  Tensor copies complete in any order.  Tensor-core products
complete in issue order, and a commit arrives once every earlier product has
completed.  Every shared-memory stage and TMEM region carries a tag for what it
holds.  A product checks its operands' tags when it completes.  A thread access
or a copy into a region that an operation in flight reads or writes is a
hazard.  Random schedules of random item lists must finish without a deadlock
or a hazard.  Mistakes planted in the model must be caught.
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
        if self.done >= phase + 2:
            raise Hazard(f"{self.name}: waiting for phase {phase} after {self.done} completed")
        return self.done >= phase + 1


def s_regions(w):
    # S's columns in quadrant w: P's low half, P's high half, the rest of S
    return (f"Slo{w}", f"Shi{w}", f"Srest{w}")


class Cta:
    def __init__(self, items, rng, faults=()):
        """items: steps per item in take order (0 = an empty list, never published)."""
        self.items, self.rng, self.faults = list(items), rng, set(faults)
        b = {}
        for s in range(SLOTS):
            b[f"list_full{s}"] = Barrier(f"list_full{s}", 1)
            b[f"list_empty{s}"] = Barrier(f"list_empty{s}", LIST_CONSUMERS)
        for name in ("q_full", "q_empty", "kfull", "kempty", "vfull", "vempty", "s_full", "o_full"):
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
    def load_warp(self):
        b = self.b
        st = {"built": 0, "taken": 0, "ended": False}

        def publish():
            slot = st["built"] % SLOTS
            if st["built"] >= SLOTS and "no_list_empty_wait" not in self.faults:
                yield ("wait", b[f"list_empty{slot}"], st["built"] // SLOTS - 1)
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

        yield from publish()
        g = nq = 0
        k = 0
        while True:
            slot = k % SLOTS
            if self.slots[slot] is None:
                break
            self.hold("load", slot)
            item, n_steps = self.slots[slot]
            if nq > 0 and "no_q_empty_wait" not in self.faults:
                yield ("wait", b["q_empty"], nq - 1)
            self.issue_copy("Q", ("Q", item), b["q_full"])
            nq += 1
            for j in range(n_steps):
                if g > 0:
                    yield ("wait", b["kempty"], g - 1)
                self.issue_copy("K", ("K", g), b["kfull"])
                yield ("yield",)
                if j == 0 and not st["ended"]:
                    yield from publish()
                if g > 0 and "no_vempty_wait" not in self.faults:
                    yield ("wait", b["vempty"], g - 1)
                self.issue_copy("V", ("V", g), b["vfull"])
                g += 1
            self.holders[slot].discard("load")
            k += 1

    def mma_warp(self):
        b, n, k = self.b, 0, 0
        while True:
            slot = k % SLOTS
            yield ("wait", b[f"list_full{slot}"], k // SLOTS)
            if self.slots[slot] is None:
                break
            self.hold("mma", slot)
            item, n_steps = self.slots[slot]
            yield ("wait", b["q_full"], k)
            for j in range(n_steps):
                last = j == n_steps - 1
                yield ("wait", b["kfull"], n)
                self.issue_mma(["Q", "K"] + [r for w in range(N_SOFT) for r in s_regions(w)],
                               self._s_product(item, n))
                self.commit(b["kempty"])
                self.commit(b["s_full"])
                if last:
                    self.commit(b["q_empty"])
                if "pv_before_p_half" not in self.faults:
                    yield ("wait", b["p_half"], n)
                yield ("wait", b["vfull"], n)
                self.issue_mma(["V"] + [f"Slo{w}" for w in range(N_SOFT)] +
                               [f"O{w}" for w in range(N_SOFT)], self._pv(item, j, n, "lo"))
                if "no_p_full_wait" not in self.faults:
                    yield ("wait", b["p_full"], n)
                self.issue_mma(["V"] + [f"Shi{w}" for w in range(N_SOFT)] +
                               [f"O{w}" for w in range(N_SOFT)], self._pv(item, j, n, "hi"))
                self.commit(b["vempty"])
                if last:
                    self.commit(b["o_full"])
                n += 1
                yield ("yield",)
            self.release("mma", slot)
            k += 1

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
            yield ("wait", b[f"list_full{slot}"], k // SLOTS)
            if self.slots[slot] is None:
                break
            self.hold(f"soft{w}", slot)
            item, n_steps = self.slots[slot]
            for j in range(n_steps):
                yield ("wait", b["s_full"], n)
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
            if "no_o_full_wait" not in self.faults:
                yield ("wait", b["o_full"], k)
            self.thread_access(f"O{w}", ("O", item, n_steps - 1, "hi"))
            self.tag[f"O{w}"] = ("free",)
            if w == 0:
                self.consumed.append(item)
            self.release(f"soft{w}", slot)
            k += 1

    # ----------------------------------------------------------- schedule
    def run(self, max_events=500000):
        actors = [self.load_warp(), self.mma_warp()] + [self.softmax_warp(w) for w in range(N_SOFT)]
        state, live = [None] * len(actors), [True] * len(actors)
        for i, a in enumerate(actors):
            try:
                state[i] = next(a)
            except StopIteration:
                live[i] = False
        for _ in range(max_events):
            runnable = [i for i in range(len(actors)) if live[i] and
                        (state[i][0] != "wait" or state[i][1].ready(state[i][2]))]
            pending = bool(self.copies or self.mma)
            if not runnable and not pending:
                if any(live):
                    raise AssertionError("deadlock: " + ", ".join(
                        f"actor {i} on {state[i][1].name} phase {state[i][2]}"
                        for i in range(len(actors)) if live[i]))
                return
            if runnable and (not pending or self.rng.random() < 0.5):
                i = self.rng.choice(runnable)
                try:
                    state[i] = next(actors[i])
                except StopIteration:
                    live[i] = False
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


@pytest.mark.parametrize("fault", ["no_vempty_wait", "no_q_empty_wait", "no_list_empty_wait",
                                   "pv_before_p_half", "no_p_full_wait", "p_half_early",
                                   "no_o_full_wait"])
def test_planted_mistakes_are_caught(fault):
    """Each fault drops one wait or moves one arrival; some schedule must expose it."""
    caught = False
    for seed in range(300):
        rng = random.Random(seed)
        cta = Cta([rng.choice([1, 2, 3, 4]) for _ in range(6)], rng, faults={fault})
        try:
            cta.run()
        except AssertionError:   # a hazard, an aliased phase or a deadlock
            caught = True
            break
    assert caught, fault
