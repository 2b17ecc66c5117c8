"""A model of the attention-backward kernel's mbarrier protocol, run under
random interleavings on the CPU.

The kernel (tile_sparse_video_b200/csrc/backward.cu, attn_bwd_kernel) has four
kinds of actors per CTA: warp 8 (lists, TMA loads, the score-side products),
warp 9 (the accumulating products), and two elementwise warpgroups, which also
run the epilogue.  The tensor core and the TMA engine complete their work
asynchronously and arrive on mbarriers.  This model replays the protocol as
written in the kernel (same barriers, same arrival counts, same waits, the
same per-item and per-half-step structure) with every asynchronous completion
and every actor step scheduled in a random order, and checks:

* no waiter ever proceeds on a barrier that has completed two or more phases
  beyond the one it waits for (the parity test would then alias);
* a TMEM buffer is overwritten by new score products only after the
  accumulating products that read its bf16 P / dS have completed;
* a load stage is refilled only after every product reading it has completed;
* the accumulators are overwritten (first product of an item) only after the
  previous item's epilogue has read them;
* the item list is rewritten only after every actor has finished with it;
* the run ends (no deadlock).

Two planted copies of the protocol must be caught: the accumulating warp left
out of the per-item hand-off (the epilogue barrier counting 8 arrivals, as
before the fix), and score products issued into a buffer without waiting for
the accumulation that reads it.
"""
import random

import pytest


class Violation(AssertionError):
    pass


class Model:
    """One CTA; `items` is the list of per-item step counts it will take."""

    def __init__(self, items, HS=2, NS=2, acc_warp_joins=True, sd_waits_for_acc=True, seed=0):
        self.items, self.HS, self.NS = items, HS, NS
        self.acc_warp_joins = acc_warp_joins
        self.sd_waits_for_acc = sd_waits_for_acc
        self.rng = random.Random(seed)
        self.done = {}          # barrier -> completed phases
        self.count = {}         # barrier -> arrivals in the current phase
        self.need = {}          # barrier -> arrivals per phase
        self.fifo = {"sd": [], "acc": [], "tma": []}   # async completions, in order per engine
        # shared state for the hazard checks
        self.acc_complete = set()      # global half-steps whose accumulating products completed
        self.sd_complete = set()
        self.epi_done_items = set()    # items whose epilogue (both warpgroups) finished
        self.list_readers_done = {}    # item -> actors done with its list
        self.list_item = None
        for b, n in [("x_full", 1), ("list_full", 1), ("acc_full", 1),
                     ("epi_done", 9 if acc_warp_joins else 8)]:
            self.need[b] = n
        for s in range(NS):
            self.need[f"y_full{s}"] = 1
        for w in range(2):
            self.need[f"s_full{w}"] = 1
            self.need[f"p_ready{w}"] = 4      # four warps of the warpgroup
            self.need[f"acc_done{w}"] = 1
        for b in self.need:
            self.done[b] = 0
            self.count[b] = 0

    # -- barrier primitives ------------------------------------------------
    def arrive(self, b, n=1):
        self.count[b] += n
        assert self.count[b] <= self.need[b], (b, self.count[b])
        if self.count[b] == self.need[b]:
            self.count[b] = 0
            self.done[b] += 1

    def ready(self, b, k):
        return self.done[b] >= k + 1

    def proceed(self, who, b, k):
        if self.done[b] > k + 1:
            raise Violation(f"{who} waits for phase {k} of {b}, which has completed {self.done[b]} phases")

    # -- actors (generators yielding ("wait", barrier, phase) or None) -----
    def issuer(self):
        G = Gs = 0
        hw = [0, 0]
        xl = 0
        for t, cnt in enumerate(self.items + [None]):
            if t > 0:
                yield ("wait", "epi_done", t - 1)
            if cnt is None:
                self.list_item = -1
                self.arrive("list_full")
                return
            prev = t - 1
            if prev >= 0:
                readers = self.list_readers_done.get(prev, set())
                need = {"wg0", "wg1", "acc"}
                if not need <= readers:
                    raise Violation(f"list of item {t} written while {need - readers} still use item {prev}")
            self.list_item = t
            self.arrive("list_full")
            U = cnt * self.HS

            def load(n):
                self.fifo["tma"].append(("y", (Gs + n) % self.NS, Gs + n))

            def sd(v):
                n, c = divmod(v, self.HS)
                w = (G + v) & 1
                if v == 0:
                    yield ("wait", "x_full", xl - 1)
                if c == 0:
                    yield ("wait", f"y_full{(Gs + n) % self.NS}", (Gs + n) // self.NS)
                # buffer w last held half-step G+v-2: its accumulating products must be done
                if G + v >= 2 and (G + v - 2) not in self.acc_complete:
                    raise Violation(f"score products of half-step {G + v} overwrite buffer {w} "
                                    f"before the accumulation of {G + v - 2} completed")
                self.fifo["sd"].append(("sd", w, G + v))
            if cnt > 0:
                self.fifo["tma"].append(("x", None, t))
                xl += 1
                for n in range(min(cnt, self.NS)):
                    # the stage was last used by step Gs+n-NS: all its products must be done
                    self.check_stage(Gs + n - self.NS)
                    load(n)
                yield from sd(0)
                if U > 1:
                    yield from sd(1)
            for u in range(U):
                n, c = divmod(u, self.HS)
                w = (G + u) & 1
                idx = hw[w]
                hw[w] += 1
                if u + 2 < U:
                    if self.sd_waits_for_acc:
                        yield ("wait", f"acc_done{w}", idx)
                    if c == self.HS - 1 and n + self.NS < cnt:
                        self.check_stage(Gs + n)
                        load(n + self.NS)
                    yield from sd(u + 2)
            G += U
            Gs += cnt

    def check_stage(self, step):
        if step < 0:
            return
        for v in range(step * self.HS, (step + 1) * self.HS):
            if v not in self.acc_complete or v not in self.sd_complete:
                raise Violation(f"stage of step {step} refilled before half-step {v} finished with it")

    def acc_warp(self):
        G = 0
        hw = [0, 0]
        for t in range(len(self.items) + 1):
            yield ("wait", "list_full", t)
            if self.list_item == -1:
                return
            item = self.list_item
            cnt = self.items[item]
            U = cnt * self.HS
            for u in range(U):
                w = (G + u) & 1
                idx = hw[w]
                hw[w] += 1
                yield ("wait", f"p_ready{w}", idx)
                if u == 0 and item > 0 and (item - 1) not in self.epi_done_items:
                    raise Violation(f"accumulators of item {item} overwritten before the epilogue of {item - 1}")
                self.fifo["acc"].append(("acc", w, G + u, u == U - 1))
            self.list_readers_done.setdefault(item, set()).add("acc")
            G += U
            if self.acc_warp_joins:
                self.arrive("epi_done")

    def warpgroup(self, wg):
        G = Gs = mine = accs = 0
        for t in range(len(self.items) + 1):
            yield ("wait", "list_full", t)
            if self.list_item == -1:
                return
            item = self.list_item
            cnt = self.items[item]
            U = cnt * self.HS
            for u in range((wg - G) & 1, U, 2):
                n = u // self.HS
                yield ("wait", f"s_full{wg}", mine)
                mine += 1
                yield ("wait", f"y_full{(Gs + n) % self.NS}", (Gs + n) // self.NS)
                self.arrive(f"p_ready{wg}", 4)
            G += U
            Gs += cnt
            if cnt > 0:
                yield ("wait", "acc_full", accs)
                accs += 1
            self.list_readers_done.setdefault(item, set()).add(f"wg{wg}")
            done = self.list_readers_done[item]
            if {"wg0", "wg1"} <= done:
                self.epi_done_items.add(item)
            self.arrive("epi_done", 4)

    # -- asynchronous completions ------------------------------------------
    def complete(self, engine):
        op = self.fifo[engine].pop(0)
        if op[0] == "x":
            self.arrive("x_full")
        elif op[0] == "y":
            self.arrive(f"y_full{op[1]}")
        elif op[0] == "sd":
            self.sd_complete.add(op[2])
            self.arrive(f"s_full{op[1]}")
        elif op[0] == "acc":
            self.acc_complete.add(op[2])
            self.arrive(f"acc_done{op[1]}")
            if op[3]:
                self.arrive("acc_full")

    def run(self, max_steps=200000):
        actors = {"issuer": self.issuer(), "acc": self.acc_warp(), "wg0": self.warpgroup(0),
                  "wg1": self.warpgroup(1)}
        pending = {name: None for name in actors}
        for name, gen in actors.items():
            pending[name] = next(gen, "end")
        for _ in range(max_steps):
            choices = [("actor", n) for n, p in pending.items()
                       if p != "end" and (p is None or self.ready(p[1], p[2]))]
            choices += [("engine", e) for e, q in self.fifo.items() if q]
            if not choices:
                if all(p == "end" for p in pending.values()):
                    return
                raise Violation(f"deadlock: {pending}")
            kind, name = self.rng.choice(choices)
            if kind == "engine":
                self.complete(name)
                continue
            p = pending[name]
            if p is not None:
                self.proceed(name, p[1], p[2])
            pending[name] = next(actors[name], "end")
        raise Violation("step limit")


ITEM_MIXES = [
    [3, 2, 4],
    [1, 1, 1, 1],
    [0, 3, 0, 0, 2, 0, 1],     # items with no steps (a key tile nobody attends)
    [5, 0, 1, 7, 0, 2],
]


@pytest.mark.parametrize("HS,NS", [(2, 2), (1, 3)], ids=["r128", "r64"])
@pytest.mark.parametrize("items", ITEM_MIXES, ids=["plain", "one_step", "empty_items", "mixed"])
def test_protocol_holds_under_random_schedules(items, HS, NS):
    for seed in range(300):
        Model(items, HS=HS, NS=NS, seed=seed).run()


def test_planted_handoff_without_the_accumulating_warp_is_caught():
    """The epilogue barrier counting only the eight elementwise warps (the
    accumulating warp not in the per-item hand-off) lets the list be rewritten,
    or the list barrier run two phases ahead of that warp, on items with no
    steps: some schedule must expose it."""
    caught = 0
    for seed in range(300):
        try:
            Model([0, 3, 0, 0, 2, 0, 1], HS=2, NS=2, acc_warp_joins=False, seed=seed).run()
        except Violation:
            caught += 1
    assert caught > 0


def test_planted_early_score_products_are_caught():
    """Score products issued into a buffer without waiting for the accumulating
    products of its previous half-step (which read the bf16 P / dS stored in
    the same columns) must be caught."""
    caught = 0
    for seed in range(100):
        try:
            Model([4, 3, 5], HS=2, NS=2, sd_waits_for_acc=False, seed=seed).run()
        except Violation as e:
            caught += "overwrite buffer" in str(e) or "refilled" in str(e)
    assert caught > 0
