"""A model of the forward attention kernel's synchronisation, run under random
interleavings on the CPU.

The kernel (tile_sparse_video_b200/csrc/sparse_attn.cu, sparse_attn_kernel) has
per CTA: a K producer warp (which also loads Q), a V producer warp, an S issuer,
a PV issuer, and eight softmax warps (two warpgroups x four TMEM lane
quadrants) that also run the epilogue.  The tensor core and the TMA engine
complete their work asynchronously and arrive on mbarriers.  The softmax warps
of one quadrant hand the running reference max from tile to tile through a
two-slot shared-memory mailbox and a per-quadrant mbarrier, and may rescale O
when it moves.  This model replays that protocol (same barriers, arrival
counts, waits and per-item / per-tile structure; the rescale decision drawn at
random) and checks:

* no waiter proceeds on a barrier two or more phases beyond the one it waits for;
* a K or V ring slot, the S tile of a warpgroup, its P tile and Q are
  overwritten only after everything reading them has completed;
* a mailbox slot is read only once its tile has been published and is
  overwritten only after it has been read;
* O is rescaled only while no PV product is in flight, read by the epilogue only
  after the item's last PV, and restarted (first PV of an item) only after the
  previous epilogue has read it;
* the item of each step is handed out through two list slots: the K producer
  takes it (from the grid's work counter) and publishes it in slot t % 2
  (list_full), every other role reads it there, and the slot is rewritten only
  after all twelve roles released the item it held two items earlier
  (list_empty); a role must never read a stale or rewritten slot, and the end
  marker (-1) stops every role;
* the 256-thread group barriers match, and the run ends (no deadlock).

Planted mistakes (P written without waiting for the warpgroup's previous PV, S
issued without waiting for the warpgroup to have loaded its previous S, O
rescaled without waiting for the partner's PV, a list slot rewritten without
waiting for its readers) must be caught.
"""
import random

import pytest


class Violation(AssertionError):
    pass


class Model:
    def __init__(self, items, NSK=3, NSV=2, seed=0, plant=None):
        self.items, self.NSK, self.NSV = items, NSK, NSV
        self.plant = plant or set()
        self.rng = random.Random(seed)
        self.need, self.done, self.count = {}, {}, {}
        for b, n in [("q_full", 1), ("q_empty", 1), ("o_full", 1), ("o_empty", 8)]:
            self.need[b] = n
        for s in range(NSK):
            self.need[f"k_full{s}"] = 1
            self.need[f"k_empty{s}"] = 1
        for s in range(NSV):
            self.need[f"v_full{s}"] = 1
            self.need[f"v_empty{s}"] = 1
        for w in range(2):
            self.need[f"s_full{w}"] = 1
            self.need[f"s_empty{w}"] = 4
            self.need[f"p_full{w}"] = 4
            self.need[f"pv_done{w}"] = 1
        for q in range(4):
            self.need[f"dec{q}"] = 1
        for sl in range(2):
            self.need[f"list_full{sl}"] = 1
            self.need[f"list_empty{sl}"] = 12   # K, V, S issuer, PV issuer, 8 softmax warps
        for b in self.need:
            self.done[b] = 0
            self.count[b] = 0
        self.fifo = {"s": [], "pv": [], "tk": [], "tv": []}
        # hazard bookkeeping (global tile indices)
        self.s_done, self.pv_done_set, self.pv_issued = set(), set(), 0
        self.s_loaded = {}           # global tile -> quadrants that loaded S
        self.k_read_done, self.v_read_done = set(), set()
        self.mbox = {}               # (quadrant, slot) -> global tile published
        self.mbox_read = set()       # (quadrant, global tile) values consumed
        self.epi = {}                # item -> warps done with the epilogue
        self.item_first = []         # global index of each item's first tile
        self.slot = [None, None]     # item published in each list slot (-1: none left)
        self.released = {}           # item -> roles that released its list slot
        G = 0
        for nk in items:
            self.item_first.append(G)
            G += nk

    def arrive(self, b, n=1):
        self.count[b] += n
        assert self.count[b] <= self.need[b], (b, self.count[b])
        if self.count[b] == self.need[b]:
            self.count[b] = 0
            self.done[b] += 1

    def ready(self, b, k):
        return self.done[b] >= k + 1

    # ---------------------------------------------------------------- list slots
    def publish(self, t):
        """K producer: item t (or the end marker) into slot t % 2."""
        if t >= 2:
            if "list_early" not in self.plant:
                yield ("wait", f"list_empty{t & 1}", (t >> 1) - 1)
            if len(self.released.get(t - 2, ())) < 12:
                raise Violation(f"list slot {t & 1} rewritten with item {t} while item {t - 2} is still "
                                f"being read ({12 - len(self.released.get(t - 2, ()))} roles)")
        self.slot[t & 1] = t if t < len(self.items) else -1
        self.arrive(f"list_full{t & 1}")

    def read_slot(self, who, t):
        """A reader: wait for slot t % 2 and check that it holds item t."""
        yield ("wait", f"list_full{t & 1}", t >> 1)
        want = t if t < len(self.items) else -1
        if self.slot[t & 1] != want:
            raise Violation(f"{who} read item {self.slot[t & 1]} from slot {t & 1}, expected {want}")

    def release(self, who, t):
        self.released.setdefault(t, set()).add(who)
        self.arrive(f"list_empty{t & 1}")

    # ---------------------------------------------------------------- actors
    def k_producer(self):
        g = 0
        for t, nk in enumerate(self.items):
            yield from self.publish(t)
            if t > 0:
                yield ("wait", "q_empty", t - 1)
                first = self.item_first[t - 1]
                if not all(x in self.s_done for x in range(first, first + self.items[t - 1])):
                    raise Violation(f"Q of item {t} loaded while an S product of item {t - 1} is in flight")
            self.fifo["tk"].append(("q", t))
            for n in range(nk):
                s = g % self.NSK
                if g >= self.NSK:
                    yield ("wait", f"k_empty{s}", g // self.NSK - 1)
                    if (g - self.NSK) not in self.k_read_done:
                        raise Violation(f"K slot {s} refilled before the S product of tile {g - self.NSK} read it")
                self.fifo["tk"].append(("k", s, g))
                g += 1
            self.release("kp", t)
        yield from self.publish(len(self.items))

    def v_producer(self):
        g = 0
        for t, nk in enumerate(self.items + [None]):
            yield from self.read_slot("vp", t)
            if nk is None:
                return
            for n in range(nk):
                s = g % self.NSV
                if g >= self.NSV:
                    yield ("wait", f"v_empty{s}", g // self.NSV - 1)
                    if (g - self.NSV) not in self.v_read_done:
                        raise Violation(f"V slot {s} refilled before the PV product of tile {g - self.NSV} read it")
                self.fifo["tv"].append(("v", s, g))
                g += 1
            self.release("vp", t)

    def s_issuer(self):
        gk = 0
        si = [0, 0]
        last_of_w = [None, None]
        for t, nk in enumerate(self.items + [None]):
            yield from self.read_slot("si", t)
            if nk is None:
                return
            self.release("si", t)
            yield ("wait", "q_full", t)
            for n in range(nk):
                w = n & 1
                if si[w] > 0 and "s_issue_early" not in self.plant:
                    yield ("wait", f"s_empty{w}", si[w] - 1)
                prev = last_of_w[w]
                if prev is not None and len(self.s_loaded.get(prev, ())) < 4:
                    raise Violation(f"S of tile {gk} overwrites S tile {w} before tile {prev} was loaded")
                s = gk % self.NSK
                yield ("wait", f"k_full{s}", gk // self.NSK)
                self.fifo["s"].append((gk, w, s, n == nk - 1))
                last_of_w[w] = gk
                gk += 1
                si[w] += 1

    def pv_issuer(self):
        gv = 0
        pf = [0, 0]
        for t, nk in enumerate(self.items + [None]):
            yield from self.read_slot("pvi", t)
            if nk is None:
                return
            self.release("pvi", t)
            for n in range(nk):
                w = n & 1
                if n == 0 and t > 0:
                    yield ("wait", "o_empty", t - 1)
                    if len(self.epi.get(t - 1, ())) < 8:
                        raise Violation(f"first PV of item {t} before the epilogue of item {t - 1} read O")
                yield ("wait", f"p_full{w}", pf[w])
                pf[w] += 1
                sv = gv % self.NSV
                yield ("wait", f"v_full{sv}", gv // self.NSV)
                self.pv_issued += 1
                self.fifo["pv"].append((gv, w, sv, n == nk - 1))
                gv += 1

    def softmax_warp(self, wg, q):
        cw = 0
        cnt = [0, 0]
        for t, nk in enumerate(self.items + [None]):
            yield from self.read_slot(f"sm{wg}{q}", t)
            if nk is None:
                return
            G = self.item_first[t]
            yield ("bar",)
            yield ("bar",)
            for n in range(wg, nk, 2):
                Gn = G + n
                yield ("wait", f"s_full{wg}", cw)
                self.s_loaded.setdefault(Gn, set()).add(q)
                self.arrive(f"s_empty{wg}")
                if Gn > 0:
                    yield ("wait", f"dec{q}", Gn - 1)
                    if n > 0:
                        got = self.mbox.get((q, (Gn - 1) & 1))
                        if got != Gn - 1:
                            raise Violation(f"tile {Gn} read mailbox slot {(Gn - 1) & 1} holding tile {got}")
                        self.mbox_read.add((q, Gn - 1))
                rescale = n > 0 and self.rng.random() < 0.3
                if cw > 0:
                    if "p_early" not in self.plant:
                        yield ("wait", f"pv_done{wg}", cw - 1)
                    # the warpgroup's previous tile (maybe in an earlier item)
                    prev_tiles = [x for x in range(Gn - 1, -1, -1) if self.tile_wg(x) == wg]
                    if prev_tiles and prev_tiles[0] not in self.pv_done_set:
                        raise Violation(f"P of tile {Gn} written before the PV of tile {prev_tiles[0]} completed")
                # publish the decision
                old = self.mbox.get((q, Gn & 1))
                if old is not None and self.reads_mailbox(old + 1) and (q, old) not in self.mbox_read:
                    raise Violation(f"mailbox slot {Gn & 1} overwritten by tile {Gn} before tile {old}'s value was read")
                self.mbox[(q, Gn & 1)] = Gn
                self.arrive(f"dec{q}")
                if rescale:
                    idx = cnt[1 - wg] + ((n - 1) >> 1)
                    if "rescale_early" not in self.plant:
                        yield ("wait", f"pv_done{1 - wg}", idx)
                    if self.pv_issued != len(self.pv_done_set):
                        raise Violation(f"O rescaled at tile {Gn} while a PV product is in flight")
                    if (Gn - 1) not in self.pv_done_set and self.pv_issued >= Gn:
                        raise Violation(f"O rescaled at tile {Gn} before PV of tile {Gn - 1}")
                self.arrive(f"p_full{wg}")
                cw += 1
            yield ("wait", "o_full", t)
            first = self.item_first[t]
            if not all(x in self.pv_done_set for x in range(first, first + nk)):
                raise Violation(f"epilogue of item {t} before its last PV completed")
            cnt[0] += (nk + 1) // 2
            cnt[1] += nk // 2
            yield ("bar",)
            self.epi.setdefault(t, set()).add((wg, q))
            self.arrive("o_empty")
            self.release(f"sm{wg}{q}", t)

    def tile_wg(self, x):
        for t, first in enumerate(self.item_first):
            if first <= x < first + self.items[t]:
                return (x - first) & 1
        return None

    def reads_mailbox(self, x):
        """Tile x reads the mailbox unless it is the first tile of its item."""
        return x < sum(self.items) and x not in self.item_first

    # ---------------------------------------------------------------- engines
    def complete(self, e):
        op = self.fifo[e].pop(0)
        if e == "tk":
            if op[0] == "q":
                self.arrive("q_full")
            else:
                self.arrive(f"k_full{op[1]}")
        elif e == "tv":
            self.arrive(f"v_full{op[1]}")
        elif e == "s":
            g, w, s, last = op
            self.s_done.add(g)
            self.k_read_done.add(g)
            self.arrive(f"s_full{w}")
            self.arrive(f"k_empty{s}")
            if last:
                self.arrive("q_empty")
        else:
            g, w, sv, last = op
            self.pv_done_set.add(g)
            self.v_read_done.add(g)
            self.arrive(f"pv_done{w}")
            self.arrive(f"v_empty{sv}")
            if last:
                self.arrive("o_full")

    def run(self, max_steps=400000):
        actors = {"kp": self.k_producer(), "vp": self.v_producer(), "si": self.s_issuer(),
                  "pvi": self.pv_issuer()}
        for wg in range(2):
            for q in range(4):
                actors[f"sm{wg}{q}"] = self.softmax_warp(wg, q)
        sm = [n for n in actors if n.startswith("sm")]
        pending = {n: next(g, "end") for n, g in actors.items()}
        at_bar = set()
        for _ in range(max_steps):
            # the group barrier releases when all eight softmax warps are at it
            if len(at_bar) == len(sm):
                for n in sm:
                    pending[n] = next(actors[n], "end")
                at_bar.clear()
                continue
            choices = []
            for n, p in pending.items():
                if p == "end" or n in at_bar:
                    continue
                if p[0] == "bar":
                    choices.append(("bar", n))
                elif self.ready(p[1], p[2]):
                    choices.append(("actor", n))
            choices += [("engine", e) for e, f in self.fifo.items() if f]
            if not choices:
                if all(p == "end" for p in pending.values()):
                    return
                raise Violation(f"deadlock: { {n: p for n, p in pending.items() if p != 'end'} }")
            kind, n = self.rng.choice(choices)
            if kind == "engine":
                self.complete(n)
            elif kind == "bar":
                at_bar.add(n)
            else:
                p = pending[n]
                if self.done[p[1]] > p[2] + 1:
                    raise Violation(f"{n} waits for phase {p[2]} of {p[1]}, which has completed "
                                    f"{self.done[p[1]]} phases")
                pending[n] = next(actors[n], "end")
        raise Violation("step limit")


ITEM_MIXES = [
    [4, 4, 4],
    [1, 3, 1, 1, 2],          # single-tile items: the second warpgroup has no tile
    [7, 2, 5],
    [2, 1, 6, 1, 3],
]


@pytest.mark.parametrize("items", ITEM_MIXES, ids=["even", "short", "long", "mixed"])
@pytest.mark.parametrize("NSK,NSV", [(3, 2), (4, 4)], ids=["r128_rings", "r64_rings"])
def test_attention_protocol_holds_under_random_schedules(items, NSK, NSV):
    for seed in range(150):
        Model(items, NSK=NSK, NSV=NSV, seed=seed).run()


@pytest.mark.parametrize("plant", ["p_early", "s_issue_early", "rescale_early", "list_early"])
def test_planted_attention_mistakes_are_caught(plant):
    caught = 0
    for seed in range(150):
        try:
            Model([4, 3, 5], seed=seed, plant={plant}).run()
        except Violation:
            caught += 1
    assert caught > 0, plant
