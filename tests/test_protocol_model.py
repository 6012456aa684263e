"""A model of the tiled GEMM's barrier protocol, run on the CPU under random
interleavings (no GPU).

Every role of `gemm_w4w8a8_kernel` is a coroutine that waits on mbarriers the
way the kernel does: try_wait.parity P passes when the barrier's current
(incomplete) phase has the other parity, i.e. when "the phase of parity P"
has completed, which is also true when the waiter is a whole phase early.
TMA copies land in any order; the MMAs of one issuing thread complete in
issue order, and its commit arrives when they have.  The model checks, at
every step, what the kernel relies on:
  * a waiter that passes sees exactly the group it asked for, fully landed
    or completed (a parity wait that passes a phase early is caught here);
  * no buffer is overwritten (TMA, unpack, MMA, scale table) before every
    consumer of its previous group is done with it;
  * no phase receives more arrivals than its count;
  * the run never deadlocks.
The ring sizes are read from the kernel's source, so a change to them is
checked here; two tests plant known mistakes (the odd stage count of the
fault the kernel's history records: two issuers on alternate groups, 5
stages, 4 accumulators; and a done ring shallower than the stage ring) and
expect the model to find them.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mixed_precision_quantized_act_b200", "csrc", "gemm_w4w8a8.cuh")


def kernel_constants():
    text = open(SRC).read()

    def num(name):
        m = re.search(r"constexpr int %s = (\d+);" % name, text)
        assert m, name
        return int(m.group(1))

    c = {k: num(k) for k in ("kStages8", "kStagesA4", "kTBufs", "kRaw", "kAccBufs", "kTabSlots",
                             "kEpiWarps", "kXformWarps")}
    max_stages = max(c["kStages8"], c["kStagesA4"])
    assert "kDone = kMaxStages > kTBufs ? kMaxStages : kTBufs" in text
    c["kDone"] = max(max_stages, c["kTBufs"])
    return c


class Violation(AssertionError):
    pass


def check(ok, what):
    if not ok:
        raise Violation(what)


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        check(self.pending >= 0, f"{self.name}: more arrivals than its count in phase {self.phase}")
        self._complete()

    def complete_tx(self, n):
        self.tx -= n
        check(self.tx >= 0, f"{self.name}: more bytes than expected in phase {self.phase}")
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


class Model:
    """One CTA of the tiled kernel on one tile of `G` groups (or a run of
    `G` groups over several tiles: the rings do not care)."""

    def __init__(self, G, is4, c, rng):
        self.G, self.is4, self.rng = G, is4, rng
        self.S = c["kStagesA4"] if is4 else c["kStages8"]
        self.c = c
        n = c
        self.full = [Bar(f"full[{s}]", 1) for s in range(max(n["kStages8"], n["kStagesA4"]))]
        self.done = [Bar(f"done[{i}]", 1) for i in range(n["kDone"])]
        self.rfull = [Bar(f"rfull[{r}]", 1) for r in range(n["kRaw"])]
        self.rempty = [Bar(f"rempty[{r}]", n["kXformWarps"]) for r in range(n["kRaw"])]
        self.tfull = [Bar(f"tfull[{b}]", n["kXformWarps"]) for b in range(n["kTBufs"])]
        self.accempty = [Bar(f"accempty[{a}]", n["kEpiWarps"]) for a in range(n["kAccBufs"])]
        self.tabfull = [Bar(f"tabfull[{i}]", 1) for i in range(n["kTabSlots"])]
        self.tabempty = [Bar(f"tabempty[{i}]", n["kEpiWarps"]) for i in range(n["kTabSlots"])]
        # contents
        self.stage = {}          # s -> [group, boxes landed]
        self.boxes = 1 if is4 else 2
        self.raw = {}            # r -> [group, landed]
        self.tbuf = {}           # b -> {warp: group}
        self.acc = {}            # a -> [group, complete]
        self.table = {}          # slot -> group
        self.mma_done = set()    # groups whose MMAs completed
        self.unpacked = {}       # group -> warps that read its packed tile
        self.drained = {}        # group -> epilogue warps that read its accumulator and table slot
        self.tma = []            # in-flight copies (callables)
        self.mmaq = [[], []]     # per issuer, in issue order
        self.roles = []

    # ---------------------------------------------------------- copies
    def load_a(self, g):
        s = g % self.S
        if g >= self.S:
            check(g - self.S in self.mma_done, f"stage {s} refilled for group {g} before group {g - self.S}'s MMAs")
        self.stage[s] = [g, 0]
        self.full[s].arrive(expect_tx=self.boxes)
        for _ in range(self.boxes):  # A_q, and W8 on 8-bit tiles
            def land(s=s, g=g):
                check(self.stage[s][0] == g, f"copy of group {g} landed in stage {s} holding {self.stage[s][0]}")
                self.stage[s][1] += 1
                self.full[s].complete_tx(1)
            self.tma.append(land)

    def load_raw(self, g):
        r = g % self.c["kRaw"]
        if g >= self.c["kRaw"]:
            prev = g - self.c["kRaw"]
            check(len(self.unpacked.get(prev, ())) == self.c["kXformWarps"],
                  f"packed slot {r} refilled for group {g} before every unpack warp read group {prev}")
        self.raw[r] = [g, False]
        self.rfull[r].arrive(expect_tx=2)
        for _ in range(2):
            def land(r=r, g=g):
                check(self.raw[r][0] == g, f"packed copy of group {g} landed in slot {r} holding {self.raw[r][0]}")
                self.raw[r][1] = True
                self.rfull[r].complete_tx(1)
            self.tma.append(land)

    # ---------------------------------------------------------- roles
    def producer(self):
        G, S, R = self.G, self.S, self.c["kRaw"]
        for g in range(min(S, G)):
            self.load_a(g)
        ga, gw = min(S, G), (0 if self.is4 else G)
        while ga < G or gw < G:
            def ready():
                raw_ok = gw < G and (gw < R or self.rempty[gw % R].passed(((gw // R) - 1) & 1))
                a_ok = ga < G and self.done[(ga - S) % self.c["kDone"]].passed(((ga - S) // self.c["kDone"]) & 1)
                return raw_ok or a_ok
            yield ready
            if gw < G and (gw < R or self.rempty[gw % R].passed(((gw // R) - 1) & 1)):
                self.load_raw(gw)
                gw += 1
            if ga < G and self.done[(ga - S) % self.c["kDone"]].passed(((ga - S) // self.c["kDone"]) & 1):
                self.load_a(ga)
                ga += 1

    def issuer(self, who):
        G, S, T, A, D = self.G, self.S, self.c["kTBufs"], self.c["kAccBufs"], self.c["kDone"]
        for g in range(who, G, 2):
            s, b, a = g % S, g % T, g % A
            yield lambda: self.full[s].passed((g // S) & 1)
            check(self.stage.get(s) == [g, self.boxes], f"issuer {who}: stage {s} holds {self.stage.get(s)} for group {g}")
            if self.is4:
                yield lambda: self.tfull[b].passed((g // T) & 1)
                parts = self.tbuf.get(b, {})
                check(len(parts) == self.c["kXformWarps"] and all(v == g for v in parts.values()),
                      f"issuer {who}: unpacked buffer {b} holds {parts} for group {g}")
            yield lambda: self.accempty[a].passed((g // A) & 1)
            if g >= A:
                check(len(self.drained.get(g - A, ())) == self.c["kEpiWarps"],
                      f"accumulator {a} reused for group {g} before group {g - A} was drained")

            def mma(g=g, s=s, b=b, a=a):
                check(self.stage.get(s) == [g, self.boxes], f"MMA of group {g}: stage {s} changed under it")
                if self.is4:
                    check(all(v == g for v in self.tbuf[b].values()), f"MMA of group {g}: buffer {b} changed under it")
                self.acc[a] = [g, True]
                self.mma_done.add(g)

            def commit(g=g):
                self.done[g % D].arrive()
            self.mmaq[who] += [mma, commit]

    def unpack(self, w):
        G, R, T, D = self.G, self.c["kRaw"], self.c["kTBufs"], self.c["kDone"]
        for g in range(G):
            r, b = g % R, g % T
            yield lambda: self.rfull[r].passed((g // R) & 1)
            check(self.raw.get(r) == [g, True], f"unpack {w}: packed slot {r} holds {self.raw.get(r)} for group {g}")
            if g >= T:
                gp = g - T
                yield lambda: self.done[gp % D].passed((gp // D) & 1)
                check(gp in self.mma_done, f"unpack {w}: buffer {b} rewritten before group {gp}'s MMAs")
            self.unpacked.setdefault(g, set()).add(w)
            self.tbuf.setdefault(b, {})[w] = g
            self.rempty[r].arrive()
            self.tfull[b].arrive()

    def scale_table(self):
        G, TS = self.G, self.c["kTabSlots"]
        for g in range(G):
            slot = g % TS
            yield lambda: self.tabempty[slot].passed(((g // TS) & 1) ^ 1)
            if g >= TS:
                check(len(self.drained.get(g - TS, ())) == self.c["kEpiWarps"],
                      f"table slot {slot} rewritten for group {g} before every epilogue warp read group {g - TS}")
            self.table[slot] = g
            self.tabfull[slot].arrive()

    def epilogue(self, e):
        G, A, D, TS = self.G, self.c["kAccBufs"], self.c["kDone"], self.c["kTabSlots"]
        for bar in self.accempty:  # the bias fill of every accumulator
            bar.arrive()
        yield lambda: True
        for g in range(G):
            a, slot = g % A, g % TS
            yield lambda: self.done[g % D].passed((g // D) & 1)
            check(self.acc.get(a) == [g, True], f"epilogue {e}: accumulator {a} holds {self.acc.get(a)} for group {g}")
            yield lambda: self.tabfull[slot].passed((g // TS) & 1)
            check(self.table.get(slot) == g, f"epilogue {e}: table slot {slot} holds {self.table.get(slot)} for group {g}")
            self.drained.setdefault(g, set()).add(e)
            self.accempty[a].arrive()
            self.tabempty[slot].arrive()

    # ---------------------------------------------------------- scheduler
    def run(self):
        roles = [self.producer(), self.issuer(0), self.issuer(1), self.scale_table()]
        roles += [self.epilogue(e) for e in range(self.c["kEpiWarps"])]
        if self.is4:
            roles += [self.unpack(w) for w in range(self.c["kXformWarps"])]
        waiting = {}
        for r in roles:
            try:
                waiting[r] = next(r)
            except StopIteration:
                pass
        steps = 0
        while waiting or self.tma or self.mmaq[0] or self.mmaq[1]:
            steps += 1
            check(steps < 2_000_000, "no end")
            choices = [("role", r) for r, p in waiting.items() if p()]
            choices += [("tma", i) for i in range(len(self.tma))]
            choices += [("mma", q) for q in (0, 1) if self.mmaq[q]]
            check(choices, "deadlock: every role waits and nothing is in flight")
            kind, x = self.rng.choice(choices)
            if kind == "role":
                try:
                    waiting[x] = x.send(None)
                except StopIteration:
                    del waiting[x]
            elif kind == "tma":
                self.tma.pop(x)()
            else:
                self.mmaq[x].pop(0)()
        check(len(self.mma_done) == self.G, "not every group ran")
        check(all(len(self.drained.get(g, ())) == self.c["kEpiWarps"] for g in range(self.G)), "not every group drained")


@pytest.mark.parametrize("is4", [True, False], ids=["4bit", "8bit"])
@pytest.mark.parametrize("G", [1, 2, 3, 7, 32, 75])
def test_kernel_protocol_holds_under_random_interleavings(G, is4):
    c = kernel_constants()
    for seed in range(40 if G < 32 else 12):
        Model(G, is4, c, random.Random(seed * 1000 + G)).run()


def test_model_finds_the_odd_stage_fault():
    """Five stages with two issuers on alternate groups, as in the fault the
    kernel's history records (then with four accumulators): consecutive
    phases of one stage's barrier are waited by different issuers, and one of
    them can pass a phase early.  The model must find it.  (With two
    accumulators the in-order drain happens to keep the issuers close enough
    together to hide it, which is no reason to allow odd rings.)"""
    c = dict(kernel_constants(), kStages8=5, kAccBufs=4)
    c["kDone"] = max(5, c["kStagesA4"], c["kTBufs"], 4)
    found = 0
    for seed in range(200):
        try:
            Model(24, False, c, random.Random(seed)).run()
        except Violation:
            found += 1
    assert found > 0


def test_model_finds_a_short_done_ring():
    """A done ring shallower than the stage ring lets the producer's wait on a
    stage's last group alias a later phase."""
    c = dict(kernel_constants())
    c["kDone"] = 2
    found = 0
    for seed in range(200):
        try:
            Model(24, True, c, random.Random(seed)).run()
        except Violation:
            found += 1
    assert found > 0
