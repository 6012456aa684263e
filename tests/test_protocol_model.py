"""A model of the tiled GEMM's barrier protocol, run on the CPU under random
interleavings (no GPU).

Every role of `gemm_w4w8a8_kernel` is a coroutine that waits on mbarriers the
way the kernel does: try_wait.parity P passes when the barrier's current
(incomplete) phase has the other parity, i.e. when "the phase of parity P"
has completed, which is also true when the waiter is a whole phase early.
Copies land in any order; the MMAs of one issuing thread complete in issue
order, and its commit arrives when they have.  The CTA runs several tiles in
a row (the persistent schedule), each split into chunks of CH groups (the
last chunk of a tile may be shorter); a stage holds one chunk's A_q tiles
and weights and is refilled once the commits of the chunk's last two groups
-- one per issuer -- have arrived.  The model checks, at every step, what the
kernel relies on:
  * a waiter that passes sees exactly the chunk or group it asked for, fully
    landed or completed (a parity wait that passes a phase early is caught);
  * no buffer (stage, unpacked TMEM buffer, accumulator, scale-table slot) is
    overwritten before every consumer of its previous contents is done;
  * no phase receives more arrivals than its count;
  * the run never deadlocks.
The ring sizes are read from the kernel's source, so a change to them is
checked here; the last tests plant mistakes (a done ring shorter than a
stage's worth of groups, a stage released by its last group's commit alone,
a scale-table slot released after the first of its groups) and expect the
model to find them; and that the unpack's own wait for its buffer's previous
MMAs matters exactly when the unpacked buffers are fewer than the groups two
stages hold.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mixed_precision_quantized_act_b200", "csrc", "gemm_w4w8a8.cuh")


def kernel_constants():
    text = open(SRC).read()

    def num(pattern, name):
        m = re.search(pattern, text)
        assert m, name
        return int(m.group(1))

    c = {}
    m = re.search(r"constexpr int kC4 = (\d+), kC8 = (\d+);", text)
    assert m, "kC4 / kC8"
    c["kC4"], c["kC8"] = int(m.group(1)), int(m.group(2))
    m = re.search(r"constexpr int kTabG = (\d+), kTabSlots = (\d+);", text)
    assert m, "kTabG / kTabSlots"
    c["kTabG"], c["kTabSlots"] = int(m.group(1)), int(m.group(2))
    for k in ("kStages", "kTBufs", "kDone", "kXformWarps"):
        c[k] = num(r"constexpr int %s = (\d+);" % k, k)
    # accumulators: one count for 128-token tiles, another for 64-token ones
    m = re.search(r"constexpr int kAccBufs = BM == 128 \? (\d+) : (\d+);", text)
    assert m, "kAccBufs"
    c["kAccBufs"], c["kAccBufs64"] = int(m.group(1)), int(m.group(2))
    c["kEpiWarps"] = num(r"#define MIXLLM_EPI_WARPS (\d+)", "MIXLLM_EPI_WARPS")
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
    """One CTA of the tiled kernel running `tiles` tiles of `G` groups."""

    def __init__(self, G, tiles, is4, c, rng, release_last_only=False, table_early=False, unpack_no_wait=False):
        self.G, self.is4, self.rng, self.c = G, is4, rng, c
        self.CH = c["kC4"] if is4 else c["kC8"]
        self.S = c["kStages"]
        self.total = G * tiles
        self.release_last_only = release_last_only
        self.table_early = table_early
        self.unpack_no_wait = unpack_no_wait
        # chunks: (first running group, number of groups)
        self.chunks = []
        for t in range(tiles):
            for g0 in range(0, G, self.CH):
                self.chunks.append((t * G + g0, min(self.CH, G - g0)))
        self.chunk_of = {}
        for ci, (gi0, ng) in enumerate(self.chunks):
            for j in range(ng):
                self.chunk_of[gi0 + j] = ci
        self.full = [Bar(f"full[{s}]", 1) for s in range(self.S)]
        self.done = [Bar(f"done[{i}]", 1) for i in range(c["kDone"])]
        self.tfull = [Bar(f"tfull[{b}]", c["kXformWarps"]) for b in range(c["kTBufs"])]
        self.accempty = [Bar(f"accempty[{a}]", c["kEpiWarps"]) for a in range(c["kAccBufs"])]
        self.tabfull = [Bar(f"tabfull[{i}]", 1) for i in range(c["kTabSlots"])]
        self.tabempty = [Bar(f"tabempty[{i}]", c["kEpiWarps"]) for i in range(c["kTabSlots"])]
        self.copies = 3 if is4 else 2   # A_q box + (W4 bulk + zero-point box | W8 box)
        self.stage = {}                 # s -> [chunk, copies landed]
        self.tbuf = {}                  # b -> {warp: group}
        self.acc = {}                   # a -> group whose MMAs completed there
        self.table = {}                 # (slot, place) -> group
        self.mma_done = set()
        self.unpacked = {}              # group -> unpack warps that read its packed bytes
        self.drained = {}               # group -> epilogue warps that drained it
        self.inflight = []              # landing copies (callables)
        self.mmaq = [[], []]            # per issuer, in issue order

    # ---------------------------------------------------------- copies
    def load_chunk(self, ci):
        s = ci % self.S
        if ci >= self.S:
            gi0, ng = self.chunks[ci - self.S]
            for gi in range(gi0, gi0 + ng):
                check(gi in self.mma_done, f"stage {s} refilled with chunk {ci} before group {gi}'s MMAs")
                if self.is4:
                    check(len(self.unpacked.get(gi, ())) == self.c["kXformWarps"],
                          f"stage {s} refilled with chunk {ci} before every unpack warp read group {gi}")
        self.stage[s] = [ci, 0]
        self.full[s].arrive(expect_tx=self.copies)
        for _ in range(self.copies):
            def land(s=s, ci=ci):
                check(self.stage[s][0] == ci, f"copy of chunk {ci} landed in stage {s} holding {self.stage[s][0]}")
                self.stage[s][1] += 1
                self.full[s].complete_tx(1)
            self.inflight.append(land)

    # ---------------------------------------------------------- roles
    def producer(self):
        D = self.c["kDone"]
        n = len(self.chunks)
        for ci in range(min(self.S, n)):
            self.load_chunk(ci)
        for ci in range(self.S, n):
            gi0, ng = self.chunks[ci - self.S]
            gl = gi0 + ng - 1
            yield lambda gl=gl: self.done[gl % D].passed((gl // D) & 1)
            if ng > 1 and not self.release_last_only:
                yield lambda gl=gl: self.done[(gl - 1) % D].passed(((gl - 1) // D) & 1)
            self.load_chunk(ci)

    def issuer(self, who):
        S, T, A, D = self.S, self.c["kTBufs"], self.c["kAccBufs"], self.c["kDone"]
        for gi in range(who, self.total, 2):
            ci = self.chunk_of[gi]
            s, b, a = ci % S, gi % T, gi % A
            yield lambda: self.full[s].passed((ci // S) & 1)
            check(self.stage.get(s) == [ci, self.copies], f"issuer {who}: stage {s} holds {self.stage.get(s)} for chunk {ci}")
            if self.is4:
                yield lambda: self.tfull[b].passed((gi // T) & 1)
                parts = self.tbuf.get(b, {})
                check(len(parts) == self.c["kXformWarps"] and all(v == gi for v in parts.values()),
                      f"issuer {who}: unpacked buffer {b} holds {parts} for group {gi}")
            yield lambda: self.accempty[a].passed((gi // A) & 1)
            if gi >= A:
                check(len(self.drained.get(gi - A, ())) == self.c["kEpiWarps"],
                      f"accumulator {a} reused for group {gi} before group {gi - A} was drained")

            def mma(gi=gi, ci=ci, s=s, b=b, a=a):
                check(self.stage.get(s) == [ci, self.copies], f"MMA of group {gi}: stage {s} changed under it")
                if self.is4:
                    check(all(v == gi for v in self.tbuf[b].values()), f"MMA of group {gi}: buffer {b} changed under it")
                self.acc[a] = gi
                self.mma_done.add(gi)

            def commit(gi=gi):
                self.done[gi % D].arrive()
            self.mmaq[who] += [mma, commit]

    def unpack(self, w):
        S, T, D = self.S, self.c["kTBufs"], self.c["kDone"]
        for gi in range(self.total):
            ci = self.chunk_of[gi]
            s, b = ci % S, gi % T
            if gi == self.chunks[ci][0]:
                yield lambda: self.full[s].passed((ci // S) & 1)
            check(self.stage.get(s) == [ci, self.copies], f"unpack {w}: stage {s} holds {self.stage.get(s)} for chunk {ci}")
            if gi >= T:
                gp = gi - T
                if not self.unpack_no_wait:
                    yield lambda: self.done[gp % D].passed((gp // D) & 1)
                check(gp in self.mma_done, f"unpack {w}: buffer {b} rewritten before group {gp}'s MMAs")
            self.unpacked.setdefault(gi, set()).add(w)
            self.tbuf.setdefault(b, {})[w] = gi
            self.tfull[b].arrive()

    def scale_table(self):
        TG, TS = self.c["kTabG"], self.c["kTabSlots"]
        for gi in range(self.total):
            slot = (gi // TG) % TS
            if gi % TG == 0:
                yield lambda: self.tabempty[slot].passed(((gi // (TG * TS)) & 1) ^ 1)
                prev = gi - TG * TS
                for gp in range(max(prev, 0), max(prev + TG, 0)):
                    check(len(self.drained.get(gp, ())) == self.c["kEpiWarps"],
                          f"table slot {slot} rewritten for group {gi} before every epilogue warp read group {gp}")
            self.table[(slot, gi % TG)] = gi
            if gi % TG == TG - 1 or gi == self.total - 1:
                self.tabfull[slot].arrive()

    def epilogue(self, e):
        A, D, TG, TS = self.c["kAccBufs"], self.c["kDone"], self.c["kTabG"], self.c["kTabSlots"]
        for bar in self.accempty:  # the preset of every accumulator
            bar.arrive()
        yield lambda: True
        for gi in range(self.total):
            a, slot = gi % A, (gi // TG) % TS
            yield lambda: self.done[gi % D].passed((gi // D) & 1)
            check(self.acc.get(a) == gi, f"epilogue {e}: accumulator {a} holds {self.acc.get(a)} for group {gi}")
            if gi % TG == 0:
                yield lambda: self.tabfull[slot].passed((gi // (TG * TS)) & 1)
            check(self.table.get((slot, gi % TG)) == gi,
                  f"epilogue {e}: table entry {(slot, gi % TG)} holds {self.table.get((slot, gi % TG))} for group {gi}")
            self.drained.setdefault(gi, set()).add(e)
            release_at = 0 if self.table_early else TG - 1
            if gi % TG == release_at or gi == self.total - 1:
                self.tabempty[slot].arrive()
            self.accempty[a].arrive()

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
        while waiting or self.inflight or self.mmaq[0] or self.mmaq[1]:
            steps += 1
            check(steps < 3_000_000, "no end")
            choices = [("role", r) for r, p in waiting.items() if p()]
            choices += [("copy", i) for i in range(len(self.inflight))]
            choices += [("mma", q) for q in (0, 1) if self.mmaq[q]]
            check(choices, "deadlock: every role waits and nothing is in flight")
            kind, x = self.rng.choice(choices)
            if kind == "role":
                try:
                    waiting[x] = x.send(None)
                except StopIteration:
                    del waiting[x]
            elif kind == "copy":
                self.inflight.pop(x)()
            else:
                self.mmaq[x].pop(0)()
        check(len(self.mma_done) == self.total, "not every group ran")
        check(all(len(self.drained.get(g, ())) == self.c["kEpiWarps"] for g in range(self.total)),
              "not every group drained")


@pytest.mark.parametrize("bm", [128, 64], ids=["tile128", "tile64"])
@pytest.mark.parametrize("is4", [True, False], ids=["4bit", "8bit"])
@pytest.mark.parametrize("G,tiles", [(1, 3), (2, 2), (3, 2), (5, 3), (7, 1), (32, 1), (32, 2), (9, 4)])
def test_kernel_protocol_holds_under_random_interleavings(G, tiles, is4, bm):
    c = kernel_constants()
    if bm == 64:
        c = dict(c, kAccBufs=c["kAccBufs64"])
    for seed in range(30 if G * tiles < 32 else 8):
        Model(G, tiles, is4, c, random.Random(seed * 1000 + G * 10 + tiles)).run()


def _finds(c, is4, release_last_only=False, table_early=False, unpack_no_wait=False, runs=120):
    found = 0
    for seed in range(runs):
        try:
            Model(8, 3, is4, c, random.Random(seed), release_last_only, table_early, unpack_no_wait).run()
        except Violation:
            found += 1
    return found


def test_model_finds_a_short_done_ring():
    """A done ring shorter than a stage's worth of groups lets the producer's
    wait on a chunk's last group pass on an older phase of the same slot."""
    c = dict(kernel_constants(), kDone=2)
    assert _finds(c, True) > 0


def test_model_finds_a_stage_released_by_one_issuer():
    """Releasing a stage on the commit of its last group alone ignores the
    other issuer's MMAs on the same stage."""
    assert _finds(kernel_constants(), False, release_last_only=True) > 0


def test_model_finds_a_table_slot_released_early():
    """An epilogue warp that releases a scale-table slot after the first of
    its groups lets the scale warp rewrite entries not yet read."""
    assert _finds(kernel_constants(), True, table_early=True) > 0


def test_unpack_wait_matters_exactly_when_buffers_are_fewer_than_staged_groups():
    """The unpack's wait for the MMAs of its buffer's previous group is
    implied by the stage ring when kTBufs >= kStages * kC4 (the chunk it
    unpacks lands only after those MMAs) and needed otherwise: dropping it is
    caught then, and harmless with the larger buffer count."""
    c = kernel_constants()
    needed = c["kTBufs"] < c["kStages"] * c["kC4"]
    assert needed == (_finds(c, True, unpack_no_wait=True) > 0)
    big = dict(c, kTBufs=c["kStages"] * c["kC4"], kDone=max(c["kDone"], c["kStages"] * c["kC4"]))
    assert _finds(big, True, unpack_no_wait=True) == 0
