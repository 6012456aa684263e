"""A model of the few-token tensor-core kernel's barrier protocol
(`gemm_small_m_kernel`), run on the CPU under random interleavings, in the
same way as the tiled kernel's model (test_protocol_model.py).

What differs from the tiled kernel: a stage holds a chunk of `gpc` groups
(4 on 4-bit tiles, 2 on 8-bit ones) loaded by one set of copies, so both MMA
issuers wait on every stage, and the producer refills a stage once the last
group of each issuer in the chunk it held is done; the scale tables are
loaded once; the unpack either runs all 8 warps on every group (shared-memory
tiles, 64 tokens) or splits the groups between two warps per TMEM lane
quadrant by parity (tensor-memory tiles, 16 and 32 tokens); 4 epilogue warps.
"""
import os
import random
import re

import pytest

from .test_protocol_model import Bar, Violation, check

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mixed_precision_quantized_act_b200", "csrc", "gemm_small_m.cuh")


def kernel_constants():
    text = open(SRC).read()

    def num(pattern):
        m = re.search(pattern, text)
        assert m, pattern
        return int(m.group(1))

    c = {
        "kTBufs": num(r"constexpr int kTBufs = (\d+);"),
        "kAccBufs": num(r"constexpr int kAccBufs = (\d+);"),
        "kMaxStages": num(r"constexpr int kMaxStages = (\d+);"),
        "kGpc4": num(r"kGpc4 = (\d+), kGpc8 = \d+;"),
        "kGpc8": num(r"kGpc4 = \d+, kGpc8 = (\d+);"),
        "kChunkWBytes": num(r"constexpr int kChunkWBytes = (\d+);"),
        "kUnpackWarps": num(r"constexpr int kSmUnpackWarps = (\d+);"),
        "kRingDuo": num(r"kRingBytes = DUO \? (\d+) \* 1024") * 1024,
        "kRingTmem": num(r"kTmemW \? (\d+) \* 1024 : \d+ \* 1024\)") * 1024,
        "kRingSmem": num(r"kTmemW \? \d+ \* 1024 : (\d+) \* 1024\)") * 1024,
    }
    assert "static constexpr int kDone = kMaxStages;" in text
    assert "static constexpr bool kTmemW = MP <= 32;" in text
    assert "nst &= ~1;  // even" in text
    c["kDone"] = c["kMaxStages"]
    return c


def stages_for(c, MP, duo=False):
    ring = c["kRingDuo"] if duo else (c["kRingTmem"] if MP <= 32 else c["kRingSmem"])
    stage = c["kChunkWBytes"] + c["kGpc4"] * MP * 128
    return min(ring // stage, c["kMaxStages"]) & ~1


class SmallMModel:
    def __init__(self, ng, is4, MP, c, rng, nst=None, duo=False):
        self.ng, self.is4, self.MP, self.c, self.rng = ng, is4, MP, c, rng
        self.tmem = MP <= 32
        self.gpc = c["kGpc4"] if is4 else c["kGpc8"]
        self.nch = (ng + self.gpc - 1) // self.gpc
        self.nst = nst if nst is not None else stages_for(c, MP, duo)
        assert self.nst >= 1
        uw = c["kUnpackWarps"]
        self.full = [Bar(f"full[{s}]", 1) for s in range(c["kMaxStages"])]
        self.done = [Bar(f"done[{i}]", 1) for i in range(c["kDone"])]
        self.tfull = [Bar(f"tfull[{b}]", uw // 2 if self.tmem else uw) for b in range(c["kTBufs"])]
        self.accempty = [Bar(f"accempty[{a}]", 4) for a in range(c["kAccBufs"])]
        self.tabready = Bar("tabready", 1)
        self.stage = {}        # s -> [chunk, copies landed]
        self.copies = 3        # token box, weights, zero points (or W8 box): counted as one phase
        self.tbuf = {}         # b -> {warp: group}
        self.acc = {}
        self.mma_done = set()
        self.drained = {}
        self.tma = []
        self.mmaq = [[], []]

    def gstage(self, i):
        return (i // self.gpc) % self.nst

    def gphase(self, i):
        return ((i // self.gpc) // self.nst) & 1

    def load(self, ch):
        s = ch % self.nst
        if ch >= self.nst:
            prev = ch - self.nst
            groups = range(prev * self.gpc, min(prev * self.gpc + self.gpc, self.ng))
            check(all(g in self.mma_done for g in groups),
                  f"stage {s} refilled with chunk {ch} before every MMA of chunk {prev}")
        self.stage[s] = [ch, 0]
        self.full[s].arrive(expect_tx=self.copies)
        for _ in range(self.copies):
            def land(s=s, ch=ch):
                check(self.stage[s][0] == ch, f"copy of chunk {ch} landed in stage {s} holding {self.stage[s][0]}")
                self.stage[s][1] += 1
                self.full[s].complete_tx(1)
            self.tma.append(land)

    def producer(self):
        nst, nch, gpc, D = self.nst, self.nch, self.gpc, self.c["kDone"]
        issued = min(nch, nst)
        for ch in range(issued):
            self.load(ch)
        for ch in range(nst, nch):
            last = (ch - nst) * gpc + gpc - 1
            yield lambda: self.done[last % D].passed((last // D) & 1)
            yield lambda: self.done[(last - 1) % D].passed(((last - 1) // D) & 1)
            self.load(ch)

    def scale_table(self):
        self.tabready.arrive()
        return
        yield

    def issuer(self, who):
        T, A, D = self.c["kTBufs"], self.c["kAccBufs"], self.c["kDone"]
        for i in range(who, self.ng, 2):
            s, b, a = self.gstage(i), i % T, i % A
            yield lambda: self.full[s].passed(self.gphase(i))
            check(self.stage.get(s) == [i // self.gpc, self.copies],
                  f"issuer {who}: stage {s} holds {self.stage.get(s)} for group {i}")
            if self.is4:
                yield lambda: self.tfull[b].passed((i // T) & 1)
                parts = self.tbuf.get(b, {})
                want = self.c["kUnpackWarps"] // 2 if self.tmem else self.c["kUnpackWarps"]
                check(len([v for v in parts.values() if v == i]) == want,
                      f"issuer {who}: unpacked buffer {b} holds {parts} for group {i}")
            yield lambda: self.accempty[a].passed((i // A) & 1)
            if i >= A:
                check(len(self.drained.get(i - A, ())) == 4, f"accumulator {a} reused for group {i} before group {i - A} was drained")

            def mma(i=i, s=s, b=b, a=a):
                check(self.stage.get(s) == [i // self.gpc, self.copies], f"MMA of group {i}: stage {s} changed under it")
                if self.is4:
                    check(all(v == i for v in self.tbuf[b].values()), f"MMA of group {i}: buffer {b} changed under it")
                self.acc[a] = i
                self.mma_done.add(i)

            def commit(i=i):
                self.done[i % D].arrive()
            self.mmaq[who] += [mma, commit]

    def unpack(self, w):
        T, D = self.c["kTBufs"], self.c["kDone"]
        if self.tmem:
            h = w // 4  # warps 4..7 and 8..11: the two halves, alternate groups
            groups = range(h, self.ng, 2)
            key = w % 4  # the lane quadrant this warp writes
        else:
            groups = range(self.ng)
            key = w
        for i in groups:
            s, b = self.gstage(i), i % T
            yield lambda: self.full[s].passed(self.gphase(i))
            check(self.stage.get(s) == [i // self.gpc, self.copies], f"unpack {w}: stage {s} holds {self.stage.get(s)} for group {i}")
            if i >= T:
                ip = i - T
                yield lambda: self.done[ip % D].passed((ip // D) & 1)
                check(ip in self.mma_done, f"unpack {w}: buffer {b} rewritten before group {ip}'s MMAs")
            self.tbuf.setdefault(b, {})[key] = i
            self.tfull[b].arrive()

    def epilogue(self, e):
        A, D = self.c["kAccBufs"], self.c["kDone"]
        for bar in self.accempty:
            bar.arrive()
        yield lambda: self.tabready.passed(0)
        for i in range(self.ng):
            a = i % A
            yield lambda: self.done[i % D].passed((i // D) & 1)
            check(self.acc.get(a) == i, f"epilogue {e}: accumulator {a} holds {self.acc.get(a)} for group {i}")
            self.drained.setdefault(i, set()).add(e)
            self.accempty[a].arrive()

    def run(self):
        roles = [self.producer(), self.issuer(0), self.issuer(1)] + [self.epilogue(e) for e in range(4)]
        self.scale_table_gen = self.scale_table()
        roles.append(self.scale_table_gen)
        if self.is4:
            roles += [self.unpack(w) for w in range(self.c["kUnpackWarps"])]
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
        check(len(self.mma_done) == self.ng, "not every group ran")
        check(all(len(self.drained.get(i, ())) == 4 for i in range(self.ng)), "not every group drained")


@pytest.mark.parametrize("MP", [16, 32, 64])
@pytest.mark.parametrize("is4", [True, False], ids=["4bit", "8bit"])
@pytest.mark.parametrize("ng", [1, 2, 3, 5, 8, 13, 32])
def test_small_m_protocol_holds_under_random_interleavings(ng, is4, MP):
    c = kernel_constants()
    for seed in range(25):
        SmallMModel(ng, is4, MP, c, random.Random(seed * 100 + ng)).run()


@pytest.mark.parametrize("is4", [True, False], ids=["4bit", "8bit"])
@pytest.mark.parametrize("ng", [1, 2, 3, 5, 8, 13, 32])
def test_two_ctas_per_sm_form_of_16_tokens(ng, is4):
    """The 16-token form that shares an SM with a second CTA: its shallower
    ring (two stages) under the same protocol."""
    c = kernel_constants()
    assert stages_for(c, 16, duo=True) == 2
    for seed in range(25):
        SmallMModel(ng, is4, 16, c, random.Random(seed * 100 + ng), duo=True).run()


@pytest.mark.parametrize("nst", [1, 3, 5])
@pytest.mark.parametrize("is4", [True, False], ids=["4bit", "8bit"])
def test_odd_stage_counts_are_safe_with_whole_chunk_stages(nst, is4):
    """Unlike per-group stages (the tiled kernel), a chunk stage is waited on
    by both issuers in turn, and refilled only after both are past it: an odd
    ring is safe here.  (The kernel still rounds to even; this records that
    a 64-token ring could use 3 stages.)"""
    c = kernel_constants()
    for seed in range(40):
        SmallMModel(17, is4, 64, c, random.Random(seed), nst=nst).run()


def test_model_finds_a_refill_after_only_one_issuer():
    """Planted mistake: the producer waits for only the chunk's last group,
    not the other issuer's last one."""
    c = kernel_constants()

    class OneWait(SmallMModel):
        def producer(self):
            nst, nch, gpc, D = self.nst, self.nch, self.gpc, self.c["kDone"]
            for ch in range(min(nch, nst)):
                self.load(ch)
            for ch in range(nst, nch):
                last = (ch - nst) * gpc + gpc - 1
                yield lambda: self.done[last % D].passed((last // D) & 1)
                self.load(ch)

    found = 0
    for seed in range(200):
        try:
            OneWait(24, False, 16, c, random.Random(seed)).run()
        except Violation:
            found += 1
    assert found > 0
