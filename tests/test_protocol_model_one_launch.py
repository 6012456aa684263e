"""A model of the grid-wide hand-off of the tiled GEMM that quantizes X
itself (`gemm_w4w8a8_kernel<..., kFuseQ = true>`, mixllm_linear_one_launch),
run on the CPU under random interleavings (no GPU).

Per CTA the kernel does, in this order:
  * every thread quantizes the CTA's share of the (token, group) pairs; after
    a CTA barrier one thread (the first epilogue thread) adds the share's
    size to qcnt[0] (release);
  * the producer and the scale warp each wait until qcnt[0] equals the total
    (acquire) before their first A_q / s_a load -- unless the CTA has no
    tiles, when they load nothing and do not wait;
  * the epilogue drains the CTA's tiles, which needs both of those loads;
  * the same first epilogue thread then adds 1 to qcnt[1]; the CTA that
    makes it the grid size zeroes both counters.
The model interleaves these steps of all CTAs at random, runs two launches
in a row on the same counters, and checks that every wait ends, that no
waiter misses the full count (a reset before it looked would leave it
waiting for ever), and that both counters are zero after each launch.  The
source is checked to still publish and count done from the same thread and
to reset only on the last arrival; the last tests plant the mistakes those
choices avoid and expect the model to find them (or, for the publishing
thread, show exactly when it matters).
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mixed_precision_quantized_act_b200", "csrc", "gemm_w4w8a8.cuh")


class Deadlock(AssertionError):
    pass


class Launch:
    """One launch of `ctas` CTAs on the shared counters q = [pairs, done]."""

    def __init__(self, q, shares, tiles, rng, reset_first=False, publish_other_thread=False,
                 done_after_producer=False):
        self.q, self.shares, self.tiles, self.rng = q, shares, tiles, rng
        self.C = len(shares)
        self.total = sum(shares)
        self.reset_first = reset_first
        self.publish_other_thread = publish_other_thread
        self.done_after_producer = done_after_producer

    def cta(self, c):
        """The CTA's threads as coroutines; each `yield` is a point where other
        threads may run.  A wait yields until its condition holds."""
        st = {"quantized": False, "prod": False, "scale": False}
        q = self.q
        share, has_tiles = self.shares[c], self.tiles[c]

        def count_done():
            old = q[1]
            q[1] += 1
            if (self.reset_first and old == 0) or (not self.reset_first and old == self.C - 1):
                q[0] = 0
                q[1] = 0

        def publisher():  # the first epilogue thread: publish, later count the CTA done
            yield
            st["quantized"] = True
            if not self.publish_other_thread and share:
                q[0] += share
            # the epilogue's tiles need the producer's and the scale warp's loads
            while has_tiles and not (st["prod"] and st["scale"]):
                yield
            yield
            if not self.done_after_producer:
                count_done()

        def other_publisher():  # thread 0, in the planted mistake
            while not st["quantized"]:
                yield
            yield
            if share:
                q[0] += share

        def waiter(key):
            while not st["quantized"]:  # the CTA barrier after the quantization
                yield
            if has_tiles:
                while q[0] < self.total:
                    yield
                check_no_overshoot(q[0], self.total)
            st[key] = True
            if key == "prod" and self.done_after_producer:
                yield
                count_done()

        threads = [publisher(), waiter("prod"), waiter("scale")]
        if self.publish_other_thread:
            threads.append(other_publisher())
        return threads

    def run(self):
        live = [t for c in range(self.C) for t in self.cta(c)]
        idle = 0
        while live:
            t = self.rng.choice(live)
            before = tuple(self.q)
            try:
                next(t)
            except StopIteration:
                live.remove(t)
                idle = 0
                continue
            idle = idle + 1 if tuple(self.q) == before else 0
            if idle > 2000 * (len(live) + 1):
                raise Deadlock(f"no progress with {len(live)} threads waiting, counters {self.q}")


def check_no_overshoot(v, total):
    if v > total:
        raise AssertionError(f"count {v} above the total {total}")


def run_launches(C, seed, n=2, empty_ctas=0, **kw):
    rng = random.Random(seed)
    q = [0, 0]
    for _ in range(n):
        npairs = rng.randint(0, 6 * C)
        shares = [npairs * (c + 1) // C - npairs * c // C for c in range(C)]
        tiles = [c >= empty_ctas for c in range(C)]
        Launch(q, shares, tiles, rng, **kw).run()
        if q != [0, 0]:
            raise AssertionError(f"counters left at {q} after the launch")


def test_source_matches_the_model():
    text = open(SRC).read()
    # publication and the done count by the same thread, the reset on the last arrival only
    assert re.search(r"if \(threadIdx\.x == 128 && p1 > p0\) \{\s*__threadfence\(\);\s*red_release_gpu_u32\(qcnt,", text)
    assert "if (threadIdx.x == 128 && atom_add_acq_rel_gpu_u32(qcnt + 1, 1u) == gridDim.x - 1) {" in text
    # both waiters skip the wait when the CTA has nothing to load
    assert "if (first == 0) {" in text and "if (nsc > 0) {" in text


@pytest.mark.parametrize("C", [1, 2, 3, 8])
@pytest.mark.parametrize("empty", [0, 1])
def test_hand_off_holds_under_random_interleavings(C, empty):
    for seed in range(60):
        run_launches(C, seed * 31 + C, empty_ctas=min(empty, C - 1) if C > 1 else 0)


def _finds(C, runs=200, **kw):
    found = 0
    for seed in range(runs):
        try:
            run_launches(C, seed, **kw)
        except AssertionError:
            found += 1
    return found


def test_model_finds_a_reset_by_the_first_cta_to_finish():
    """Zeroing the counters when the first CTA finishes strands the waiters
    of CTAs that have not looked yet."""
    assert _finds(4, reset_first=True) > 0


def test_publishing_thread_matters_only_when_no_cta_waits():
    """With the pairs published by one thread and the CTA counted done by
    another, a CTA can be counted done before its publication lands.  While
    some CTA has tiles that cannot reach the reset (its waiters need every
    share first), so the kernel's choice of one thread for both is a second
    guard; with no CTA waiting, the late publication survives the reset and
    the model catches it."""
    assert _finds(3, publish_other_thread=True, empty_ctas=1) == 0
    assert _finds(3, publish_other_thread=True, empty_ctas=3) > 0


def test_model_finds_a_done_count_before_the_scale_warp_waited():
    """Counting the CTA done as soon as its producer has waited lets the last
    CTA zero the counter while another CTA's scale warp still waits on it."""
    assert _finds(4, done_after_producer=True) > 0
