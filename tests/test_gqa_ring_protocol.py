"""Protocol check of the GQA-family decode kernels' stage rings (race
detection without a GPU).

The GQA, GTA, fp8 GQA and MQA kernels (csrc/decode_gqa.cu,
csrc/decode_gqa_fp8.cu, csrc/decode_mqa_mma.cu) share one pipeline: a single
producer thread walks the part's pages, waits on a slot's `empty` barrier
before reusing it, writes the slot's skip flag (a page id out of range loads
nothing), and either arrives on `full` alone (skipped page) or arrives with
the expected transaction bytes and issues TMA loads that land later, in any
order.  Each consumer warp waits on `full` with the parity of the slot's use
count, reads the skip flag and the tile, and arrives on `empty`: the bf16
kernels after the page's MMAs (they read the tile throughout), the fp8 kernel
as soon as its bytes are in registers.  Tied pages (GTA) use twice as many
one-tile slots as the bf16 kernel has stages.  After the loop the stage ring
serves as scratch for the merge.

The model runs those agents under random interleavings (warps, the producer
and each TMA landing advance in any order) with the mbarrier phase rules and
checks that every agent finishes, that no parity wait aliases a later phase,
that no slot or skip flag is overwritten while a reader of the previous page
is pending, that every read sees the page it expects, and that no load is
in flight when the ring becomes merge scratch.  Planted mistakes must each
be caught.
"""

import random
import zlib

import pytest

CW = 4


class Bar:
    """mbarrier: `count` arrivals and the expected transaction units complete a phase."""

    def __init__(self, name, count):
        self.name, self.count, self.arrivals, self.tx, self.phase = name, count, 0, 0, 0

    def arrive(self, expect_tx=0):
        self.arrivals += 1
        self.tx += expect_tx
        self._complete()

    def complete_tx(self, units):
        self.tx -= units
        self._complete()

    def _complete(self):
        if self.arrivals == self.count and self.tx == 0:
            self.arrivals = 0
            self.phase += 1

    def done(self, k):
        assert self.phase <= k + 1, f"{self.name}: waiting on phase {k} but {self.phase} completed (aliasing)"
        return self.phase > k


class Ring:
    def __init__(self, n, nslots, early_release, bad, mistake=None, consumer_slots=None, empty_count=CW):
        self.n, self.nslots, self.early, self.bad, self.mistake = n, nslots, early_release, bad, mistake
        self.cslots = consumer_slots or nslots
        self.full = [Bar(f"full{s}", 1) for s in range(max(nslots, self.cslots))]
        self.empty = [Bar(f"empty{s}", empty_count) for s in range(max(nslots, self.cslots))]
        self.slot_page = [None] * len(self.full)     # page whose tile the slot holds (after landing)
        self.skip_page = [None] * len(self.full)     # page whose skip flag the slot holds
        self.skip_val = [None] * len(self.full)
        self.readers = [0] * len(self.full)          # consumers reading the tile now
        self.skip_reads = [CW] * len(self.full)      # consumers that read the current skip flag
        self.inflight = []                           # (slot, page) loads issued, not landed
        self.consumers_done = 0

    # ---------------------------------------------------------------- agents
    def producer(self):
        for i in range(self.n):
            st = i % self.nslots
            if i >= self.nslots and self.mistake != "no_empty_wait":
                k = i // self.nslots - 1
                yield lambda st=st, k=k: self.empty[st].done(k)
            assert self.skip_reads[st] == CW, f"skip flag of slot {st} rewritten before every warp read it"
            self.skip_page[st], self.skip_val[st], self.skip_reads[st] = i, i in self.bad, 0
            if i in self.bad:
                self.full[st].arrive()
                continue
            assert self.readers[st] == 0, f"slot {st} loaded while {self.readers[st]} warp(s) still read it"
            self.full[st].arrive(expect_tx=1)
            self.inflight.append((st, i))
            yield None

    def land(self):
        """One TMA load lands (any of those in flight)."""
        st, i = self.inflight.pop(self.rng.randrange(len(self.inflight)))
        assert self.readers[st] == 0, f"slot {st} written by a landing load while being read"
        self.slot_page[st] = i
        self.full[st].complete_tx(1)

    def consumer(self):
        for i in range(self.n):
            st = i % self.cslots
            k = i // self.cslots
            yield lambda st=st, k=k: self.full[st].done(k)
            if self.mistake == "release_before_read":
                self.empty[st].arrive()
                yield None
            assert self.skip_page[st] == i, f"warp read the skip flag of page {self.skip_page[st]} for page {i}"
            bad = self.skip_val[st]
            self.skip_reads[st] += 1
            if not bad:
                assert self.slot_page[st] == i, f"warp read page {self.slot_page[st]} for page {i}"
                self.readers[st] += 1
            if self.early:
                # the fp8 kernel: bytes in registers, then the warp frees the slot
                if not bad:
                    self.readers[st] -= 1
                yield None
                if self.mistake != "release_before_read":
                    self.empty[st].arrive()
                yield None                                   # the page's math, no shared-memory reads
            else:
                yield None                                   # the MMAs read the tile
                if not bad:
                    assert self.slot_page[st] == i, f"tile of page {i} replaced while its MMAs read it"
                    self.readers[st] -= 1
                if self.mistake != "release_before_read":
                    self.empty[st].arrive()
        self.consumers_done += 1
        if self.consumers_done == CW:
            assert not self.inflight, "ring used as merge scratch while a load is in flight"

    # ---------------------------------------------------------------- scheduler
    def run(self, rng):
        self.rng = rng
        agents = [self.producer()] + [self.consumer() for _ in range(CW)]
        waits = [None] * len(agents)
        live = list(range(len(agents)))
        steps = 0
        while live or self.inflight:
            ready = [a for a in live if waits[a] is None or waits[a]()]
            choices = ready + (["land"] if self.inflight else [])
            assert choices, "deadlock: every agent waits and no load is in flight"
            c = rng.choice(choices)
            if c == "land":
                self.land()
            else:
                try:
                    waits[c] = next(agents[c])
                except StopIteration:
                    live.remove(c)
            steps += 1
            assert steps < 100000, "no progress"


CONFIGS = {
    "gqa_bf16": dict(nslots=2, early_release=False),      # two 32 KB stages
    "gta_tied_slots": dict(nslots=4, early_release=False),  # four 16 KB one-tile slots
    "gqa_fp8": dict(nslots=4, early_release=True),         # four 16 KB stages, early release
    "mqa_bf16": dict(nslots=3, early_release=False),      # three 64 KB stages
}


def _cases(seed, count):
    rng = random.Random(seed)
    for _ in range(count):
        n = rng.choice([1, 2, 3, 5, 9, 17])
        bad = {i for i in range(n) if rng.random() < 0.15}
        yield n, bad, random.Random(rng.random())


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_ring_protocol_holds(name):
    for n, bad, rng in _cases(zlib.crc32(name.encode()), 300):
        Ring(n, bad=bad, **CONFIGS[name]).run(rng)


def _caught(make):
    for n, bad, rng in _cases(7, 300):
        try:
            make(n, bad).run(rng)
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_producer_without_empty_wait_is_caught(name):
    assert _caught(lambda n, bad: Ring(n, bad=bad, mistake="no_empty_wait", **CONFIGS[name]))


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_release_before_reading_is_caught(name):
    assert _caught(lambda n, bad: Ring(n, bad=bad, mistake="release_before_read", **CONFIGS[name]))


def test_tied_slots_read_with_the_stage_count_is_caught():
    """Producer on four one-tile slots, consumers still counting two stages."""
    assert _caught(lambda n, bad: Ring(n, bad=bad, nslots=4, early_release=False, consumer_slots=2))


def test_empty_barrier_expecting_an_extra_arrival_is_caught():
    assert _caught(lambda n, bad: Ring(n, bad=bad, nslots=2, early_release=False, empty_count=CW + 1))
