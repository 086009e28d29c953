"""Protocol check of the MLA pair kernel (race detection without a GPU).

The MLA decode kernel (csrc/decode_mla_pair.cu) runs on a 2-CTA cluster.
Each CTA has a TMA producer, one MMA-issuing thread, an in-order tensor pipe
and the softmax warps, and the two CTAs talk through distributed shared
memory:
  * each page's row maxima (and at the end the row sums) go to the partner by
    st.async, counted on the partner's exchange barrier (xbar, one per page
    parity);
  * each CTA's probabilities P_j go into the partner's buffer pp[j & 1] by
    st.async once both CTAs' P.V of page j - 2 has completed (pv_done, a
    multicast tcgen05.commit that arrives on both CTAs), counted on the
    partner's pp_full[j & 1], which the partner's MMA thread armed before its
    own P.V of page j - 2.

This test models those agents for both CTAs with the kernel's issue
conditions and the mbarrier rules (phases, arrival counts, transaction
bytes that may land before the arm), delivers TMA copies and DSMEM stores in
any order, and checks under many random interleavings that
  * both CTAs finish (no deadlock) and nothing is still in flight at exit;
  * no parity wait can alias a later phase;
  * no transaction lands in a phase other than the one it belongs to;
  * every read (by an MMA or a softmax step) sees the page it expects, and no
    buffer is overwritten while an issued MMA that reads it is pending.
Planted mistakes must each be caught.
"""

import random

import pytest


class ProtocolError(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise ProtocolError(msg)


class Bar:
    """An mbarrier: `count` arrivals and zero outstanding transaction units
    complete a phase.  Units may land before the arrival that expects them
    (negative count), but never for another phase."""

    def __init__(self, name, count=1):
        self.name, self.count = name, count
        self.pending, self.tx, self.phase = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, expect=0):
        check(self.pending > 0, f"{self.name}: arrival beyond the phase's count (phase {self.phase})")
        self.tx += expect
        self.pending -= 1
        self._maybe_complete()

    def complete_tx(self, units, phase):
        check(phase == self.phase, f"{self.name}: transaction of phase {phase} landed in phase {self.phase}")
        self.tx -= units
        self._maybe_complete()

    def done(self, k):
        """Has phase k completed?  A parity wait cannot tell k from k + 2."""
        check(self.phase <= k + 1, f"{self.name}: waiting on phase {k} but {self.phase} completed (aliasing)")
        return self.phase > k


class Buffers:
    """Tagged buffers: a tag names the page (and kind) the buffer holds; None
    while a copy into it is in flight.  Issued MMAs register as readers."""

    def __init__(self):
        self.tag, self.readers = {}, {}

    def read(self, key, expect, who):
        check(self.tag.get(key) == expect, f"{who}: read {key} expecting {expect}, found {self.tag.get(key)}")

    def write(self, key, tag, who, ordered=False):
        """`ordered`: a write by the tensor pipe itself, which runs its MMAs in
        issue order, so MMAs still queued behind it are no hazard."""
        if not ordered:
            check(self.readers.get(key, 0) == 0,
                  f"{who}: {key} overwritten while {self.readers.get(key)} reader(s) pending")
        self.tag[key] = tag

    def hold(self, key):
        self.readers[key] = self.readers.get(key, 0) + 1

    def release(self, key):
        self.readers[key] -= 1


E_STAGES, V_STAGES = 2, 3


class Pair:
    """Both CTAs of one cluster decoding n pages."""

    def __init__(self, n, rng, rescale_rate=0.3):
        self.n, self.rng, self.rescale_rate = n, rng, rescale_rate
        self.buf = Buffers()
        self.bars = [self._make_bars(r) for r in range(2)]
        self.pipe = [[], []]        # in-order tensor pipe of each CTA
        self.flight = []            # TMA landings and DSMEM stores / remote arrivals in flight
        for r in range(2):
            self.buf.tag[(r, "O")] = ("O", -1)

    @staticmethod
    def _make_bars(r):
        b = {}
        for s in range(E_STAGES):
            b[f"e_full{s}"], b[f"e_empty{s}"] = Bar(f"{r}.e_full{s}"), Bar(f"{r}.e_empty{s}")
        for s in range(V_STAGES):
            b[f"v_full{s}"], b[f"v_empty{s}"] = Bar(f"{r}.v_full{s}"), Bar(f"{r}.v_empty{s}")
        for i in range(2):
            for name in ("s_full", "p_full", "pp_full", "xbar"):
                b[f"{name}{i}"] = Bar(f"{r}.{name}{i}")
            b[f"pv_done{i}"] = Bar(f"{r}.pv_done{i}", count=2)
        b["o_ready"], b["mma_done"] = Bar(f"{r}.o_ready"), Bar(f"{r}.mma_done")
        return b

    def bar(self, r, name):
        return self.bars[r][name]

    # ------------------------------------------------------------ actions
    def mma(self, r, reads, writes, who):
        for key, _ in reads:
            self.buf.hold(key)
        self.pipe[r].append(("mma", reads, writes, who))

    def commit(self, r, targets):
        self.pipe[r].append(("commit", targets))

    def pipe_step(self, r):
        op = self.pipe[r].pop(0)
        if op[0] == "mma":
            _, reads, writes, who = op
            for key, expect in reads:
                self.buf.read(key, expect, who)
                self.buf.release(key)
            for key, tag in writes:
                self.buf.write(key, tag, who, ordered=True)
        else:
            for c, name in op[1]:
                if c == r:
                    self.bar(c, name).arrive()
                else:                                   # multicast arrival on the other CTA
                    self.flight.append(lambda c=c, name=name: self.bar(c, name).arrive())

    def tma(self, r, kind, stage, page, barname, phase, who):
        key = (r, kind, stage)
        self.buf.write(key, None, who)                  # the copy starts overwriting the stage
        self.bar(r, barname).arrive(expect=1)

        def land():
            self.buf.write(key, (kind, page), "tma")
            self.bar(r, barname).complete_tx(1, phase)
        self.flight.append(land)

    def send(self, r, to, kind, idx, tag, barname, phase):
        key = (to, kind, idx)
        self.buf.write(key, None, f"{r}.softmax st.async")

        def land():
            self.buf.write(key, tag, "dsmem")
            self.bar(to, barname).complete_tx(1, phase)
        self.flight.append(land)

    # ------------------------------------------------------------- agents
    def producer(self, r):
        who = f"{r}.producer"
        for j in range(self.n):
            es, vs = j % E_STAGES, j % V_STAGES
            if j >= E_STAGES:
                while not self.bar(r, f"e_empty{es}").done(j // E_STAGES - 1):
                    yield
            self.tma(r, "E", es, j, f"e_full{es}", j // E_STAGES, who)
            yield
            if j >= V_STAGES:
                while not self.bar(r, f"v_empty{vs}").done(j // V_STAGES - 1):
                    yield
            self.tma(r, "V", vs, j, f"v_full{vs}", j // V_STAGES, who)
            yield

    def mma_thread(self, r):
        who = f"{r}.mma"
        n = self.n
        for t in range(min(2, n)):
            self.bar(r, f"pp_full{t}").arrive(expect=1)     # the partner's P of pages 0 and 1 may land
        for j in range(n + 1):
            if j < n:
                es, vs = j % E_STAGES, j % V_STAGES
                while not (self.bar(r, f"v_full{vs}").done(j // V_STAGES) and
                           self.bar(r, f"e_full{es}").done(j // E_STAGES)):
                    yield
                # zero the value rows past the context (generic stores into the V stage)
                self.buf.read((r, "V", vs), ("V", j), who)
                self.buf.write((r, "V", vs), ("V", j), who)
                self.mma(r, [((r, "E", es), ("E", j)), ((r, "V", vs), ("V", j))], [((r, "T", j & 1), ("S", j))],
                         f"{r}.S_{j}")
                self.commit(r, [(r, f"s_full{j & 1}")])
                self.commit(r, [(r, f"e_empty{es}")])
                yield
            if j >= 1:
                t = j - 1
                while not (self.bar(r, f"p_full{t & 1}").done(t >> 1) and self.bar(r, f"pp_full{t & 1}").done(t >> 1)):
                    yield
                if t + 2 < n:
                    self.bar(r, f"pp_full{t & 1}").arrive(expect=1)   # armed before this P.V can free the partner
                self.mma(r, [((r, "T", t & 1), ("P", t)), ((r, "pp", t & 1), ("P", t)),
                             ((r, "V", t % V_STAGES), ("V", t)), ((r, "O"), ("O", t - 1))],
                         [((r, "O"), ("O", t))], f"{r}.PV_{t}")
                self.commit(r, [(r, "o_ready")])
                self.commit(r, [(r, f"v_empty{t % V_STAGES}")])
                self.commit(r, [(0, f"pv_done{t & 1}"), (1, f"pv_done{t & 1}")])
                yield
        self.commit(r, [(r, "mma_done")])
        while not self.bar(r, "mma_done").done(0):
            yield
        for t in range(max(0, n - 2), n):
            while not self.bar(r, f"pv_done{t & 1}").done(t >> 1):
                yield

    def exchange(self, r, j, who):
        """This CTA's row value to the partner (st.async counted on its xbar),
        the local arrival, then the wait and the read of the partner's."""
        sb = j & 1
        self.send(r, 1 - r, "xch", sb, ("X", j), f"xbar{sb}", j >> 1)
        self.bar(r, f"xbar{sb}").arrive(expect=1)
        while not self.bar(r, f"xbar{sb}").done(j >> 1):
            yield
        self.buf.read((r, "xch", sb), ("X", j), who)

    def softmax(self, r):
        who = f"{r}.softmax"
        n = self.n
        for j in range(n):
            sb = j & 1
            while not self.bar(r, f"s_full{sb}").done(j >> 1):
                yield
            self.buf.read((r, "T", sb), ("S", j), who)
            yield from self.exchange(r, j, who)
            if j >= 2:
                while not self.bar(r, f"pv_done{sb}").done((j - 2) >> 1):
                    yield
            self.send(r, 1 - r, "pp", sb, ("P", j), f"pp_full{sb}", j >> 1)
            self.buf.write((r, "T", sb), ("P", j), who)
            if j >= 1 and self.rng.random() < self.rescale_rate:
                while not self.bar(r, "o_ready").done(j - 1):
                    yield
                self.buf.read((r, "O"), ("O", j - 1), who)
                self.buf.write((r, "O"), ("O", j - 1), who)
            self.bar(r, f"p_full{sb}").arrive()
            yield
        yield from self.exchange(r, n, who)             # the row sums
        if n:
            while not self.bar(r, "o_ready").done(n - 1):
                yield
            self.buf.read((r, "O"), ("O", n - 1), who)

    # ---------------------------------------------------------------- run
    def run(self, steps=400000):
        alive = [g for r in range(2) for g in (self.producer(r), self.mma_thread(r), self.softmax(r))]
        for _ in range(steps):
            choices = list(alive)
            choices += [("pipe", r) for r in range(2) if self.pipe[r]]
            if self.flight:
                choices.append(("flight",))
            if not choices:
                return
            pick = self.rng.choice(choices)
            if isinstance(pick, tuple) and pick[0] == "pipe":
                self.pipe_step(pick[1])
            elif isinstance(pick, tuple):
                self.flight.pop(self.rng.randrange(len(self.flight)))()
            else:
                try:
                    next(pick)
                except StopIteration:
                    alive.remove(pick)
                    if not alive:
                        # the final cluster barrier: nothing may still be headed for either CTA
                        check(not self.flight and not self.pipe[0] and not self.pipe[1],
                              f"exit with {len(self.flight)} transfer(s) in flight")
        raise ProtocolError(f"no progress: deadlock (n={self.n})")


def test_pair_protocol_random_interleavings():
    rng = random.Random(2024)
    for _ in range(400):
        Pair(rng.randint(0, 9), rng).run()


def _caught(cls, n, seed, needle, trials=200):
    rng = random.Random(seed)
    msgs = []
    for _ in range(trials):
        try:
            cls(n, rng).run()
        except ProtocolError as e:
            msgs.append(str(e))
    return any(needle in m for m in msgs), msgs[:3]


class _NoPvDoneWait(Pair):
    """The P store into the partner's buffer without the pv_done wait; with
    `early` also before this page's maximum exchange."""
    early = False

    def softmax(self, r):
        who = f"{r}.softmax"
        for j in range(self.n):
            sb = j & 1
            while not self.bar(r, f"s_full{sb}").done(j >> 1):
                yield
            self.buf.read((r, "T", sb), ("S", j), who)
            if self.early:
                self.send(r, 1 - r, "pp", sb, ("P", j), f"pp_full{sb}", j >> 1)
            yield from self.exchange(r, j, who)
            if not self.early:
                self.send(r, 1 - r, "pp", sb, ("P", j), f"pp_full{sb}", j >> 1)
            self.buf.write((r, "T", sb), ("P", j), who)
            self.bar(r, f"p_full{sb}").arrive()
            yield
        yield from self.exchange(r, self.n, who)


def test_the_maximum_exchange_already_orders_the_p_buffer():
    """The exchange of page j needs the partner's scores of page j, which its
    in-order pipe completes only after its P.V of page j - 2 (the reader of
    the buffer P_j goes into): the pv_done wait before the store is implied."""
    rng = random.Random(7)
    for _ in range(300):
        _NoPvDoneWait(rng.randint(0, 9), rng).run()


def test_catches_p_sent_before_the_exchange_without_the_pv_done_wait():
    class Broken(_NoPvDoneWait):
        early = True

    ok, msgs = _caught(Broken, 8, 1, "pp")
    assert ok, msgs


def test_catches_the_buffer_armed_before_its_phase_completed():
    """Arming pp_full for page t + 2 before the wait for page t's P."""

    class Broken(Pair):
        def mma_thread(self, r):
            n = self.n
            for t in range(min(2, n)):
                self.bar(r, f"pp_full{t}").arrive(expect=1)
            for j in range(n + 1):
                if j < n:
                    es, vs = j % E_STAGES, j % V_STAGES
                    while not (self.bar(r, f"v_full{vs}").done(j // V_STAGES) and
                               self.bar(r, f"e_full{es}").done(j // E_STAGES)):
                        yield
                    self.mma(r, [((r, "E", es), ("E", j)), ((r, "V", vs), ("V", j))], [((r, "T", j & 1), ("S", j))],
                             f"{r}.S_{j}")
                    self.commit(r, [(r, f"s_full{j & 1}")])
                    self.commit(r, [(r, f"e_empty{es}")])
                    yield
                if j >= 1:
                    t = j - 1
                    if t + 2 < n:
                        self.bar(r, f"pp_full{t & 1}").arrive(expect=1)       # planted: armed before the wait
                    while not (self.bar(r, f"p_full{t & 1}").done(t >> 1) and
                               self.bar(r, f"pp_full{t & 1}").done(t >> 1)):
                        yield
                    self.mma(r, [((r, "T", t & 1), ("P", t)), ((r, "pp", t & 1), ("P", t)),
                                 ((r, "V", t % V_STAGES), ("V", t)), ((r, "O"), ("O", t - 1))],
                             [((r, "O"), ("O", t))], f"{r}.PV_{t}")
                    self.commit(r, [(r, "o_ready")])
                    self.commit(r, [(r, f"v_empty{t % V_STAGES}")])
                    self.commit(r, [(0, f"pv_done{t & 1}"), (1, f"pv_done{t & 1}")])
                    yield
            self.commit(r, [(r, "mma_done")])
            while not self.bar(r, "mma_done").done(0):
                yield

    ok, msgs = _caught(Broken, 8, 2, "pp_full")
    assert ok, msgs


def test_catches_a_v_stage_reused_before_its_pv():
    class Broken(Pair):
        def producer(self, r):
            who = f"{r}.producer"
            for j in range(self.n):
                es, vs = j % E_STAGES, j % V_STAGES
                if j >= E_STAGES:
                    while not self.bar(r, f"e_empty{es}").done(j // E_STAGES - 1):
                        yield
                self.tma(r, "E", es, j, f"e_full{es}", j // E_STAGES, who)
                yield
                self.tma(r, "V", vs, j, f"v_full{vs}", j // V_STAGES, who)    # planted: no v_empty wait
                yield

    ok, msgs = _caught(Broken, 9, 3, "V")
    assert ok, msgs


def test_catches_the_partner_maximum_read_before_it_landed():
    class Broken(Pair):
        def exchange(self, r, j, who):
            sb = j & 1
            self.send(r, 1 - r, "xch", sb, ("X", j), f"xbar{sb}", j >> 1)
            self.buf.read((r, "xch", sb), ("X", j), who)                    # planted: read before the wait
            self.bar(r, f"xbar{sb}").arrive(expect=1)
            while not self.bar(r, f"xbar{sb}").done(j >> 1):
                yield

    ok, msgs = _caught(Broken, 6, 4, "xch")
    assert ok, msgs


def test_catches_a_rescale_without_the_output_wait():
    class Broken(Pair):
        def __init__(self, n, rng):
            super().__init__(n, rng, rescale_rate=1.0)

        def softmax(self, r):
            who = f"{r}.softmax"
            for j in range(self.n):
                sb = j & 1
                while not self.bar(r, f"s_full{sb}").done(j >> 1):
                    yield
                self.buf.read((r, "T", sb), ("S", j), who)
                yield from self.exchange(r, j, who)
                if j >= 2:
                    while not self.bar(r, f"pv_done{sb}").done((j - 2) >> 1):
                        yield
                self.send(r, 1 - r, "pp", sb, ("P", j), f"pp_full{sb}", j >> 1)
                self.buf.write((r, "T", sb), ("P", j), who)
                if j >= 1:
                    self.buf.read((r, "O"), ("O", j - 1), who)                # planted: no o_ready wait
                self.bar(r, f"p_full{sb}").arrive()
                yield
            yield from self.exchange(r, self.n, who)

    ok, msgs = _caught(Broken, 6, 5, "'O'")
    assert ok, msgs
