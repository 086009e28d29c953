"""Protocol check of the latent decode kernel's pipeline (race detection
without a GPU).

The tensor-core latent kernel coordinates a TMA producer, one MMA-issuing
thread, the tensor pipe (which runs MMAs in issue order and signals commits
when everything issued before them has completed) and the softmax warps
through mbarriers, and reuses shared-memory stages and two TMEM score
buffers.  This test models those agents with the same issue conditions as
the kernel (csrc/decode_latent_tc.cu) and the mbarrier phase rules (a wait
on parity k & 1 returns once phase k has completed), runs them under many
random interleavings, and checks that

* every agent finishes (no deadlock),
* no parity wait is issued on a barrier that is already a full phase past
  the awaited one (parity aliasing),
* no buffer is overwritten while an operation that reads it is pending:
  a stage's E boxes before the score MMAs that read them completed, its V
  boxes before P.V completed, a TMEM score buffer before the P.V that reads
  the probabilities in it completed, O before the previous P.V completed.

Both ring modes are covered: the split-release ring (E and V groups with their
own barriers, readiness-ordered MMA issue) and the whole-stage ring.
"""

import random

import pytest


class Bar:
    """mbarrier: `count` arrivals complete a phase."""

    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.phase = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1

    def done(self, k):
        """Has phase k completed?  Asserts the wait cannot alias."""
        assert self.phase <= k + 1, f"{self.name}: waiting on phase {k} but {self.phase} completed (aliasing)"
        return self.phase > k


class Model:
    def __init__(self, n, stages, split, rng):
        self.n, self.S, self.split, self.rng = n, stages, split, rng
        self.e_full = [Bar(f"e_full{s}") for s in range(stages)]
        self.v_full = [Bar(f"v_full{s}") for s in range(stages)]
        self.e_empty = [Bar(f"e_empty{s}") for s in range(stages)]
        self.v_empty = [Bar(f"v_empty{s}") for s in range(stages)]
        self.s_full = [Bar(f"s_full{i}") for i in range(2)]
        self.p_full = [Bar(f"p_full{i}") for i in range(2)]
        self.o_ready = Bar("o_ready")
        self.pipe = []            # in-order tensor pipe: ("mma", reads, writes) or ("commit", bar)
        self.inflight_tma = []    # (group key, bar)
        # readers still pending per buffer: stage E/V groups, TMEM score buffers, O
        self.readers = {}
        self.log = []

    # ------------------------------------------------------------ resources
    def _read(self, key):
        self.readers[key] = self.readers.get(key, 0) + 1

    def _unread(self, key):
        self.readers[key] -= 1

    def _write(self, key):
        assert self.readers.get(key, 0) == 0, f"{key} overwritten while {self.readers[key]} reader(s) pending"

    def mma(self, reads, writes):
        for w in writes:
            self._write(w) if w.startswith(("E", "V")) else None
        for r in reads:
            self._read(r)
        self.pipe.append(("mma", reads, writes))

    def commit(self, bar):
        self.pipe.append(("commit", bar))

    def pipe_step(self):
        kind, *rest = self.pipe.pop(0)
        if kind == "mma":
            reads, writes = rest
            for w in writes:          # TMEM write hazards are checked at completion order
                if w.startswith("T"):
                    self._write(w)
            for r in reads:
                self._unread(r)
        else:
            rest[0].arrive()

    # ------------------------------------------------------------- agents
    def producer(self):
        S, split = self.S, self.split
        for j in range(self.n):
            st, eph = j % S, j // S - 1
            if j >= S:
                while not self.e_empty[st].done(eph):
                    yield
            self._write(f"E{st}")
            if not split:
                self._write(f"V{st}")
            self.inflight_tma.append(self.e_full[st])
            yield
            if split:
                if j >= S:
                    while not self.v_empty[st].done(eph):
                        yield
                self._write(f"V{st}")
                self.inflight_tma.append(self.v_full[st])
                yield

    def issue_s(self, j, part):
        st, buf = j % self.S, f"T{j & 1}"
        groups = {"E": [f"E{st}"], "V": [f"V{st}"], "all": [f"E{st}", f"V{st}"]}[part]
        self.mma(groups, [buf])

    def issue_pv(self, t):
        st = t % self.S
        self.mma([f"T{t & 1}", f"V{st}", "O"], ["O"])      # O is read-modify-write
        self.commit(self.o_ready)
        self.commit(self.v_empty[st] if self.split else self.e_empty[st])

    def mma_thread(self):
        n, S = self.n, self.S
        if not self.split:
            for j in range(n):
                st = j % S
                while not self.e_full[st].done(j // S):
                    yield
                self.issue_s(j, "all")
                self.commit(self.s_full[j & 1])
                yield
                if j >= 1:
                    while not self.p_full[(j - 1) & 1].done((j - 1) >> 1):
                        yield
                    self.issue_pv(j - 1)
                    yield
            if n:
                while not self.p_full[(n - 1) & 1].done((n - 1) >> 1):
                    yield
                self.issue_pv(n - 1)
            return
        jpv = jsv = jse = 0
        while jpv < n:
            if jsv < jse and self.v_full[jsv % S].done(jsv // S):
                self.issue_s(jsv, "V")
                self.commit(self.s_full[jsv & 1])
                jsv += 1
            elif jpv < jsv and self.p_full[jpv & 1].done(jpv >> 1):
                self.issue_pv(jpv)
                jpv += 1
            elif jse < n and jse == jsv and jpv >= jse - 1 and self.e_full[jse % S].done(jse // S):
                self.issue_s(jse, "E")
                self.commit(self.e_empty[jse % S])
                jse += 1
            yield

    def softmax(self):
        for j in range(self.n):
            while not self.s_full[j & 1].done(j >> 1):
                yield
            buf = f"T{j & 1}"
            self._write(buf)              # P_j written over the scores (read by PV_j later)
            if self.rng.random() < 0.3 and j >= 1:    # a rescale of O this tile
                while not self.o_ready.done(j - 1):
                    yield
                self._write("O")
            self.p_full[j & 1].arrive()
            yield
        if self.n:
            while not self.o_ready.done(self.n - 1):
                yield

    def run(self):
        agents = [self.producer(), self.mma_thread(), self.softmax()]
        alive = list(agents)
        for _ in range(200000):
            choices = alive + (["pipe"] if self.pipe else []) + (["tma"] if self.inflight_tma else [])
            if not choices:
                return
            pick = self.rng.choice(choices)
            if pick == "pipe":
                self.pipe_step()
            elif pick == "tma":
                self.inflight_tma.pop(self.rng.randrange(len(self.inflight_tma))).arrive()
            else:
                try:
                    next(pick)
                except StopIteration:
                    alive.remove(pick)
        raise AssertionError(f"no progress: deadlock (n={self.n}, stages={self.S}, split={self.split})")


@pytest.mark.parametrize("split,stages", [(True, 2), (False, 4), (False, 2), (True, 4)])
def test_pipeline_protocol_random_interleavings(split, stages):
    rng = random.Random(1234 + stages + 10 * split)
    for trial in range(300):
        n = rng.randint(0, 11)
        Model(n, stages, split, rng).run()


def test_model_catches_a_planted_hazard():
    """The checker itself: issuing S_t(E) without waiting for PV_{t-2} (the
    TMEM score buffer is still being read) must be reported."""

    class Broken(Model):
        def mma_thread(self):
            n, S = self.n, self.S
            jpv = jsv = jse = 0
            while jpv < n:
                if jsv < jse and self.v_full[jsv % S].done(jsv // S):
                    self.issue_s(jsv, "V")
                    self.commit(self.s_full[jsv & 1])
                    jsv += 1
                elif jpv < jsv and self.p_full[jpv & 1].done(jpv >> 1):
                    self.issue_pv(jpv)
                    jpv += 1
                elif jse < n and jse <= jsv + 1 and self.e_full[jse % S].done(jse // S):   # planted: no PV_{t-2} wait
                    self.issue_s(jse, "E")
                    self.commit(self.e_empty[jse % S])
                    jse += 1
                yield

    rng = random.Random(7)
    messages = []
    for _ in range(200):
        try:
            Broken(8, 2, True, rng).run()
        except AssertionError as e:
            messages.append(str(e))
    assert any("overwritten" in m and m.startswith("T") for m in messages), messages[:3]


def test_model_catches_a_producer_that_skips_the_value_slot_wait():
    class Broken(Model):
        def producer(self):
            S = self.S
            for j in range(self.n):
                st, eph = j % S, j // S - 1
                if j >= S:
                    while not self.e_empty[st].done(eph):
                        yield
                self._write(f"E{st}")
                self.inflight_tma.append(self.e_full[st])
                yield
                self._write(f"V{st}")            # planted: no v_empty wait
                self.inflight_tma.append(self.v_full[st])
                yield

    rng = random.Random(11)
    messages = []
    for _ in range(200):
        try:
            Broken(9, 2, True, rng).run()
        except AssertionError as e:
            messages.append(str(e))
    assert any(m.startswith("V") and "overwritten" in m for m in messages), messages[:3]


def test_model_catches_a_rescale_without_the_output_wait():
    class Broken(Model):
        def softmax(self):
            for j in range(self.n):
                while not self.s_full[j & 1].done(j >> 1):
                    yield
                self._write(f"T{j & 1}")
                if j >= 1:
                    self._write("O")             # planted: rescale without waiting for PV_{j-1}
                self.p_full[j & 1].arrive()
                yield

    rng = random.Random(13)
    messages = []
    for _ in range(200):
        try:
            Broken(8, 4, False, rng).run()
        except AssertionError as e:
            messages.append(str(e))
    assert any(m.startswith("O") and "overwritten" in m for m in messages), messages[:3]
