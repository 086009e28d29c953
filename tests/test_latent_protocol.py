"""Protocol check of the latent decode kernel's pipeline (race detection
without a GPU).

The tensor-core latent kernel (GLA, MLRA) coordinates a TMA producer, one
MMA-issuing thread, the tensor pipe (which runs MMAs in issue order and
signals commits when everything issued before them has completed) and the
softmax warps through mbarriers, and reuses shared-memory stages and two TMEM
score buffers.  This test models those agents with the same issue conditions
as the kernel (csrc/decode_latent_tc.cu) and the mbarrier phase rules (a wait
on parity k & 1 returns once phase k has completed), runs them under many
random interleavings, and checks that

* every agent finishes (no deadlock),
* no parity wait is issued on a barrier that is already a full phase past
  the awaited one (parity aliasing),
* no buffer is overwritten while an operation that reads it is pending: a
  stage before the score MMAs and the P.V that read it completed, a TMEM
  score buffer before the P.V that reads the probabilities in it completed,
  O before the previous P.V completed.

Planted mistakes (a producer that skips its empty wait, an MMA thread that
runs the score MMAs two tiles ahead, a rescale without the output wait) must
each be caught.
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
    def __init__(self, n, stages, rng):
        self.n, self.S, self.rng = n, stages, rng
        self.full = [Bar(f"full{s}") for s in range(stages)]
        self.empty = [Bar(f"empty{s}") for s in range(stages)]
        self.s_full = [Bar(f"s_full{i}") for i in range(2)]
        self.p_full = [Bar(f"p_full{i}") for i in range(2)]
        self.o_ready = Bar("o_ready")
        self.pipe = []            # in-order tensor pipe: ("mma", reads, writes) or ("commit", bar)
        self.inflight_tma = []    # barriers of loads in flight
        self.readers = {}         # readers still pending per buffer: stages, TMEM score buffers, O

    # ------------------------------------------------------------ resources
    def _read(self, key):
        self.readers[key] = self.readers.get(key, 0) + 1

    def _unread(self, key):
        self.readers[key] -= 1

    def _write(self, key):
        assert self.readers.get(key, 0) == 0, f"{key} overwritten while {self.readers[key]} reader(s) pending"

    def mma(self, reads, writes, consumes=()):
        # `consumes`: buffers whose reader was reserved when their data was
        # written (P_j in a score buffer is reserved for PV_j)
        for r in reads:
            self._read(r)
        self.pipe.append(("mma", list(reads) + list(consumes), writes))

    def commit(self, bar):
        self.pipe.append(("commit", bar))

    def pipe_step(self):
        kind, *rest = self.pipe.pop(0)
        if kind == "mma":
            reads, writes = rest
            for r in reads:
                self._unread(r)
            for w in writes:
                # a score buffer written while a P.V that reads it is pending;
                # O is read and written by P.V MMAs in pipe order
                if w.startswith("T"):
                    self._write(w)
        else:
            rest[0].arrive()

    # ------------------------------------------------------------- agents
    def producer(self):
        S = self.S
        for j in range(self.n):
            st = j % S
            if j >= S:
                while not self.empty[st].done(j // S - 1):
                    yield
            self._write(f"K{st}")
            self.inflight_tma.append(self.full[st])
            yield

    def issue_s(self, j):
        self.mma([f"K{j % self.S}"], [f"T{j & 1}"])

    def issue_pv(self, t):
        self.mma([f"K{t % self.S}", "O"], ["O"], consumes=[f"T{t & 1}"])   # O is read-modify-write
        self.commit(self.o_ready)
        self.commit(self.empty[t % self.S])

    def mma_thread(self):
        n, S = self.n, self.S
        for j in range(n):
            while not self.full[j % S].done(j // S):
                yield
            self.issue_s(j)
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

    def softmax(self):
        for j in range(self.n):
            while not self.s_full[j & 1].done(j >> 1):
                yield
            self._write(f"T{j & 1}")      # P_j written over the scores ...
            self._read(f"T{j & 1}")       # ... and held for PV_j
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
        raise AssertionError(f"no progress: deadlock (n={self.n}, stages={self.S})")


@pytest.mark.parametrize("stages", [2, 4])
def test_pipeline_protocol_random_interleavings(stages):
    rng = random.Random(1234 + stages)
    for trial in range(300):
        n = rng.randint(0, 11)
        Model(n, stages, rng).run()


def _caught(cls, n, stages, seed, prefix):
    rng = random.Random(seed)
    messages = []
    for _ in range(200):
        try:
            cls(n, stages, rng).run()
        except AssertionError as e:
            messages.append(str(e))
    return any(m.startswith(prefix) and "overwritten" in m for m in messages), messages[:3]


def test_model_catches_score_mmas_two_tiles_ahead():
    """Issuing S_{j+1} before PV_{j-1} (the TMEM score buffer still holds
    P_{j-1}) must be reported."""

    class Broken(Model):
        def mma_thread(self):
            n, S = self.n, self.S
            for j in range(n):
                while not self.full[j % S].done(j // S):
                    yield
                self.issue_s(j)
                self.commit(self.s_full[j & 1])
                yield
            for t in range(n):                    # planted: every P.V after every score tile
                while not self.p_full[t & 1].done(t >> 1):
                    yield
                self.issue_pv(t)
                yield

    ok, msgs = _caught(Broken, 8, 4, 7, "T")
    assert ok, msgs


def test_model_catches_a_producer_that_skips_the_empty_wait():
    class Broken(Model):
        def producer(self):
            for j in range(self.n):
                self._write(f"K{j % self.S}")     # planted: no empty wait
                self.inflight_tma.append(self.full[j % self.S])
                yield

    ok, msgs = _caught(Broken, 9, 2, 11, "K")
    assert ok, msgs


def test_model_catches_a_rescale_without_the_output_wait():
    class Broken(Model):
        def softmax(self):
            for j in range(self.n):
                while not self.s_full[j & 1].done(j >> 1):
                    yield
                self._write(f"T{j & 1}")
                self._read(f"T{j & 1}")
                if j >= 1:
                    self._write("O")             # planted: rescale without waiting for PV_{j-1}
                self.p_full[j & 1].arrive()
                yield

    ok, msgs = _caught(Broken, 8, 4, 13, "O")
    assert ok, msgs
