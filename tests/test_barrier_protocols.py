"""Randomised-interleaving models of two kernels' barrier protocols (host only).

Each model runs the kernel's roles as Python generators over a model of the
mbarrier (arrival count, transaction bytes, phase parity; a wait on parity P
is satisfied once the barrier's current phase parity differs from P), with
the asynchronous completions (TMA copies landing, tensor-core commits) as
separate events taken in a random order. They check that no role waits
forever and that every consumer sees the stage, accumulator and tile it
expects:

* the tensor-core mixing GEMM (premix_kernel) whose tiles come from a global
  counter: the producer publishes each tile index in a 16-entry ring and
  closes the sequence with an end entry that reuses a stage barrier;
* the persistent convolution (tc_conv_persist_kernel): two operand rings,
  double-buffered accumulators, eight epilogue warps.

A planted defect (the mixing GEMM's final drain waiting again on the stage
the end entry reused) must make the first model report a stuck role.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0

    def arrive(self, n=1):
        self.pending -= n
        self._check()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.pending -= 1
        self._check()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._check()

    def _check(self):
        assert self.pending >= 0 and self.tx >= 0
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


def _schedule(roles, rng, tma, mma_events, on_tma, on_mma, limit=200000):
    alive = list(range(len(roles)))
    steps = 0
    while alive or tma or mma_events:
        steps += 1
        if steps > limit:
            return False
        pick = rng.random()
        if tma and pick < 0.25:
            on_tma(tma.pop(rng.randrange(len(tma))))
            continue
        if mma_events and pick < 0.45:
            on_mma(mma_events.pop(0))  # commits complete in issue order
            continue
        if not alive:
            continue
        r = rng.choice(alive)
        try:
            next(roles[r])
        except StopIteration:
            alive.remove(r)
    return True


def mixing_gemm_model(ntiles, S, seed, skip_reused_stage=True):
    """premix_kernel with the tile counter: returns (finished, tiles seen by the epilogue)."""
    rng = random.Random(seed)
    full = [Bar(1) for _ in range(S)]
    empty = [Bar(1) for _ in range(S)]
    tfull = [Bar(1) for _ in range(2)]
    tempty = [Bar(8) for _ in range(2)]
    ring = [None] * 16
    tma, mma_events, seen = [], [], []
    counter = [0]

    def producer():
        issued, s, ph, ended, j = 0, 0, 0, False, 0
        while True:
            while not empty[s].done(ph ^ 1):
                yield
            t = counter[0]
            counter[0] += 1
            if t >= ntiles:
                t = -1
            ring[j % 16] = (j, t)
            if t < 0:
                full[s].arrive()  # the end entry
                ended = True
                break
            full[s].expect_tx(4)
            tma.append(s)
            issued += 1
            s += 1
            if s == S:
                s, ph = 0, ph ^ 1
            j += 1
        start = max(issued - S, 0)
        if skip_reused_stage and ended and issued >= S:
            start += 1
        for jj in range(start, issued):
            while not full[jj % S].done((jj // S) & 1):
                yield

    def mma():
        s, ph, j = 0, 0, 0
        while True:
            ab = j & 1
            while not full[s].done(ph):
                yield
            jt, t = ring[j % 16]
            assert jt == j
            while not tempty[ab].done(((j >> 1) & 1) ^ 1):
                yield
            if t < 0:
                tfull[ab].arrive()
                break
            mma_events.append((s, ab))
            s += 1
            if s == S:
                s, ph = 0, ph ^ 1
            j += 1

    def epilogue(w):
        j = 0
        while True:
            ab = j & 1
            while not tfull[ab].done((j >> 1) & 1):
                yield
            jt, t = ring[j % 16]
            assert jt == j
            if t < 0:
                break
            if w == 0:
                seen.append(t)
            yield
            tempty[ab].arrive()
            j += 1

    def on_mma(ev):
        s, ab = ev
        empty[s].arrive()
        tfull[ab].arrive()

    roles = [producer(), mma()] + [epilogue(w) for w in range(8)]
    ok = _schedule(roles, rng, tma, mma_events, lambda s: full[s].complete_tx(4), on_mma)
    return ok, seen


def persistent_conv_model(units, k_steps, kc, SA, SB, seed):
    """tc_conv_persist_kernel: activation ring (SB), mixed-kernel ring (SA), two accumulators."""
    rng = random.Random(seed)
    spc = k_steps // kc
    fullA = [Bar(1) for _ in range(SA)]
    emptyA = [Bar(1) for _ in range(SA)]
    fullB = [Bar(1) for _ in range(SB)]
    emptyB = [Bar(1) for _ in range(SB)]
    tfull = [Bar(1) for _ in range(2)]
    tempty = [Bar(8) for _ in range(2)]
    A, Bst, T = [None] * SA, [None] * SB, [None] * 2
    tma, mma_events = [], []

    def x_producer():
        issued = 0
        for i in range(units):
            for cc in range(kc):
                s, ph = issued % SB, (issued // SB) & 1
                while not emptyB[s].done(ph ^ 1):
                    yield
                fullB[s].expect_tx(1)
                tma.append(("B", s, (i, cc)))
                issued += 1

    def w_producer():
        issued = 0
        for i in range(units):
            for k in range(k_steps):
                s, ph = issued % SA, (issued // SA) & 1
                while not emptyA[s].done(ph ^ 1):
                    yield
                fullA[s].expect_tx(1)
                tma.append(("A", s, (i, k)))
                issued += 1

    def mma():
        s = ph = sbi = phb = 0
        for i in range(units):
            ab = i & 1
            while not tempty[ab].done(((i >> 1) & 1) ^ 1):
                yield
            assert T[ab] is None or T[ab][1] == "read"
            while not fullB[sbi].done(phb):
                yield
            while not fullA[s].done(ph):
                yield
            t = 0
            for k in range(k_steps):
                assert A[s] == (i, k) and Bst[sbi] == (i, k // spc)
                s_cur, sbi_cur, chunk_end = s, sbi, False
                t += 1
                if t == spc:
                    t, chunk_end = 0, True
                    sbi += 1
                    if sbi == SB:
                        sbi, phb = 0, phb ^ 1
                s += 1
                if s == SA:
                    s, ph = 0, ph ^ 1
                if k + 1 < k_steps:
                    if chunk_end:
                        while not fullB[sbi].done(phb):
                            yield
                    while not fullA[s].done(ph):
                        yield
                mma_events.append(("eA", s_cur))
                if chunk_end:
                    mma_events.append(("eB", sbi_cur))
            T[ab] = (i, "acc")
            mma_events.append(("tf", ab))

    def epilogue(w):
        for i in range(units):
            ab = i & 1
            while not tfull[ab].done((i >> 1) & 1):
                yield
            assert T[ab] in ((i, "acc"), (i, "read"))
            yield
            tempty[ab].arrive()
            if tempty[ab].pending == 8:
                T[ab] = (i, "read")

    def on_tma(ev):
        kind, s, tag = ev
        if kind == "A":
            A[s] = tag
            fullA[s].complete_tx(1)
        else:
            Bst[s] = tag
            fullB[s].complete_tx(1)

    def on_mma(ev):
        kind, x = ev
        if kind == "eA":
            A[x] = None
            emptyA[x].arrive()
        elif kind == "eB":
            Bst[x] = None
            emptyB[x].arrive()
        else:
            tfull[x].arrive()

    roles = [x_producer(), w_producer(), mma()] + [epilogue(w) for w in range(8)]
    return _schedule(roles, rng, tma, mma_events, on_tma, on_mma, limit=10**6)


@pytest.mark.parametrize("S", [2, 3, 4])
def test_mixing_gemm_counter_protocol(S):
    for ntiles in range(0, 11):
        for seed in range(12):
            ok, seen = mixing_gemm_model(ntiles, S, seed * 131 + ntiles)
            assert ok, (ntiles, S, seed)
            assert seen == list(range(ntiles)), (ntiles, S, seed, seen)


def test_mixing_gemm_model_catches_the_drain_defect():
    """The drain that also waits on the stage the end entry reused gets stuck."""
    stuck = 0
    for ntiles in (2, 3, 5, 8):
        for seed in range(4):
            ok, _ = mixing_gemm_model(ntiles, 2, seed, skip_reused_stage=False)
            stuck += not ok
    assert stuck > 0


@pytest.mark.parametrize("shape", [(3, 18, 2, 8, 2), (5, 1, 1, 2, 1), (4, 36, 4, 8, 2),
                                   (2, 9, 1, 3, 1), (7, 2, 2, 2, 2)])
def test_persistent_convolution_protocol(shape):
    units, k_steps, kc, SA, SB = shape
    for seed in range(25):
        assert persistent_conv_model(units, k_steps, kc, SA, SB, seed), (shape, seed)
