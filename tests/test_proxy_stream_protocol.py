"""The mbarrier protocol of the persistent proxy kernel (kap_stream.cu), simulated on the CPU.

The kernel's roles hand work to each other through mbarriers: the Q producer
fills a ring of QS chunk slots (q_full / q_empty; the four pooling warps of
the chunk's parity release a slot); the key producer fills a ring of 3
key-tile slots (k_full / k_empty, released by the MMAs' commit); eight pooling
warps (two per head: the even and the odd sub-rows, meeting at the head's
named barrier before the block vector) fill one of two B-operand buffers per
tile (a_full, eight arrivals; a_empty, the MMAs' commit after the tile's last
key tile); two epilogue groups of four warps take alternate tiles, and the
MMA issuer fills, for each key tile, one of the two TMEM accumulators of the
tile's group (acc_full by commit; acc_empty, the group's four warps); a
group's warps meet at its named barrier between the phases of a tile.  This
model replays each role's waits (with the kernel's parities) and arrivals
over a CTA's sequence of tiles with random key-tile counts, with copies and
MMAs completing asynchronously (MMAs in issue order).  Every run must
complete, and each wait must be satisfied by exactly the phase it intends.
"""
import random

import pytest

KS = 3


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0   # phase = completed phases

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def ready(self, parity, want_phase):
        # try_wait.parity(P) succeeds iff the phase with parity P has completed
        ok = (self.phase & 1) != parity
        if ok:
            assert self.phase == want_phase + 1, (self.phase, want_phase)   # exactly the intended phase
        return ok


class NamedBarrier:
    """bar.sync among n warps: generation counter."""

    def __init__(self, n):
        self.n, self.waiting, self.gen = n, 0, 0

    def sync(self):
        g = self.gen
        self.waiting += 1
        if self.waiting == self.n:
            self.waiting = 0
            self.gen += 1
        while self.gen == g:
            yield


def run(ntk, R, QS, rng):
    """ntk[x]: key tiles of the CTA's x-th tile; R chunks (sub-rows) per tile."""
    q_full = [Bar(1) for _ in range(QS)]
    q_empty = [Bar(4) for _ in range(QS)]
    k_full = [Bar(1) for _ in range(KS)]
    k_empty = [Bar(1) for _ in range(KS)]
    a_full, a_empty = [Bar(8), Bar(8)], [Bar(1), Bar(1)]
    acc_full, acc_empty = [Bar(1) for _ in range(4)], [Bar(4) for _ in range(4)]   # [2 group + buffer]
    drain = Bar(1)
    epi_bar = [NamedBarrier(4), NamedBarrier(4)]
    head_bar = [NamedBarrier(2) for _ in range(4)]
    pending = []                        # async completions, ('copy', bar) or ('mma', [bars])

    def q_producer():
        qc = 0
        for _ in ntk:
            for _v in range(R):
                slot, use = qc % QS, qc // QS
                if use >= 1:
                    while not q_empty[slot].ready((use - 1) & 1, use - 1):
                        yield
                pending.append(("copy", q_full[slot]))
                qc += 1
        for c in range(max(0, qc - QS), qc):                    # drain
            while not q_full[c % QS].ready((c // QS) & 1, c // QS):
                yield

    def k_producer():
        kc = 0
        for n in ntk:
            for _kt in range(n):
                slot, use = kc % KS, kc // KS
                if use >= 1:
                    while not k_empty[slot].ready((use - 1) & 1, use - 1):
                        yield
                pending.append(("copy", k_full[slot]))
                kc += 1
        for c in range(max(0, kc - KS), kc):
            while not k_full[c % KS].ready((c // KS) & 1, c // KS):
                yield

    def pooling(mt, half):
        qc = 0
        for tcount, _ in enumerate(ntk):
            buf = tcount & 1
            if tcount >= 2:
                while not a_empty[buf].ready(((tcount >> 1) - 1) & 1, (tcount >> 1) - 1):
                    yield
            for v in range(R):
                if (v & 1) != half:
                    continue
                c = qc + v
                slot = c % QS
                while not q_full[slot].ready((c // QS) & 1, c // QS):
                    yield
                yield                                           # sums the chunk, writes the vector
                q_empty[slot].arrive()
            qc += R
            yield from head_bar[mt].sync()                      # the odd sums are written
            yield                                               # the block vector (even warp)
            a_full[buf].arrive()

    def mma():
        kc = 0
        accg = [0, 0]
        for tcount, n in enumerate(ntk):
            buf, eg = tcount & 1, tcount & 1
            while not a_full[buf].ready((tcount >> 1) & 1, tcount >> 1):
                yield
            for _kt in range(n):
                slot = kc % KS
                u = accg[eg]
                ab = 2 * eg + (u & 1)
                while not k_full[slot].ready((kc // KS) & 1, kc // KS):
                    yield
                if u >= 2:
                    while not acc_empty[ab].ready(((u >> 1) - 1) & 1, (u >> 1) - 1):
                        yield
                pending.append(("mma", [k_empty[slot], acc_full[ab]]))
                kc += 1
                accg[eg] += 1
            pending.append(("mma", [a_empty[buf]]))
        pending.append(("mma", [drain]))
        while not drain.ready(0, 0):
            yield

    def epilogue(eg):
        u = 0
        for kloc, n in enumerate(ntk):
            if (kloc & 1) != eg:
                continue
            yield                                               # key scales of the row
            yield from epi_bar[eg].sync()
            for _kt in range(n):
                ab = 2 * eg + (u & 1)
                while not acc_full[ab].ready((u >> 1) & 1, u >> 1):
                    yield
                acc_empty[ab].arrive()
                yield                                           # score bits and argmax of its 32 key blocks
                u += 1
            yield from epi_bar[eg].sync()                       # sub-row maxima reduced
            yield                                               # HRM blocks written
            yield from epi_bar[eg].sync()                       # scales and maxima free for the next tile

    alive = ([q_producer(), k_producer(), mma()] + [pooling(mt, half) for half in (0, 1) for mt in range(4)] +
             [epilogue(eg) for eg in (0, 1) for _ in range(4)])
    steps = 0
    while alive or pending:
        steps += 1
        assert steps < 400000, "deadlock"
        if pending and (not alive or rng.random() < 0.35):
            copies = [k for k, p in enumerate(pending) if p[0] == "copy"]
            mmas = [k for k, p in enumerate(pending) if p[0] == "mma"]
            choice = rng.choice(copies + mmas[:1])           # copies land in any order; MMAs in issue order
            kind, what = pending.pop(choice)
            for bar in (what if kind == "mma" else [what]):
                bar.arrive()
            continue
        r = rng.choice(alive)
        try:
            next(r)
        except StopIteration:
            alive.remove(r)


@pytest.mark.parametrize("QS", [4, 6, 8])
@pytest.mark.parametrize("R", [4, 8])
def test_proxy_stream_protocol_completes_on_its_intended_phases(QS, R):
    rng = random.Random(QS * 10 + R)
    for _ in range(40):
        tiles = rng.randint(1, 7)
        ntk = [rng.randint(1, 9) for _ in range(tiles)]
        run(ntk, R, QS, rng)


def test_a_wrong_parity_is_caught():
    """The model is sensitive: the MMA's accumulator wait with the parity one off fails."""
    import inspect
    src = inspect.getsource(run).replace("acc_empty[ab].ready(((u >> 1) - 1) & 1",
                                         "acc_empty[ab].ready((u >> 1) & 1")
    assert src != inspect.getsource(run)
    ns = dict(globals())
    exec(compile(src, "mutant", "exec"), ns)
    with pytest.raises(AssertionError):
        rng = random.Random(0)
        for _ in range(20):
            ns["run"]([3, 5, 2, 7], 8, 4, rng)


def test_an_odd_q_ring_is_caught():
    """With an odd ring a slot serves both parities in turn, and the even-chunk warps can
    wait on a slot's next use before the odd warps' chunk in it has landed: the model
    reports the aliased phase (the kernel takes an even ring only)."""
    with pytest.raises(AssertionError):
        rng = random.Random(1)
        for _ in range(40):
            run([rng.randint(1, 9) for _ in range(5)], 8, 3, rng)
