"""The mbarrier protocol of the attention kernel (osk.cu), simulated on the CPU.

The kernel's producer warp (K and V copies into one slot each), MMA warp
(S = Q K^T into one TMEM buffer, P V into O) and softmax warps (reading S,
writing P in place, voting on the skip) hand work to each other through
mbarriers: q_full; k_full / k_empty and v_full / v_empty for the two slots;
s_full for S; p_full[2] (one arrival per softmax warp) for P and the skip flag;
o_done[2] for P V; and the MMA drain.  This model replays each role's waits
(with the kernel's parities) and arrivals, with copies and MMAs completing
asynchronously (MMAs in issue order), for random keep masks and skip
decisions.  Every run must complete, and each wait must be satisfied by
exactly the phase it intends.
"""
import random

import pytest


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


def run(keep, skip, rescale, rng):
    """keep[t]: list entry t is computed; skip[c] / rescale[c]: the softmax's
    decisions for the c-th computed entry (c = 0 is never skipped)."""
    n_comp = sum(keep)
    q_full, k_full, k_empty, v_full, v_empty = Bar(1), Bar(1), Bar(1), Bar(1), Bar(1)
    s_full, drain = Bar(1), Bar(1)
    p_full = [Bar(1), Bar(1)]          # the softmax warps arrive together: one arrival here
    o_done = [Bar(1), Bar(1)]
    pending = []                       # async completions, ('copy', bar) or ('mma', [bars])
    armed = {"k": -1, "v": -1}
    pending.append(("copy", q_full))   # Q is requested in the prologue

    def producer():
        ncopy = 0
        for t in range(len(keep)):
            if not keep[t]:
                continue
            use = ncopy
            for name, full, empty in (("k", k_full, k_empty), ("v", v_full, v_empty)):
                if use >= 1:
                    while not empty.ready((use - 1) & 1, use - 1):
                        yield
                pending.append(("copy", full))
                armed[name] = use
            ncopy += 1
        # drain: every copy this role started has landed
        while not q_full.ready(0, 0):
            yield
        for name, full in (("k", k_full), ("v", v_full)):
            if armed[name] >= 0:
                while not full.ready(armed[name] & 1, armed[name]):
                    yield

    def mma():
        while not q_full.ready(0, 0):
            yield
        kept = 0
        if n_comp:
            while not k_full.ready(0, 0):
                yield
            pending.append(("mma", [s_full, k_empty]))            # S(0); the K slot is free after it
        for u in range(n_comp):
            while not p_full[u & 1].ready((u >> 1) & 1, u >> 1):
                yield
            while not v_full.ready(u & 1, u):
                yield
            bars = []
            if not skip[u]:
                pending.append(("mma", []))                       # P V(u), committed below
                bars += [v_empty, o_done[kept & 1]]
                kept += 1
            else:
                v_empty.arrive()
            if u + 1 < n_comp:
                # S(u + 1) is issued right behind P V(u), before the commits
                while not k_full.ready((u + 1) & 1, u + 1):
                    yield
                bars += [s_full, k_empty]
            pending.append(("mma", bars))                         # the commits: after every MMA so far
        pending.append(("mma", [drain]))
        while not drain.ready(0, 0):
            yield

    def softmax():
        n_pv = 0
        for c in range(n_comp):
            sb = c & 1
            while not s_full.ready(sb, c):
                yield
            yield                                                  # reads S, votes
            if skip[c]:
                p_full[sb].arrive()
                continue
            if rescale[c] and n_pv >= 1:                           # O must be complete before re-basing
                while not o_done[(n_pv - 1) & 1].ready(((n_pv - 1) >> 1) & 1, (n_pv - 1) >> 1):
                    yield
            p_full[sb].arrive()
            n_pv += 1
        if n_pv >= 1:                                              # epilogue reads O
            while not o_done[(n_pv - 1) & 1].ready(((n_pv - 1) >> 1) & 1, (n_pv - 1) >> 1):
                yield

    alive = [producer(), mma(), softmax()]
    steps = 0
    while alive or pending:
        steps += 1
        assert steps < 200000, "deadlock"
        if pending and (not alive or rng.random() < 0.35):
            copies = [k for k, p in enumerate(pending) if p[0] == "copy"]
            mmas = [k for k, p in enumerate(pending) if p[0] == "mma"]
            # copies land in any order; MMAs complete in issue order
            choice = rng.choice(copies + mmas[:1])
            kind, what = pending.pop(choice)
            for bar in (what if kind == "mma" else [what]):
                bar.arrive()
            continue
        r = rng.choice(alive)
        try:
            next(r)
        except StopIteration:
            alive.remove(r)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 13])
def test_attention_pipeline_protocol_completes_on_its_intended_phases(n):
    rng = random.Random(n)
    for _ in range(300):
        keep = [1] * n if rng.random() < 0.5 else [int(rng.random() < 0.7) for _ in range(n)]
        if not any(keep):
            keep[rng.randrange(n)] = 1
        n_comp = sum(keep)
        skip = [0] + [int(rng.random() < 0.4) for _ in range(n_comp - 1)]
        rescale = [int(rng.random() < 0.3) for _ in range(n_comp)]
        run(keep, skip, rescale, rng)


def test_a_wrong_parity_is_caught():
    """The model is sensitive: the MMA's P wait with the parity one off fails."""
    import inspect
    src = inspect.getsource(run).replace("p_full[u & 1].ready((u >> 1) & 1", "p_full[u & 1].ready(((u >> 1) + 1) & 1")
    ns = dict(globals())
    exec(compile(src, "mutant", "exec"), ns)
    with pytest.raises(AssertionError):
        rng = random.Random(0)
        for n in (3, 5, 8):
            ns["run"]([1] * n, [0] * n, [0] * n, rng)
