"""A model of the mbarrier protocol of pruned attention over a packed past,
run over random interleavings on the CPU.

Roles, as in the kernel: the producer TMA-loads the local tiles
j = n_past .. n-1 (those below the stage count without a wait); the
converters fill the past tiles 0 .. n_past-1, K then V; the MMA thread
consumes tiles in order and releases a stage (K after S(j), V after PV(j))
through an asynchronous commit when a later tile will use it.  Barriers are
modelled the way the hardware decides a parity wait: a wait for parity P
returns once the count of completed phases c has (c & 1) != P.

The model checks that every wait that returns was for a phase that had
really completed (no stale-parity success), that each stage's "full" phases
receive their arrivals in tile order (one per tile), and that the run ends.
With the producer's converters-done wait removed -- the protocol of an
earlier variant -- the model finds a stale-parity success once the past spans
4 or more tiles, which is the fault that variant raised."""
import random

import pytest

STAGES = 2


class Bar:
    """One-arrival mbarrier; `first` and `step` name the tile each phase
    belongs to (tile first + step * phase), so out-of-order arrivals show."""

    def __init__(self, first=0, step=STAGES, log=None):
        self.done = 0          # completed phases
        self.first, self.step, self.log = first, step, log

    def arrive(self, tile=None):
        if tile is not None and tile != self.first + self.step * self.done:
            self.log.append(("arrival", tile, self.first + self.step * self.done))
        self.done += 1

    def ready(self, phase):
        """The hardware answer of a parity wait for `phase`, and whether it is right."""
        ok = (self.done & 1) != (phase & 1)
        return ok, (not ok) or self.done >= phase + 1


def run(n_past, n, seed, conv_done_wait=True):
    rng = random.Random(seed)
    stale = []
    full = {w: [Bar(st, STAGES, stale) for st in range(STAGES)] for w in "KV"}
    empty = {w: [Bar() for _ in range(STAGES)] for w in "KV"}
    conv_done = Bar()

    def wait(bar, phase, who):
        ok, right = bar.ready(phase)
        if ok and not right:
            stale.append(who)
        return ok

    # ---- producer: local tiles; the first kStages tiles' loads need no wait
    def producer():
        j0 = n_past
        for j in range(j0, n):
            st = j % STAGES
            if j >= STAGES:
                if conv_done_wait and n_past > 0:
                    while not wait(conv_done, 0, ("P", "done")):
                        yield
                while not wait(empty["K"][st], j // STAGES - 1, ("P", "K", j)):
                    yield
            full["K"][st].arrive(j)
            yield
            if j >= STAGES:
                while not wait(empty["V"][st], j // STAGES - 1, ("P", "V", j)):
                    yield
            full["V"][st].arrive(j)
            yield

    # ---- converters: K then V of each past tile
    def converter():
        for u in range(2 * n_past):
            j, w = u // 2, "KV"[u % 2]
            st = j % STAGES
            if j >= STAGES:
                while not wait(empty[w][st], j // STAGES - 1, ("C", w, j)):
                    yield
            if u == 2 * n_past - 1:
                conv_done.arrive()
            yield                      # the expansion takes a while
            full[w][st].arrive(j)
            yield

    # ---- MMA thread with asynchronous commits (completing in order, later)
    commits = []

    def mma():
        for j in range(n):
            st, pst = j % STAGES, (j + STAGES - 1) % STAGES
            while not wait(full["K"][st], j // STAGES, ("M", "K", j)):
                yield
            if j > 0:
                while not wait(full["V"][pst], (j - 1) // STAGES, ("M", "V", j - 1)):
                    yield
            if j + STAGES < n:
                commits.append(empty["K"][st])
            if j > 0 and (j - 1) + STAGES < n:
                commits.append(empty["V"][pst])
            yield
        if n > 0:
            while not wait(full["V"][(n - 1) % STAGES], (n - 1) // STAGES, ("M", "V", n - 1)):
                yield

    def completer():
        while True:
            if commits and rng.random() < 0.5:
                commits.pop(0).arrive()
            yield

    roles = [producer(), converter(), mma()]
    comp = completer()
    live = list(range(3))
    for _ in range(20000):
        if not live:
            break
        i = rng.choice(live + [-1])
        if i < 0:
            next(comp)
            continue
        try:
            next(roles[i])
        except StopIteration:
            live.remove(i)
    return not live, stale


@pytest.mark.parametrize("n_past", range(0, 9))
@pytest.mark.parametrize("n_local", [1, 2, 3, 5])
def test_protocol_waits_are_exact_and_finish(n_past, n_local):
    for seed in range(40):
        finished, stale = run(n_past, n_past + n_local, seed)
        assert finished, (n_past, n_local, seed)
        assert not stale, (n_past, n_local, seed, stale[:3])


def test_without_the_converters_done_wait_a_stale_parity_succeeds():
    found = {}
    for n_past in range(0, 9):
        found[n_past] = any(run(n_past, n_past + 3, seed, conv_done_wait=False)[1] for seed in range(60))
    assert not any(found[k] for k in range(0, 4))      # short pasts: the old protocol was sound
    assert all(found[k] for k in range(4, 9))          # 4 or more past tiles: stale parity
