"""A model of the fused QKV output stage's rotary-row staging protocol, run over random
interleavings: one filler thread, eight output warps, one shared-memory buffer, two mbarriers
(rope_full: one arrival with a byte count, completed when the copy lands; rope_empty: eight
arrivals). A wait on parity P returns once the barrier's phase of that parity has completed,
i.e. when (completed phases) mod 2 != P, which is ambiguous once a waiter falls two phases
behind; the model checks that this never happens, that no schedule deadlocks, that every read
sees exactly the pass it waited for, and that tiles without Q/K heads are skipped on both sides.
The protocol is the one the K2 QKNR kernel runs (per tile: pass A = column pairs 0-31 with
parity 0, pass B = pairs 32-63 with parity 1)."""
import random

import pytest

WARPS = 8


class Barrier:
    """mbarrier: a phase completes when its arrivals are all in and its transaction count is 0."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phases = count, count, 0, 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phases += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        assert self.pending >= 0, "arrival on a completed phase"
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        assert self.tx >= 0
        self._check()

    def done(self, parity):
        return (self.phases & 1) != parity


def run(tiles, rope_tile, seed, early_arrivals=False):
    rng = random.Random(seed)
    full, empty = Barrier(1), Barrier(WARPS)
    buf = {"pass": None}
    inflight = []  # copies issued, not landed: pass ids

    def filler():
        p = 0
        for t in range(tiles):
            if not rope_tile(t):
                continue
            for _ph in range(2):
                if p > 0:
                    while not empty.done((p - 1) & 1):
                        yield
                    # the phase waited for is the latest one (never two behind)
                    assert empty.phases == p
                full.arrive(expect_tx=1)  # the phase completes only when the copy lands
                inflight.append(p)
                p += 1
                yield

    def warp(w):
        seen = 0
        for t in range(tiles):
            if not rope_tile(t):
                yield
                continue
            for ph in range(2):
                if early_arrivals and w >= WARPS // 2:
                    # a warp whose head needs no rotation reporting without waiting for the pass
                    empty.arrive()
                    seen += 1
                    yield
                    continue
                while not full.done(ph):
                    yield
                assert full.phases == seen + 1, "waited on a phase two behind"
                assert buf["pass"] == seen, (w, t, ph, buf["pass"], seen)
                yield  # reading
                assert buf["pass"] == seen, "buffer overwritten while being read"
                empty.arrive()
                seen += 1
                yield

    agents = [filler()] + [warp(w) for w in range(WARPS)]
    live = list(range(len(agents)))
    steps = 0
    while live or inflight:
        choices = list(live) + (["land"] if inflight else [])
        c = rng.choice(choices)
        steps += 1
        assert steps < 200000, "no progress"
        if c == "land":
            p = inflight.pop(0)
            buf["pass"] = p
            full.complete_tx(1)
            continue
        try:
            next(agents[c])
        except StopIteration:
            live.remove(c)
    n_rope = sum(1 for t in range(tiles) if rope_tile(t))
    assert full.phases == 2 * n_rope and empty.phases == 2 * n_rope


@pytest.mark.parametrize("seed", range(200))
def test_protocol_random_interleavings(seed):
    # 9 tiles of a pair: two of every three hold Q/K heads (QKV: N = 3 x 3072, 256-column tiles)
    run(9, lambda t: t % 3 != 2, seed)


def test_protocol_all_tiles_and_none():
    run(5, lambda t: True, 1)
    run(4, lambda t: False, 2)


def test_model_catches_early_arrivals():
    # the reason every output warp waits for each pass, even where its head is in V: reports
    # that run ahead let the filler overwrite rows still being read, or arrive on a completed
    # phase
    failures = 0
    for seed in range(100):
        try:
            run(9, lambda t: True, seed, early_arrivals=True)
        except AssertionError:
            failures += 1
    assert failures > 0
