"""A model of the awq_w4a16 GEMV's per-warp copy ring, run over random interleavings. One warp
owns SLOTS shared-memory slots, each with an mbarrier (count 1): it requests a step's tiles into
the slot at its ring position (an arrival with the expected bytes, then copies that complete the
bytes when they land) and moves on, flipping its phase parity when it wraps; it consumes the step
in the slot at its position once the slot's barrier shows the phase of that parity complete, then
requests the step SLOTS ahead into the same slot. The prologue requests the first SLOTS steps,
which wraps the ring once, so the parity is set back to 0 before the first wait. A wait on parity
P returns once the barrier's phase of that parity has completed ((completed phases) mod 2 != P),
which holds at once for P = 1 on a fresh barrier: without the reset the first pass would read
slots before their copies land. A warp whose wait gives up walks the remaining requested slots
and waits for each, so that no copy lands in shared memory after the warp is gone.

The model checks that every consumed step finds its own tiles landed in its slot, that no copy
lands in a slot whose previous step is still unread, that the barriers' arrivals never overrun a
phase, and that the drain after a lost wait leaves no copy in flight."""
import random

import pytest


class Barrier:
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


def run(slots, total, seed, reset_parity=True, give_up_at=None):
    """One schedule. total: steps of the warp (units x steps per unit); give_up_at: the step at
    which the warp's wait gives up (None: it never does). Returns the steps consumed."""
    rng = random.Random(seed)
    bars = [Barrier(1) for _ in range(slots)]
    holds = [None] * slots    # step whose tiles have landed in the slot
    unread = [False] * slots  # the slot holds a landed step not consumed yet
    in_flight = []            # (slot, step) copies requested, not landed
    st = {"pos": 0, "ph": 0, "left": total, "next": 0}

    def issue():
        if st["left"] > 0:
            s = st["pos"]
            bars[s].arrive(expect_tx=1)
            in_flight.append((s, st["next"]))
            st["next"] += 1
            st["left"] -= 1
        if st["pos"] + 1 == slots:
            st["pos"] = 0
            st["ph"] ^= 1
        else:
            st["pos"] += 1

    def land(k):
        s, step = in_flight.pop(k)
        assert not unread[s], f"copy of step {step} lands over unread step {holds[s]} in slot {s}"
        holds[s], unread[s] = step, True
        bars[s].complete_tx(1)

    consumed = []

    def warp():
        for _ in range(slots):
            issue()
        if reset_parity:
            st["ph"] = 0
        for i in range(total):
            if give_up_at is not None and i == give_up_at:
                break
            while not bars[st["pos"]].done(st["ph"]):
                yield
            s = st["pos"]
            assert holds[s] == i and unread[s], f"step {i} read from slot {s} holding {holds[s]}"
            unread[s] = False
            consumed.append(i)
            issue()
        else:
            return
        # the lost wait: wait for every requested, unconsumed copy before leaving
        for _ in range(len(consumed), total - st["left"]):
            while not bars[st["pos"]].done(st["ph"]):
                yield
            unread[st["pos"]] = False
            if st["pos"] + 1 == slots:
                st["pos"] = 0
                st["ph"] ^= 1
            else:
                st["pos"] += 1
        assert not in_flight, "copies still in flight when the warp leaves"

    g = warp()
    alive = True
    for _ in range(100000):
        if alive and (not in_flight or rng.random() < 0.5):
            try:
                next(g)
            except StopIteration:
                alive = False
        elif in_flight:
            land(rng.randrange(len(in_flight)))
        if not alive and not in_flight:
            break
    assert not alive, "the warp never finished (deadlock)"
    return consumed


@pytest.mark.parametrize("slots", [2, 4, 8, 16])
@pytest.mark.parametrize("total", [0, 1, 3, 8, 24, 37])
def test_every_step_reads_its_own_tiles(slots, total):
    for seed in range(40):
        assert run(slots, total, seed) == list(range(total))


@pytest.mark.parametrize("slots", [2, 4, 16])
def test_drain_after_a_lost_wait_leaves_no_copy_in_flight(slots):
    for seed in range(60):
        total = 5 + seed % 30
        give_up = seed % (total + 1)
        assert run(slots, total, seed, give_up_at=give_up) == list(range(min(give_up, total)))


@pytest.mark.parametrize("slots", [2, 4, 8])
def test_without_the_parity_reset_the_first_pass_reads_early(slots):
    failures = 0
    for seed in range(40):
        try:
            run(slots, 3 * slots, seed, reset_parity=False)
        except AssertionError:
            failures += 1
    assert failures > 0
