"""A model of K1's split-K reduction across the CTAs of a cluster, run over random interleavings.
Each CTA initialises its receive barrier (expecting the bytes of the rows it owns from every other
CTA), then arrives on the cluster barrier early (relaxed); its reduction warps wait for the local
MMAs, wait on the cluster barrier (every CTA has initialised its receive barrier), send the
partial sums of rows another CTA owns into that CTA's slots (asynchronous stores that count their
bytes on the owner's barrier, landing in any order), write their own rows' partials locally, wait
for their barrier, and add the slots in cluster-rank order. The model checks that no store
targets an uninitialised barrier, that the owner adds only complete slots, that the sums equal the
direct ones bit for bit whatever the landing order (fixed order of the adds), and that no schedule
deadlocks."""
import random

import numpy as np
import pytest


def run(nsplit, rows, seed, send_before_wait=False):
    rng = random.Random(seed)
    nrng = np.random.default_rng(seed)
    partial = nrng.normal(size=(nsplit, rows)).astype(np.float32)  # CTA j's partial of each row
    rows_per = -(-rows // nsplit)
    owner = [min(r // rows_per, nsplit - 1) for r in range(rows)]
    inited = [False] * nsplit
    expect = [0] * nsplit
    landed = [0] * nsplit
    slots = [dict() for _ in range(nsplit)]  # (src, row) -> value
    arrived = [False] * nsplit
    in_flight = []  # (dst, src, row, value)
    results = {}

    def cta(j):
        own = [r for r in range(rows) if owner[r] == j]
        expect[j] = (nsplit - 1) * len(own)
        inited[j] = True
        yield
        arrived[j] = True  # early, relaxed cluster arrive
        yield  # the MMAs finish
        if not send_before_wait:
            while not all(arrived):
                yield  # cluster wait
        for r in range(rows):
            if owner[r] == j:
                slots[j][(j, r)] = partial[j, r]
            else:
                assert inited[owner[r]], "store to an uninitialised barrier"
                in_flight.append((owner[r], j, r, partial[j, r]))
            yield
        while landed[j] < expect[j]:
            yield
        for r in own:
            acc = np.float32(0.0)
            for src in range(nsplit):  # rank order
                assert (src, r) in slots[j], "slot read before it landed"
                acc = np.float32(acc + slots[j][(src, r)])
            results[r] = acc

    agents = [cta(j) for j in range(nsplit)]
    # the CTAs of a cluster start together but run at their own pace
    live = list(range(nsplit))
    n = 0
    while live or in_flight:
        choices = list(live) + (["land"] if in_flight else [])
        c = rng.choice(choices)
        n += 1
        assert n < 100000, "no progress"
        if c == "land":
            dst, src, r, v = in_flight.pop(rng.randrange(len(in_flight)))
            assert inited[dst]
            slots[dst][(src, r)] = v
            landed[dst] += 1
            continue
        try:
            next(agents[c])
        except StopIteration:
            live.remove(c)
    want = {}
    for r in range(rows):
        acc = np.float32(0.0)
        for src in range(nsplit):
            acc = np.float32(acc + partial[src, r])
        want[r] = acc
    assert results == want


@pytest.mark.parametrize("nsplit,rows", [(2, 64), (3, 64), (4, 64), (8, 64), (2, 5)])
@pytest.mark.parametrize("seed", range(20))
def test_reduction_random_interleavings(nsplit, rows, seed):
    run(nsplit, rows, seed)


def test_sending_before_the_cluster_wait_can_hit_an_uninitialised_barrier():
    # why the send waits on the cluster barrier: a CTA that has not yet initialised its receive
    # barrier may be the owner
    failures = 0
    for seed in range(50):
        try:
            run(4, 16, seed, send_before_wait=True)
        except AssertionError:
            failures += 1
    assert failures > 0
