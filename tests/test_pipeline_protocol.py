"""The stage-ring protocol of the bulk-staged kernels, simulated on the CPU.

A producer fills S shared-memory stages in order; consumers wait on a stage's
"full" barrier with a parity wait and release it on its "empty" barrier.  An
mbarrier parity wait only tells the last two phases apart: it returns as soon
as the phase *before the current one* has the requested parity.  So a waiter
that is two phases ahead of the barrier goes on early and reads a stage that is
still being filled.  The simulation runs the protocol under random
interleavings and asynchronous copy completion, and reports every read of a
stage that does not yet hold the consumer's chunk.

The absmean and ternarize kernels give consumer warp w the stage w (as many
consumer warps as stages): never early.  Spreading chunks round-robin over
more warps than stages is caught early — the design the kernels do not use.
"""
import random

import pytest


class Barrier:
    """Phase counter of an mbarrier (arrival count 1 per phase)."""

    def __init__(self):
        self.completed = 0   # number of completed phases

    def try_wait_parity(self, parity):
        # true iff the phase just before the current one has this parity
        # (before any phase completes, the "previous phase" counts as parity 1)
        return (self.completed + 1) % 2 == parity

    def complete(self):
        self.completed += 1


def simulate(n_chunks, stages, consumers, owner_of, seed, copy_delay=(1, 6), max_steps=20000):
    """Returns the list of early reads (chunk, completed phases seen); a run
    that stops making progress (a consequence of early releases) adds
    ("stuck", step)."""
    rng = random.Random(seed)
    full = [Barrier() for _ in range(stages)]
    empty = [Barrier() for _ in range(stages)]
    stage_holds = [None] * stages          # chunk whose data has landed in the stage
    in_flight = []                          # (ready_time, stage, chunk)
    queues = {c: [j for j in range(n_chunks) if owner_of(j) == c] for c in range(consumers)}
    pos = {c: 0 for c in range(consumers)}
    reading = {}                            # consumer -> (chunk, remaining steps)
    prod_j = 0
    t = 0
    early = []
    while prod_j < n_chunks or in_flight or any(pos[c] < len(queues[c]) for c in queues) or reading:
        t += 1
        if t > max_steps:
            early.append(("stuck", t))
            break
        for item in [x for x in in_flight if x[0] <= t]:   # copies land
            in_flight.remove(item)
            _, s, j = item
            stage_holds[s] = j
            full[s].complete()
        actors = ["p"] + list(queues)
        rng.shuffle(actors)
        for a in actors:
            if a == "p":
                if prod_j < n_chunks:
                    s, ph = prod_j % stages, (prod_j // stages) & 1
                    if empty[s].try_wait_parity(ph ^ 1):
                        in_flight.append((t + rng.randint(*copy_delay), s, prod_j))
                        prod_j += 1
                continue
            c = a
            if c in reading:
                j, left = reading[c]
                if left > 1:
                    reading[c] = (j, left - 1)
                else:
                    del reading[c]
                    empty[j % stages].complete()          # release the stage
                continue
            if pos[c] < len(queues[c]) and rng.random() < 0.7:
                j = queues[c][pos[c]]
                s, ph = j % stages, (j // stages) & 1
                if full[s].try_wait_parity(ph):
                    if stage_holds[s] != j:
                        early.append((j, full[s].completed))
                    reading[c] = (j, rng.randint(1, 4))
                    pos[c] += 1
    return early


@pytest.mark.parametrize("seed", range(20))
def test_owned_stages_never_read_early(seed):
    S = 6
    assert simulate(200, S, S, lambda j: j % S, seed) == []


def test_round_robin_over_more_warps_than_stages_reads_early():
    """8 consumer warps taking chunks round-robin over 5 stages: some warp
    waits two phases ahead and reads a stage that is still being filled."""
    hits = sum(len(simulate(200, 5, 8, lambda j: j % 8, seed)) for seed in range(20))
    assert hits > 0


@pytest.mark.parametrize("seed", range(5))
def test_single_consumer_in_order(seed):
    """One consumer taking every chunk in order (the GEMM's roles) is safe."""
    assert simulate(100, 4, 1, lambda j: 0, seed) == []
