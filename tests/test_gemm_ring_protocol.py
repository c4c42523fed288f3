"""The ring protocol of the one-SM tensor-core GEMM, simulated on the CPU.

The kernel streams three rings through shared memory; two of them have more
than one waiter, and this simulation runs those under random interleavings
with asynchronous copy completion:

  - packed tiles (kSP stages, four k-blocks each): the TMA thread fills them in
    order, each after a parity wait on the stage's "empty" barrier, which
    completes once the four k-blocks of the previous tile there have been
    expanded (four arrivals);
  - expanded int8 tiles (kSB stages, one k-block each): expansion warp v takes
    the k-blocks with index v mod kExp; for each it waits for its expanded
    stage to be empty, then for the packed tile to be full, writes the stage
    and arrives on both barriers; the MMA thread takes the expanded stages in
    order and releases each one.

An mbarrier parity wait only tells the last two phases apart, so a waiter two
phases ahead of a barrier goes on early.  The kernel states the depths that
keep every waiter at most one phase ahead: kSB >= kExp and kSB + 3 <= 4 kSP.
The simulation reports every read of a stage that does not hold the waiter's
data and every write over data not yet consumed: none for the kernel's own
ring depths, and some for depths that break the conditions far enough (fewer
expanded stages than expansion warps; a single packed stage).  The second
condition is sufficient, not tight: an expansion warp at k-block kb needs the
MMA to have taken kb - kSB, so it runs at most about kSB / 4 tiles ahead of
the TMA thread.
"""
import random

import pytest


class Barrier:
    """mbarrier with an arrival count per phase."""

    def __init__(self, count=1):
        self.count = count
        self.pending = count
        self.completed = 0   # completed phases

    def try_wait_parity(self, parity):
        # true iff the phase just before the current one has this parity
        # (before any phase completes, the "previous phase" counts as parity 1)
        return (self.completed + 1) % 2 == parity

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


GROUP = 4  # k-blocks per packed tile


def simulate(n_kblocks, k_exp, s_b, s_p, seed, copy_delay=(1, 6), max_steps=40000):
    """Returns a list of violations: ("early-read", ...), ("overwrite", ...),
    or ("stuck", step) when the run stops making progress."""
    assert n_kblocks % GROUP == 0
    rng = random.Random(seed)
    n_tiles = n_kblocks // GROUP
    pfull = [Barrier(1) for _ in range(s_p)]
    pempty = [Barrier(GROUP) for _ in range(s_p)]
    bfull = [Barrier(1) for _ in range(s_b)]
    bempty = [Barrier(1) for _ in range(s_b)]
    p_holds = [None] * s_p       # tile whose data has landed in the stage
    p_reads_left = {}            # tile -> k-blocks of it not yet expanded
    b_holds = [None] * s_b       # k-block expanded into the stage
    b_consumed = set()           # k-blocks the MMA has read
    in_flight = []               # (ready_time, stage, tile)
    tma_t = 0
    exp_next = {v: v for v in range(k_exp)}   # next k-block of each expansion warp
    exp_phase = {v: 0 for v in range(k_exp)}  # 0: wait empty, 1: wait packed, 2..: writing
    mma_k = 0
    bad = []
    t = 0
    while mma_k < n_kblocks:
        t += 1
        if t > max_steps:
            bad.append(("stuck", t))
            break
        for item in [x for x in in_flight if x[0] <= t]:  # TMA copies land
            in_flight.remove(item)
            _, s, tile = item
            p_holds[s] = tile
            pfull[s].arrive()
        actors = ["tma", "mma"] + list(range(k_exp))
        rng.shuffle(actors)
        for a in actors:
            if a == "tma":
                if tma_t < n_tiles:
                    s, ph = tma_t % s_p, (tma_t // s_p) & 1
                    if pempty[s].try_wait_parity(ph ^ 1):
                        old = tma_t - s_p
                        if old >= 0 and p_reads_left.get(old, 0) > 0:
                            bad.append(("overwrite", "packed", old, tma_t))
                        p_reads_left[tma_t] = GROUP
                        in_flight.append((t + rng.randint(*copy_delay), s, tma_t))
                        tma_t += 1
            elif a == "mma":
                b, ph = mma_k % s_b, (mma_k // s_b) & 1
                if bfull[b].try_wait_parity(ph) and rng.random() < 0.8:
                    if b_holds[b] != mma_k:
                        bad.append(("early-read", "expanded", mma_k, b_holds[b]))
                    b_consumed.add(mma_k)
                    bempty[b].arrive()
                    mma_k += 1
            else:
                v = a
                kb = exp_next[v]
                if kb >= n_kblocks or rng.random() < 0.3:
                    continue
                b, tile = kb % s_b, kb // GROUP
                sp = tile % s_p
                if exp_phase[v] == 0:
                    if bempty[b].try_wait_parity(((kb // s_b) & 1) ^ 1):
                        exp_phase[v] = 1
                elif exp_phase[v] == 1:
                    if pfull[sp].try_wait_parity((tile // s_p) & 1):
                        if p_holds[sp] != tile:
                            bad.append(("early-read", "packed", tile, p_holds[sp]))
                        old = kb - s_b
                        if old >= 0 and old not in b_consumed:
                            bad.append(("overwrite", "expanded", old, kb))
                        exp_phase[v] = 2
                else:  # the write takes a step or two, then both arrivals
                    if rng.random() < 0.5:
                        b_holds[b] = kb
                        p_reads_left[tile] = p_reads_left.get(tile, GROUP) - 1
                        bfull[b].arrive()
                        pempty[sp].arrive()
                        exp_next[v] = kb + k_exp
                        exp_phase[v] = 0
    return bad


# (k_exp, s_b, s_p) of the kernel for 16..32, 64 and 128 tokens per tile
KERNEL_RINGS = [(8, 8, 3), (8, 8, 4), (4, 5, 4), (4, 4, 4)]


@pytest.mark.parametrize("rings", KERNEL_RINGS)
@pytest.mark.parametrize("seed", range(6))
def test_kernel_ring_depths_never_read_early(rings, seed):
    k_exp, s_b, s_p = rings
    assert s_b >= k_exp and s_b + 3 <= 4 * s_p  # the kernel's static_assert
    assert simulate(96, k_exp, s_b, s_p, seed) == []


def test_fewer_expanded_stages_than_warps_goes_wrong():
    """kSB < kExp: some expansion warp waits two phases ahead on an empty
    barrier and overwrites a tile the MMA has not read."""
    hits = [x for seed in range(20) for x in simulate(96, 8, 5, 4, seed)]
    assert any(x[:2] == ("overwrite", "expanded") for x in hits)


def test_shallow_packed_ring_goes_wrong():
    """One packed stage for eight expanded ones (kSB + 3 > 4 kSP by far): an
    expansion warp gets two phases ahead of the packed stage's full barrier
    and reads a tile that is still being filled."""
    hits = [x for seed in range(20) for x in simulate(96, 8, 8, 1, seed)]
    assert any(x[:2] == ("early-read", "packed") for x in hits)
