"""The ring protocol of the two-SM tensor-core GEMM, simulated on the CPU.

A cluster of two CTAs shares one accumulator tile: each CTA's TMA thread
loads, per k-block, its half of the activation tile (both halves count on the
leader CTA's "x full" barrier) and its 128 packed weight rows (its own
"packed full" barrier) into stage it mod A of its TMA ring; its four
expansion warps wait for the packed tile and for expanded stage it mod B to be
empty, read the packed rows (one arrival each on the CTA's "A empty" barrier),
write their share of the expanded tile and arrive on the leader's "expanded"
barrier (eight arrivals: four warps in each CTA); the leader's MMA thread
waits for both, issues the MMAs and, when they complete, arrives on the
"A empty" and "B empty" barriers of both CTAs.  "A empty" counts five
arrivals per phase (the MMAs' and the four expansion warps'), "B empty" one.

Every waiter takes its stages in order with parity waits (an mbarrier tells
only the last two phases apart).  The simulation runs random interleavings
with asynchronous copy landing and MMA completion and reports every read of a
stage that does not hold the waiter's k-block and every write over data not
yet consumed: none for the kernel's ring depths.
"""
import random

import pytest


class Barrier:
    """mbarrier with an arrival count per phase."""

    def __init__(self, count=1):
        self.count = count
        self.pending = count
        self.completed = 0

    def try_wait_parity(self, parity):
        return (self.completed + 1) % 2 == parity

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


WARPS = 4  # expansion warps per CTA


def simulate(n_kblocks, A, B, seed, max_steps=60000, skip_b_wait=False):
    rng = random.Random(seed)
    xfull = [Barrier(2) for _ in range(A)]  # leader: both CTAs' x halves (modelled as one arrival each)
    pfull = [[Barrier(1) for _ in range(A)] for _ in range(2)]
    emptyA = [[Barrier(1 + WARPS) for _ in range(A)] for _ in range(2)]
    expd = [Barrier(2 * WARPS) for _ in range(B)]
    emptyB = [[Barrier(1) for _ in range(B)] for _ in range(2)]
    x_holds = [[None] * A for _ in range(2)]   # k-block whose x half landed in the stage
    p_holds = [[None] * A for _ in range(2)]   # k-block whose packed rows landed
    p_reads = [dict() for _ in range(2)]       # k-block -> expansion warps still to read its packed rows
    e_parts = [dict() for _ in range(B)]       # stage -> {(cta, warp): k-block written}
    consumed = set()                           # k-blocks whose MMAs have completed
    in_flight = []                             # (time, kind, cta, stage, k-block)
    tma_it = [0, 0]
    exp_it = {(c, v): 0 for c in range(2) for v in range(WARPS)}
    exp_phase = {w: 0 for w in exp_it}
    mma_it = 0
    bad = []
    t = 0
    while len(consumed) < n_kblocks:
        t += 1
        if t > max_steps:
            bad.append(("stuck", t))
            break
        for item in [x for x in in_flight if x[0] <= t]:
            in_flight.remove(item)
            _, kind, c, s, kb = item
            if kind == "x":
                x_holds[c][s] = kb
                xfull[s].arrive()
            elif kind == "p":
                p_holds[c][s] = kb
                pfull[c][s].arrive()
            else:  # the MMAs of k-block kb completed
                consumed.add(kb)
                for cc in range(2):
                    emptyA[cc][kb % A].arrive()
                    emptyB[cc][kb % B].arrive()
        actors = ["tma0", "tma1", "mma"] + list(exp_it)
        rng.shuffle(actors)
        for a in actors:
            if a in ("tma0", "tma1"):
                c = int(a[-1])
                it = tma_it[c]
                if it < n_kblocks:
                    s, ph = it % A, (it // A) & 1
                    if emptyA[c][s].try_wait_parity(ph ^ 1):
                        old = it - A
                        if old >= 0 and (old not in consumed or p_reads[c].get(old, 0) > 0):
                            bad.append(("overwrite", "tma", c, old, it))
                        p_reads[c][it] = WARPS
                        in_flight.append((t + rng.randint(1, 6), "x", c, s, it))
                        in_flight.append((t + rng.randint(1, 6), "p", c, s, it))
                        tma_it[c] += 1
            elif a == "mma":
                it = mma_it
                if it < n_kblocks and rng.random() < 0.7:
                    sa, sb = it % A, it % B
                    if xfull[sa].try_wait_parity((it // A) & 1) and expd[sb].try_wait_parity((it // B) & 1):
                        if any(x_holds[c][sa] != it for c in range(2)):
                            bad.append(("early-read", "x", it))
                        parts = e_parts[sb]
                        if len(parts) != 2 * WARPS or any(k != it for k in parts.values()):
                            bad.append(("early-read", "expanded", it))
                        in_flight.append((t + rng.randint(2, 12), "done", 0, 0, it))
                        mma_it += 1
            else:
                c, v = a
                it = exp_it[a]
                if it >= n_kblocks or rng.random() < 0.3:
                    continue
                sa, sb = it % A, it % B
                if exp_phase[a] == 0:
                    if pfull[c][sa].try_wait_parity((it // A) & 1) and \
                            (skip_b_wait or emptyB[c][sb].try_wait_parity(((it // B) & 1) ^ 1)):
                        if p_holds[c][sa] != it:
                            bad.append(("early-read", "packed", c, it))
                        p_reads[c][it] -= 1
                        emptyA[c][sa].arrive()  # the packed rows have been read
                        old = it - B
                        if old >= 0 and old not in consumed:
                            bad.append(("overwrite", "expanded", c, old, it))
                        exp_phase[a] = 1
                else:  # the write takes a step or two, then the arrival at the leader
                    if rng.random() < 0.5:
                        e_parts[sb][a] = it
                        expd[sb].arrive()
                        exp_it[a] = it + 1
                        exp_phase[a] = 0
    return bad


# (TMA stages, expanded stages): the kernel's, and the earlier depths
@pytest.mark.parametrize("depths", [(5, 5), (7, 3), (4, 6)])
@pytest.mark.parametrize("seed", range(5))
def test_two_sm_rings_never_read_early(depths, seed):
    A, B = depths
    assert simulate(60, A, B, seed) == []


def test_simulation_sees_a_missing_wait():
    """Planted in the model: the expansion warps skip the 'B empty' wait.  With
    more TMA stages than expanded ones (7 and 3) the packed tile's arrival no
    longer implies that the expanded stage's last k-block was consumed, and
    some warp writes over it.  (With as many or fewer TMA stages the packed
    wait alone would guard the expanded stage, which is why the kernel's
    depths are checked with the wait in place.)"""
    hits = [h for seed in range(10) for h in simulate(40, 7, 3, seed, max_steps=8000, skip_b_wait=True)]
    assert any(h[:2] == ("overwrite", "expanded") for h in hits)
