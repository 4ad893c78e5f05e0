"""A host model of the tensor-core kernel's stage-ring handshake.

The kernel's roles meet on mbarriers and wait with phase-parity tests: a wait
for phase k passes when the barrier's current phase parity differs from
k & 1.  So a waiter that is a whole phase ahead of the barrier (the barrier
still in phase k-1) sees the parity of phase k-2 and passes at once.

Modelled here, with copies that land in any order:
  producer   issues the fill of iteration j into stage j mod S once empty(s)
             completed the phase of iteration j - S
  decoders   group g takes iterations i = g (mod G) in order, parity-waits on
             full(i mod S), reads the stage, arrives on empty
  MMA        takes every iteration in order, parity-waits on full and on the
             decoder's hand-off, arrives on empty
A decoder that passes its wait while the stage does not hold iteration i's
data is a violation.  The ring rule of the kernel (S a multiple of G, a
static_assert in its Cfg) must never produce one; rings that break it must
produce some, which shows the model can see the failure.
"""
import random

import pytest


def run_ring(S: int, G: int, iters: int, seed: int) -> int:
    rng = random.Random(seed)
    full_done = [0] * S                 # completed phases of full(s)
    stage_tag = [-1] * S                # iteration whose data a stage holds
    dec_arr = [0] * S                   # decoder arrivals on empty(s)
    mma_arr = [0] * S                   # MMA arrivals on empty(s)
    next_fill = 0
    in_flight = []                      # fills issued, not landed
    dec_next = list(range(G))           # next iteration of each group
    dec_done = [False] * iters
    mma_next = 0
    violations = 0

    def passes(done: int, k: int) -> bool:      # mbarrier try_wait.parity for phase k
        return (done & 1) != (k & 1)

    while mma_next < iters:
        moves = []
        if next_fill < iters:
            s = next_fill % S
            if min(dec_arr[s], mma_arr[s]) >= next_fill // S:
                moves.append("issue")
        if in_flight:
            moves.append("land")
        for g in range(G):
            i = dec_next[g]
            if i < iters and passes(full_done[i % S], i // S):
                moves.append(("dec", g))
        if mma_next < iters and dec_done[mma_next] and passes(full_done[mma_next % S], mma_next // S):
            moves.append("mma")
        if not moves:
            return violations + 1000            # stuck: counted as a failure too
        mv = rng.choice(moves)
        if mv == "issue":
            in_flight.append(next_fill)
            next_fill += 1
        elif mv == "land":
            j = in_flight.pop(rng.randrange(len(in_flight)))    # any landing order
            stage_tag[j % S] = j
            full_done[j % S] += 1
        elif mv == "mma":
            mma_arr[mma_next % S] += 1
            mma_next += 1
        else:
            g = mv[1]
            i = dec_next[g]
            if stage_tag[i % S] != i:
                violations += 1
                return violations             # stale stage read: the race
            dec_done[i] = True
            dec_arr[i % S] += 1
            dec_next[g] += G
    return violations


@pytest.mark.parametrize("S,G", [(3, 3), (6, 3), (9, 3), (2, 2), (4, 2), (6, 2)])
def test_whole_round_rings_never_read_a_stale_stage(S, G):
    assert all(run_ring(S, G, 60, seed) == 0 for seed in range(400))


@pytest.mark.parametrize("S,G", [(4, 3), (5, 3), (7, 3), (10, 3)])
def test_other_rings_can_read_a_stale_stage(S, G):
    assert any(run_ring(S, G, 60, seed) > 0 for seed in range(400))
