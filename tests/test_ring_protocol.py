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


def run_a_ring(A: int, G: int, iters: int, seed: int) -> int:
    """The TMEM A-slot ring: decoder group g writes slot i mod A for its
    iterations i = g (mod G) after a parity wait on aempty; the MMA reads the
    slots in order and its commits complete in issue order, at random times.
    Returns the number of overwrites of a slot an unfinished MMA still reads
    (or of reads of a slot that does not hold the MMA's iteration)."""
    rng = random.Random(seed)
    aempty_done = [0] * A               # completed phases of aempty(a)
    slot_tag = [-1] * A                 # iteration whose weights a slot holds
    dec_next = list(range(G))
    written = [False] * iters
    mma_next = 0                        # next iteration the MMA issues
    mma_done = 0                        # MMAs completed (in issue order)
    bad = 0

    def passes(done: int, k: int) -> bool:
        return (done & 1) != (k & 1)

    while mma_done < iters:
        moves = []
        for g in range(G):
            i = dec_next[g]
            # the wait for the slot's previous use (iteration i - A): phase i//A - 1
            if i < iters and passes(aempty_done[i % A], i // A - 1):
                moves.append(("dec", g))
        if mma_next < iters and written[mma_next]:
            moves.append("issue")
        if mma_done < mma_next:
            moves.append("complete")
        if not moves:
            return bad + 1000
        mv = rng.choice(moves)
        if mv == "issue":
            if slot_tag[mma_next % A] != mma_next:
                bad += 1
            mma_next += 1
        elif mv == "complete":
            aempty_done[mma_done % A] += 1
            mma_done += 1
        else:
            g = mv[1]
            i = dec_next[g]
            if i - A >= 0 and mma_done <= i - A:       # previous user of the slot still in flight
                bad += 1
            slot_tag[i % A] = i
            written[i] = True
            dec_next[g] += G
    return bad


@pytest.mark.parametrize("A,G", [(3, 3), (4, 3), (7, 3), (2, 2), (3, 2)])
def test_a_ring_at_least_as_deep_as_the_groups_is_safe(A, G):
    assert all(run_a_ring(A, G, 60, seed) == 0 for seed in range(400))


@pytest.mark.parametrize("A,G", [(2, 3), (1, 2)])
def test_a_ring_shallower_than_the_groups_is_not(A, G):
    assert any(run_a_ring(A, G, 60, seed) > 0 for seed in range(400))


def run_split_ring(S: int, G: int, iters: int, seed: int, pre: int) -> int:
    """The stage ring with a stage's codes and activations on separate
    barriers: code(s) completes when the codes land (decoder group g parity-
    waits on it for its iterations i = g mod G), full(s) when the activation
    boxes land (the MMA parity-waits on it, in order, after the decoders'
    hand-off).  The two copies of a fill land independently, in any order
    across stages.  The codes of the first `pre` iterations are issued before
    anything else may move (before the dependency wait); their activation
    boxes, and every later fill, only once empty(s) saw both the decoders'
    and the MMA's arrivals for the stage's previous round.  Returns the
    number of stale reads (a waiter passing while the stage holds another
    iteration's codes or activations); 1000 more if the model gets stuck."""
    rng = random.Random(seed)
    code_done = [0] * S
    act_done = [0] * S
    code_tag = [-1] * S
    act_tag = [-1] * S
    dec_arr = [0] * S
    mma_arr = [0] * S
    in_code, in_act = [], []
    next_code = min(pre, S, iters)      # codes already issued before the wait
    in_code.extend(range(next_code))
    next_act = 0
    dec_next = list(range(G))
    dec_done = [False] * iters
    mma_next = 0
    bad = 0

    def passes(done: int, k: int) -> bool:
        return (done & 1) != (k & 1)

    while mma_next < iters:
        moves = []
        # a fill (codes + activations, or activations alone for a pre-issued
        # iteration) once the stage's previous round is released
        j = next_act
        if j < iters and min(dec_arr[j % S], mma_arr[j % S]) >= j // S:
            moves.append("fill")
        if in_code:
            moves.append("land_code")
        if in_act:
            moves.append("land_act")
        for g in range(G):
            i = dec_next[g]
            if i < iters and passes(code_done[i % S], i // S):
                moves.append(("dec", g))
        if mma_next < iters and dec_done[mma_next] and passes(act_done[mma_next % S], mma_next // S):
            moves.append("mma")
        if not moves:
            return bad + 1000
        mv = rng.choice(moves)
        if mv == "fill":
            if j >= next_code:
                in_code.append(j)
                next_code = j + 1
            in_act.append(j)
            next_act += 1
        elif mv == "land_code":
            c = in_code.pop(rng.randrange(len(in_code)))
            code_tag[c % S] = c
            code_done[c % S] += 1
        elif mv == "land_act":
            a = in_act.pop(rng.randrange(len(in_act)))
            act_tag[a % S] = a
            act_done[a % S] += 1
        elif mv == "mma":
            if act_tag[mma_next % S] != mma_next:
                bad += 1
            mma_arr[mma_next % S] += 1
            mma_next += 1
        else:
            g = mv[1]
            i = dec_next[g]
            if code_tag[i % S] != i:
                bad += 1
            dec_done[i] = True
            dec_arr[i % S] += 1
            dec_next[g] += G
    return bad


@pytest.mark.parametrize("S,G", [(3, 3), (6, 3), (9, 3), (2, 2), (4, 2), (6, 2)])
@pytest.mark.parametrize("pre", [0, 1, 100])
def test_split_barrier_rings_never_read_a_stale_stage(S, G, pre):
    assert all(run_split_ring(S, G, 60, seed, pre) == 0 for seed in range(300))


@pytest.mark.parametrize("S,G", [(4, 3), (5, 3), (7, 3)])
def test_split_barrier_rings_off_whole_rounds_can(S, G):
    assert any(run_split_ring(S, G, 60, seed, 100) > 0 for seed in range(400))
