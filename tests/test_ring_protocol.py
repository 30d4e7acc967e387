"""Model check of the decode kernel's page ring (CPU).

The partial-attention kernel streams pages through NST shared-memory stages: the producer
fills page i into stage i % NST once page i - NST has been released; consumer warp w takes
pages w, w + PW, ...; a consumer waits for fill f = i // NST of its stage with an mbarrier
parity wait on f & 1.  A parity wait cannot tell fill f from fill f - 2: it returns at once
whenever the barrier's completed-phase count has the other parity -- including when fill
f - 1 has not completed yet.  The kernel therefore requires that fill f - 1 of a stage was
consumed by the same warp (NST a multiple of PW), so it has always completed.  This test
replays random interleavings and checks that no wait is ever ambiguous for the ring shapes
the kernel uses, and that a shape violating the rule is caught."""
import random

import pytest

# (stages, page-parallel warps): FP8 and TQ3 rings for 1, 2 and 4 warps per n-tile
KERNEL_RINGS = [(8, 4), (16, 4), (8, 2), (16, 2), (8, 1), (16, 1)]


def replay(count, nst, pw, seed):
    """Random interleaving; returns True if some consumer started a wait for fill f of a stage
    whose fill f-1 had not completed (an ambiguous parity wait)."""
    rng = random.Random(seed)
    completed = [0] * nst        # completed fills per stage
    released = [False] * count
    issued = 0
    in_flight = []               # pages copied but not landed
    nxt = list(range(pw))        # next page of each consumer warp
    ambiguous = False
    waiting = {}
    while not all(released):
        moves = []
        if issued < count and (issued < nst or released[issued - nst]):
            moves.append("issue")
        if in_flight:
            moves.append("land")
        for w in range(pw):
            if nxt[w] < count:
                moves.append(w)
        if not moves:
            raise AssertionError("deadlock")
        m = rng.choice(moves)
        if m == "issue":
            in_flight.append(issued)
            issued += 1
        elif m == "land":
            i = in_flight.pop(rng.randrange(len(in_flight)))
            completed[i % nst] += 1
        else:
            i = nxt[m]
            s, f = i % nst, i // nst
            if m not in waiting:
                waiting[m] = i
                if completed[s] < f:          # fill f-1 not complete: parity is ambiguous
                    ambiguous = True
            if completed[s] > f:              # fill f complete: consume and release
                released[i] = True
                nxt[m] += pw
                del waiting[m]
    return ambiguous


@pytest.mark.parametrize("nst,pw", KERNEL_RINGS)
def test_kernel_rings_never_wait_ambiguously(nst, pw):
    for seed in range(60):
        for count in (1, 5, nst - 1, nst, nst + 3, 3 * nst + 1, 45):
            assert not replay(count, nst, pw, seed), (nst, pw, count, seed)


def test_ring_shape_that_violates_the_rule_is_detected():
    # six stages shared by four warps: some stage is consumed by two different warps
    assert any(replay(45, 6, 4, seed) for seed in range(200))
