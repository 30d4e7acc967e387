"""Model check of the decode kernel's page ring (CPU).

The partial-attention kernel streams pages through NST shared-memory stages: the producer
fills page i into stage i % NST once page i - NST has been released; consumer warp w takes
pages w, w + PW, ...; a consumer waits for fill f = i // NST of its stage with an mbarrier
parity wait on f & 1.  A parity wait cannot tell fill f from fill f - 2: it returns at once
whenever the barrier's completed-phase count has the other parity -- including when fill
f - 1 has not completed yet.  The kernel therefore requires that fill f - 1 of a stage was
consumed by the same warp (NST a multiple of PW), so it has always completed.  This test
replays random interleavings and checks that no wait is ever ambiguous for the ring shapes
the kernel uses, that a shape violating the rule is caught, and that a unit ends with every copy
landed and consumed (so a CTA can re-initialise its barriers for its next unit)."""
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
    # a unit ends with no copy in flight and every copy consumed: the kernel may then
    # invalidate and re-initialise the stage barriers for the CTA's next unit
    assert issued == count and not in_flight and not waiting
    return ambiguous


@pytest.mark.parametrize("nst,pw", KERNEL_RINGS)
def test_kernel_rings_never_wait_ambiguously(nst, pw):
    for seed in range(60):
        for count in (1, 5, nst - 1, nst, nst + 3, 3 * nst + 1, 45):
            assert not replay(count, nst, pw, seed), (nst, pw, count, seed)


def test_ring_shape_that_violates_the_rule_is_detected():
    # six stages shared by four warps: some stage is consumed by two different warps
    assert any(replay(45, 6, 4, seed) for seed in range(200))


def replay_team(count, nst, tw, seed):
    """Team layout (more than 8 query columns): pages go in batches of tw; warp w first waits
    for page b + w of batch b (its K page), then all warps meet at the batch barrier, then every
    warp consumes every page of the batch (V) without waiting: the K warps' waits before the
    barrier cover them, which the model asserts.  A batch's stages are released at the next
    batch's barrier (every warp has consumed them by then) and refilled with the pages nst
    ahead.  Returns True if some wait started for fill f of a stage whose fill f-1 had not
    completed."""
    rng = random.Random(seed)
    completed = [0] * nst
    releases = [0] * count
    issued = 0
    in_flight = []
    batch = [0] * tw           # first page of each warp's current batch
    step = ["k"] * tw          # "k": K page, "bar": at the barrier, int q: V page b + q
    waiting = [None] * tw
    ambiguous = False

    def start_wait(w, i):
        nonlocal ambiguous
        if waiting[w] != i:
            waiting[w] = i
            if completed[i % nst] < i // nst:
                ambiguous = True
        return completed[i % nst] > i // nst

    while any(b < count for b in batch):
        moves = []
        if issued < count and (issued < nst or releases[issued - nst] == tw):
            moves.append("issue")
        if in_flight:
            moves.append("land")
        arrived = [w for w in range(tw) if step[w] == "bar"]
        if len(arrived) == tw:
            moves.append("barrier")
        ready = []                 # warps whose wait would end (or who have no K page)
        for w in range(tw):
            if batch[w] < count and step[w] != "bar":
                moves.append(w)
                i = batch[w] + (w if step[w] == "k" else step[w])
                if step[w] != "k" or i >= count or completed[i % nst] > i // nst:
                    ready.append(w)
        if not (ready or "issue" in moves or "land" in moves or "barrier" in moves):
            raise AssertionError("deadlock")
        m = rng.choice(moves)
        if m == "issue":
            in_flight.append(issued)
            issued += 1
        elif m == "land":
            i = in_flight.pop(rng.randrange(len(in_flight)))
            completed[i % nst] += 1
        elif m == "barrier":
            b = batch[0]
            for i in range(max(0, b - tw), min(b, count)):   # the previous batch is released
                releases[i] = tw
            step = [0] * tw
        else:
            w, b = m, batch[m]
            if step[w] == "k":
                i = b + w
                if i >= count or start_wait(w, i):
                    waiting[w] = None
                    step[w] = "bar"
            else:
                i = b + step[w]
                # a V read: the page's K warp saw its copy complete before the barrier
                assert completed[i % nst] > i // nst, "V read of a page not yet landed"
                step[w] += 1
                if step[w] == min(tw, count - b):
                    batch[w] += tw
                    step[w] = "k"
    assert issued == count and not in_flight   # as above: the barriers can be re-initialised
    return ambiguous


@pytest.mark.parametrize("nst,tw", [(8, 4), (4, 2), (8, 2)])   # the kernel's team rings
def test_team_ring_never_waits_ambiguously(nst, tw):
    for seed in range(60):
        for count in (1, 3, tw, nst - 1, nst, nst + 3, 3 * nst + 1, 45):
            assert not replay_team(count, nst, tw, seed), (nst, tw, count, seed)


def test_team_ring_needs_a_stage_per_page_of_a_batch():
    # Every warp consumes every page, so a warp never waits on a fill whose predecessor it has
    # not consumed itself.  Stages are released a batch late, so the ring needs two batches:
    # with one, a K page waits for a stage released only at the barrier that K page gates, and
    # the model reports the deadlock.
    assert not any(replay_team(45, 8, 4, seed) for seed in range(100))
    with pytest.raises(AssertionError, match="deadlock"):
        for seed in range(20):
            replay_team(45, 4, 4, seed)
