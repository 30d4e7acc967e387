"""The decode work-unit cut (mkv_decode_plan) on host-only pools.

The cut is host logic.  A grid's pages -- every sequence's pages of its format (or of both, for
the fused grid), in call order -- form a line that is cut into CTAs of equal cost; a CTA takes one
unit (pages of one format inside a logical page range of one sequence) per sequence its share
touches.  These tests check what any correct cut must satisfy -- each page of a format in exactly
one unit of that format, TQ3 ranges tiling each table in logical order, the page limits per unit,
the one-wave budget, units listed CTA by CTA -- and that the costliest CTA is within a few pages of
the average.
"""
import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import Pool

FP8, TQ3 = 0, 1
MAX_PAGES, MIN_PAGES = 512, {FP8: 4, TQ3: 8}
PAGE_COST = {FP8: 11, TQ3: 10}   # relative time of one page per CTA, as the planner weighs them
UNIT_COST = 60                   # and of starting a unit
LINE_CUT_BELOW = 0.85            # the line cut replaces a per-group cut this far from balance
FP8_RUN_GAP = 2048               # FP8 pages farther apart than this start a new run


def mixed_pool(lens, Hkv=4, sink=1, window=64, protect_frac=0.03, seed=0):
    """Host-only pool whose sequences hold FP8 anchors (sink pages, the window, random protected
    pages) among TQ3 pages."""
    rng = np.random.default_rng(seed)
    pages = [-(-n // 16) for n in lens]
    pool = Pool(Hkv, 128, len(lens), max(pages) + 1, sum(pages) + 8, sum(pages) + 8,
                sink_pages=sink, host_only=True)
    seqs = list(range(len(lens)))
    pool.append(seqs, list(lens))
    for s, n in zip(seqs, pages):
        for p in rng.choice(n, size=int(protect_frac * n), replace=False):
            pool.set_protected(s, int(p), True)
    pool.demote(seqs, window)
    return pool, seqs


def formats(pool, s):
    table, _ = pool.block_table(s)
    return np.array([e >> 30 for e in table])


def check_cut(pool, seqs, units, wave, Hkv):
    units = np.asarray(units)
    assert units.ndim == 2 and units.shape[1] == 6
    cta = units[:, 5]
    # CTA by CTA, numbered 0, 1, 2, ... with at least one unit each
    assert cta[0] == 0 and np.all(np.diff(cta) >= 0) and np.all(np.diff(cta) <= 1)
    for pos, s in enumerate(seqs):
        fm = formats(pool, s)
        mine = units[units[:, 0] == pos]
        for f in (FP8, TQ3):
            idx = np.nonzero(fm == f)[0]
            us = mine[mine[:, 1] == f]
            if idx.size == 0:
                assert us.size == 0
                continue
            us = us[np.argsort(us[:, 2], kind="stable")]
            # runs: FP8 pages split where the gap exceeds FP8_RUN_GAP pages; TQ3 pages form one
            run = np.zeros(idx.size, dtype=np.int64)
            if f == FP8:
                run[1:] = np.cumsum(np.diff(idx) > FP8_RUN_GAP)
            covered = []
            for _, _, first, end, cnt, _ in us:
                inside = idx[(idx >= first) & (idx < end)]
                assert inside.size == cnt > 0
                r = run[np.searchsorted(idx, inside[0])]
                assert cnt <= MAX_PAGES and cnt >= min(MIN_PAGES[f], int((run == r).sum()))
                covered.extend(inside.tolist())
            assert covered == idx.tolist(), f"seq {s} fmt {f}: pages not covered exactly once"
            if f == TQ3:
                # ranges tile the table; each after the first starts on a TQ3 page
                assert us[0, 2] == 0 and us[-1, 3] == fm.size
                assert np.array_equal(us[1:, 2], us[:-1, 3])
                assert np.all(fm[us[1:, 2]] == TQ3)
            else:
                # ranges start and end on FP8 pages
                assert np.all(fm[us[:, 2]] == FP8) and np.all(fm[us[:, 3] - 1] == FP8)
    n_ctas = int(cta[-1]) + 1
    budget = max(1, wave // Hkv)
    min_units = 0   # at least one unit per group and per 512 pages
    for s in seqs:
        fm = formats(pool, s)
        for f in (FP8, TQ3):
            min_units += -(-int((fm == f).sum()) // MAX_PAGES)
    if len(seqs) <= 256 and min_units <= budget:
        assert n_ctas <= budget, (n_ctas, budget)
    return units


def cta_costs(units):
    """Cost of each CTA as the planner weighs it: its pages, and a unit cost for every unit
    that starts a run (the planner charges a run's start once, to the CTA that starts it; a
    unit that continues a run another CTA started costs that CTA nothing extra here)."""
    units = np.asarray(units)
    cost = units[:, 4] * np.where(units[:, 1] == TQ3, PAGE_COST[TQ3], PAGE_COST[FP8])
    return np.bincount(units[:, 5], weights=cost)


@pytest.mark.parametrize("lens,Hkv,window", [
    ((131072,) * 4, 4, 512),
    ((8192,) * 8, 8, 256),
    ((2048, 32768, 5000, 17, 16, 4, 900, 12000), 4, 512),
    ((65536, 100, 40000), 2, 64),
])
def test_cut_covers_every_page_once_within_one_wave(lens, Hkv, window):
    pool, seqs = mixed_pool(lens, Hkv=Hkv, window=window, seed=len(lens))
    for q_len in (1, 4):
        units, wave = pool.decode_plan(seqs, q_len, 2 * Hkv)
        check_cut(pool, seqs, units, wave, Hkv)


@pytest.mark.parametrize("seed", range(8))
def test_ctas_are_balanced(seed):
    """The costliest CTA is within a few pages of the line's average: a cut point moves at most
    a few pages to keep units from being shorter than the minimum, and a CTA has two."""
    rng = np.random.default_rng(100 + seed)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    lens = rng.integers(16, 40000, size=int(rng.integers(1, 40))).tolist()
    pool, seqs = mixed_pool(lens, Hkv=Hkv, window=int(rng.choice([0, 64, 512])),
                            protect_frac=float(rng.choice([0.0, 0.05, 0.3])), seed=seed)
    units, wave = pool.decode_plan(seqs, 1, Hkv)
    units = check_cut(pool, seqs, units, wave, Hkv)
    costs = cta_costs(units)
    U = max(1, wave // Hkv)
    if units[-1, 5] + 1 > U:
        return  # more groups than the wave holds: one unit per group, the scheduler balances
    total_pages = int(units[:, 4].sum())
    k = max(1, min(U, total_pages // MIN_PAGES[TQ3]))
    runs = n_runs(pool, seqs)
    slack = 2 * MIN_PAGES[TQ3] * PAGE_COST[FP8] + PAGE_COST[FP8]
    # the per-group cut where its longest unit is within 1 / 0.85 of the average, else the
    # line cut, within a few pages of it
    bound = max(costs.sum() / U / LINE_CUT_BELOW + PAGE_COST[FP8],
                (costs.sum() + runs * UNIT_COST) / k + slack)
    assert costs.max() <= bound, (costs.max(), costs.sum() / U)


def n_runs(pool, seqs):
    total = 0
    for s in seqs:
        fm = formats(pool, s)
        idx = np.nonzero(fm == FP8)[0]
        total += (idx.size > 0) + int((np.diff(idx) > FP8_RUN_GAP).sum()) + int((fm == TQ3).any())
    return total


def test_a_ragged_batch_fills_the_wave_evenly():
    """32 sequences of 2K-32K tokens in a wave of 148 CTAs: cutting each sequence into whole
    shares would leave the longest CTA far above the average, so the planner takes the line cut,
    whose CTAs (some starting several units) stay within a few pages of it."""
    rng = np.random.default_rng(7)
    lens = rng.integers(2048, 32769, size=32).tolist()
    pool, seqs = mixed_pool(lens, Hkv=1, window=512, protect_frac=0.02, seed=7)
    units, wave = pool.decode_plan(seqs, 1, 6)
    units = check_cut(pool, seqs, units, wave, 1)
    costs = cta_costs(units)
    assert len(costs) == wave and np.bincount(units[:, 5]).max() >= 2
    assert costs.max() <= 1.05 * costs.mean() + 2 * MIN_PAGES[TQ3] * PAGE_COST[FP8] + UNIT_COST


def test_one_long_tq3_run_splits_evenly():
    pool, seqs = mixed_pool((16 * 8192,), Hkv=4, window=0, protect_frac=0.0)
    units, wave = pool.decode_plan(seqs, 1, 4)
    units = check_cut(pool, seqs, units, wave, 4)
    tq3 = units[units[:, 1] == TQ3]
    budget = wave // 4
    assert units[-1, 5] + 1 <= budget
    # the first CTA also holds the FP8 page 0; every other takes an equal TQ3 share
    assert tq3[1:, 4].max() - tq3[1:, 4].min() <= 1 and tq3[:, 4].sum() == 8191


def test_call_positions_beyond_int16():
    n = 33000
    pool = Pool(1, 64, n, 1, n, 1, host_only=True)
    seqs = list(range(n))[::-1]
    pool.append(seqs, [16] * n)
    units, _ = pool.decode_plan(seqs, 1, 1)
    assert units.shape == (n, 6)
    assert np.array_equal(units[:, 0], np.arange(n))
    assert np.all(units[:, 1:5] == [FP8, 0, 1, 1])
    # launches of at most 256 sequences, CTA numbers running on across them
    assert units[0, 5] == 0 and np.all(np.diff(units[:, 5]) >= 0)


def test_plan_count_query_and_small_buffer():
    from mixed_format_paged_mkv_b200.api import MkvError, lib, _I32P
    import ctypes
    pool, seqs = mixed_pool((4096, 4096), Hkv=2)
    units, _ = pool.decode_plan(seqs, 1, 2)
    assert len(units) > 1
    s = np.array(seqs, dtype=np.int32)
    buf = np.zeros((len(units) - 1, 6), dtype=np.int32)
    n = ctypes.c_int32()
    rc = lib().mkv_decode_plan(pool.handle, s.ctypes.data_as(_I32P), s.size, 1, 2,
                               buf.ctypes.data_as(_I32P), len(units) - 1, ctypes.byref(n), None)
    assert rc == -1 and n.value == len(units) and not buf.any()
    with pytest.raises(MkvError):
        pool.decode_plan(seqs, 1, 3)          # 3 query heads over 2 KV heads
    with pytest.raises(MkvError):
        pool.decode_plan([0, 0, 5], 1, 2)     # sequence outside the pool


def test_a_sequence_beyond_one_launch_is_rejected():
    # 512 pages per unit at most and 1536 units per launch: a sequence of 786,433+ pages of one
    # format cannot be decoded in one launch group, and the planner says so up front
    pages = 1536 * 512 + 1
    pool = Pool(1, 64, 1, pages, pages, 1, host_only=True)
    pool.append([0], [16 * pages])
    from mixed_format_paged_mkv_b200.api import MkvError
    with pytest.raises(MkvError) as e:
        pool.decode_plan([0], 1, 1)
    assert e.value.name == "UNSUPPORTED"
    pool.reset(0)
    pool.append([0], [16 * (pages - 1)])
    units, _ = pool.decode_plan([0], 1, 1)
    assert len(units) == 1536 and units[:, 4].max() == 512



def test_decode_sms_caps_the_wave():
    """set_decode_sms plans the cut for fewer SMs: the CTA budget of the wave shrinks with it and
    the cut still covers every page once."""
    pool, seqs = mixed_pool((16 * 8192, 5000), Hkv=2, window=64)
    units, wave = pool.decode_plan(seqs, 1, 2)
    pool.set_decode_sms(8)
    small, small_wave = pool.decode_plan(seqs, 1, 2)
    assert small_wave <= wave and small_wave <= 8 * 8
    check_cut(pool, seqs, small, small_wave, 2)
    assert len(small) <= len(units)
    pool.set_decode_sms(0)
    assert pool.decode_plan(seqs, 1, 2)[1] == wave
    from mixed_format_paged_mkv_b200.api import MkvError
    with pytest.raises(MkvError):
        pool.set_decode_sms(-1)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("sms", [1, 2, 3])
def test_tiny_wave_still_covers_both_formats(fused, sms):
    """A wave of one or two CTAs per KV head: each grid still gets a CTA, so both formats'
    pages are covered."""
    pool, seqs = mixed_pool((3000, 700, 45, 1600), Hkv=4, window=64, protect_frac=0.1)
    pool.set_decode_kernels(fused)
    pool.set_decode_sms(sms)
    units, wave = pool.decode_plan(seqs, 1, 4)
    check_cut(pool, seqs, units, max(wave, 2 * 4), 4)
    assert set(units[:, 1].tolist()) == {FP8, TQ3}


def test_launches_split_where_units_would_overflow():
    """200 sequences of 4000 pages need at least 8 units of at most 512 pages each: the call is
    planned as launches of at most 1536 units (192 sequences, then the other 8, which fit one
    wave and get finer units); CTA numbers run on across launches."""
    n, pages = 200, 4000
    pool = Pool(1, 64, n, pages, n * pages, 1, host_only=True)
    seqs = list(range(n))
    pool.append(seqs, [16 * pages] * n)
    units, wave = pool.decode_plan(seqs, 1, 1)
    assert units[:, 4].max() <= MAX_PAGES
    first = units[units[:, 0] < 192]
    assert len(first) == 192 * 8 and first[-1, 5] + 1 == 192 * 8
    check_cut(pool, seqs, units, wave, 1)
