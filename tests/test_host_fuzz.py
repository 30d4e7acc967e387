"""Differential test of the host logic: random streams of pool operations applied to a host-only
library pool and to the oracle's pool must give the same block tables, lengths, footprint and
demotion counts after every operation, and the same error (with nothing changed) whenever one of
them rejects an operation.

The streams mix appends of random sizes (sometimes over a sequence's page limit or the FP8
slab), protection flags, demotions with random windows, prefill of empty sequences, copies,
resets and new slot orders, with repeated and out-of-range sequence ids among them.  Every
tenth step the decode cut of the live sequences is checked as in test_plan."""
import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import MkvError, Pool
from oracle import pool as P

from test_plan import check_cut

LAST_OP = [None]   # named in assertion messages


def state(lp, op, n_seqs):
    for s in range(n_seqs):
        t, ctx = lp.block_table(s)
        assert t == op.block_table(s), s
        assert ctx == op.ctx[s], s
    live, n8, n3, bpt = lp.stats()
    olive, on8, on3, obpt = op.stats()
    assert (live, n8, n3) == (olive, on8, on3)
    assert bpt == pytest.approx(obpt, rel=1e-12, abs=0)


def both(fn_lib, fn_ora):
    """Run the operation on both pools; they must agree on success or on the error code."""
    err_l = err_o = None
    res_l = res_o = None
    try:
        res_l = fn_lib()
    except MkvError as e:
        err_l = e.name
    try:
        res_o = fn_ora()
    except P.PoolError as e:
        err_o = e.code
    assert err_l == err_o, (err_l, err_o, LAST_OP[0])
    return res_l, res_o, err_l


@pytest.mark.parametrize("seed", range(8))
def test_random_operation_streams_match_the_oracle(seed):
    HKV, D = [(1, 64), (2, 128), (4, 256)][seed % 3]
    rng = np.random.default_rng(1000 + seed)
    n_seqs = int(rng.integers(2, 6))
    max_pages = int(rng.integers(3, 12))
    fp8_slots = int(rng.integers(4, 3 * max_pages))
    tq3_slots = int(rng.integers(0, 3 * max_pages))
    sink = int(rng.integers(0, 3))
    lp = Pool(HKV, D, n_seqs, max_pages, fp8_slots, tq3_slots, sink_pages=sink, host_only=True)
    op = P.RefPool(HKV, D, n_seqs, max_pages, fp8_slots, tq3_slots, sink_pages=sink)
    if rng.random() < 0.5:
        for fmt, n in ((P.FP8, fp8_slots), (P.TQ3, tq3_slots)):
            order = rng.permutation(n).tolist()
            lp.set_slot_order(fmt, order)
            op.set_slot_order(fmt, order)
    seq_pool = list(range(n_seqs)) + [n_seqs]          # one id out of range

    def seqs():
        k = int(rng.integers(1, 4))
        ids = [int(x) for x in rng.choice(seq_pool, size=k)]
        if rng.random() < 0.8:                            # mostly distinct and in range
            ids = sorted(set(i for i in ids if i < n_seqs)) or [0]
        return ids

    for step in range(250):
        kind = rng.choice(["append", "append", "append", "protect", "demote", "demote",
                           "prefill", "copy", "reset", "order"])
        LAST_OP[0] = kind
        if kind == "append":
            ids = seqs()
            counts = [int(rng.integers(0, 40)) for _ in ids]
            if rng.random() < 0.05:
                counts[0] = -1
            rows = max(sum(c for c in counts if c > 0), 0)
            z = np.zeros((rows, HKV, D))
            both(lambda: lp.append(ids, counts), lambda: op.append(ids, counts, z, z))
        elif kind == "protect":
            s = int(rng.integers(0, n_seqs))
            page = int(rng.integers(-1, max_pages + 1))
            flag = int(rng.integers(0, 2))
            both(lambda: lp.set_protected(s, page, flag), lambda: op.set_protected(s, page, flag))
        elif kind == "demote":
            ids = seqs()
            W = int(rng.choice([0, 16, 40, 100, -1 if rng.random() < 0.05 else 64]))
            nl, no, err = both(lambda: lp.demote(ids, W), lambda: op.demote(ids, W))
            if err is None:
                assert nl == len(no)
        elif kind == "prefill":
            ids = seqs()
            counts = [int(rng.integers(0, 80)) for _ in ids]
            W = int(rng.choice([0, 16, 64]))
            rows = max(sum(c for c in counts if c > 0), 0)
            z = np.zeros((rows, HKV, D))
            both(lambda: lp.prefill(ids, counts, window=W), lambda: op.prefill(ids, counts, z, z, W))
        elif kind == "copy":
            src, dst = (int(x) for x in rng.integers(0, n_seqs, size=2))
            both(lambda: lp.copy(src, dst), lambda: op.seq_copy(src, dst))
        elif kind == "reset":
            s = int(rng.integers(0, n_seqs))
            both(lambda: lp.reset(s), lambda: op.seq_reset(s))
        else:
            fmt, n = (P.FP8, fp8_slots) if rng.random() < 0.5 else (P.TQ3, tq3_slots)
            order = rng.permutation(n).tolist()
            if n > 1 and rng.random() < 0.1:
                order[0] = order[1]                       # not a permutation
            both(lambda: lp.set_slot_order(fmt, order), lambda: op.set_slot_order(fmt, order))
        state(lp, op, n_seqs)
        if step % 10 == 9:
            # the decode cut of every non-empty sequence covers its pages once
            live = [q for q in range(n_seqs) if op.ctx[q] > 0]
            if live:
                units, wave = lp.decode_plan(live, 1, HKV)
                check_cut(lp, live, units, wave, HKV)
