"""CPU tests of the library's host logic and ABI (no GPU): every declared symbol is exported,
and a host-only pool makes exactly the oracle's allocation, policy and table decisions."""
import os
import re

import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import MkvError, Pool, api
from mixed_format_paged_mkv_b200.workloads import WORKLOADS
from oracle import pool as P

from harness import lib_pool, oracle_pool

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "mkv.h")).read()
    return re.findall(r"MKV_API\s+[\w\s\*]+?\b(mkv_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 20
    L = api.lib()
    for n in names:
        assert hasattr(L, n), n
        assert n in api.SIGNATURES, n
    assert set(api.SIGNATURES) == set(names)


def tables_equal(lp, op, n_seqs):
    for s in range(n_seqs):
        t, ctx = lp.block_table(s)
        assert t == op.block_table(s), s
        assert ctx == op.ctx[s]


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(B=3, ctx=(700, 1290, 1024))),
    (3, dict(B=5, ctx_range=(300, 2500), window=128, protect_frac=0.1)),
    (5, dict(B=6, ctx_range=(100, 900))),
])
def test_host_only_pool_matches_oracle_tables(cfg, kw):
    w = WORKLOADS[cfg].scaled(**kw)
    lp = lib_pool(w, host_only=True)
    op = oracle_pool(w) if cfg in (1,) else oracle_pool_tables_only(w)
    tables_equal(lp, op, w.B)
    live, n8, n3, _ = lp.stats()
    assert (live, n8, n3) == op.stats()[:3]


def oracle_pool_tables_only(w):
    # same replay with zero-valued inputs: tables do not depend on values
    shape = w.pool_shape()
    pool = P.RefPool(shape["num_kv_heads"], 32, shape["max_seqs"], shape["max_pages_per_seq"],
                     shape["fp8_slots"], shape["tq3_slots"])
    for fmt, key in ((P.FP8, "fp8_slots"), (P.TQ3, "tq3_slots")):
        order = w.slot_permutation(fmt, shape[key])
        if order is not None:
            pool.set_slot_order(fmt, order)
    for op in w.build_ops():
        if op[0] == "append":
            z = np.zeros((op[2], shape["num_kv_heads"], 32))
            pool.append([op[1]], [op[2]], z, z)
        elif op[0] == "protect":
            for p in op[2]:
                pool.set_protected(op[1], p, 1)
        else:
            pool.demote([op[1]], op[2])
    return pool


def test_steady_state_steps_match_oracle():
    rng = np.random.default_rng(0)
    lp = Pool(4, 128, 6, 64, 80, 200, host_only=True)
    op = P.RefPool(4, 32, 6, 64, 80, 200)
    lens = [37, 16, 1, 100, 0]
    lp.append([0, 1, 2, 3], lens[:4])
    op.append([0, 1, 2, 3], lens[:4], *(np.zeros((sum(lens), 4, 32)),) * 2)
    for step in range(60):
        seqs = [int(s) for s in rng.permutation(5)[:3]]
        n = [int(x) for x in rng.integers(0, 4, 3)]
        lp.append(seqs, n)
        op.append(seqs, n, *(np.zeros((sum(n), 4, 32)),) * 2)
        if step % 7 == 3:
            lp.set_protected(seqs[0], 0, True)
            op.set_protected(seqs[0], 0, 1)
        assert lp.demote(seqs, 24) == len(op.demote(seqs, 24))
        tables_equal(lp, op, 6)
    lp.copy(3, 5)
    op.seq_copy(3, 5)
    lp.reset(0)
    op.seq_reset(0)
    lp.append([0], [50])
    op.append([0], [50], *(np.zeros((50, 4, 32)),) * 2)
    tables_equal(lp, op, 6)


def test_errors_leave_pool_unchanged():
    lp = Pool(2, 128, 3, 4, 3, 2, host_only=True)
    lp.append([0], [20])
    before = lp.block_table(0)
    with pytest.raises(MkvError) as e:
        lp.append([7], [1])
    assert e.value.name == "BAD_SEQ"
    with pytest.raises(MkvError) as e:
        lp.append([0, 0], [1, 1])
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(MkvError) as e:
        lp.append([1], [40])            # 3 pages needed, 1 FP8 slot left
    assert e.value.name == "OUT_OF_PAGES"
    with pytest.raises(MkvError) as e:
        lp.append([0], [60])            # 5 pages > max_pages_per_seq 4
    assert e.value.name == "OUT_OF_PAGES"
    assert lp.block_table(0) == before and lp.block_table(1) == ([], 0)
    with pytest.raises(MkvError) as e:
        lp.workspace_bytes([1], 1, 2)
    assert e.value.name == "EMPTY_CONTEXT"
    with pytest.raises(MkvError) as e:
        lp.workspace_bytes([0], 5, 14)  # q_len * g = 35 > 32
    assert e.value.name == "UNSUPPORTED"
    with pytest.raises(MkvError) as e:
        lp.workspace_bytes([0], 1, 3)
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(MkvError) as e:
        lp.set_protected(0, 9, True)
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(MkvError) as e:
        lp.set_slot_order(0, [0, 0, 1])
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(MkvError) as e:
        Pool(2, 96, 1, 1, 1, 1, host_only=True)
    assert e.value.name == "UNSUPPORTED"
    with pytest.raises(MkvError) as e:
        Pool(1, 64, 1, 2 ** 27, 1, 1, host_only=True)   # 16 x pages would overflow int32 tokens
    assert e.value.name == "INVALID_ARG"
    Pool(1, 64, 1, 2 ** 27 - 1, 1, 1, host_only=True)
    lp.append([1], [16])                # FP8 slab now full (3 of 3)
    with pytest.raises(MkvError) as e:
        lp.append([2], [1])
    assert e.value.name == "OUT_OF_PAGES"
    assert lp.demote([0, 1], 0) == 0      # page 0 is a sink; page 1 of seq 0 is not full
    with pytest.raises(MkvError) as e:
        lp.copy(0, 1)
    assert e.value.name == "INVALID_ARG"
    lp2 = Pool(2, 128, 2, 8, 8, 1, host_only=True)
    lp2.append([0], [64])
    t0 = lp2.block_table(0)
    with pytest.raises(MkvError) as e:
        lp2.demote([0], 0)                 # 3 candidates, 1 TQ3 slot
    assert e.value.name == "OUT_OF_PAGES"
    assert lp2.block_table(0) == t0


def test_workspace_grows_with_context_and_is_small():
    lp = Pool(4, 256, 4, 9000, 9000, 9000, host_only=True)
    lp.append([0], [131072])
    lp.demote([0], 512)
    ws = lp.workspace_bytes([0], 1, 24)
    kv = 8192 * 4 * (14 * 256)  # TQ3 bytes of the sequence (upper bound)
    assert 0 < ws < 0.1 * kv      # no dense shadow: page lists and partial states only
    assert lp.workspace_bytes([0], 4, 24) > ws


def test_stats_footprint_formula():
    lp = Pool(4, 256, 1, 100, 100, 100, host_only=True)
    lp.append([0], [1600])
    lp.demote([0], 512)
    live, n8, n3, bpt = lp.stats()
    assert (live, n8, n3) == (1600, 1 + 32, 67)
    assert bpt == pytest.approx((33 * 4 * (32 * 256 + 16) + 67 * 4 * 14 * 256) / 1600)


@pytest.mark.parametrize("window,sink", [(0, 1), (48, 1), (1000, 1), (16, 0), (32, 3)])
def test_host_only_prefill_tables_match_oracle(window, sink):
    """Slot allocation of the direct prefill pack (pages ascending, each from its format's
    slab, sequences in list order) matches the oracle's block tables."""
    rng = np.random.default_rng(window + sink)
    lens = [0, 1, 15, 16, 17, 200, 333]
    Hkv, D = 2, 64
    lp = Pool(Hkv, D, len(lens) + 1, 32, 80, 80, sink_pages=sink, host_only=True)
    op = P.RefPool(Hkv, D, len(lens) + 1, 32, 80, 80, sink_pages=sink)
    for fmt in (0, 1):
        order = rng.permutation(80).astype(np.int32)
        lp.set_slot_order(fmt, order)
        op.set_slot_order(fmt, order)
    lp.append([len(lens)], [5])
    op.append([len(lens)], [5], np.zeros((5, Hkv, D)), np.zeros((5, Hkv, D)))
    seqs = list(range(len(lens)))
    lp.prefill(seqs, lens, window=window)
    x = np.zeros((sum(lens), Hkv, D))
    op.prefill(seqs, lens, x, x, window)
    for s in seqs + [len(lens)]:
        t, ctx = lp.block_table(s)
        assert t == op.block_table(s) and ctx == op.ctx[s], s
    with pytest.raises(MkvError) as e:
        lp.prefill([len(lens)], [16], window=0)          # not empty
    assert e.value.name == "INVALID_ARG"


def test_prefill_and_materialise_errors_leave_the_pool_unchanged():
    lp = Pool(1, 64, 3, 8, 3, 8, host_only=True)
    op = P.RefPool(1, 64, 3, 8, 3, 8)
    with pytest.raises(MkvError) as e:
        lp.prefill([0], [16], window=-1)
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(MkvError) as e:
        lp.prefill([0, 0], [16, 16], window=0)
    assert e.value.name == "INVALID_ARG"
    # 100 tokens, window 100: all 7 pages stay FP8, 3 FP8 slots -> nothing may change
    with pytest.raises(MkvError) as e:
        lp.prefill([1], [100], window=100)
    assert e.value.name == "OUT_OF_PAGES"
    assert lp.block_table(1) == ([], 0)
    # the same call with window 0 packs pages 1..5 to TQ3 and keeps page 0 and the partial
    # page 6 as FP8
    lp.prefill([1], [100], window=0)
    x = np.zeros((100, 1, 64))
    op.prefill([1], [100], x, x, 0)
    assert lp.block_table(1) == (op.block_table(1), 100)
    assert [e >> 30 for e in lp.block_table(1)[0]] == [0, 1, 1, 1, 1, 1, 0]
    with pytest.raises(MkvError) as e:
        lp.materialise(1)
    assert e.value.name == "INVALID_ARG"
