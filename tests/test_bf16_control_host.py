"""Host logic of the BF16 control pool (CPU, host-only pools): the library makes the oracle's
table, allocation and footprint decisions -- every page BF16, nothing ever demoted."""
import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import MkvError, Pool
from mixed_format_paged_mkv_b200.workloads import WORKLOADS
from oracle import pool as P

from harness import lib_pool, oracle_pool


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (3, dict(B=4, ctx_range=(300, 2500), window=128, protect_frac=0.1)),
])
def test_control_pool_tables_match_oracle(cfg, kw):
    w = WORKLOADS[cfg].scaled(**kw)
    shape = dict(w.pool_shape(), fp8_slots=sum(w.pages()) + 8)  # every page stays in slab 0
    lp = lib_pool(w, shape=shape, host_only=True, bf16_control=True)
    op = oracle_pool(w, shape=shape, bf16_control=True)
    for s in range(w.B):
        t, ctx = lp.block_table(s)
        assert t == op.block_table(s) and ctx == op.ctx[s]
        assert all((e >> 30) & 3 == P.BF16 for e in t)
    live, n8, n3, bpt = lp.stats()
    assert (live, n8, n3) == op.stats()[:3] and n3 == 0
    assert bpt == pytest.approx(op.stats()[3])


def test_control_pool_never_demotes_and_copies_prefills_resets():
    lp = Pool(2, 64, 4, 64, 200, 0, host_only=True, bf16_control=True)
    op = P.RefPool(2, 64, 4, 64, 200, 0, bf16_control=True)
    z = np.zeros((900, 2, 64))
    lp.append([0], [900])
    op.append([0], [900], z, z)
    assert lp.demote([0], 0) == 0 and op.demote([0], 0) == []
    lp.prefill([1], [500], window=0)
    op.prefill([1], [500], z[:500], z[:500], 0)
    lp.copy(0, 2)
    op.seq_copy(0, 2)
    lp.reset(1)
    op.seq_reset(1)
    lp.append([3], [17])
    op.append([3], [17], z[:17], z[:17])
    for s in range(4):
        assert lp.block_table(s)[0] == op.block_table(s)
    assert lp.slot_bytes(P.BF16) == 2 * (2 * 16 * 64 * 2)   # Hkv x (K, V) x 16 tokens x D x 2 B
    with pytest.raises(MkvError):
        lp.slot_bytes(P.FP8)                    # a control pool holds no FP8 pages
