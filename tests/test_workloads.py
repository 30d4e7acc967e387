"""The synthetic input recipe, checked against its written description: context lengths, the
anchor pages each workload ends up with (page 0, the pages holding the last W tokens, and the
protected share), the outlier channels of K, and bf16 rounding.  Built on host-only pools, so
only the allocation and policy logic runs (no device work)."""
import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import Pool
from mixed_format_paged_mkv_b200.workloads import WORKLOADS, bf16_bits


def built_tables(w):
    pool = Pool(**w.pool_shape(), host_only=True)
    for op in w.build_ops(0):
        if op[0] == "append":
            pool.append([op[1]], [op[2]])
        elif op[0] == "protect":
            for p in op[2]:
                pool.set_protected(op[1], p, True)
        else:
            pool.demote([op[1]], op[2])
    return [pool.block_table(s) for s in range(w.B)]


def anchor_pages(L, W):
    """page 0 and every page holding one of the last W tokens"""
    n = -(-L // 16)
    return {0} | {p for p in range(n) if 16 * p + 16 > L - W}


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_anchor_pages_follow_the_recipe(idx):
    w = WORKLOADS[idx]
    lens = w.lengths()
    if idx == 3:
        assert all(2048 <= L <= 32768 for L in lens)
    elif idx == 5:
        assert all(4096 <= L <= 65536 for L in lens)
    for s, (table, ctx) in enumerate(built_tables(w)):
        assert ctx == lens[s] and len(table) == -(-ctx // 16)
        fp8 = {p for p, e in enumerate(table) if e >> 30 == 0}
        base = anchor_pages(ctx, w.window)
        assert base <= fp8, s
        extra = fp8 - base
        older = (ctx - w.window) // 16 - 1          # full pages before the window, page 0 excluded
        if idx == 3:
            assert len(extra) == round(0.02 * max(older, 0)), s
        elif idx == 4:
            assert len(fp8) == round(0.04 * len(table)) == 328, s
        else:
            assert not extra, s
        assert all(p not in base for p in extra)


def test_tiny_and_batch_shapes():
    assert [len(t) for t, _ in built_tables(WORKLOADS[1])] == [64]
    t1, _ = built_tables(WORKLOADS[1])[0]
    assert {p for p, e in enumerate(t1) if e >> 30 == 0} == {0, 60, 61, 62, 63}
    t2 = built_tables(WORKLOADS[2])
    assert all({p for p, e in enumerate(t) if e >> 30 == 0} == {0} | set(range(496, 512))
               for t, _ in t2)


def test_outlier_channels_of_k():
    w = WORKLOADS[2]
    oc = np.asarray(w.outlier_channels(0))
    assert oc.shape == (w.Hkv, 4) and all(len(set(r.tolist())) == 4 for r in oc)
    k, v = w.kv(0, 0)
    kf = (k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    vf = (v.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for h in range(w.Hkv):
        sd = kf[:, h, :].std(axis=0)
        assert set(np.argsort(sd)[-4:].tolist()) == set(oc[h].tolist())
        assert 6 < sd[oc[h]].mean() / np.delete(sd, oc[h]).mean() < 10
        assert vf[:, h, :].std(axis=0).max() < 1.3              # V has no outliers


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 3.0e38], dtype=np.float32)
    b = bf16_bits(x)
    back = (b.astype(np.uint32) << 16).view(np.float32)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1); 1 + 3*2^-8 rounds up to 1 + 2^-6
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2 ** -6 and back[3] == -1.0
    assert np.isfinite(back[4])
