"""The oracle's direct prefill pack, pinned by the anchor rule and by the FP8 path: on inputs that
FP8 holds exactly, packing a page straight from bf16 must give the very page that appending it
as FP8 and demoting it gives."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import pool as P


def fp8_exact_tokens(rng, n, Hkv, D):
    """bf16-representable values that an FP8 page of 16 tokens stores exactly: E4M3 grid values
    times 2^e, with one |x| = 448 * 2^e per (page, head) so the page scale is exactly 2^e."""
    codes = rng.integers(0, 256, size=(n, Hkv, D)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38          # no NaN codes
    x = F.e4m3_decode(codes)
    for p0 in range(0, n, 16):
        for h in range(Hkv):
            t = p0 + int(rng.integers(0, min(16, n - p0)))
            x[t, h, int(rng.integers(0, D))] = 448.0 * (1 if rng.random() < 0.5 else -1)
            e = int(rng.integers(-6, 3))
            x[p0:p0 + 16, h, :] *= 2.0 ** e
    return x


def pages_of(pool, s):
    out = []
    for fmt, slot in pool.table[s]:
        store = pool.fp8 if fmt == P.FP8 else pool.tq3
        out.append((fmt, [np.asarray(a) for a in store[slot]]))
    return out


@pytest.mark.parametrize("n,W,sink", [(16 * 9, 32, 1), (16 * 6 + 5, 0, 1), (40, 16, 0),
                                      (16 * 12, 100, 2), (10, 0, 1), (16 * 5, 1000, 1)])
def test_prefill_equals_append_then_demote_on_fp8_exact_inputs(n, W, sink):
    rng = np.random.default_rng(n + W + sink)
    Hkv, D = 2, 64
    K = fp8_exact_tokens(rng, n, Hkv, D)
    V = fp8_exact_tokens(rng, n, Hkv, D)
    a = P.RefPool(Hkv, D, 2, 16, 32, 32, sink_pages=sink)
    b = P.RefPool(Hkv, D, 2, 16, 32, 32, sink_pages=sink)
    a.prefill([1], [n], K, V, W)
    b.append([1], [n], K, V)
    b.demote([1], W)
    assert a.ctx[1] == b.ctx[1] == n
    pa, pb = pages_of(a, 1), pages_of(b, 1)
    assert [f for f, _ in pa] == [f for f, _ in pb]
    for (f, xa), (_, xb) in zip(pa, pb):
        for u, w in zip(xa, xb):
            assert np.array_equal(u, w)


@pytest.mark.parametrize("n,W,sink", [(16 * 20 + 3, 64, 1), (16 * 20, 0, 3), (7, 0, 0)])
def test_prefill_page_formats_follow_the_anchor_rule(n, W, sink):
    rng = np.random.default_rng(3)
    Hkv, D = 1, 32
    K = rng.standard_normal((n, Hkv, D))
    pool = P.RefPool(Hkv, D, 1, 32, 32, 32, sink_pages=sink)
    pool.prefill([0], [n], K, K, W)
    fmts = [f for f, _ in pool.table[0]]
    want = [P.TQ3 if (p >= sink and 16 * p + 16 <= n - W) else P.FP8 for p in range(-(-n // 16))]
    assert fmts == want
    # nothing the demotion policy would still convert
    assert pool.demote_candidates(0, W) == []


def test_prefill_errors_leave_the_pool_unchanged():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((64, 1, 32))
    pool = P.RefPool(1, 32, 2, 8, 2, 8)
    pool.append([0], [1], K[:1], K[:1])
    with pytest.raises(P.PoolError) as e:
        pool.prefill([0], [16], K[:16], K[:16], 0)        # not empty
    assert e.value.code == "INVALID_ARG"
    with pytest.raises(P.PoolError) as e:
        pool.prefill([1], [64], K, K, 64)                 # 4 FP8 pages, 1 FP8 slot left
    assert e.value.code == "OUT_OF_PAGES"
    assert pool.table[1] == [] and pool.ctx[1] == 0 and len(pool.alloc[P.FP8].free) == 1
