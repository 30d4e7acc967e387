"""Pins of the oracle's pool model and attention against invariants and closed forms.

Pool: the anchor policy reproduces the workloads' stated FP8 page sets, slots are unique,
every live page is mapped, allocation follows the slot order.  Attention: merge of any page
partition equals single-pass attention, the per-format partials merged equal the materialised
dense attention, the dequantised sequence equals the raw slot bytes parsed by layout, equal keys
give mean(V), one token gives V, the first query of a q_len-4 causal call equals a q_len-1 call
three tokens earlier, and a 50-digit Decimal brute force agrees on tiny inputs.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

from oracle import attention as A
from oracle import formats as F
from oracle import pool as P
from mixed_format_paged_mkv_b200.workloads import WORKLOADS, bf16_bits


def build(w, layer=0, shape=None):
    """Replay a workload's build calls on a fresh oracle pool."""
    shape = shape or w.pool_shape()
    pool = P.RefPool(shape["num_kv_heads"], shape["head_dim"], shape["max_seqs"],
                     shape["max_pages_per_seq"], shape["fp8_slots"], shape["tq3_slots"])
    for fmt in (P.FP8, P.TQ3):
        order = w.slot_permutation(fmt, shape["fp8_slots" if fmt == P.FP8 else "tq3_slots"])
        if order is not None:
            pool.set_slot_order(fmt, order)
    for op in w.build_ops(layer):
        if op[0] == "append":
            k, v = w.kv(op[1], layer)
            pool.append([op[1]], [op[2]], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
        elif op[0] == "protect":
            for p in op[2]:
                pool.set_protected(op[1], p, 1)
        else:
            pool.demote([op[1]], op[2])
    return pool


def check_invariants(pool):
    used = {P.FP8: set(), P.TQ3: set()}
    for s in range(pool.max_seqs):
        assert len(pool.table[s]) == -(-pool.ctx[s] // 16)
        for fmt, slot in pool.table[s]:
            assert slot not in used[fmt]
            used[fmt].add(slot)
            assert slot not in pool.alloc[fmt].free
    for fmt in (P.FP8, P.TQ3):
        assert used[fmt] | pool.alloc[fmt].free == set(range(pool.alloc[fmt].n))


def test_tiny_workload_fp8_pages_are_page0_and_last4():
    w = WORKLOADS[1]
    pool = build(w)
    fmts = [f for f, _ in pool.table[0]]
    assert [p for p, f in enumerate(fmts) if f == P.FP8] == [0, 60, 61, 62, 63]
    assert fmts.count(P.TQ3) == 59
    check_invariants(pool)
    # first FP8 slot handed out is the first of the slot order
    order = w.slot_permutation(P.FP8, 128)
    assert pool.table[0][0] == (P.FP8, int(order[0]))


def test_policy_windows_and_protection():
    w = WORKLOADS[3].scaled(B=3, ctx_range=(700, 1500), window=128, protect_frac=0.2)
    pool = build(w)
    check_invariants(pool)
    for s, L in enumerate(w.lengths()):
        prot = set(w.protected(s))
        for p, (fmt, _) in enumerate(pool.table[s]):
            full = 16 * (p + 1) <= L
            anchor = p == 0 or 16 * p + 16 > L - 128 or p in prot
            assert fmt == (P.FP8 if (anchor or not full) else P.TQ3), (s, p)


def test_demote_is_idempotent_and_frees_fp8_slots():
    w = WORKLOADS[1]
    pool = build(w)
    free8 = len(pool.alloc[P.FP8].free)
    assert pool.demote([0], 64) == []
    assert len(pool.alloc[P.FP8].free) == free8 == 128 - 5


def test_append_then_demote_token_by_token():
    w = WORKLOADS[1].scaled(ctx=(40,))
    pool = P.RefPool(2, 128, 2, 16, 16, 16)
    k, v = w.kv(0)
    K, V = F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v)
    for t in range(40):
        pool.append([0], [1], K[t:t + 1], V[t:t + 1])
        pool.demote([0], 8)
    fmts = [f for f, _ in pool.table[0]]
    assert fmts == [P.FP8, P.TQ3, P.FP8]     # L=40, W=8: page 1 (tokens 16..31) is old
    check_invariants(pool)
    with pytest.raises(P.PoolError):
        pool.append([5], [1], K[:1], V[:1])


def test_seq_copy_and_reset():
    w = WORKLOADS[1].scaled(ctx=(100,))
    pool = P.RefPool(2, 128, 3, 16, 32, 32)
    k, v = w.kv(0)
    pool.append([0], [100], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
    pool.demote([0], 32)
    pool.seq_copy(0, 2)
    K0, V0 = pool.dequant_seq(0)
    K2, V2 = pool.dequant_seq(2)
    assert np.array_equal(K0, K2) and np.array_equal(V0, V2)
    check_invariants(pool)
    pool.seq_reset(0)
    check_invariants(pool)
    assert pool.ctx[0] == 0 and pool.ctx[2] == 100


# ------------------------------------------------------------------ attention
def small_pool(seed=0, L=200, Hkv=2, D=64, W=48):
    rng = np.random.default_rng(seed)
    k = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((L, Hkv, D), dtype=np.float32)))
    v = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((L, Hkv, D), dtype=np.float32)))
    pool = P.RefPool(Hkv, D, 1, 64, 64, 64)
    pool.append([0], [L], k, v)
    pool.demote([0], W)
    return pool


def test_merge_of_any_page_partition_equals_single_pass():
    pool = small_pool()
    K, V = pool.dequant_seq(0)
    rng = np.random.default_rng(1)
    q = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((2, 6, 64), dtype=np.float32)))
    ref = A.attention(K, V, q, 0.125)
    n_pages = len(pool.table[0])
    for trial in range(5):
        labels = rng.integers(0, 4, n_pages)
        parts = []
        for part in range(4):
            toks = [t for p in np.nonzero(labels == part)[0] for t in range(16 * p, min(16 * p + 16, K.shape[0]))]
            parts.append(A.partial_state(K, V, q, 0.125, toks))
        out = A.merge(parts)
        assert np.max(np.abs(out - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_per_format_partials_merge_to_the_materialised_attention():
    # the method's identity: attention computed separately over the FP8 pages and over the TQ3
    # pages, then merged with global normalisation, is the attention over the dense
    # materialised cache (the pages' "materialising profile")
    pool = small_pool(seed=5, L=203, W=40)
    pool.set_protected(0, 3, 1)
    fmts = [f for f, _ in pool.table[0]]
    assert P.FP8 in fmts and P.TQ3 in fmts
    K, V = pool.dequant_seq(0)
    L = K.shape[0]
    rng = np.random.default_rng(6)
    q = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((2, 6, 64), dtype=np.float32)))
    dense = A.materialise_and_attend(pool, 0, q, 0.125)
    parts = []
    for fmt in (P.FP8, P.TQ3):
        toks = [t for p, f in enumerate(fmts) if f == fmt for t in range(16 * p, min(16 * p + 16, L))]
        parts.append(A.partial_state(K, V, q, 0.125, toks))
    merged = A.merge(parts)
    assert np.max(np.abs(merged - dense)) <= 1e-12 * np.max(np.abs(dense))


def test_dequantised_sequence_matches_the_raw_slot_bytes():
    # dequant_seq reads the stored codes; the same values must come back from each page's raw
    # slot bytes parsed by layout, page by page in table order
    pool = small_pool(seed=7, L=150, W=32)
    K, V = pool.dequant_seq(0)
    Hkv, D = pool.Hkv, pool.D
    for p, (fmt, slot) in enumerate(pool.table[0]):
        raw = pool.slot_bytes((fmt << 30) | slot)
        rows = slice(16 * p, min(16 * p + 16, K.shape[0]))
        n = rows.stop - rows.start
        if fmt == P.FP8:
            kc, vc, ks, vs = F.parse_fp8_slot(raw, Hkv, D)
            kd = F.e4m3_decode(kc) * ks[:, None, None]
            vd = F.e4m3_decode(vc) * vs[:, None, None]
        else:
            kq, ks, vq, vs = F.parse_tq3_slot(raw, Hkv, D)
            kd = (kq.reshape(Hkv, 16, -1, 32) - 3.5) * ks[..., None]
            vd = (vq.reshape(Hkv, 16, -1, 32) - 3.5) * vs[..., None]
        assert np.array_equal(K[rows], kd.reshape(Hkv, 16, D).transpose(1, 0, 2)[:n])
        assert np.array_equal(V[rows], vd.reshape(Hkv, 16, D).transpose(1, 0, 2)[:n])


def test_equal_keys_give_mean_of_values():
    # keys on the grid {+-0.5, +-1.5, +-2.5, +-3.5} * 2^-2 are exact in E4M3 pages (codes
    # +-64/192/320/448 with scale 2^-9) and in TQ3 pages (s = 2^-2), so every page -- FP8 or
    # TQ3 -- dequantises to the same key and the softmax is uniform.
    L, Hkv, D = 96, 1, 64
    rng = np.random.default_rng(2)
    row = rng.choice([-3.5, -2.5, -1.5, -0.5, 0.5, 1.5, 2.5, 3.5], size=D) * 0.25
    row[::32] = 3.5 * 0.25
    k = np.broadcast_to(row, (L, Hkv, D)).copy()
    v = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((L, Hkv, D), dtype=np.float32)))
    pool = P.RefPool(Hkv, D, 1, 16, 16, 16)
    pool.append([0], [L], k, v)
    pool.demote([0], 16)
    assert sum(f == P.TQ3 for f, _ in pool.table[0]) == 4
    K, V = pool.dequant_seq(0)
    assert np.array_equal(K, k)
    q = rng.standard_normal((1, 3, D))
    out = A.attention(K, V, q, 1.0 / 8)
    assert np.allclose(out[0], V[:, 0].mean(axis=0)[None, :], rtol=0, atol=1e-13)


def test_one_token_context_returns_its_value():
    rng = np.random.default_rng(3)
    k = rng.standard_normal((1, 2, 64))
    v = rng.standard_normal((1, 2, 64))
    q = rng.standard_normal((1, 4, 64))
    out = A.attention(k, v, q, 0.3)
    assert np.array_equal(out[0, :2], np.broadcast_to(v[0, 0], (2, 64)))
    assert np.array_equal(out[0, 2:], np.broadcast_to(v[0, 1], (2, 64)))


def test_causal_multi_token_query0_equals_shorter_single_query():
    pool = small_pool(seed=4, L=150)
    K, V = pool.dequant_seq(0)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 4, 64))
    out4 = A.attention(K, V, q, 0.125)
    out1 = A.attention(K[:147], V[:147], q[:1], 0.125)
    assert np.array_equal(out4[0], out1[0])
    last = A.attention(K, V, q[3:4], 0.125)
    assert np.array_equal(out4[3], last[0])


def _decimal_attention(K, V, q, scale):
    getcontext().prec = 50
    L, Hkv, D = K.shape
    Hq = q.shape[1]
    g = Hq // Hkv
    out = np.empty((Hq, D))
    for hq in range(Hq):
        h = hq // g
        s = [Decimal(scale) * sum(Decimal(float(q[0, hq, d])) * Decimal(float(K[t, h, d]))
                                  for d in range(D)) for t in range(L)]
        e = [x.exp() for x in s]
        tot = sum(e)
        for d in range(D):
            out[hq, d] = float(sum(e[t] * Decimal(float(V[t, h, d])) for t in range(L)) / tot)
    return out


def test_brute_force_decimal_on_tiny_cache():
    pool = small_pool(seed=6, L=40, Hkv=1, D=32, W=8)
    K, V = pool.dequant_seq(0)
    rng = np.random.default_rng(7)
    q = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((1, 2, 32), dtype=np.float32)))
    ref = _decimal_attention(K, V, q, 1 / np.sqrt(32))
    out = A.attention(K, V, q, 1 / np.sqrt(32))
    assert np.max(np.abs(out[0] - ref)) <= 1e-13


def test_scipy_softmax_cross_check():
    from scipy.special import softmax
    pool = small_pool(seed=8, L=130)
    K, V = pool.dequant_seq(0)
    q = np.random.default_rng(9).standard_normal((1, 4, 64))
    out = A.attention(K, V, q, 0.1)
    for hq in range(4):
        p = softmax(0.1 * K[:, hq // 2] @ q[0, hq])
        assert np.allclose(out[0, hq], p @ V[:, hq // 2], rtol=1e-13, atol=1e-15)


def test_empty_parts_and_empty_context():
    pool = small_pool(seed=10, L=64)
    K, V = pool.dequant_seq(0)
    q = np.random.default_rng(11).standard_normal((1, 2, 64))
    empty = A.partial_state(K, V, q, 0.1, [])
    full = A.partial_state(K, V, q, 0.1, range(64))
    assert np.all(np.isneginf(empty[0])) and np.all(empty[1] == 0)
    assert np.array_equal(A.merge([empty, full]), A.merge([full]))
    with pytest.raises(ValueError):
        A.attention(K[:0], V[:0], q, 0.1)
