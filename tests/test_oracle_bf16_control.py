"""Pins of the oracle's BF16 control pages (CPU).

The control keeps every page's bf16 values as they are (the comparator of the pages' "KV bytes
per live token versus BF16" and of their canary against a control).  Pinned against hand-derived
slot bytes, the identity it must be (values out = values in), the pool rules it must keep (no
demotion, slots and tables as for FP8 pages) and dense softmax attention on the raw inputs."""
import numpy as np
import pytest
from scipy.special import softmax

from mixed_format_paged_mkv_b200.workloads import bf16_bits
from oracle import attention as A
from oracle import formats as F
from oracle import pool as P


def test_slot_bytes_hand_derived():
    """One KV head, D 32: token 0 of K = (1, -2, 0.5, 0, ...), token 1 of V = (-0.0, 3.0, ...).
    bf16 bits: 1 -> 3F80, -2 -> C000, 0.5 -> 3F00, -0 -> 8000, 3 -> 4040, little-endian."""
    pool = P.RefPool(1, 32, 1, 4, 4, 0, bf16_control=True)
    k = np.zeros((2, 1, 32))
    v = np.zeros((2, 1, 32))
    k[0, 0, :3] = (1.0, -2.0, 0.5)
    v[1, 0, :2] = (-0.0, 3.0)
    pool.append([0], [2], k, v)
    e = pool.block_table(0)[0]
    assert (e >> 30) & 3 == P.BF16
    raw = pool.slot_bytes(e)
    assert raw.size == F.bf16_head_bytes(32) == 2048
    assert raw[:6].tolist() == [0x80, 0x3F, 0x00, 0xC0, 0x00, 0x3F]
    v_token1 = 16 * 32 * 2 + 32 * 2          # V rows start after 16 K rows; token 1
    assert raw[v_token1:v_token1 + 4].tolist() == [0x00, 0x80, 0x40, 0x40]
    expected_nonzero = {0, 1, 3, 5, v_token1 + 1, v_token1 + 2, v_token1 + 3}
    assert set(np.nonzero(raw)[0].tolist()) == expected_nonzero
    kb, vb = F.parse_bf16_slot(raw, 1, 32)
    assert kb[0, 0, 1] == 0xC000 and vb[0, 1, 1] == 0x4040


def test_values_round_trip_exactly_across_pages():
    rng = np.random.default_rng(0)
    Hkv, D = 2, 64
    pool = P.RefPool(Hkv, D, 2, 16, 40, 0, bf16_control=True)
    parts = []
    for n in (5, 11, 16, 1, 40):
        x = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((n, Hkv, D)) * 7))
        y = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((n, Hkv, D))))
        pool.append([1], [n], x, y)
        parts.append((x, y))
    K, V = pool.dequant_seq(1)
    assert np.array_equal(K, np.concatenate([a for a, _ in parts]))
    assert np.array_equal(V, np.concatenate([b for _, b in parts]))
    assert pool.demote([1], 0) == []                       # a control page is never converted
    assert all((e >> 30) & 3 == P.BF16 for e in pool.block_table(1))
    live, n8, n3, bpt = pool.stats()
    assert (live, n8, n3) == (73, 5, 0)
    assert bpt == pytest.approx(5 * Hkv * 4 * 16 * D / 73)


def test_attention_equals_dense_softmax_of_the_inputs():
    rng = np.random.default_rng(1)
    Hkv, D, g, L = 2, 32, 3, 70
    pool = P.RefPool(Hkv, D, 1, 8, 8, 0, bf16_control=True)
    k = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((L, Hkv, D))))
    v = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((L, Hkv, D))))
    pool.append([0], [L], k, v)
    q = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((1, Hkv * g, D))))
    K, V = pool.dequant_seq(0)
    out = A.attention(K, V, q, 0.2)
    for hq in range(Hkv * g):
        h = hq // g
        w = softmax(0.2 * k[:, h] @ q[0, hq])
        assert np.allclose(out[0, hq], w @ v[:, h], rtol=1e-12, atol=1e-13)


def test_prefill_and_copy_reset_keep_bf16_pages():
    rng = np.random.default_rng(2)
    pool = P.RefPool(1, 32, 3, 8, 12, 0, bf16_control=True)
    x = F.bf16_bits_to_f64(bf16_bits(rng.standard_normal((50, 1, 32))))
    pool.prefill([0], [50], x, x, window_tokens=0)        # all pages written as bf16
    assert [(e >> 30) & 3 for e in pool.block_table(0)] == [P.BF16] * 4
    pool.seq_copy(0, 1)
    assert np.array_equal(pool.dequant_seq(1)[0], x)
    pool.seq_reset(0)
    assert pool.block_table(0) == [] and len(pool.alloc[0].free) == 12 - 4


def test_bf16_bits_rejects_values_bf16_cannot_hold():
    with pytest.raises(ValueError):
        F.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -10]))
    # 2^-130 is an fp32 subnormal: 2^-149 * 2^19, bits 0x00080000, so bf16 bits 0x0008
    assert F.f64_to_bf16_bits(np.array([-0.0, 1.5, 2.0 ** -130])).tolist() == [0x8000, 0x3FC0, 0x0008]
