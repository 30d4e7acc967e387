"""GPU parity of the page writers: FP8 append (with rescale-on-grow), FP8 -> TQ3 demotion and
slot copies must reproduce the oracle's slot bytes and block tables bit for bit."""
import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import Pool
from mixed_format_paged_mkv_b200.workloads import WORKLOADS, Workload, bf16_bits
from oracle import formats as F
from oracle import pool as P

from harness import lib_pool, oracle_pool, to_bf16_tensor

pytestmark = pytest.mark.gpu


def compare(lp, op, seqs):
    for s in seqs:
        t, ctx = lp.block_table(s)
        assert t == op.block_table(s), s
        assert ctx == op.ctx[s]
        for p, e in enumerate(t):
            got, want = lp.read_slot(e), op.slot_bytes(e)
            if not np.array_equal(got, want):
                bad = np.nonzero(got != want)[0]
                raise AssertionError(f"seq {s} page {p} entry {e:#x}: {bad.size} bytes differ, "
                                     f"first at {bad[0]}: got {got[bad[0]]:#x} want {want[bad[0]]:#x}")
    lp.device_status()


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(B=2, ctx=(600, 1000))),
    (3, dict(B=3, ctx_range=(300, 1500), window=128, protect_frac=0.1)),
])
def test_workload_pages_bit_exact(cfg, kw):
    w = WORKLOADS[cfg].scaled(**kw)
    compare(lib_pool(w), oracle_pool(w), range(w.B))


def test_head_dim_64():
    w = Workload("d64", 9, B=2, Hq=4, Hkv=2, D=64, q_len=1, window=32, ctx=(90, 200), outliers=True)
    compare(lib_pool(w), oracle_pool(w), range(w.B))


def _tokens(rng, n, Hkv, D, scale=1.0):
    return bf16_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32) * np.float32(scale))


def test_token_by_token_appends_with_rescale_and_demotion():
    rng = np.random.default_rng(1)
    Hkv, D = 2, 128
    lp = Pool(Hkv, D, 2, 16, 16, 16)
    op = P.RefPool(Hkv, D, 2, 16, 16, 16)
    for t in range(70):
        # growing magnitudes force rescale-on-grow inside partially filled pages
        k = _tokens(rng, 1, Hkv, D, 1.0 + t / 7.0)
        v = _tokens(rng, 1, Hkv, D, 3.0 - t / 40.0)
        lp.append([0], [1], to_bf16_tensor(k), to_bf16_tensor(v))
        op.append([0], [1], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
        assert lp.demote([0], 20) == len(op.demote([0], 20))
        if t % 9 == 0 or t == 69:
            compare(lp, op, [0])


def test_mixed_append_sizes_two_sequences():
    rng = np.random.default_rng(2)
    Hkv, D = 4, 256
    lp = Pool(Hkv, D, 3, 32, 40, 40)
    op = P.RefPool(Hkv, D, 3, 32, 40, 40)
    for n0, n1 in [(37, 5), (5, 0), (1, 16), (16, 30), (0, 1), (30, 13)]:
        k = _tokens(rng, n0 + n1, Hkv, D, 2.0)
        v = _tokens(rng, n0 + n1, Hkv, D)
        lp.append([1, 0], [n0, n1], to_bf16_tensor(k), to_bf16_tensor(v))
        op.append([1, 0], [n0, n1], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
        lp.demote([0, 1], 16)
        op.demote([0, 1], 16)
    compare(lp, op, [0, 1])


def test_zero_tokens_and_signed_zero():
    Hkv, D = 1, 64
    lp = Pool(Hkv, D, 1, 8, 8, 8)
    op = P.RefPool(Hkv, D, 1, 8, 8, 8)
    z = np.zeros((16, Hkv, D), np.uint16)
    z[3, 0, 5] = 0x8000                      # bf16 -0.0 on an all-zero page
    k = np.concatenate([z, _tokens(np.random.default_rng(3), 16, Hkv, D)])
    k[20, 0, 7] = 0x8000                     # -0.0 on a page with a nonzero scale
    v = k[::-1].copy()
    lp.append([0], [32], to_bf16_tensor(k), to_bf16_tensor(v))
    op.append([0], [32], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
    lp.append([0], [16], to_bf16_tensor(k[:16]), to_bf16_tensor(v[:16]))
    op.append([0], [16], F.bf16_bits_to_f64(k[:16]), F.bf16_bits_to_f64(v[:16]))
    lp.demote([0], 0)
    op.demote([0], 0)
    compare(lp, op, [0])


def test_copy_reset_and_slot_reuse():
    rng = np.random.default_rng(4)
    Hkv, D = 2, 128
    lp = Pool(Hkv, D, 3, 16, 12, 12)
    op = P.RefPool(Hkv, D, 3, 16, 12, 12)
    k, v = _tokens(rng, 90, Hkv, D), _tokens(rng, 90, Hkv, D)
    lp.append([0], [90], to_bf16_tensor(k), to_bf16_tensor(v))
    op.append([0], [90], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
    lp.demote([0], 30)
    op.demote([0], 30)
    lp.copy(0, 2)
    op.seq_copy(0, 2)
    compare(lp, op, [0, 2])
    lp.reset(0)
    op.seq_reset(0)
    # reused FP8 slots must come back with zeroed rows beyond the written tokens
    k2, v2 = _tokens(rng, 21, Hkv, D), _tokens(rng, 21, Hkv, D)
    lp.append([1], [21], to_bf16_tensor(k2), to_bf16_tensor(v2))
    op.append([1], [21], F.bf16_bits_to_f64(k2), F.bf16_bits_to_f64(v2))
    compare(lp, op, [0, 1, 2])


@pytest.mark.parametrize("D", [64, 256])
def test_extreme_magnitudes_bit_exact(D):
    """Pages whose values sit at bf16's extremes (subnormals near 1e-40, values near 1e38) and in
    between: the TQ3 coder takes its exact fallback for page scales outside [2^-100, 2^100) and
    the source-domain path elsewhere; both must give the oracle's bytes, for demotion and for
    direct prefill packing."""
    rng = np.random.default_rng(5)
    Hkv, n = 2, 16 * 12
    mags = np.array([1e-40, 3e-39, 1e-35, 1e-20, 1.0, 1e20, 1e30, 1e37, 4e37], np.float32)
    k = np.empty((n, Hkv, D), np.uint16)
    v = np.empty((n, Hkv, D), np.uint16)
    for p in range(n // 16):
        for h in range(Hkv):
            sk, sv = mags[(p + h) % mags.size], mags[(3 * p + h) % mags.size]
            k[16 * p:16 * p + 16, h] = _tokens(rng, 16, 1, D, sk)[:, 0]
            v[16 * p:16 * p + 16, h] = _tokens(rng, 16, 1, D, sv)[:, 0]
    k[5, 0, :7] = 0x8000                          # signed zeros among tiny values
    v[40, 1, 3] = 0x0001                          # the smallest bf16 subnormal
    lp = Pool(Hkv, D, 2, 16, 32, 32)
    op = P.RefPool(Hkv, D, 2, 16, 32, 32)
    lp.append([0], [n], to_bf16_tensor(k), to_bf16_tensor(v))
    op.append([0], [n], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
    assert lp.demote([0], 16) == len(op.demote([0], 16))
    lp.prefill([1], [n], to_bf16_tensor(k), to_bf16_tensor(v), window=16)
    op.prefill([1], [n], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v), window_tokens=16)
    compare(lp, op, [0, 1])
