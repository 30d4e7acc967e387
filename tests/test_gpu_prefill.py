"""GPU parity of the direct prefill pack (mkv_prefill_kv): slot bytes and block tables bit-exact
against the oracle, and decode over the prefilled cache within the attention tolerance."""
import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200 import Pool
from mixed_format_paged_mkv_b200.workloads import Workload, bf16_bits
from oracle import attention as A
from oracle import formats as F
from oracle import pool as P

from harness import assert_close, to_bf16_tensor

pytestmark = pytest.mark.gpu


def prefilled(Hkv, D, lens, window, sink=1, seed=0, outliers=True):
    rng = np.random.default_rng(seed)
    rows = sum(lens)
    k = rng.standard_normal((rows, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((rows, Hkv, D), dtype=np.float32)
    if outliers:
        k[:, :, :4] *= 8
    kb, vb = bf16_bits(k), bf16_bits(v)
    pages = sum(-(-n // 16) for n in lens)
    shape = (Hkv, D, len(lens), max(-(-n // 16) for n in lens) + 4, pages + 16, pages + 16)
    lp = Pool(*shape, sink_pages=sink)
    op = P.RefPool(*shape, sink_pages=sink)
    seqs = list(range(len(lens)))
    lp.prefill(seqs, lens, to_bf16_tensor(kb), to_bf16_tensor(vb), window=window)
    op.prefill(seqs, lens, F.bf16_bits_to_f64(kb), F.bf16_bits_to_f64(vb), window)
    torch.cuda.synchronize()
    return lp, op


def compare_pages(lp, op, seqs):
    n3 = 0
    for s in seqs:
        t, ctx = lp.block_table(s)
        assert t == op.block_table(s) and ctx == op.ctx[s], s
        for p, e in enumerate(t):
            n3 += (e >> 30) == 1
            got, want = lp.read_slot(e), op.slot_bytes(e)
            if not np.array_equal(got, want):
                bad = np.nonzero(got != want)[0]
                raise AssertionError(f"seq {s} page {p} entry {e:#x}: {bad.size} bytes differ, "
                                     f"first at {bad[0]}")
    lp.device_status()
    return n3


@pytest.mark.parametrize("Hkv,D,lens,window,sink", [
    (2, 128, (1000, 17, 16, 1), 64, 1),
    (4, 256, (700, 300), 512, 1),
    (2, 64, (500, 129), 0, 0),
    (1, 128, (400,), 32, 3),
])
def test_prefill_pages_bit_exact(Hkv, D, lens, window, sink):
    lp, op = prefilled(Hkv, D, lens, window, sink, seed=D + window)
    assert compare_pages(lp, op, range(len(lens))) > 0


def test_prefill_then_decode_and_later_demotion():
    Hkv, D, Hq, lens, W = 2, 128, 8, (900, 333), 64
    lp, op = prefilled(Hkv, D, lens, W, seed=7)
    rng = np.random.default_rng(8)
    q = bf16_bits(rng.standard_normal((len(lens), 1, Hq, D), dtype=np.float32))
    out = lp.decode(list(range(len(lens))), to_bf16_tensor(q)).cpu().numpy()
    for s in range(len(lens)):
        K, V = op.dequant_seq(s)
        ref = A.attention(K, V, F.bf16_bits_to_f64(q[s]), 1 / np.sqrt(D))
        assert_close(out[s], ref, what=f"seq {s}")
    # the window pages stay FP8 and demote later like appended ones
    k1 = bf16_bits(rng.standard_normal((2 * 48, Hkv, D), dtype=np.float32))
    lp.append([0, 1], [48, 48], to_bf16_tensor(k1), to_bf16_tensor(k1))
    op.append([0, 1], [48, 48], F.bf16_bits_to_f64(k1), F.bf16_bits_to_f64(k1))
    assert lp.demote([0, 1], W) == len(op.demote([0, 1], W))
    compare_pages(lp, op, range(len(lens)))
