"""GPU checks of the BF16 control pool: page bytes and tables bit for bit against the oracle,
the dense fp32 view exact, and decode attention over the bf16 pages within the tolerance."""
import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200.workloads import WORKLOADS, Workload
from oracle import pool as P

from harness import assert_close, lib_pool, oracle_decode, oracle_pool, to_bf16_tensor

pytestmark = pytest.mark.gpu

CASES = [
    WORKLOADS[1],
    WORKLOADS[3].scaled(B=3, ctx_range=(200, 2500), window=256),
    Workload("ctl128", 61, B=2, Hq=12, Hkv=2, D=128, q_len=3, window=32, ctx=(700, 45)),
    Workload("ctl64", 62, B=3, Hq=8, Hkv=4, D=64, q_len=1, window=16, ctx=(1, 17, 300)),
]


def pools(w):
    shape = dict(w.pool_shape(), fp8_slots=sum(w.pages()) + 8)   # every page stays BF16
    return (lib_pool(w, shape=shape, bf16_control=True),
            oracle_pool(w, shape=shape, bf16_control=True))


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_control_pages_and_decode_match_oracle(w):
    lp, op = pools(w)
    for s in range(w.B):
        table, ctx = lp.block_table(s)
        assert table == op.block_table(s) and ctx == op.ctx[s]
        for e in table:
            assert (e >> 30) & 3 == P.BF16
            assert np.array_equal(lp.read_slot(e), op.slot_bytes(e)), f"seq {s} entry {e:#x}"
    q = to_bf16_tensor(np.stack([w.q(s) for s in range(w.B)]))
    out = lp.decode(list(range(w.B)), q).cpu().numpy()
    torch.cuda.synchronize()
    lp.device_status()
    for s in range(w.B):
        assert_close(out[s], oracle_decode(op, w, s), what=f"{w.name} seq {s}")


def test_control_materialise_is_exact():
    w = CASES[1]
    lp, op = pools(w)
    for s in range(w.B):
        k, v = lp.materialise(s)
        K, V = op.dequant_seq(s)
        assert np.array_equal(k.cpu().numpy().astype(np.float64), K)
        assert np.array_equal(v.cpu().numpy().astype(np.float64), V)
    lp.device_status()


@pytest.mark.parametrize("D,Hq,Hkv,q_len", [(128, 8, 2, 1), (256, 24, 4, 2)])
def test_control_decode_with_ctas_spanning_sequences(D, Hq, Hkv, q_len):
    """The BF16 control kernel under the line cut: unequal sequences and a small SM budget give
    CTAs that take the pieces of several sequences one after another."""
    w = Workload("ctlspan", 63, B=5, Hq=Hq, Hkv=Hkv, D=D, q_len=q_len, window=32,
                 ctx=(1500, 1300, 120, 60, 33))
    lp, op = pools(w)
    for sms in range(1, 64):
        lp.set_decode_sms(sms)
        units, _ = lp.decode_plan(list(range(w.B)), q_len, Hq)
        if np.bincount(units[:, 5]).max() >= 2:
            break
    else:
        pytest.fail("no plan with a CTA that starts several units")
    q = to_bf16_tensor(np.stack([w.q(s) for s in range(w.B)]))
    out = lp.decode(list(range(w.B)), q).cpu().numpy()
    torch.cuda.synchronize()
    lp.device_status()
    for s in range(w.B):
        assert_close(out[s], oracle_decode(op, w, s), what=f"{w.name} seq {s}")
