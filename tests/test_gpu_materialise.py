"""GPU parity of the materialising profile: the dense fp32 K and V that mkv_materialise_kv writes
must equal, bit for bit, the oracle's exact dequantised values rounded to fp32 (TQ3 values are
exact in fp32; FP8 values are the fp32 product dec(code) * scale)."""
import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200 import MkvError
from mixed_format_paged_mkv_b200.workloads import WORKLOADS, Workload

from harness import lib_pool, oracle_pool

pytestmark = pytest.mark.gpu


def check_bit_exact(lp, op, seqs):
    for s in seqs:
        k, v = lp.materialise(s)
        torch.cuda.synchronize()
        K, V = op.dequant_seq(s)
        for got, ref, name in ((k, K, "K"), (v, V, "V")):
            got = got.cpu().numpy()
            want = ref.astype(np.float32)
            assert got.shape == want.shape, (s, name, got.shape, want.shape)
            if not np.array_equal(got.view(np.uint32), want.view(np.uint32)):
                bad = np.argwhere(got.view(np.uint32) != want.view(np.uint32))
                t, h, d = bad[0]
                raise AssertionError(f"seq {s} {name}: {len(bad)} values differ, first at token {t} "
                                     f"head {h} channel {d}: got {got[t, h, d]!r} want {want[t, h, d]!r}")
    lp.device_status()


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (3, dict(B=3, ctx_range=(300, 1500), window=128, protect_frac=0.1)),
    (4, dict(B=2, ctx=(2500, 1001), layers=1)),
])
def test_materialise_matches_oracle(cfg, kw):
    w = WORKLOADS[cfg].scaled(**kw)
    check_bit_exact(lib_pool(w), oracle_pool(w), range(w.B))


@pytest.mark.parametrize("D,ctx", [(64, (1, 17, 90)), (128, (16, 333)), (256, (15, 48))])
def test_head_dims_and_ragged_tails(D, ctx):
    w = Workload("mat", 21, B=len(ctx), Hq=4, Hkv=2, D=D, q_len=1, window=16, ctx=ctx,
                 outliers=True)
    check_bit_exact(lib_pool(w), oracle_pool(w), range(w.B))


def test_materialise_rejects_small_outputs_and_empty_is_a_no_op():
    w = Workload("mat", 22, B=2, Hq=4, Hkv=2, D=128, q_len=1, window=16, ctx=(40, 1))
    lp = lib_pool(w)
    small = torch.empty((39, 2, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(MkvError) as e:
        lp.materialise(0, small, small)
    assert e.value.name == "INVALID_ARG"
    lp.reset(1)
    k, v = lp.materialise(1)
    assert k.shape == (0, 2, 128) and v.shape == (0, 2, 128)
    lp.device_status()
