"""GPU parity of decode attention when K and V are far from unit scale.

The oracle handles any finite bf16 input, so the library must too: K and V scaled by 1e-4, 1e3
and 3e4, and caches whose 32-channel groups and tokens mix those scales.  Attention outputs are
convex combinations of V rows, so their error is judged in units of V's scale: the outputs and
the oracle's are both divided by the V multiplier before the usual bounds (max-abs 2e-3, rel-L2
1e-3) are applied.  With mixed scales every 32-channel group of the output is judged against the
largest dequantised |V| of that group in the sequence, and the whole output by rel-L2.

The inputs with K scaled by 4 make the logits climb by more than 8 (log2 units) after the first
pages, so probabilities reach 2^8 relative to the running reference maximum.
"""
import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200.workloads import Workload

from harness import ATOL, REL_L2, assert_close, lib_pool, oracle_pool, to_bf16_tensor
from oracle import attention as A
from oracle import formats as F

pytestmark = pytest.mark.gpu


def _base(**kw):
    args = dict(name="range", cfg=40, B=2, Hq=8, Hkv=2, D=256, q_len=1, window=32,
                ctx=(700, 1500), outliers=False)
    args.update(kw)
    return Workload(**args)


def _decode(w):
    lp = lib_pool(w)
    op = oracle_pool(w)
    q = to_bf16_tensor(np.stack([w.q(s) for s in range(w.B)]))
    out = lp.decode(list(range(w.B)), q).cpu().numpy()
    torch.cuda.synchronize()
    lp.device_status()
    refs, vmax = [], []
    for s in range(w.B):
        K, V = op.dequant_seq(s)
        qs = F.bf16_bits_to_f64(w.q(s))
        refs.append(A.attention(K, V, qs, 1.0 / np.sqrt(w.D)))
        vmax.append(np.abs(V).max(axis=0))     # [Hkv, D]
    return out, refs, vmax


@pytest.mark.parametrize("k_scale,v_scale", [
    (1.0, 1e-4), (1e-4, 1.0), (1e-4, 1e-4),
    (1.0, 1e3), (4.0, 1e3), (1e3, 1.0), (1e3, 1e3),
    (1.0, 3e4), (4.0, 3e4), (3e4, 3e4),
])
@pytest.mark.parametrize("D", [128, 256])
def test_uniform_scales(k_scale, v_scale, D):
    w = _base(D=D, k_scale=k_scale, v_scale=v_scale, cfg=41 + D)
    out, refs, _ = _decode(w)
    for s in range(w.B):
        assert_close(out[s] / v_scale, refs[s] / v_scale,
                     what=f"K x{k_scale:g} V x{v_scale:g} D {D} seq {s}")


@pytest.mark.parametrize("k_scale,v_scale", [(1.0, 1e-4), (4.0, 1e3), (4.0, 3e4), (1e3, 1e3)])
@pytest.mark.parametrize("D", [64, 256])
def test_uniform_scales_many_query_columns(k_scale, v_scale, D):
    """q_len 4 with 6 query heads per KV head: 24 query columns, the team layout (each page
    decoded once for three n-tiles; two warps for D 64, four for D 256)."""
    w = _base(D=D, Hq=12, Hkv=2, q_len=4, k_scale=k_scale, v_scale=v_scale, cfg=45 + D,
              ctx=(900, 260))
    out, refs, _ = _decode(w)
    for s in range(w.B):
        assert_close(out[s] / v_scale, refs[s] / v_scale,
                     what=f"q_len 4 K x{k_scale:g} V x{v_scale:g} D {D} seq {s}")


@pytest.mark.parametrize("D,q_len,k_scale", [(256, 1, 1.0), (128, 1, 4.0), (256, 3, 1.0),
                                             (64, 2, 1.0), (64, 4, 4.0)])
def test_mixed_group_and_token_scales(D, q_len, k_scale):
    """Every (token, KV head, 32-channel group) of K and V has its own multiplier from 1e-4 to
    3e4, so one page mixes scales across groups and tokens."""
    w = _base(D=D, q_len=q_len, k_scale=k_scale, scale_mix=True, cfg=50 + D + q_len,
              ctx=(900, 333))
    out, refs, vmax = _decode(w)
    g = w.g
    for s in range(w.B):
        got = out[s].astype(np.float64)
        ref = refs[s]
        assert np.all(np.isfinite(got)), f"seq {s}: non-finite output"
        for hq in range(w.Hq):
            h = hq // g
            for grp in range(w.D // 32):
                sl = slice(32 * grp, 32 * grp + 32)
                unit = max(vmax[s][h, sl].max(), 1e-30)
                err = np.abs(got[:, hq, sl] - ref[:, hq, sl]).max() / unit
                assert err <= ATOL, (f"seq {s} head {hq} group {grp}: max-abs {err:.3e} of the "
                                     f"group's largest |V| ({unit:.3e})")
        rl2 = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
        assert rl2 <= REL_L2, f"seq {s}: rel-L2 {rl2:.3e}"
