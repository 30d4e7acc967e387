"""GPU parity of decode attention over the mixed-format cache against the float64 oracle on
identical quantised inputs: max-abs error <= 2e-3 and rel-L2 <= 1e-3 per sequence."""
import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200 import Pool
from mixed_format_paged_mkv_b200.workloads import WORKLOADS, Workload, bf16_bits, long_qlen4
from oracle import attention as A
from oracle import formats as F
from oracle import pool as P

from harness import assert_close, lib_pool, oracle_decode, oracle_pool, to_bf16_tensor

pytestmark = pytest.mark.gpu


def q_tensor(w, layer=0, seqs=None):
    seqs = range(w.B) if seqs is None else seqs
    return to_bf16_tensor(np.stack([w.q(s, layer) for s in seqs]))


def run_and_check(w, lp=None, op=None, sm_scale=None):
    lp = lp or lib_pool(w)
    op = op or oracle_pool(w)
    out = lp.decode(list(range(w.B)), q_tensor(w), sm_scale=sm_scale)
    torch.cuda.synchronize()
    lp.device_status()
    out = out.cpu().numpy()
    for s in range(w.B):
        assert_close(out[s], oracle_decode(op, w, s, sm_scale=sm_scale), what=f"{w.name} seq {s}")
    return lp


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(B=3, ctx=(800, 2048, 1500))),
    (3, dict(B=4, ctx_range=(200, 3000), window=256, protect_frac=0.05)),
    (4, dict(B=2, ctx=(4096, 2500), layers=1)),
    (5, dict(B=5, ctx_range=(300, 2000))),
])
def test_workloads_scaled(cfg, kw):
    run_and_check(WORKLOADS[cfg].scaled(**kw))


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("w", [
    WORKLOADS[2].scaled(B=3, ctx=(800, 2048, 1500)),
    WORKLOADS[3].scaled(B=4, ctx_range=(200, 3000), window=256, protect_frac=0.3),
    Workload("fp8heavy", 17, B=2, Hq=8, Hkv=2, D=256, q_len=1, window=2000, ctx=(2500, 900)),
    Workload("multitok", 18, B=2, Hq=12, Hkv=2, D=128, q_len=3, window=48, ctx=(1200, 77)),
], ids=["batch", "ragged", "fp8heavy", "multitok"])
def test_split_and_fused_partial_kernels(w, fused):
    """The per-format grids (TQ3 grid, then the FP8 grid as its programmatic dependent) and the
    fused grid both match the oracle."""
    lp = lib_pool(w)
    lp.set_decode_kernels(fused)
    run_and_check(w, lp=lp)


def test_decode_planned_for_fewer_sms():
    """A cut planned for 8 SMs (longer units, full page lists) matches the oracle too."""
    w = Workload("fewsms", 19, B=2, Hq=8, Hkv=2, D=128, q_len=1, window=64, ctx=(12000, 900),
                 outliers=True)
    lp = lib_pool(w)
    full, _ = lp.decode_plan([0, 1], 1, 8)
    lp.set_decode_sms(8)
    units, _ = lp.decode_plan([0, 1], 1, 8)
    assert units[:, 4].max() > full[:, 4].max()
    run_and_check(w, lp=lp)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("D,Hq,Hkv,q_len", [(128, 8, 2, 1), (256, 12, 2, 1), (64, 16, 2, 2),
                                            (256, 24, 4, 4)])
def test_ctas_spanning_many_sequences(D, Hq, Hkv, q_len, fused):
    """Sequences of very unequal length, planned for few SMs: the planner takes the line cut,
    and some CTAs take the pieces of several sequences (and, fused, of both formats) one after
    another, re-initialising their ring between them; every piece's partial state reaches the
    merge.  One-tile and team layouts."""
    w = Workload("span", 23, B=5, Hq=Hq, Hkv=Hkv, D=D, q_len=q_len, window=64,
                 ctx=(1500, 1300, 120, 60, 33), protect_frac=0.1, outliers=True)
    lp = lib_pool(w)
    lp.set_decode_kernels(fused)
    for sms in range(1, 64):
        lp.set_decode_sms(sms)
        units, _ = lp.decode_plan(list(range(w.B)), q_len, Hq)
        if np.bincount(units[:, 5]).max() >= 2:
            break
    else:
        pytest.fail("no plan with a CTA that starts several units")
    run_and_check(w, lp=lp)


@pytest.mark.parametrize("fused", [False, True])
def test_fp8_runs_far_apart(fused):
    """Under the line cut, the sink page and the recent window, more than 2048 pages apart, are
    separate FP8 runs, each its own unit (a short scan range); the result still matches the
    oracle.  Unequal lengths and a small SM budget make the planner take the line cut."""
    w = Workload("runs", 29, B=3, Hq=8, Hkv=2, D=128, q_len=1, window=64,
                 ctx=(40000, 36011, 300), outliers=True)
    lp = lib_pool(w)
    lp.set_decode_kernels(fused)
    for sms in range(1, 148):
        lp.set_decode_sms(sms)
        units, _ = lp.decode_plan([0, 1, 2], 1, 8)
        fp8 = units[(units[:, 0] == 0) & (units[:, 1] == 0)]
        if len(fp8) >= 2:
            break
    else:
        pytest.fail("no plan split the FP8 pages into runs")
    assert fp8[:, 2].min() == 0 and fp8[:, 3].max() - fp8[:, 2].max() < 16
    run_and_check(w, lp=lp)


def test_long_qlen4_scaled():
    run_and_check(long_qlen4().scaled(B=2, ctx=(3001, 1200), layers=1))


@pytest.mark.parametrize("Hq,Hkv,q_len", [(2, 2, 1), (4, 2, 3), (8, 1, 4), (12, 2, 2), (6, 6, 5),
                                          (16, 2, 1), (16, 4, 8)])
def test_gqa_widths_and_multi_token(Hq, Hkv, q_len):
    w = Workload("gqa", 11, B=2, Hq=Hq, Hkv=Hkv, D=128, q_len=q_len, window=48,
                 ctx=(333, 70), outliers=True)
    run_and_check(w)


@pytest.mark.parametrize("D,Hq,Hkv,q_len", [(64, 16, 2, 3), (64, 8, 1, 4), (128, 24, 4, 4),
                                            (256, 24, 2, 1)])
def test_team_layout_shapes(D, Hq, Hkv, q_len):
    """More than 8 query columns per KV head (the team layout: one page decoded once for all
    n-tiles) at every head size, and 12 query heads per KV head at q_len 1 (two n-tiles)."""
    w = Workload("team", 20 + D + q_len, B=2, Hq=Hq, Hkv=Hkv, D=D, q_len=q_len, window=48,
                 ctx=(1100, 123), outliers=True)
    for fused in (False, True):
        lp = lib_pool(w)
        lp.set_decode_kernels(fused)
        run_and_check(w, lp=lp)


@pytest.mark.parametrize("ctx", [(1,), (15,), (16,), (17,), (33,), (4, 300)])
def test_short_and_ragged_contexts(ctx):
    w = Workload("short", 12, B=len(ctx), Hq=8, Hkv=2, D=128, q_len=1, window=16, ctx=ctx)
    run_and_check(w)


def test_all_tokens_new_causal():
    w = Workload("allnew", 13, B=2, Hq=4, Hkv=2, D=256, q_len=7, window=0, ctx=(7, 40))
    run_and_check(w)


def test_all_fp8_and_almost_all_tq3():
    base = Workload("fmt", 14, B=2, Hq=8, Hkv=2, D=128, q_len=1, window=10**6, ctx=(700, 301))
    run_and_check(base)                                   # window covers everything: all FP8
    run_and_check(base.scaled(window=0, cfg=15))          # only page 0 and partial tails FP8


def test_head_dim_64_and_custom_scale():
    w = Workload("d64", 16, B=3, Hq=8, Hkv=4, D=64, q_len=2, window=32, ctx=(100, 257, 64),
                 outliers=True)
    run_and_check(w, sm_scale=0.3)


def test_steady_state_append_demote_decode():
    w = WORKLOADS[5].scaled(B=4, ctx_range=(100, 600))
    shape = w.pool_shape(extra_pages_per_seq=4)
    lp = lib_pool(w, shape=shape)
    op = oracle_pool(w, shape=shape)
    rng = np.random.default_rng(5)
    seqs = list(range(w.B))
    for step in range(40):
        k = bf16_bits(rng.standard_normal((w.B, w.Hkv, w.D), dtype=np.float32))
        v = bf16_bits(rng.standard_normal((w.B, w.Hkv, w.D), dtype=np.float32))
        lp.append(seqs, [1] * w.B, to_bf16_tensor(k), to_bf16_tensor(v))
        op.append(seqs, [1] * w.B, F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
        assert lp.demote(seqs, w.window) == len(op.demote(seqs, w.window))
        if step % 13 == 12:
            q = bf16_bits(rng.standard_normal((w.B, 1, w.Hq, w.D), dtype=np.float32))
            out = lp.decode(seqs, to_bf16_tensor(q)).cpu().numpy()
            for s in seqs:
                K, V = op.dequant_seq(s)
                ref = A.attention(K, V, F.bf16_bits_to_f64(q[s]), 1 / np.sqrt(w.D))
                assert_close(out[s], ref, what=f"step {step} seq {s}")
    lp.device_status()


def test_repeated_sequence_rows_and_order():
    w = WORKLOADS[2].scaled(B=3, ctx=(500, 900, 130))
    shape = dict(w.pool_shape(), max_seqs=6)     # a call may list at most max_seqs rows
    lp = lib_pool(w, shape=shape)
    op = oracle_pool(w, shape=shape)
    order = [2, 0, 2, 1]
    q = to_bf16_tensor(np.stack([w.q(s) for s in order]))
    out = lp.decode(order, q).cpu().numpy()
    for i, s in enumerate(order):
        assert_close(out[i], oracle_decode(op, w, s), what=f"row {i}")


def _full_size_reference(args):
    """Oracle output of one (sequence, KV head) of the full-size long-context layer (run in a
    spawned worker: pages of a head depend only on that head's inputs)."""
    s, h = args
    w = WORKLOADS[4].scaled(layers=1)
    op = oracle_pool(w, seqs=[s], heads=[h], shape=dict(w.pool_shape(), num_kv_heads=1))
    return oracle_decode(op, w, s, heads=[h])


@pytest.mark.slow
def test_long_context_full_size_sampled():
    """The long-context workload at full size (4 x 131072 tokens, 24/4 heads, D 256), in the
    launch configuration the benchmark times; the oracle checks one KV-head group of every
    sequence, every KV head index once (24 of the 96 query-head outputs)."""
    import multiprocessing as mp
    pairs = [(0, 0), (1, 2), (2, 1), (3, 3)]
    # the oracle workers start (spawned) before the first GPU call of this test
    with mp.get_context("spawn").Pool(len(pairs)) as workers:
        pending = workers.map_async(_full_size_reference, pairs)
        w = WORKLOADS[4].scaled(layers=1)
        lp = lib_pool(w)
        out = lp.decode(list(range(w.B)), q_tensor(w)).cpu().numpy()
        lp.device_status()
        refs = pending.get(timeout=900)
    assert np.all(np.isfinite(out))
    for (s, h), ref in zip(pairs, refs):
        assert_close(out[s][:, h * w.g:(h + 1) * w.g], ref, what=f"full-size seq {s} head {h}")


def test_more_sequences_than_one_launch_holds():
    """300 sequences (more than a launch's 256) are split into launch groups; every row must
    still come out right, in call order."""
    rng = np.random.default_rng(30)
    n = 300
    ctx = tuple(int(x) for x in rng.integers(1, 60, size=n))
    w = Workload("many", 30, B=n, Hq=4, Hkv=2, D=64, q_len=1, window=16, ctx=ctx)
    lp = lib_pool(w)
    op = oracle_pool(w)
    order = list(rng.permutation(n))
    q = to_bf16_tensor(np.stack([w.q(s) for s in order]))
    out = lp.decode(order, q).cpu().numpy()
    lp.device_status()
    for i, s in enumerate(order):
        assert_close(out[i], oracle_decode(op, w, s), what=f"row {i} seq {s}")


def test_bounded_wait_reports_a_timeout_and_the_context_survives():
    """Failure detection without a fault: a wait that nothing completes gives up after its limit
    and is reported as DEVICE_TIMEOUT; the same context then decodes correctly."""
    from mixed_format_paged_mkv_b200 import MkvError
    w = Workload("wait", 31, B=1, Hq=4, Hkv=2, D=64, q_len=1, window=16, ctx=(100,))
    lp = lib_pool(w)
    lp.device_status()
    lp.selftest_wait(1_000_000)
    with pytest.raises(MkvError) as e:
        lp.device_status()
    assert e.value.name == "DEVICE_TIMEOUT"
    lp.device_status()  # reading cleared it
    run_and_check(w, lp=lp)


def test_corrupted_device_table_entry_is_flagged():
    """A table entry corrupted on the device (slot beyond the slab) is caught by the kernels'
    checks (the page is skipped, not read) and reported as DEVICE_CHECK; restoring it restores
    the result."""
    from mixed_format_paged_mkv_b200 import MkvError
    w = Workload("corrupt", 32, B=2, Hq=4, Hkv=2, D=64, q_len=1, window=16, ctx=(300, 90))
    shape = w.pool_shape()
    lp = lib_pool(w, shape=shape)
    tables = lp.buffers[2].view(torch.int32)
    idx = 0 * shape["max_pages_per_seq"] + 3          # sequence 0, page 3 (TQ3)
    good = int(tables[idx].item())
    assert good >> 30 == 1
    tables[idx] = (1 << 30) | (shape["tq3_slots"] + 7)
    lp.decode([0, 1], q_tensor(w))
    with pytest.raises(MkvError) as e:
        lp.device_status()
    assert e.value.name == "DEVICE_CHECK"
    lp.materialise(0)
    with pytest.raises(MkvError) as e:
        lp.device_status()
    assert e.value.name == "DEVICE_CHECK"
    tables[idx] = good
    run_and_check(w, lp=lp)


def test_decode_argument_errors_are_caught_before_any_launch():
    """A workspace below the planned size, a workspace that is not 256-byte aligned and a
    non-finite sm_scale are rejected by the host before anything is launched; the pool then
    decodes normally."""
    from mixed_format_paged_mkv_b200 import MkvError
    w = Workload("args", 31, B=2, Hq=4, Hkv=2, D=128, q_len=1, window=16, ctx=(300, 45))
    lp = lib_pool(w)
    op = oracle_pool(w)
    seqs = [0, 1]
    q = q_tensor(w)
    need = lp.workspace_bytes(seqs, 1, w.Hq)
    launches = lp.launch_count()
    small = torch.empty(need // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(MkvError) as e:
        lp.decode(seqs, q, workspace=small)
    assert e.value.name == "WORKSPACE_TOO_SMALL"
    big = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(MkvError) as e:
        lp.decode(seqs, q, workspace=big[16:])
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(MkvError) as e:
        lp.decode(seqs, q, sm_scale=float("nan"), workspace=big)
    assert e.value.name == "INVALID_ARG"
    assert lp.launch_count() == launches
    out = lp.decode(seqs, q, workspace=big).cpu().numpy()
    lp.device_status()
    for s in seqs:
        assert_close(out[s], oracle_decode(op, w, s), what=f"seq {s}")
