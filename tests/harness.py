"""Shared helpers of the tests: replay a workload's pool calls on the oracle and on the
CUDA library, and compare outputs with the attention tolerance (max-abs 2e-3, rel-L2 1e-3)."""
from __future__ import annotations

import numpy as np

from mixed_format_paged_mkv_b200.workloads import Workload
from oracle import attention as A
from oracle import formats as F
from oracle import pool as P

ATOL = 2e-3
REL_L2 = 1e-3


def oracle_pool(w: Workload, layer: int = 0, shape: dict | None = None, seqs=None, heads=None,
                bf16_control: bool = False):
    """Oracle pool after the workload's build calls.  ``seqs`` restricts the build to some
    sequences (their contents do not depend on the others); ``heads`` keeps only some KV
    heads (pages of one head depend only on that head's inputs).  ``bf16_control`` builds the
    BF16 control pool instead (pages keep their bf16 values, nothing is demoted)."""
    shape = shape or w.pool_shape()
    Hkv = shape["num_kv_heads"] if heads is None else len(heads)
    pool = P.RefPool(Hkv, shape["head_dim"], shape["max_seqs"], shape["max_pages_per_seq"],
                     shape["fp8_slots"], shape["tq3_slots"], bf16_control=bf16_control)
    if seqs is None and heads is None:
        for fmt, key in ((P.FP8, "fp8_slots"), (P.TQ3, "tq3_slots")):
            order = w.slot_permutation(fmt, shape[key])
            if order is not None:
                pool.set_slot_order(fmt, order)
    for op in w.build_ops(layer):
        if seqs is not None and op[1] not in seqs:
            continue
        if op[0] == "append":
            k, v = w.kv(op[1], layer)
            if heads is not None:
                k, v = k[:, heads], v[:, heads]
            pool.append([op[1]], [op[2]], F.bf16_bits_to_f64(k), F.bf16_bits_to_f64(v))
        elif op[0] == "protect":
            for p in op[2]:
                pool.set_protected(op[1], p, 1)
        else:
            pool.demote([op[1]], op[2])
    return pool


def to_bf16_tensor(bits, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def lib_pool(w: Workload, layer: int = 0, shape: dict | None = None, host_only: bool = False,
             bf16_control: bool = False):
    """Library pool after the same build calls (inputs copied to the device per call)."""
    from mixed_format_paged_mkv_b200 import Pool
    shape = shape or w.pool_shape()
    pool = Pool(**shape, host_only=host_only, bf16_control=bf16_control)
    for fmt, key in ((0, "fp8_slots"), (1, "tq3_slots")):
        order = w.slot_permutation(fmt, shape[key])
        if order is not None:
            pool.set_slot_order(fmt, order)
    for op in w.build_ops(layer):
        if op[0] == "append":
            if host_only:
                pool.append([op[1]], [op[2]])
            else:
                k, v = w.kv(op[1], layer)
                pool.append([op[1]], [op[2]], to_bf16_tensor(k), to_bf16_tensor(v))
        elif op[0] == "protect":
            for p in op[2]:
                pool.set_protected(op[1], p, True)
        else:
            pool.demote([op[1]], op[2])
    return pool


def oracle_decode(pool, w: Workload, seq: int, layer: int = 0, sm_scale=None, heads=None):
    """float64 attention of one sequence: [q_len, Hq, D] (only the query heads of ``heads``'
    groups when given, in order)."""
    q = F.bf16_bits_to_f64(w.q(seq, layer))
    if heads is not None:
        q = np.concatenate([q[:, h * w.g:(h + 1) * w.g] for h in heads], axis=1)
    K, V = pool.dequant_seq(seq)
    scale = 1.0 / np.sqrt(w.D) if sm_scale is None else sm_scale
    return A.attention(K, V, q, scale)


def assert_close(got, ref, atol=ATOL, rel=REL_L2, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    rl2 = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= atol, f"{what}: max-abs {err.max():.3e} > {atol}"
    assert rl2 <= rel, f"{what}: rel-L2 {rl2:.3e} > {rel}"
    return float(err.max()), float(rl2)
