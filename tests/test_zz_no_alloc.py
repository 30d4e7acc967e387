"""GPU test of mkv_decode_attention_noalloc, the decode entry point for callers that cannot
allocate device memory (for example code under stream capture, or a runtime that owns the
whole device-memory budget): it keeps its partial states in a static device array inside the
library instead of a caller workspace.

Calls the entry point through the C ABI twice in a row (the second call finds the first call's
contents in the shared array) and checks each output against mkv_decode_attention on the same
inputs, with the attention tolerance of the other tests; also checks that a call needing more
scratch than the static array holds is rejected with MKV_ERR_WORKSPACE_TOO_SMALL.  Kept in a
file of its own, collected last."""
import ctypes
import math

import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200 import Pool, api
from mixed_format_paged_mkv_b200.workloads import WORKLOADS

from harness import assert_close, lib_pool, to_bf16_tensor

pytestmark = pytest.mark.gpu


def noalloc_decode(pool, seq_ids, q, sm_scale, out):
    s = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
    n, q_len, Hq, _ = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return api.lib().mkv_decode_attention_noalloc(
        pool.handle, s.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), s.size, q_len,
        ctypes.c_void_p(q.data_ptr()), Hq, ctypes.c_float(sm_scale),
        ctypes.c_void_p(out.data_ptr()), stream)


def test_noalloc_matches_workspace_decode_twice():
    w = WORKLOADS[4].scaled(B=3, ctx=(9000, 4100, 700), layers=1)
    lp = lib_pool(w)
    seqs = list(range(w.B))
    scale = 1.0 / math.sqrt(w.D)
    rng = np.random.default_rng(21)
    for call in range(2):
        q = torch.from_numpy(rng.standard_normal((w.B, 1, w.Hq, w.D), dtype=np.float32)).to(
            torch.bfloat16).cuda()
        ref = lp.decode(seqs, q, sm_scale=scale).cpu().numpy()
        out = torch.full((w.B, 1, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
        rc = noalloc_decode(lp, seqs, q, scale, out)
        assert rc == 0, api.lib().mkv_last_error().decode()
        got = out.cpu().numpy()
        lp.device_status()
        for s in seqs:
            assert_close(got[s], ref[s], what=f"call {call} seq {s}")


def test_noalloc_rejects_calls_beyond_the_static_scratch():
    # many short sequences: at least two partial states each (FP8 page 0 and the TQ3 rest), so
    # the call needs more than the 32 MiB static scratch whatever the unit cut
    Hkv, D, B, L = 8, 256, 80, 512
    pool = Pool(Hkv, D, B, L // 16 + 1, L // 16 + B + 64, B * (L // 16) + 8)
    z = torch.zeros((L, Hkv, D), dtype=torch.bfloat16, device="cuda")
    for s in range(B):
        pool.append([s], [L], z, z)
        pool.demote([s], 0)
    q = torch.zeros((B, 4, 8 * Hkv, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, 4, 8 * Hkv, D), dtype=torch.float32, device="cuda")
    assert pool.workspace_bytes(list(range(B)), 4, 8 * Hkv) > (32 << 20)
    rc = noalloc_decode(pool, list(range(B)), q, 0.0625, out)
    assert api.ERRORS[rc] == "WORKSPACE_TOO_SMALL", api.lib().mkv_last_error().decode()
    assert b"static scratch" in api.lib().mkv_last_error()
