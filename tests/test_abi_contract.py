"""The C ABI's documented argument contract, called directly through ctypes on the CPU.

Every int-returning entry point rejects a NULL pool with MKV_ERR_INVALID_ARG and leaves a
message in mkv_last_error(); a successful call clears it.  Pool creation validates the
configuration and the buffers' presence and 256-byte alignment before any CUDA call; device-only
calls reject host-only pools; inspection calls follow their NULL-output conventions.
"""
import ctypes

import numpy as np
import pytest

from mixed_format_paged_mkv_b200.api import POOL_HOST_ONLY, PoolConfig, lib

OK, INVALID_ARG, BAD_SEQ, UNSUPPORTED = 0, -1, -2, -10


def last_error():
    return lib().mkv_last_error().decode()


def cfg(**kw):
    c = dict(num_kv_heads=2, head_dim=64, page_size=16, max_seqs=4, max_pages_per_seq=8,
             fp8_slots=8, tq3_slots=8, sink_pages=1, flags=POOL_HOST_ONLY)
    c.update(kw)
    return PoolConfig(**c)


def host_pool():
    h = ctypes.c_void_p()
    c = cfg()
    assert lib().mkv_pool_create(ctypes.byref(c), None, None, None, None, ctypes.byref(h)) == OK
    return h


def i32p(*v):
    a = (ctypes.c_int32 * max(len(v), 1))(*v)
    return ctypes.cast(a, ctypes.POINTER(ctypes.c_int32)), a


def test_null_pool_is_rejected_everywhere():
    L = lib()
    seqs, _keep = i32p(0)
    n = ctypes.c_int32()
    sz = ctypes.c_size_t()
    i64 = ctypes.c_int64()
    calls = {
        "mkv_pool_set_slot_order": (None, 0, seqs, 1),
        "mkv_append_kv": (None, seqs, seqs, 1, None, None, None),
        "mkv_set_protected": (None, 0, 0, 1),
        "mkv_demote_pages": (None, seqs, 1, 0, ctypes.byref(n), None),
        "mkv_decode_workspace_bytes": (None, seqs, 1, 1, 2, ctypes.byref(sz)),
        "mkv_decode_plan": (None, seqs, 1, 1, 2, None, 0, ctypes.byref(n), None),
        "mkv_decode_attention": (None, seqs, 1, 1, None, 2, ctypes.c_float(1.0), None, None, 0,
                                 None),
        "mkv_decode_attention_noalloc": (None, seqs, 1, 1, None, 2, ctypes.c_float(1.0), None,
                                         None),
        "mkv_seq_reset": (None, 0, None),
        "mkv_seq_copy": (None, 0, 1, None),
        "mkv_materialise_kv": (None, 0, None, None, 0, None),
        "mkv_prefill_kv": (None, seqs, seqs, 1, None, None, 0, None),
        "mkv_selftest_wait": (None, 1000, None),
        "mkv_selftest_tc_logits": (None, None, None, None, None),
        "mkv_get_block_table": (None, 0, None, 0, ctypes.byref(n), None),
        "mkv_slot_bytes": (None, 0, ctypes.byref(sz)),
        "mkv_read_slot": (None, 0, None, 0, None),
        "mkv_pool_stats": (None, None, None, None, None),
        "mkv_get_device_status": (None, None),
        "mkv_timing_enable": (None, 1),
        "mkv_timing_read": (None, None, None, None),
        "mkv_launch_count": (None, ctypes.byref(i64)),
    }
    for name, args in calls.items():
        assert getattr(L, name)(*args) == INVALID_ARG, name
        assert last_error(), name
    L.mkv_pool_destroy(None)  # ignored


def test_config_validation_and_required_bytes():
    L = lib()
    sizes = [ctypes.c_size_t() for _ in range(4)]
    c = cfg(flags=0)
    assert L.mkv_pool_required_bytes(ctypes.byref(c), *[ctypes.byref(s) for s in sizes]) == OK
    assert last_error() == ""
    assert [s.value for s in sizes] == [8 * 2 * (32 * 64 + 16), 8 * 2 * 14 * 64, 4 * 8 * 4, 256]
    assert L.mkv_pool_required_bytes(ctypes.byref(c), None, None, None, None) == OK
    assert L.mkv_pool_required_bytes(None, None, None, None, None) == INVALID_ARG
    ctl = cfg(flags=2)      # BF16 control pool: the first slab holds 64*D bytes per head
    assert L.mkv_pool_required_bytes(ctypes.byref(ctl), *[ctypes.byref(s) for s in sizes]) == OK
    assert sizes[0].value == 8 * 2 * 64 * 64
    for bad, code in ((dict(head_dim=96), UNSUPPORTED), (dict(page_size=32), INVALID_ARG),
                      (dict(num_kv_heads=0), INVALID_ARG), (dict(max_seqs=0), INVALID_ARG),
                      (dict(fp8_slots=0), INVALID_ARG), (dict(tq3_slots=-1), INVALID_ARG),
                      (dict(sink_pages=-1), INVALID_ARG), (dict(flags=4), INVALID_ARG),
                      (dict(max_seqs=1 << 16, max_pages_per_seq=1 << 16), INVALID_ARG)):
        c = cfg(**bad)
        assert L.mkv_pool_required_bytes(ctypes.byref(c), None, None, None, None) == code, bad


def test_create_checks_buffers_before_any_device_call():
    L = lib()
    h = ctypes.c_void_p()
    c = cfg()
    assert L.mkv_pool_create(ctypes.byref(c), None, None, None, None, None) == INVALID_ARG
    # host-only pools take no buffers
    assert L.mkv_pool_create(ctypes.byref(c), ctypes.c_void_p(4096), None, None, None,
                             ctypes.byref(h)) == INVALID_ARG
    dev = cfg(flags=0)
    # device pools need every buffer (the TQ3 slab only when it has slots) ...
    assert L.mkv_pool_create(ctypes.byref(dev), None, ctypes.c_void_p(4096), ctypes.c_void_p(8192),
                             ctypes.c_void_p(12288), ctypes.byref(h)) == INVALID_ARG
    # ... each 256-byte aligned; these addresses are never dereferenced: the checks come first
    assert L.mkv_pool_create(ctypes.byref(dev), ctypes.c_void_p(4096 + 16), ctypes.c_void_p(8192),
                             ctypes.c_void_p(12288), ctypes.c_void_p(16384),
                             ctypes.byref(h)) == INVALID_ARG
    assert "aligned" in last_error()
    assert h.value is None


def test_device_only_calls_reject_host_only_pools():
    L = lib()
    p = host_pool()
    try:
        seqs, _k = i32p(0)
        cnt, _c = i32p(20)
        assert L.mkv_append_kv(p, seqs, cnt, 1, None, None, None) == OK
        assert L.mkv_decode_attention(p, seqs, 1, 1, None, 2, ctypes.c_float(0.1), None, None, 0,
                                      None) == INVALID_ARG
        assert L.mkv_decode_attention_noalloc(p, seqs, 1, 1, None, 2, ctypes.c_float(0.1), None,
                                              None) == INVALID_ARG
        assert L.mkv_read_slot(p, 0, None, 0, None) == INVALID_ARG
        assert L.mkv_selftest_wait(p, 1000, None) == INVALID_ARG
        assert L.mkv_selftest_tc_logits(p, None, None, None, None) == INVALID_ARG
        assert L.mkv_materialise_kv(p, 0, None, None, 32, None) == INVALID_ARG
        # host-only pools have nothing on a device to report
        assert L.mkv_get_device_status(p, None) == OK
        assert last_error() == ""
    finally:
        L.mkv_pool_destroy(p)


def test_inspection_output_conventions():
    L = lib()
    p = host_pool()
    try:
        seqs, _k = i32p(1)
        cnt, _c = i32p(40)
        assert L.mkv_append_kv(p, seqs, cnt, 1, None, None, None) == OK
        n, ctx = ctypes.c_int32(), ctypes.c_int32()
        assert L.mkv_get_block_table(p, 1, None, 0, ctypes.byref(n), ctypes.byref(ctx)) == OK
        assert (n.value, ctx.value) == (3, 40)
        out = (ctypes.c_int32 * 2)(-7, -7)
        # a short buffer receives the first entries; the count still says 3
        assert L.mkv_get_block_table(p, 1, out, 2, ctypes.byref(n), None) == OK
        assert n.value == 3 and list(out) == [0, 1]
        assert L.mkv_get_block_table(p, 1, None, 2, None, None) == INVALID_ARG
        assert L.mkv_get_block_table(p, 9, None, 0, None, None) == BAD_SEQ
        sz = ctypes.c_size_t()
        assert L.mkv_slot_bytes(p, 0, ctypes.byref(sz)) == OK and sz.value == 2 * (32 * 64 + 16)
        assert L.mkv_slot_bytes(p, 1, ctypes.byref(sz)) == OK and sz.value == 2 * 14 * 64
        assert L.mkv_slot_bytes(p, 2, ctypes.byref(sz)) == INVALID_ARG
        assert L.mkv_slot_bytes(p, 0, None) == INVALID_ARG
        live, n8, n3 = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        bpt = ctypes.c_double()
        assert L.mkv_pool_stats(p, None, None, None, None) == OK
        assert L.mkv_pool_stats(p, ctypes.byref(live), ctypes.byref(n8), ctypes.byref(n3),
                                ctypes.byref(bpt)) == OK
        assert (live.value, n8.value, n3.value) == (40, 3, 0)
        assert bpt.value == pytest.approx(3 * 2 * (32 * 64 + 16) / 40)
        launches = ctypes.c_int64(-1)
        assert L.mkv_launch_count(p, ctypes.byref(launches)) == OK and launches.value == 0
        assert L.mkv_launch_count(p, None) == INVALID_ARG
        calls = ctypes.c_int64(-1)
        assert L.mkv_timing_enable(p, 1) == OK
        assert L.mkv_timing_read(p, None, None, ctypes.byref(calls)) == OK and calls.value == 0
        assert L.mkv_set_protected(p, 1, 3, 1) == INVALID_ARG      # page 3 not mapped
        assert L.mkv_set_protected(p, 1, 2, 1) == OK
        assert L.mkv_pool_set_slot_order(p, 2, None, 0) == INVALID_ARG
        order, _o = i32p(*range(7))
        assert L.mkv_pool_set_slot_order(p, 0, order, 7) == INVALID_ARG   # 8 slots
    finally:
        L.mkv_pool_destroy(p)
