"""Python binding of ``libmkv.so`` (the C ABI in ``include/mkv.h``): argument marshalling only.

PyTorch supplies device memory and the current CUDA stream; every step of append, demotion
and decode runs in the library's kernels.  There is no fallback: if the library is missing or
a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmkv.so")

FMT_FP8, FMT_TQ3, FMT_BF16 = 0, 1, 2
POOL_HOST_ONLY, POOL_BF16_CONTROL = 1, 2
ERRORS = {0: "OK", -1: "INVALID_ARG", -2: "BAD_SEQ", -3: "OUT_OF_PAGES", -4: "EMPTY_CONTEXT",
          -5: "PAGE_NOT_FULL", -6: "WORKSPACE_TOO_SMALL", -7: "CUDA", -8: "DEVICE_CHECK",
          -9: "DEVICE_TIMEOUT", -10: "UNSUPPORTED"}

# exported symbol -> (restype, argtypes)
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I32P = ctypes.POINTER(ctypes.c_int32)
_SZP = ctypes.POINTER(ctypes.c_size_t)


class PoolConfig(ctypes.Structure):
    _fields_ = [("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("max_seqs", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("fp8_slots", ctypes.c_int32),
                ("tq3_slots", ctypes.c_int32), ("sink_pages", ctypes.c_int32),
                ("flags", ctypes.c_int32)]


SIGNATURES = {
    "mkv_pool_required_bytes": (ctypes.c_int, [ctypes.POINTER(PoolConfig), _SZP, _SZP, _SZP, _SZP]),
    "mkv_pool_create": (ctypes.c_int, [ctypes.POINTER(PoolConfig), _P, _P, _P, _P,
                                       ctypes.POINTER(_P)]),
    "mkv_pool_destroy": (None, [_P]),
    "mkv_pool_set_slot_order": (ctypes.c_int, [_P, _I32, _I32P, _I32]),
    "mkv_append_kv": (ctypes.c_int, [_P, _I32P, _I32P, _I32, _P, _P, _P]),
    "mkv_set_protected": (ctypes.c_int, [_P, _I32, _I32, _I32]),
    "mkv_demote_pages": (ctypes.c_int, [_P, _I32P, _I32, _I32, _I32P, _P]),
    "mkv_decode_workspace_bytes": (ctypes.c_int, [_P, _I32P, _I32, _I32, _I32, _SZP]),
    "mkv_decode_plan": (ctypes.c_int, [_P, _I32P, _I32, _I32, _I32, _I32P, _I32, _I32P, _I32P]),
    "mkv_decode_attention": (ctypes.c_int, [_P, _I32P, _I32, _I32, _P, _I32, ctypes.c_float,
                                            _P, _P, ctypes.c_size_t, _P]),
    "mkv_decode_attention_noalloc": (ctypes.c_int, [_P, _I32P, _I32, _I32, _P, _I32,
                                                    ctypes.c_float, _P, _P]),
    "mkv_seq_reset": (ctypes.c_int, [_P, _I32, _P]),
    "mkv_seq_copy": (ctypes.c_int, [_P, _I32, _I32, _P]),
    "mkv_materialise_kv": (ctypes.c_int, [_P, _I32, _P, _P, ctypes.c_int64, _P]),
    "mkv_prefill_kv": (ctypes.c_int, [_P, _I32P, _I32P, _I32, _P, _P, _I32, _P]),
    "mkv_selftest_wait": (ctypes.c_int, [_P, ctypes.c_int64, _P]),
    "mkv_selftest_tc_logits": (ctypes.c_int, [_P, _P, _P, _P, _P]),
    "mkv_get_block_table": (ctypes.c_int, [_P, _I32, _I32P, _I32, _I32P, _I32P]),
    "mkv_slot_bytes": (ctypes.c_int, [_P, _I32, _SZP]),
    "mkv_read_slot": (ctypes.c_int, [_P, _I32, _P, ctypes.c_size_t, _P]),
    "mkv_pool_stats": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int64), _I32P, _I32P,
                                      ctypes.POINTER(ctypes.c_double)]),
    "mkv_get_device_status": (ctypes.c_int, [_P, _P]),
    "mkv_timing_enable": (ctypes.c_int, [_P, _I32]),
    "mkv_timing_read": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int64)]),
    "mkv_launch_count": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int64)]),
    "mkv_test_fail_launch": (ctypes.c_int, [_P, _I32]),
    "mkv_set_decode_kernels": (ctypes.c_int, [_P, _I32]),
    "mkv_set_decode_sms": (ctypes.c_int, [_P, _I32]),
    "mkv_last_error": (ctypes.c_char_p, []),
}

_lib = None


class MkvError(RuntimeError):
    def __init__(self, code: int, fn: str, msg: str):
        super().__init__(f"{fn} -> {ERRORS.get(code, code)}: {msg}")
        self.code = code
        self.name = ERRORS.get(code, str(code))


def lib():
    """Load libmkv.so (built in-tree by ``_build.py``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run "
                               "`python -m mixed_format_paged_mkv_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int, fn: str):
    if rc != 0:
        raise MkvError(rc, fn, lib().mkv_last_error().decode())


def _i32_array(xs):
    a = np.ascontiguousarray(np.asarray(xs, dtype=np.int32))
    return a, a.ctypes.data_as(_I32P)


def _stream_ptr(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class Pool:
    """A mixed-format paged KV cache over device buffers owned by this object (torch)."""

    def __init__(self, num_kv_heads, head_dim, max_seqs, max_pages_per_seq, fp8_slots,
                 tq3_slots, sink_pages=1, device=None, host_only=False, bf16_control=False):
        flags = (POOL_HOST_ONLY if host_only else 0) | (POOL_BF16_CONTROL if bf16_control else 0)
        self.cfg = PoolConfig(num_kv_heads, head_dim, 16, max_seqs, max_pages_per_seq,
                              fp8_slots, tq3_slots, sink_pages, flags)
        self.bf16_control = bf16_control
        self.Hkv, self.D = num_kv_heads, head_dim
        self.host_only = host_only
        L = lib()
        sizes = [ctypes.c_size_t() for _ in range(4)]
        _check(L.mkv_pool_required_bytes(ctypes.byref(self.cfg), *[ctypes.byref(s) for s in sizes]),
               "mkv_pool_required_bytes")
        self.bytes = [s.value for s in sizes]
        handle = ctypes.c_void_p()
        if host_only:
            self.buffers = None
            ptrs = [None, None, None, None]
        else:
            import torch
            dev = torch.device(device or "cuda")
            self.buffers = [torch.empty(max(b, 256), dtype=torch.uint8, device=dev)
                            for b in self.bytes]
            ptrs = [ctypes.c_void_p(b.data_ptr()) for b in self.buffers]
        _check(L.mkv_pool_create(ctypes.byref(self.cfg), *ptrs, ctypes.byref(handle)),
               "mkv_pool_create")
        self.handle = handle

    # ------------------------------------------------------------------ lifecycle
    def close(self):
        if getattr(self, "handle", None) and self.handle.value:
            lib().mkv_pool_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ calls
    def set_slot_order(self, fmt, order):
        a, p = _i32_array(order)
        _check(lib().mkv_pool_set_slot_order(self.handle, fmt, p, a.size), "mkv_pool_set_slot_order")

    def append(self, seq_ids, n_new, k=None, v=None, stream=None):
        import torch
        s, sp = _i32_array(seq_ids)
        n, np_ = _i32_array(n_new)
        if self.host_only:
            kp = vp = None
            st = None
        else:
            kp = _dev_ptr(k, torch.bfloat16, "k")
            vp = _dev_ptr(v, torch.bfloat16, "v")
            rows = int(n.sum())
            if tuple(k.shape) != (rows, self.Hkv, self.D) or tuple(v.shape) != (rows, self.Hkv, self.D):
                raise ValueError(f"k, v must be [{rows}, {self.Hkv}, {self.D}]")
            st = _stream_ptr(stream)
        _check(lib().mkv_append_kv(self.handle, sp, np_, s.size, kp, vp, st), "mkv_append_kv")

    def prefill(self, seq_ids, n_tokens, k=None, v=None, window=0, stream=None):
        """First tokens of empty sequences; full pages the anchor policy would demote at once
        are packed to TQ3 straight from bf16 (mkv_prefill_kv)."""
        import torch
        s, sp = _i32_array(seq_ids)
        n, np_ = _i32_array(n_tokens)
        if self.host_only:
            kp = vp = None
            st = None
        else:
            kp = _dev_ptr(k, torch.bfloat16, "k")
            vp = _dev_ptr(v, torch.bfloat16, "v")
            rows = int(n.sum())
            if tuple(k.shape) != (rows, self.Hkv, self.D) or tuple(v.shape) != (rows, self.Hkv, self.D):
                raise ValueError(f"k, v must be [{rows}, {self.Hkv}, {self.D}]")
            st = _stream_ptr(stream)
        _check(lib().mkv_prefill_kv(self.handle, sp, np_, s.size, kp, vp, int(window), st),
               "mkv_prefill_kv")

    def selftest_wait(self, limit_ns=1_000_000, stream=None):
        """Launch the bounded-wait self-test; the next device_status() raises DEVICE_TIMEOUT."""
        st = None if self.host_only else _stream_ptr(stream)
        _check(lib().mkv_selftest_wait(self.handle, int(limit_ns), st), "mkv_selftest_wait")

    def selftest_tc_logits(self, a, q, stream=None):
        """fp32 [128, 8] = a [128, 256] . q [8, 256]^T (f16 device tensors) through tensor memory
        and tcgen05.mma (mkv_selftest_tc_logits)."""
        import torch
        if tuple(a.shape) != (128, 256) or tuple(q.shape) != (8, 256):
            raise ValueError("a must be [128, 256] and q [8, 256]")
        d = torch.empty((128, 8), dtype=torch.float32, device=a.device)
        _check(lib().mkv_selftest_tc_logits(self.handle, _dev_ptr(a, torch.float16, "a"),
                                            _dev_ptr(q, torch.float16, "q"),
                                            _dev_ptr(d, torch.float32, "d"), _stream_ptr(stream)),
               "mkv_selftest_tc_logits")
        return d

    def set_protected(self, seq, page, flag=True):
        _check(lib().mkv_set_protected(self.handle, seq, page, 1 if flag else 0), "mkv_set_protected")

    def demote(self, seq_ids, window_tokens, stream=None):
        s, sp = _i32_array(seq_ids)
        n = ctypes.c_int32(0)
        st = None if self.host_only else _stream_ptr(stream)
        _check(lib().mkv_demote_pages(self.handle, sp, s.size, window_tokens, ctypes.byref(n), st),
               "mkv_demote_pages")
        return n.value

    def workspace_bytes(self, seq_ids, q_len, num_q_heads):
        s, sp = _i32_array(seq_ids)
        b = ctypes.c_size_t()
        _check(lib().mkv_decode_workspace_bytes(self.handle, sp, s.size, q_len, num_q_heads,
                                                ctypes.byref(b)), "mkv_decode_workspace_bytes")
        return b.value

    def decode_plan(self, seq_ids, q_len, num_q_heads):
        """The work units a decode call would cut (mkv_decode_plan): int32 [units, 6] rows of
        (call position, format, first logical page, end logical page, pages of that format, CTA),
        CTA by CTA, and the CTA budget of one wave."""
        s, sp = _i32_array(seq_ids)
        n, wave = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().mkv_decode_plan(self.handle, sp, s.size, q_len, num_q_heads, None, 0,
                                     ctypes.byref(n), ctypes.byref(wave)), "mkv_decode_plan")
        u = np.zeros((max(n.value, 1), 6), dtype=np.int32)
        _check(lib().mkv_decode_plan(self.handle, sp, s.size, q_len, num_q_heads,
                                     u.ctypes.data_as(_I32P), n.value, ctypes.byref(n), None),
               "mkv_decode_plan")
        return u[:n.value], wave.value

    def decode(self, seq_ids, q, sm_scale=None, out=None, workspace=None, stream=None):
        """q: bf16 [n, q_len, Hq, D] on the device -> fp32 [n, q_len, Hq, D]."""
        import torch
        s, sp = _i32_array(seq_ids)
        n, q_len, Hq, D = q.shape
        if n != s.size or D != self.D:
            raise ValueError("q must be [len(seq_ids), q_len, Hq, head_dim]")
        qp = _dev_ptr(q, torch.bfloat16, "q")
        if out is None:
            out = torch.empty((n, q_len, Hq, D), dtype=torch.float32, device=q.device)
        op = _dev_ptr(out, torch.float32, "out")
        if workspace is None:   # the library checks a caller-given workspace's size itself
            workspace = torch.empty(self.workspace_bytes(s, q_len, Hq), dtype=torch.uint8,
                                    device=q.device)
        wp = _dev_ptr(workspace, torch.uint8, "workspace")
        scale = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
        _check(lib().mkv_decode_attention(self.handle, sp, s.size, q_len, qp, Hq,
                                          ctypes.c_float(scale), op, wp, workspace.numel(),
                                          _stream_ptr(stream)), "mkv_decode_attention")
        return out

    def reset(self, seq, stream=None):
        st = None if self.host_only else _stream_ptr(stream)
        _check(lib().mkv_seq_reset(self.handle, seq, st), "mkv_seq_reset")

    def copy(self, src, dst, stream=None):
        st = None if self.host_only else _stream_ptr(stream)
        _check(lib().mkv_seq_copy(self.handle, src, dst, st), "mkv_seq_copy")

    def materialise(self, seq, k_out=None, v_out=None, stream=None):
        """Dense fp32 dequantised K and V of a sequence, [ctx, Hkv, D] each (a debugging and
        quality-control path; decode never uses it)."""
        if self.host_only:  # the library rejects it (no device pages)
            _check(lib().mkv_materialise_kv(self.handle, seq, None, None, 0, None),
                   "mkv_materialise_kv")
        import torch
        _, ctx = self.block_table(seq)
        dev = self.buffers[0].device
        shape = (ctx, self.Hkv, self.D)
        k_out = torch.empty(shape, dtype=torch.float32, device=dev) if k_out is None else k_out
        v_out = torch.empty(shape, dtype=torch.float32, device=dev) if v_out is None else v_out
        kp = _dev_ptr(k_out, torch.float32, "k_out")
        vp = _dev_ptr(v_out, torch.float32, "v_out")
        cap = min(k_out.numel(), v_out.numel()) // (self.Hkv * self.D)
        _check(lib().mkv_materialise_kv(self.handle, seq, kp, vp, cap, _stream_ptr(stream)),
               "mkv_materialise_kv")
        return k_out, v_out

    def block_table(self, seq):
        n = ctypes.c_int32()
        ctx = ctypes.c_int32()
        _check(lib().mkv_get_block_table(self.handle, seq, None, 0, ctypes.byref(n), ctypes.byref(ctx)),
               "mkv_get_block_table")
        a = np.zeros(max(n.value, 1), dtype=np.int32)
        _check(lib().mkv_get_block_table(self.handle, seq, a.ctypes.data_as(_I32P), n.value, None, None),
               "mkv_get_block_table")
        return a[:n.value].tolist(), ctx.value

    def slot_bytes(self, fmt):
        b = ctypes.c_size_t()
        _check(lib().mkv_slot_bytes(self.handle, fmt, ctypes.byref(b)), "mkv_slot_bytes")
        return b.value

    def read_slot(self, entry, stream=None):
        nb = self.slot_bytes((entry >> 30) & 3)  # format tag (a BF16 entry is negative)
        buf = np.zeros(nb, dtype=np.uint8)
        _check(lib().mkv_read_slot(self.handle, entry, buf.ctypes.data_as(_P), nb,
                                   _stream_ptr(stream)), "mkv_read_slot")
        return buf

    def stats(self):
        live = ctypes.c_int64()
        n8 = ctypes.c_int32()
        n3 = ctypes.c_int32()
        bpt = ctypes.c_double()
        _check(lib().mkv_pool_stats(self.handle, ctypes.byref(live), ctypes.byref(n8),
                                    ctypes.byref(n3), ctypes.byref(bpt)), "mkv_pool_stats")
        return live.value, n8.value, n3.value, bpt.value

    def device_status(self, stream=None):
        """Raise MkvError if a kernel flagged an invalid entry/input or a timed-out wait."""
        _check(lib().mkv_get_device_status(self.handle, _stream_ptr(stream)), "mkv_get_device_status")

    def timing(self, enable=True):
        _check(lib().mkv_timing_enable(self.handle, 1 if enable else 0), "mkv_timing_enable")

    def timing_read(self):
        """{'partial_ms', 'merge_ms': summed device time of each decode kernel, 'calls'}."""
        v = [ctypes.c_double(), ctypes.c_double()]
        n = ctypes.c_int64()
        _check(lib().mkv_timing_read(self.handle, ctypes.byref(v[0]), ctypes.byref(v[1]),
                                     ctypes.byref(n)), "mkv_timing_read")
        return dict(partial_ms=v[0].value, merge_ms=v[1].value, calls=n.value)

    def set_decode_kernels(self, fused):
        """Decode with one fused partial grid (True), a grid per page format (False) or the
        automatic per-call choice (None, the default)."""
        mode = 2 if fused is None else (1 if fused else 0)
        _check(lib().mkv_set_decode_kernels(self.handle, mode), "mkv_set_decode_kernels")

    def set_decode_sms(self, sms):
        """Plan later decode calls for at most ``sms`` SMs (0: all of the device's)."""
        _check(lib().mkv_set_decode_sms(self.handle, int(sms)), "mkv_set_decode_sms")

    def test_fail_launch(self, after):
        """Make the device operation after the next ``after`` ones fail (test hook; -1: off)."""
        _check(lib().mkv_test_fail_launch(self.handle, int(after)), "mkv_test_fail_launch")

    def launch_count(self):
        n = ctypes.c_int64()
        _check(lib().mkv_launch_count(self.handle, ctypes.byref(n)), "mkv_launch_count")
        return n.value
