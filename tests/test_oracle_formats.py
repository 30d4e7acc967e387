"""Pins of the oracle's number formats against what the format definitions fix.

E4M3 is checked against torch's float8_e4m3fn conversion (a library routine), a brute-force
nearest search over all finite codes, and hand-derived vectors; TQ3 against exact rational
arithmetic, an independent big-integer packer, hand-derived bytes and its error bound.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


# ------------------------------------------------------------------ E4M3
def test_e4m3_table_matches_torch_for_all_codes():
    bits = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = bits.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.E4M3_TABLE
    assert np.array_equal(np.isnan(ref), np.isnan(ours))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], ours[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(ours[ok]))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_decode_roundtrip():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes)), codes)


def test_e4m3_golden_vectors():
    for line in _golden_lines("e4m3_vectors.txt"):
        val, code = line.split()[:2]
        assert int(F.e4m3_encode(float(val))) == int(code, 16), line


def test_fp8_page_write_golden_vectors():
    codes = np.zeros((16, 4), dtype=np.uint8)
    scale = 0.0
    lines = [l for l in _golden_lines("fp8_page_vectors.txt")]
    assert len(lines) == 8
    for wl, el in zip(lines[0::2], lines[1::2]):
        head, vals = wl.split(":")
        assert head.split()[0] == "write"
        n_old = int(head.split()[1])
        x = np.array([[float(v) for v in vals.split()]])
        codes, scale = F.fp8_write(codes, scale, n_old, x)
        ehead, rows = el.split(":")
        assert float(ehead.split()[1]) == scale, wl
        want = [[int(c, 16) for c in r.split()] for r in rows.split("|")]
        assert codes[:len(want)].tolist() == want, wl
        assert not codes[len(want):].any()


def _brute_nearest(x):
    """Nearest finite E4M3 value by exhaustive search; ties -> even code; saturating."""
    best = None
    for c in range(256):
        v = F.E4M3_TABLE[c]
        if np.isnan(v) or (np.signbit(v) != np.signbit(x)):
            continue
        d = abs(x - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def test_e4m3_encode_matches_brute_force():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(300) * 50, rng.standard_normal(200) * 0.01,
                        rng.uniform(-460, 460, 200), np.array([449.0, -447.99, 1e-9, -3e-3])])
    x = F.f32(x)
    got = F.e4m3_encode(x)
    for xi, gi in zip(x, got):
        assert gi == _brute_nearest(np.clip(xi, -448, 448)), xi


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 1e-2])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(x.astype(np.float64)), ref)


# ------------------------------------------------------------------ FP8 page write
def test_fp8_fresh_page_scale_and_bound():
    rng = np.random.default_rng(3)
    x = F.f32(rng.standard_normal((16, 64)) * 3)
    codes, scale = F.fp8_write(np.zeros((16, 64), np.uint8), 0.0, 0, x)
    assert scale == float(np.float32(np.abs(x).max() / 448.0))
    xhat = F.fp8_dequant(codes, scale)
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * scale) * (1 + 2.0 ** -20)
    assert np.all(np.abs(x - xhat) <= bound)
    # the largest element lands on (or next to) the top code
    assert np.max(F.e4m3_decode(codes & 0x7F)) >= 416.0


def test_fp8_partial_page_growth_rules():
    rng = np.random.default_rng(4)
    a = F.f32(rng.standard_normal((5, 32)))
    c1, s1 = F.fp8_write(np.zeros((16, 32), np.uint8), 0.0, 0, a)
    # smaller values: scale and existing codes unchanged
    b = a[:3] * 0.25
    c2, s2 = F.fp8_write(c1, s1, 5, b)
    assert s2 == s1 and np.array_equal(c2[:5], c1[:5]) and np.all(c2[8:] == 0)
    # larger values: scale grows to the new candidate, old values re-encoded within bound
    big = F.f32(rng.standard_normal((2, 32)) * 10)
    c3, s3 = F.fp8_write(c2, s2, 8, big)
    assert s3 == float(np.float32(np.abs(big).max() / 448.0)) and s3 > s2
    old = F.fp8_dequant(c3[:5], s3)
    bound = 2 * (np.maximum(2.0 ** -4 * np.abs(a), 2.0 ** -10 * s3)) * (1 + 2.0 ** -20)
    assert np.all(np.abs(old - a) <= bound)
    assert np.all(c3[10:] == 0)


def test_fp8_zero_page():
    c, s = F.fp8_write(np.zeros((16, 32), np.uint8), 0.0, 0, np.zeros((16, 32)) * -1.0)
    assert s == 0.0 and np.all(c == 0)


# ------------------------------------------------------------------ TQ3
def test_tq3_golden_pack_vectors():
    for line in _golden_lines("tq3_pack_vectors.txt"):
        parts = [p.strip() for p in line.split("|")]
        if parts[0].startswith("codes"):
            q = np.array([int(c) for c in parts[0].split()[1].split(",")], np.uint8)
            want = bytes.fromhex(parts[1])
            assert F.tq3_pack(q).tobytes() == want
            assert np.array_equal(F.tq3_unpack(np.frombuffer(want, np.uint8)), q)
        else:
            x = np.arange(32) - 15.5
            q, s = F.tq3_quantize(x)
            assert int(np.float16(s).view(np.uint16)) == int(parts[1].split()[1], 16)
            assert q.tolist() == [int(c) for c in parts[2].split()[1].split(",")]
            assert F.tq3_pack(q).tobytes() == bytes.fromhex(parts[3])
            assert np.max(np.abs(F.tq3_dequant(q, s) - x)) == float(parts[4].split()[1])


def _bigint_pack(q):
    v = 0
    for j, c in enumerate(q):
        v |= int(c) << (3 * j)
    return v.to_bytes(12, "little")


def test_tq3_pack_matches_bigint_packer():
    rng = np.random.default_rng(5)
    q = rng.integers(0, 8, size=(200, 32)).astype(np.uint8)
    packed = F.tq3_pack(q)
    for i in range(q.shape[0]):
        assert packed[i].tobytes() == _bigint_pack(q[i])
    assert np.array_equal(F.tq3_unpack(packed), q)


def test_tq3_codes_equal_exact_floor_clamp():
    rng = np.random.default_rng(6)
    x = F.f32(rng.standard_normal((300, 32)) * rng.uniform(0.01, 20, (300, 1)))
    # plant exact threshold hits: x = k*s for the group's own s
    q, s = F.tq3_quantize(x)
    x[:50, 0] = s[:50] * rng.integers(-3, 4, 50)
    x[:50, 1] = -0.0
    q, s = F.tq3_quantize(x)
    for i in range(x.shape[0]):
        sf = Fraction(float(s[i]))
        for j in range(32):
            xf = Fraction(float(x[i, j]))
            if sf == 0:
                want = 7 if xf >= 0 else 0
            else:
                want = min(7, max(0, (xf / sf).__floor__() + 4))
            assert q[i, j] == want, (i, j)


def test_tq3_scale_definition_and_error_bound():
    rng = np.random.default_rng(8)
    x = F.f32(rng.standard_normal((500, 32)))
    q, s = F.tq3_quantize(x)
    amax = np.abs(x).max(axis=1)
    # s is the fp16 rounding of the fp32 quotient, computed here through torch's casts
    want = torch.from_numpy(amax.astype(np.float32)).div(3.5).to(torch.float16).double().numpy()
    assert np.array_equal(s, want)
    err = np.abs(F.tq3_dequant(q, s) - x)
    assert np.all(err <= s[:, None] / 2 + np.maximum(amax - 3.5 * s, 0)[:, None] + 1e-12)


def test_tq3_scale_saturates_at_the_largest_f16():
    # fp16 holds at most 65504; plain round-to-nearest-even sends 65520 and above to infinity,
    # the scale rule clamps instead, so a group with a huge amax keeps a finite scale
    assert F.f16_satfinite(65504.0) == 65504.0
    assert F.f16_satfinite(65519.99) == 65504.0
    assert F.f16_satfinite(65520.0) == 65504.0
    assert F.f16_satfinite(1e30) == 65504.0 and F.f16_satfinite(-1e30) == -65504.0
    assert F.f16_satfinite(65505.0) == 65504.0          # nearest f16 (spacing 32 there)
    x = np.zeros(32)
    x[0], x[1], x[2], x[3] = 1e9, -1e9, 3 * 65504.0, -3 * 65504.0 - 1
    q, s = F.tq3_quantize(x[None])
    assert s[0] == 65504.0
    # code = number of thresholds k * s (k = -3..3) that x reaches
    assert q[0, 0] == 7 and q[0, 1] == 0 and q[0, 2] == 7 and q[0, 3] == 0 and q[0, 4] == 4


def test_tq3_zero_group():
    q, s = F.tq3_quantize(np.zeros((1, 32)))
    assert s[0] == 0.0 and np.all(q == 7)
    assert np.all(F.tq3_dequant(q, s) == 0.0)


def test_slot_layouts_roundtrip():
    rng = np.random.default_rng(9)
    Hkv, D = 3, 64
    kc = rng.integers(0, 256, (Hkv, 16, D)).astype(np.uint8)
    vc = rng.integers(0, 256, (Hkv, 16, D)).astype(np.uint8)
    ks, vs = rng.random(Hkv).astype(np.float32), rng.random(Hkv).astype(np.float32)
    raw = F.fp8_slot_bytes(kc, vc, ks, vs)
    assert raw.size == Hkv * F.fp8_head_bytes(D)
    r = F.parse_fp8_slot(raw, Hkv, D)
    assert np.array_equal(r[0], kc) and np.array_equal(r[1], vc)
    assert np.array_equal(r[2], ks) and np.array_equal(r[3], vs)
    # head h, K row t, channel d sits at byte h*(32D+16) + t*D + d
    assert raw[1 * F.fp8_head_bytes(D) + 5 * D + 7] == kc[1, 5, 7]
    kq = rng.integers(0, 8, (Hkv, 16, D)).astype(np.uint8)
    vq = rng.integers(0, 8, (Hkv, 16, D)).astype(np.uint8)
    kss = rng.random((Hkv, 16, D // 32)).astype(np.float16).astype(np.float64)
    vss = rng.random((Hkv, 16, D // 32)).astype(np.float16).astype(np.float64)
    raw3 = F.tq3_slot_bytes(kq, kss, vq, vss)
    assert raw3.size == Hkv * F.tq3_head_bytes(D) == Hkv * 14 * D
    r3 = F.parse_tq3_slot(raw3, Hkv, D)
    for a, b in zip(r3, (kq, kss, vq, vss)):
        assert np.array_equal(a, b)
    # record (group 1, token 3) of head 0's K codes starts at byte 12*(1*16+3)
    rec = raw3[12 * 19:12 * 20]
    assert rec.tobytes() == _bigint_pack(kq[0, 3, 32:64])
