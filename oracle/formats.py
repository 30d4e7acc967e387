"""Number formats of the mixed-format paged KV cache, written from their definitions.

ORACLE -- test infrastructure only.  Nothing in the library imports this module; only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` may use it.  It shares no code, table or constant generator with the CUDA path.

Source of the method: "Minima-KV: Retention-Preserving KV Cache Compression with
Mixed-Format Paged Attention" as summarised on brainszone.ai (pt page, section "Ancoras em
FP8, arquivo em TQ3"; fr page, section "Des ancres en FP8, une archive en TQ3"): recent and
protected pages are held in FP8, older pages are converted to a denser packed 3-bit format
("packed TQ3").  The pages fix neither bit layout; the readings used here are:

* FP8 is OCP FP8 E4M3 ("E4M3FN": bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN,
  largest finite 448), one fp32 scale per (page, KV head, K-or-V).
* TQ3 stores 3-bit codes q in 0..7 that dequantise to (q - 3.5) * s, with one fp16 scale s
  per 32 channels per token per KV head; the 32 codes of a group are packed into 12 bytes,
  code j occupying bits 3j..3j+2 of the little-endian 96-bit integer formed by the 12 bytes.

All arithmetic is float64 numpy; where a step is defined by an fp32 or fp16 rounding the
rounding is applied explicitly (numpy's float64->float32 and float64->float16 casts are
IEEE round-to-nearest-even).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
F16_MAX = 65504.0
TQ3_GROUP = 32          # channels per TQ3 scale group
TQ3_GROUP_BYTES = 12    # 32 codes x 3 bits
PAGE_TOKENS = 16


# --------------------------------------------------------------------------- rounding
def f32(x):
    """Round float64 values to the nearest fp32 value (ties to even); result as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def f16_satfinite(x):
    """fp16 round-to-nearest-even with saturation to +-65504 instead of infinity.

    Clamping to the largest finite fp16 before rounding gives the same result as a
    saturating conversion: every value in (65504, 65520) rounds to 65504 anyway.
    """
    x = np.clip(np.asarray(x, dtype=np.float64), -F16_MAX, F16_MAX)
    return x.astype(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits):
    """Interpret uint16 bf16 bit patterns as float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- E4M3
def _e4m3_value(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:                                   # subnormal: m/8 * 2^(1-7)
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
_E4M3_POS = E4M3_TABLE[:0x7F].copy()            # codes 0x00..0x7E: 0 .. 448, ascending


def e4m3_decode(codes):
    """Code bytes -> float64 values (exact)."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x):
    """Nearest E4M3 code, ties to the even code, saturating to +-448; sign of zero kept.

    ``x`` must be values that are already what is to be encoded (e.g. an fp32 quotient);
    NaN encodes to 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    code = np.where(d_hi < d_lo, hi, lo)
    tie = d_hi == d_lo
    code = np.where(tie, np.where(hi % 2 == 0, hi, lo), code)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = code.astype(np.uint8) | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------- FP8 page write
def fp8_write(old_codes, old_scale, n_old, x_new):
    """Write new tokens of one (page, KV head, K-or-V) into an FP8 page.

    old_codes: uint8 [16, D] current code rows (rows >= n_old are zero);
    old_scale: the page's fp32 scale (ignored when n_old == 0);
    x_new:     float64 [n_new, D], the new tokens' bf16 values, landing at rows n_old..

    Per-page scale with rescale-on-grow (the pages say only "FP8"; one fp32 scale per page,
    KV head and tensor is the reading):
      a = max|x_new|; cand = fp32(a / 448)
      empty page      -> scale = cand
      cand > old      -> existing codes re-encoded: enc(fp32(fp32(dec(c) * old) / cand)),
                         scale = cand
      otherwise       -> scale kept
      new codes       =  enc(fp32(x / scale)), or 0x00 when scale == 0.
    Returns (codes uint8 [16, D], scale float).
    """
    codes = np.array(old_codes, dtype=np.uint8, copy=True)
    x_new = np.asarray(x_new, dtype=np.float64)
    n_new = x_new.shape[0]
    a = float(np.max(np.abs(x_new))) if n_new else 0.0
    cand = float(f32(a / E4M3_MAX))
    if n_old == 0:
        scale = cand
    elif cand > old_scale:
        prev = f32(e4m3_decode(codes[:n_old]) * old_scale)
        codes[:n_old] = e4m3_encode(f32(prev / cand))
        scale = cand
    else:
        scale = float(old_scale)
    if scale == 0.0:
        codes[n_old:n_old + n_new] = 0
    else:
        codes[n_old:n_old + n_new] = e4m3_encode(f32(x_new / scale))
    return codes, scale


def fp8_dequant(codes, scale):
    """Dequantised FP8 page values, exact in float64."""
    return e4m3_decode(codes) * float(scale)


# --------------------------------------------------------------------------- TQ3
def tq3_quantize(x):
    """Quantise groups of 32 fp32 values: x float64 [..., 32] -> (q uint8 [..., 32], s [...]).

    s = fp16_satfinite(fp32(amax / 3.5)) (absmax scaling, no rotation);
    q = #{k in -3..3 : x >= k*s}; the products k*s are exact, so no division or rounding
    enters the code decision.  Equivalently q = clamp(floor(x/s) + 4, 0, 7) with ties
    (x exactly on a threshold) going up.
    """
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[-1] == TQ3_GROUP
    amax = np.max(np.abs(x), axis=-1)
    s = f16_satfinite(f32(amax / 3.5))
    thresholds = np.arange(-3, 4, dtype=np.float64) * s[..., None]        # [..., 7]
    q = np.sum(x[..., :, None] >= thresholds[..., None, :], axis=-1)
    return q.astype(np.uint8), s


def tq3_dequant(q, s):
    """(q - 3.5) * s, exact in float64. q [..., 32], s [...]"""
    return (np.asarray(q, dtype=np.float64) - 3.5) * np.asarray(s, dtype=np.float64)[..., None]


def tq3_pack(q):
    """Codes [..., 32] -> bytes [..., 12]; bit i of code j is stream bit 3j+i, LSB first."""
    q = np.asarray(q, dtype=np.uint8)
    bits = (q[..., :, None] >> np.arange(3, dtype=np.uint8)) & 1              # [..., 32, 3]
    bits = bits.reshape(q.shape[:-1] + (96,))
    return np.packbits(bits, axis=-1, bitorder="little")


def tq3_unpack(b):
    """Bytes [..., 12] -> codes [..., 32] (inverse of tq3_pack)."""
    b = np.asarray(b, dtype=np.uint8)
    bits = np.unpackbits(b, axis=-1, bitorder="little").reshape(b.shape[:-1] + (32, 3))
    return (bits * np.array([1, 2, 4], dtype=np.uint8)).sum(axis=-1).astype(np.uint8)


# --------------------------------------------------------------------------- page layouts
def fp8_head_bytes(D: int) -> int:
    """Bytes of one KV head inside an FP8 slot: K rows, V rows, sK, sV, 8 pad bytes."""
    return 2 * PAGE_TOKENS * D + 16


def tq3_head_bytes(D: int) -> int:
    """Bytes of one KV head inside a TQ3 slot: (codes + fp16 scales) for K then V."""
    G = D // TQ3_GROUP
    return 2 * (G * PAGE_TOKENS * TQ3_GROUP_BYTES + G * PAGE_TOKENS * 2)


def fp8_slot_bytes(kcodes, vcodes, kscale, vscale):
    """Raw bytes of an FP8 slot.

    kcodes, vcodes uint8 [Hkv, 16, D]; kscale, vscale fp32 values [Hkv].
    Per KV head, in order: K codes (token-major, 16 x D), V codes (16 x D),
    K scale (fp32 LE), V scale (fp32 LE), 8 zero bytes.
    """
    out = []
    for h in range(kcodes.shape[0]):
        out.append(np.asarray(kcodes[h], dtype=np.uint8).reshape(-1))
        out.append(np.asarray(vcodes[h], dtype=np.uint8).reshape(-1))
        out.append(np.array([kscale[h], vscale[h]], dtype="<f4").view(np.uint8))
        out.append(np.zeros(8, dtype=np.uint8))
    return np.concatenate(out)


def tq3_slot_bytes(kq, ks, vq, vs):
    """Raw bytes of a TQ3 slot.

    kq, vq uint8 codes [Hkv, 16, D]; ks, vs fp16 scale values [Hkv, 16, G].
    Per KV head, in order: K code records [G][16 tokens][12 B], K scales [G][16] fp16 LE,
    V code records [G][16][12 B], V scales [G][16] fp16 LE.  Records and scales are stored
    group-major so that 16 consecutive tokens of one group are contiguous.
    """
    Hkv, T, D = kq.shape
    G = D // TQ3_GROUP
    out = []
    for h in range(Hkv):
        for q, s in ((kq[h], ks[h]), (vq[h], vs[h])):
            rec = tq3_pack(np.asarray(q).reshape(T, G, TQ3_GROUP))          # [16, G, 12]
            out.append(np.ascontiguousarray(rec.transpose(1, 0, 2)).reshape(-1))
            sc = np.asarray(s, dtype=np.float64).astype("<f2")              # [16, G]
            out.append(np.ascontiguousarray(sc.T).view(np.uint8).reshape(-1))
    return np.concatenate(out)


# --------------------------------------------------------------------------- BF16 control pages
# The control format the pages compare against ("Memória e compressão": KV bytes versus BF16):
# the bf16 values stored as they are.  Slot per KV head: K rows [16 tokens][D] then V rows
# [16][D], bf16 little-endian; rows of tokens not yet written are zero.
def bf16_head_bytes(D: int) -> int:
    return 2 * PAGE_TOKENS * D * 2


def f64_to_bf16_bits(x):
    """float64 values that bf16 holds exactly -> their uint16 bit patterns."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    if not np.array_equal(f.astype(np.float64), x, equal_nan=True):
        raise ValueError("value not representable in fp32")
    u = f.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("value not representable in bf16")
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_slot_bytes(kbits, vbits):
    """Raw bytes of a BF16 slot: kbits, vbits uint16 [Hkv, 16, D]; per KV head K rows then V
    rows, each element little-endian."""
    out = []
    for h in range(kbits.shape[0]):
        out.append(np.asarray(kbits[h], dtype="<u2").reshape(-1).view(np.uint8))
        out.append(np.asarray(vbits[h], dtype="<u2").reshape(-1).view(np.uint8))
    return np.concatenate(out)


def parse_bf16_slot(raw, Hkv, D):
    """Inverse of bf16_slot_bytes: -> (kbits, vbits) uint16 [Hkv, 16, D]."""
    raw = np.asarray(raw, dtype=np.uint8)
    b = raw[:Hkv * bf16_head_bytes(D)].view("<u2").reshape(Hkv, 2, PAGE_TOKENS, D)
    return b[:, 0].astype(np.uint16), b[:, 1].astype(np.uint16)


def parse_fp8_slot(raw, Hkv, D):
    """Inverse of fp8_slot_bytes: -> (kcodes, vcodes [Hkv,16,D], kscale, vscale [Hkv])."""
    raw = np.asarray(raw, dtype=np.uint8)
    hb = fp8_head_bytes(D)
    kc = np.empty((Hkv, PAGE_TOKENS, D), np.uint8)
    vc = np.empty_like(kc)
    ksc = np.empty(Hkv)
    vsc = np.empty(Hkv)
    for h in range(Hkv):
        b = raw[h * hb:(h + 1) * hb]
        kc[h] = b[:PAGE_TOKENS * D].reshape(PAGE_TOKENS, D)
        vc[h] = b[PAGE_TOKENS * D:2 * PAGE_TOKENS * D].reshape(PAGE_TOKENS, D)
        sc = b[2 * PAGE_TOKENS * D:2 * PAGE_TOKENS * D + 8].view("<f4")
        ksc[h], vsc[h] = float(sc[0]), float(sc[1])
    return kc, vc, ksc, vsc


def parse_tq3_slot(raw, Hkv, D):
    """Inverse of tq3_slot_bytes: -> (kq, ks, vq, vs)."""
    raw = np.asarray(raw, dtype=np.uint8)
    G = D // TQ3_GROUP
    hb = tq3_head_bytes(D)
    rec_b = G * PAGE_TOKENS * TQ3_GROUP_BYTES
    sc_b = G * PAGE_TOKENS * 2
    res = [np.empty((Hkv, PAGE_TOKENS, D), np.uint8), np.empty((Hkv, PAGE_TOKENS, G)),
           np.empty((Hkv, PAGE_TOKENS, D), np.uint8), np.empty((Hkv, PAGE_TOKENS, G))]
    for h in range(Hkv):
        b = raw[h * hb:(h + 1) * hb]
        for t in range(2):
            off = t * (rec_b + sc_b)
            rec = b[off:off + rec_b].reshape(G, PAGE_TOKENS, TQ3_GROUP_BYTES)
            q = tq3_unpack(rec).transpose(1, 0, 2).reshape(PAGE_TOKENS, D)
            s = b[off + rec_b:off + rec_b + sc_b].view("<f2").astype(np.float64)
            res[2 * t][h] = q
            res[2 * t + 1][h] = s.reshape(G, PAGE_TOKENS).T
    return tuple(res)
