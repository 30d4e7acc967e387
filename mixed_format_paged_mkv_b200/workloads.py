"""Seeded synthetic decode workloads shaped like the pages' long-context decode.

This module only draws inputs: random bf16 tensors, context lengths, protected-page picks and
slot orders, plus the sequence of pool calls that builds each workload's cache.  It holds none
of the method's arithmetic (no quantisation, policy or attention) and serves both the CUDA
library's tests/bench and the CPU oracle, so both see bit-identical inputs.

Recipe (all values bf16 from fp32 N(0,1) draws rounded to nearest even):
  RNG      numpy PCG64, seed = 1000*cfg + stream, with a spawn key per (layer, sequence);
           streams: 0 Q, 1 K, 2 V, 3 slot order, 4 outlier channels, 5 protected pages,
           6 context lengths, 7 per-step decode inputs.
  K        N(0,1); with ``outliers`` 4 distinct channels per (layer, KV head) are scaled x8
           before rounding (the same channels for every token and sequence).
  V, Q     N(0,1).
  scales   optional value-range variants multiply the fp32 draws before rounding: K by
           ``k_scale``, V by ``v_scale``, and with ``scale_mix`` every (token, KV head,
           32-channel group) of K and of V by a level drawn from ``MIX_LEVELS`` (stream 8).
  cache    per sequence, in order: append all L tokens as FP8 in one call, mark protected
           pages, demote with the anchor window W; then decode the last q_len tokens.

The five workloads (context lengths include the q_len new tokens):
  1 tiny      B=1, Hq 8 / Hkv 2, D 128, L 1024, W 64 (page 0 + last 4 pages FP8),
              pools of 128 slots filled in a random slot order.
  2 batch8    B=8, 32/8, D 128, L 8192, W 256, outlier K, permuted shared pool.
  3 ragged32  B=32, 24/4, D 256, L ~ U[2048, 32768], W 512, 2% of older pages protected.
  4 long      B=4, 24/4, D 256, L 131072, W 512, protected pages bring the FP8 share of
              pages to 4% (96% TQ3); 48 layers' worth of pages; q_len 1 and a q_len 4 variant.
  5 steady    B=64, 32/8, D 128, L ~ U[4096, 65536], W 256; each step appends one token per
              sequence, demotes and decodes.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np

PAGE = 16
S_Q, S_K, S_V, S_SLOT, S_OUTLIER, S_PROTECT, S_CTX, S_STEP, S_MIX = range(9)
# multipliers of the mixed-scale variant: from far below to far above N(0,1)
MIX_LEVELS = np.array([1e-4, 1e-2, 1.0, 1e3, 3e4], dtype=np.float32)


def bf16_bits(x) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return u.astype(np.uint16)


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: int
    B: int
    Hq: int
    Hkv: int
    D: int
    q_len: int
    window: int                      # anchor window W in tokens
    ctx: tuple = ()                  # fixed context lengths (empty -> drawn from ctx_range)
    ctx_range: tuple = ()            # (lo, hi) inclusive, uniform integers
    protect_frac: float = 0.0        # fraction of older pages marked protected
    fp8_page_frac: float = 0.0       # alternatively: protect until FP8 pages are this share
    outliers: bool = False
    layers: int = 1
    slot_order: bool = True          # random slot order (permuted block tables)
    pool_slots: int = 0              # fixed slots per format (0 -> sized from the workload)
    k_scale: float = 1.0             # multiplier of every K draw (value-range variants)
    v_scale: float = 1.0             # multiplier of every V draw
    scale_mix: bool = False          # per-(token, KV head, group) levels from MIX_LEVELS

    # ------------------------------------------------------------------ derived
    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    def seed(self, stream: int) -> int:
        return 1000 * self.cfg + stream

    def rng(self, stream: int, *key: int) -> np.random.Generator:
        ss = np.random.SeedSequence(self.seed(stream), spawn_key=tuple(int(k) for k in key))
        return np.random.Generator(np.random.PCG64(ss))

    def lengths(self) -> list:
        if self.ctx:
            return [int(x) for x in self.ctx]
        lo, hi = self.ctx_range
        return [int(x) for x in self.rng(S_CTX).integers(lo, hi, size=self.B, endpoint=True)]

    def pages(self) -> list:
        return [-(-L // PAGE) for L in self.lengths()]

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # ------------------------------------------------------------------ draws
    def outlier_channels(self, layer: int = 0) -> np.ndarray:
        """[Hkv, 4] distinct channel indices per KV head."""
        r = self.rng(S_OUTLIER, layer)
        return np.stack([r.choice(self.D, size=4, replace=False) for _ in range(self.Hkv)])

    def kv(self, seq: int, layer: int = 0, lo: int = 0, hi: int | None = None):
        """bf16 bits of K and V for tokens [lo, hi) of a sequence: uint16 [n, Hkv, D] each.
        Drawn in blocks of 4096 tokens so any token range can be regenerated alone."""
        L = self.lengths()[seq]
        hi = L if hi is None else hi
        ks, vs = [], []
        blk = 4096
        for b0 in range(lo // blk * blk, hi, blk):
            n = min(blk, L - b0)
            rk = self.rng(S_K, layer, seq, b0 // blk)
            rv = self.rng(S_V, layer, seq, b0 // blk)
            k = rk.standard_normal((n, self.Hkv, self.D), dtype=np.float32)
            v = rv.standard_normal((n, self.Hkv, self.D), dtype=np.float32)
            if self.outliers:
                oc = self.outlier_channels(layer)
                for h in range(self.Hkv):
                    k[:, h, oc[h]] *= np.float32(8.0)
            k, v = self._rescale(k, v, self.rng(S_MIX, layer, seq, b0 // blk))
            a, b = max(lo, b0) - b0, min(hi, b0 + n) - b0
            ks.append(bf16_bits(k[a:b]))
            vs.append(bf16_bits(v[a:b]))
        return np.concatenate(ks), np.concatenate(vs)

    def q(self, seq: int, layer: int = 0) -> np.ndarray:
        """bf16 bits of the queries of a sequence: uint16 [q_len, Hq, D]."""
        r = self.rng(S_Q, layer, seq)
        return bf16_bits(r.standard_normal((self.q_len, self.Hq, self.D), dtype=np.float32))

    def step_inputs(self, step: int, layer: int = 0):
        """Inputs of one decode step of one layer: the new token's K and V for every sequence
        (uint16 bf16 bits [B, Hkv, D] each, outlier channels as in ``kv``) and the queries
        (uint16 [B, q_len, Hq, D])."""
        r = self.rng(S_STEP, layer, step)
        k = r.standard_normal((self.B, self.Hkv, self.D), dtype=np.float32)
        v = r.standard_normal((self.B, self.Hkv, self.D), dtype=np.float32)
        q = r.standard_normal((self.B, self.q_len, self.Hq, self.D), dtype=np.float32)
        if self.outliers:
            oc = self.outlier_channels(layer)
            for h in range(self.Hkv):
                k[:, h, oc[h]] *= np.float32(8.0)
        k, v = self._rescale(k, v, self.rng(S_MIX, layer, 1 << 20, step))
        return bf16_bits(k), bf16_bits(v), bf16_bits(q)

    def _rescale(self, k, v, r):
        """Value-range variants: scale fp32 K, V [n, Hkv, D] draws before rounding."""
        if self.k_scale != 1.0:
            k = k * np.float32(self.k_scale)
        if self.v_scale != 1.0:
            v = v * np.float32(self.v_scale)
        if self.scale_mix:
            n, G = k.shape[0], self.D // 32
            for which in (0, 1):
                lv = MIX_LEVELS[r.integers(0, MIX_LEVELS.size, size=(n, self.Hkv, G))]
                m = np.repeat(lv, 32, axis=2)
                if which == 0:
                    k = k * m
                else:
                    v = v * m
        return k, v

    def protected(self, seq: int) -> list:
        """Logical pages the caller marks protected (sorted).  Candidates are the full pages
        that lie wholly before the last W tokens, page 0 excluded."""
        L = self.lengths()[seq]
        n_pages = -(-L // PAGE)
        last_old = (L - self.window) // PAGE          # pages < last_old end before L - W
        cand = np.arange(1, max(1, last_old))
        if cand.size == 0:
            return []
        if self.fp8_page_frac:
            anchors = 1 + (n_pages - last_old)
            k = max(0, int(round(self.fp8_page_frac * n_pages)) - anchors)
        else:
            k = int(round(self.protect_frac * cand.size))
        k = min(k, cand.size)
        if k == 0:
            return []
        return sorted(int(p) for p in self.rng(S_PROTECT, seq).choice(cand, size=k, replace=False))

    def slot_permutation(self, fmt: int, n_slots: int) -> np.ndarray | None:
        if not self.slot_order:
            return None
        return self.rng(S_SLOT, fmt).permutation(n_slots).astype(np.int32)

    # ------------------------------------------------------------------ pool sizing / build
    def pool_shape(self, extra_pages_per_seq: int = 0) -> dict:
        """Slots and table sizes for building one layer of the workload sequence by sequence
        (peak FP8 use = one sequence's pages plus every sequence's anchors)."""
        pages = self.pages()
        mp = max(pages) + extra_pages_per_seq + 1
        if self.pool_slots:
            n8 = n3 = self.pool_slots
        else:
            n3 = sum(pages) + self.B * (extra_pages_per_seq + 1)
            n8 = max(pages) + sum(min(p, self.window // PAGE + 2) + len(self.protected(s)) + 1
                                  for s, p in enumerate(pages)) + self.B * (extra_pages_per_seq + 2)
        return dict(num_kv_heads=self.Hkv, head_dim=self.D, max_seqs=self.B * self.layers,
                    max_pages_per_seq=mp, fp8_slots=n8, tq3_slots=n3)

    def build_ops(self, layer: int = 0):
        """The pool calls that build one layer's cache, as tuples:
        ("append", seq, n_tokens) -> append tokens [0, L) of ``seq`` (bulk)
        ("protect", seq, [pages])
        ("demote", seq, W)"""
        for s in range(self.B):
            yield ("append", s, self.lengths()[s])
            prot = self.protected(s)
            if prot:
                yield ("protect", s, prot)
            yield ("demote", s, self.window)


WORKLOADS = {
    1: Workload("tiny_b1_h8kv2_d128_ctx1k", 1, B=1, Hq=8, Hkv=2, D=128, q_len=1, window=64,
                ctx=(1024,), pool_slots=128),
    2: Workload("batch8_h32kv8_d128_ctx8k", 2, B=8, Hq=32, Hkv=8, D=128, q_len=1, window=256,
                ctx=(8192,) * 8, outliers=True),
    3: Workload("ragged32_h24kv4_d256_ctx2k-32k", 3, B=32, Hq=24, Hkv=4, D=256, q_len=1,
                window=512, ctx_range=(2048, 32768), protect_frac=0.02, outliers=True),
    4: Workload("long_b4_h24kv4_d256_ctx128k", 4, B=4, Hq=24, Hkv=4, D=256, q_len=1,
                window=512, ctx=(131072,) * 4, fp8_page_frac=0.04, outliers=True, layers=48),
    5: Workload("steady_b64_h32kv8_d128_ctx4k-64k", 5, B=64, Hq=32, Hkv=8, D=128, q_len=1,
                window=256, ctx_range=(4096, 65536), outliers=True),
}


def long_qlen4() -> Workload:
    """The q_len 4 variant of the long-context workload (4 new tokens, causal among them)."""
    return WORKLOADS[4].scaled(name="long_b4_h24kv4_d256_ctx128k_q4", q_len=4)


def default_sm_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
