"""Reference model of the mixed-format page pool: allocator, block tables, anchor policy.

ORACLE -- test infrastructure only (see ``oracle/formats.py`` for the rule on who may use it).

Written from the pages' description of the page hierarchy ("Minima-KV ..." summary,
brainszone.ai pt page, sections "O que os autores propõem" and "Âncoras em FP8, arquivo em
TQ3"): every page of a live request stays addressable through the request's page table;
recently used pages and pages marked protected ("anchor") stay FP8; older non-anchor pages
are converted to packed TQ3.  Readings of what the pages leave open:

* Page = 16 tokens.  A page p of a sequence of length L is an anchor iff
  p < sink_pages (page 0 by default), or 16p + 16 > L - W (it holds one of the last W
  tokens), or it is flagged protected.  Demotion converts every full FP8 page that is not
  an anchor; the TQ3 page is computed from the FP8 page (pages are *converted*).
* Slots are handed out lowest rank first (rank = position in a per-format slot order,
  identity unless set), sequences in the order the call lists them, pages ascending.
  Slots freed by a call return to the free list at the end of that call.
* Block-table entry: -1 unmapped, else (format << 30) | slot with format 0 = FP8, 1 = TQ3,
  2 = BF16.
* A call that fails changes nothing.

A control pool (``bf16_control=True``) models the comparator the pages measure the method
against ("Memória e compressão", "Verificação canário"): every page holds its bf16 values as
they are (format BF16, taken from the first slab), no page is ever demoted, and attention runs
over those values.
"""
from __future__ import annotations

import heapq

import numpy as np

from . import formats as F

FP8, TQ3, BF16 = 0, 1, 2
PAGE = F.PAGE_TOKENS


def _slab(fmt):
    """Slab (and allocator) of a format: BF16 control pages use the first slab, as FP8."""
    return 1 if fmt == TQ3 else 0


class PoolError(Exception):
    """Raised for the error cases of the pool API; ``code`` names the case."""

    def __init__(self, code: str, msg: str = ""):
        super().__init__(f"{code}: {msg}")
        self.code = code


class _Allocator:
    def __init__(self, n: int):
        self.n = n
        self.rank = np.arange(n, dtype=np.int64)
        self.heap = [(i, i) for i in range(n)]
        self.free = set(range(n))

    def set_order(self, order):
        order = np.asarray(order, dtype=np.int64)
        if sorted(order.tolist()) != list(range(self.n)):
            raise PoolError("INVALID_ARG", "slot order must be a permutation")
        self.rank = np.empty(self.n, dtype=np.int64)
        self.rank[order] = np.arange(self.n)
        self.heap = [(int(self.rank[s]), s) for s in self.free]
        heapq.heapify(self.heap)

    def take(self) -> int:
        while True:
            r, s = heapq.heappop(self.heap)
            if s in self.free:
                self.free.discard(s)
                return s

    def give(self, s: int):
        self.free.add(s)
        heapq.heappush(self.heap, (int(self.rank[s]), s))


class RefPool:
    """The pool's whole observable state: tables, lengths, flags and every slot's contents."""

    def __init__(self, Hkv, D, max_seqs, max_pages_per_seq, fp8_slots, tq3_slots,
                 sink_pages=1, bf16_control=False):
        if D % F.TQ3_GROUP:
            raise PoolError("INVALID_ARG", "head_dim must be a multiple of 32")
        self.Hkv, self.D, self.G = Hkv, D, D // F.TQ3_GROUP
        self.max_seqs, self.max_pages = max_seqs, max_pages_per_seq
        self.sink_pages = sink_pages
        self.alloc = [_Allocator(fp8_slots), _Allocator(tq3_slots)]
        self.table = [[] for _ in range(max_seqs)]      # per seq: list of (fmt, slot)
        self.ctx = [0] * max_seqs
        self.protected = [set() for _ in range(max_seqs)]
        self.fp8 = {}   # slot -> [kcodes [Hkv,16,D], vcodes, kscale [Hkv], vscale [Hkv]]
        self.tq3 = {}   # slot -> [kq [Hkv,16,D], ks [Hkv,16,G], vq, vs]
        self.bf16_control = bf16_control
        self.bf16 = {}  # slot -> [kbits [Hkv,16,D] uint16, vbits]  (control pools)
        self.page_fmt = BF16 if bf16_control else FP8   # format of written (unconverted) pages

    # ------------------------------------------------------------------ helpers
    def _check_seq(self, s):
        if not (0 <= s < self.max_seqs):
            raise PoolError("BAD_SEQ", f"sequence {s}")

    def set_slot_order(self, fmt, order):
        self.alloc[_slab(fmt)].set_order(order)

    def _store(self, fmt):
        return {FP8: self.fp8, TQ3: self.tq3, BF16: self.bf16}[fmt]

    def _new_page(self, seq):
        """Take a slot for a fresh written page (FP8, or BF16 in a control pool)."""
        slot = self.alloc[0].take()
        z = np.zeros((self.Hkv, PAGE, self.D), np.uint8)
        if self.bf16_control:
            zb = np.zeros((self.Hkv, PAGE, self.D), np.uint16)
            self.bf16[slot] = [zb, zb.copy()]
        else:
            self.fp8[slot] = [z, z.copy(), np.zeros(self.Hkv), np.zeros(self.Hkv)]
        self.table[seq].append((self.page_fmt, slot))
        return slot

    def _write_rows(self, slot, off, k, v):
        """Write rows [off, off + n) of a written page from k, v float64 [n, Hkv, D]."""
        if self.bf16_control:
            st = self.bf16[slot]
            for which, src in ((0, k), (1, v)):
                st[which][:, off:off + src.shape[0], :] = F.f64_to_bf16_bits(
                    np.transpose(src, (1, 0, 2)))
            return
        st = self.fp8[slot]
        for h in range(self.Hkv):
            for which, src in ((0, k), (1, v)):
                codes, sc = F.fp8_write(st[which][h], st[2 + which][h], off, src[:, h, :])
                st[which][h] = codes
                st[2 + which][h] = sc

    def entry(self, seq, page) -> int:
        """The int32 table entry (format 2 sets the sign bit)."""
        fmt, slot = self.table[seq][page]
        e = (fmt << 30) | slot
        return e - (1 << 32) if e >= 1 << 31 else e

    def block_table(self, seq):
        return [self.entry(seq, p) for p in range(len(self.table[seq]))]

    # ------------------------------------------------------------------ append
    def append(self, seq_ids, n_new, k, v):
        """Append tokens: k, v float64 [sum(n_new), Hkv, D] (bf16 values), rows grouped by
        sequence in ``seq_ids`` order."""
        seq_ids = [int(s) for s in seq_ids]
        n_new = [int(n) for n in n_new]
        for s in seq_ids:
            self._check_seq(s)
        if len(set(seq_ids)) != len(seq_ids) or any(n < 0 for n in n_new):
            raise PoolError("INVALID_ARG", "repeated sequence or negative count")
        need = 0
        for s, n in zip(seq_ids, n_new):
            pages_after = -(-(self.ctx[s] + n) // PAGE)
            if pages_after > self.max_pages:
                raise PoolError("OUT_OF_PAGES", f"sequence {s} exceeds max pages")
            need += pages_after - len(self.table[s])
        if need > len(self.alloc[FP8].free):
            raise PoolError("OUT_OF_PAGES", "FP8 pool exhausted")
        row = 0
        for s, n in zip(seq_ids, n_new):
            L0 = self.ctx[s]
            pages_after = -(-(L0 + n) // PAGE)
            for _ in range(len(self.table[s]), pages_after):
                self._new_page(s)
            t = 0
            while t < n:
                pos = L0 + t
                page, off = divmod(pos, PAGE)
                cnt = min(PAGE - off, n - t)
                fmt, slot = self.table[s][page]
                assert fmt == self.page_fmt
                self._write_rows(slot, off, k[row + t:row + t + cnt], v[row + t:row + t + cnt])
                t += cnt
            self.ctx[s] = L0 + n
            row += n

    # ------------------------------------------------------------------ prefill (direct pack)
    def prefill(self, seq_ids, n_tokens, k, v, window_tokens):
        """Write the first tokens of empty sequences: k, v float64 [sum(n_tokens), Hkv, D]
        (bf16 values), rows grouped by sequence in ``seq_ids`` order.  A full page that the
        anchor policy would demote at once (p >= sink_pages and 16p + 16 <= L - W, with L the
        sequence's new length; new pages carry no protection) is packed to TQ3 straight from
        the bf16 values, as ``convert`` packs an FP8 page's values; every other page is written
        as a fresh FP8 page, as by ``append``.  Pages take slots of their own format, in
        ascending page order, sequences in list order."""
        seq_ids = [int(s) for s in seq_ids]
        n_tokens = [int(n) for n in n_tokens]
        for s in seq_ids:
            self._check_seq(s)
        if (len(set(seq_ids)) != len(seq_ids) or any(n < 0 for n in n_tokens)
                or window_tokens < 0):
            raise PoolError("INVALID_ARG", "repeated sequence, negative count or window")
        if any(self.table[s] or self.ctx[s] for s in seq_ids):
            raise PoolError("INVALID_ARG", "prefill needs empty sequences")
        direct = []
        need = [0, 0]
        for s, n in zip(seq_ids, n_tokens):
            pages = -(-n // PAGE)
            if pages > self.max_pages:
                raise PoolError("OUT_OF_PAGES", f"sequence {s} exceeds max pages")
            d = [not self.bf16_control and p >= self.sink_pages
                 and PAGE * p + PAGE <= n - window_tokens for p in range(pages)]
            direct.append(d)
            need[TQ3] += sum(d)
            need[FP8] += pages - sum(d)
        for fmt in (FP8, TQ3):
            if need[fmt] > len(self.alloc[fmt].free):
                raise PoolError("OUT_OF_PAGES", "pool exhausted")
        row = 0
        for s, n, d in zip(seq_ids, n_tokens, direct):
            for p, is_tq3 in enumerate(d):
                r0, cnt = row + PAGE * p, min(PAGE, n - PAGE * p)
                if is_tq3:
                    slot = self.alloc[TQ3].take()
                    res = []
                    for src in (k, v):
                        x = np.transpose(src[r0:r0 + PAGE], (1, 0, 2))          # [Hkv,16,D]
                        q, sc = F.tq3_quantize(x.reshape(self.Hkv, PAGE, self.G, F.TQ3_GROUP))
                        res += [q.reshape(self.Hkv, PAGE, self.D), sc]
                    self.tq3[slot] = res
                    self.table[s].append((TQ3, slot))
                else:
                    slot = self._new_page(s)
                    self._write_rows(slot, 0, k[r0:r0 + cnt], v[r0:r0 + cnt])
            self.ctx[s] = n
            row += n

    # ------------------------------------------------------------------ policy
    def is_anchor(self, seq, page, window_tokens) -> bool:
        L = self.ctx[seq]
        return (page < self.sink_pages or PAGE * page + PAGE > L - window_tokens
                or page in self.protected[seq])

    def set_protected(self, seq, page, flag):
        self._check_seq(seq)
        if not (0 <= page < len(self.table[seq])):
            raise PoolError("INVALID_ARG", "page not mapped")
        if flag:
            self.protected[seq].add(page)
        else:
            self.protected[seq].discard(page)

    def demote_candidates(self, seq, window_tokens):
        L = self.ctx[seq]
        out = []
        for p, (fmt, _) in enumerate(self.table[seq]):
            if fmt == FP8 and PAGE * (p + 1) <= L and not self.is_anchor(seq, p, window_tokens):
                out.append(p)
        return out

    def demote(self, seq_ids, window_tokens):
        """Convert every full, non-anchor FP8 page of the listed sequences to TQ3.
        Returns [(seq, page, fp8_slot, tq3_slot)] in processing order."""
        seq_ids = [int(s) for s in seq_ids]
        for s in seq_ids:
            self._check_seq(s)
        if len(set(seq_ids)) != len(seq_ids) or window_tokens < 0:
            raise PoolError("INVALID_ARG", "repeated sequence or negative window")
        work = [] if self.bf16_control else [
            (s, p) for s in seq_ids for p in self.demote_candidates(s, window_tokens)]
        if len(work) > len(self.alloc[TQ3].free):
            raise PoolError("OUT_OF_PAGES", "TQ3 pool exhausted")
        done, freed = [], []
        for s, p in work:
            _, src = self.table[s][p]
            dst = self.alloc[TQ3].take()
            self.tq3[dst] = self.convert(src)
            self.table[s][p] = (TQ3, dst)
            done.append((s, p, src, dst))
            freed.append(src)
        for src in freed:
            del self.fp8[src]
            self.alloc[FP8].give(src)
        return done

    def convert(self, fp8_slot):
        """TQ3 contents of a full FP8 page: x = fp32(dec(code) * scale), then per group of
        32 channels of each (token, head, K-or-V) quantise to 3 bits."""
        kc, vc, ks, vs = self.fp8[fp8_slot]
        res = []
        for codes, scales in ((kc, ks), (vc, vs)):
            x = F.f32(F.e4m3_decode(codes) * scales[:, None, None])       # [Hkv,16,D]
            q, s = F.tq3_quantize(x.reshape(self.Hkv, PAGE, self.G, F.TQ3_GROUP))
            res += [q.reshape(self.Hkv, PAGE, self.D), s]
        return res

    # ------------------------------------------------------------------ lifecycle
    def seq_reset(self, seq):
        self._check_seq(seq)
        for fmt, slot in self.table[seq]:
            self._store(fmt).pop(slot)
            self.alloc[_slab(fmt)].give(slot)
        self.table[seq] = []
        self.ctx[seq] = 0
        self.protected[seq] = set()

    def seq_copy(self, src, dst):
        """Give ``dst`` (empty) its own copy of every page of ``src``; formats kept."""
        self._check_seq(src)
        self._check_seq(dst)
        if src == dst or self.table[dst] or self.ctx[dst]:
            raise PoolError("INVALID_ARG", "destination must be a different, empty sequence")
        need = [0, 0]
        for fmt, _ in self.table[src]:
            need[_slab(fmt)] += 1
        for slab in (0, 1):
            if need[slab] > len(self.alloc[slab].free):
                raise PoolError("OUT_OF_PAGES", "pool exhausted")
        for fmt, slot in self.table[src]:
            new = self.alloc[_slab(fmt)].take()
            store = self._store(fmt)
            store[new] = [np.array(a, copy=True) for a in store[slot]]
            self.table[dst].append((fmt, new))
        self.ctx[dst] = self.ctx[src]
        self.protected[dst] = set(self.protected[src])

    # ------------------------------------------------------------------ views
    def slot_bytes(self, entry: int):
        fmt, slot = (entry >> 30) & 3, entry & ((1 << 30) - 1)
        if fmt == FP8:
            kc, vc, ks, vs = self.fp8[slot]
            return F.fp8_slot_bytes(kc, vc, ks, vs)
        if fmt == BF16:
            kb, vb = self.bf16[slot]
            return F.bf16_slot_bytes(kb, vb)
        kq, ks, vq, vs = self.tq3[slot]
        return F.tq3_slot_bytes(kq, ks, vq, vs)

    def dequant_seq(self, seq, heads=None):
        """Dequantised K and V of a sequence: float64 [L, Hkv, D] each (exact values)."""
        L = self.ctx[seq]
        heads = range(self.Hkv) if heads is None else heads
        nh = len(list(heads))
        K = np.zeros((len(self.table[seq]) * PAGE, nh, self.D))
        V = np.zeros_like(K)
        for p, (fmt, slot) in enumerate(self.table[seq]):
            rows = slice(p * PAGE, (p + 1) * PAGE)
            for j, h in enumerate(heads):
                if fmt == FP8:
                    kc, vc, ks, vs = self.fp8[slot]
                    K[rows, j] = F.fp8_dequant(kc[h], ks[h])
                    V[rows, j] = F.fp8_dequant(vc[h], vs[h])
                elif fmt == BF16:
                    kb, vb = self.bf16[slot]
                    K[rows, j] = F.bf16_bits_to_f64(kb[h])
                    V[rows, j] = F.bf16_bits_to_f64(vb[h])
                else:
                    kq, kscale, vq, vscale = self.tq3[slot]
                    K[rows, j] = F.tq3_dequant(kq[h].reshape(PAGE, self.G, F.TQ3_GROUP),
                                               kscale[h]).reshape(PAGE, self.D)
                    V[rows, j] = F.tq3_dequant(vq[h].reshape(PAGE, self.G, F.TQ3_GROUP),
                                               vscale[h]).reshape(PAGE, self.D)
        return K[:L], V[:L]

    def stats(self):
        live = sum(self.ctx)
        n8 = sum(1 for t in self.table for f, _ in t if f == self.page_fmt)
        n3 = sum(1 for t in self.table for f, _ in t if f == TQ3)
        head = F.bf16_head_bytes(self.D) if self.bf16_control else F.fp8_head_bytes(self.D)
        kv_bytes = n8 * self.Hkv * head + n3 * self.Hkv * F.tq3_head_bytes(self.D)
        return live, n8, n3, (kv_bytes / live if live else 0.0)
