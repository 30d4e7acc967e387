// Host side of the mixed-format paged KV cache: allocator, block tables, anchor policy,
// decode planning and the C ABI declared in include/mkv.h.
//
// "Minima-KV ..." (brainszone.ai pt page, sections "O que os autores propõem" and "Âncoras em
// FP8, arquivo em TQ3"): pages of a live request stay addressable; recent and protected pages
// are FP8 anchors; older non-anchor pages are converted to packed TQ3.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <string>
#include <vector>

#include "mkv.h"
#include "mkv_internal.h"
#include "selftest.h"

using namespace mkv;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return MKV_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Free slots handed out lowest rank first; rank = position in the slot order.
struct Allocator {
  int32_t n = 0;
  std::vector<int32_t> rank;
  std::vector<uint8_t> is_free;
  std::vector<uint64_t> heap;  // (rank << 32) | slot, min-heap
  int32_t n_free = 0;

  void init(int32_t slots) {
    n = slots;
    rank.resize(n);
    is_free.assign(n, 1);
    for (int32_t i = 0; i < n; ++i) rank[i] = i;
    rebuild();
  }
  void rebuild() {
    heap.clear();
    n_free = 0;
    for (int32_t s = 0; s < n; ++s)
      if (is_free[s]) {
        heap.push_back((static_cast<uint64_t>(rank[s]) << 32) | static_cast<uint32_t>(s));
        ++n_free;
      }
    std::make_heap(heap.begin(), heap.end(), std::greater<uint64_t>());
  }
  int32_t take() {
    std::pop_heap(heap.begin(), heap.end(), std::greater<uint64_t>());
    const int32_t s = static_cast<int32_t>(heap.back() & 0xffffffffu);
    heap.pop_back();
    is_free[s] = 0;
    --n_free;
    return s;
  }
  void give(int32_t s) {
    is_free[s] = 1;
    ++n_free;
    heap.push_back((static_cast<uint64_t>(rank[s]) << 32) | static_cast<uint32_t>(s));
    std::push_heap(heap.begin(), heap.end(), std::greater<uint64_t>());
  }
};

struct Seq {
  std::vector<int32_t> table;     // block-table entries
  std::vector<int32_t> fp8_pages; // logical pages currently FP8 (BF16 in a control pool), ascending
  std::vector<uint8_t> prot;      // protected flag per logical page
  int32_t ctx = 0;
  int32_t n3 = 0;
};

inline int32_t entry_of(int fmt, int32_t slot) {
  return static_cast<int32_t>((static_cast<uint32_t>(fmt) << kFmtShift) | static_cast<uint32_t>(slot));
}
inline int fmt_of(int32_t e) { return static_cast<int>(static_cast<uint32_t>(e) >> kFmtShift); }
// Slab (and allocator) of a format: TQ3 pages have their own; FP8 pages, or the BF16 pages of a
// control pool, use the first.
inline int slab_of(int fmt) { return fmt == MKV_FMT_TQ3 ? 1 : 0; }
inline int32_t slot_of(int32_t e) { return static_cast<int32_t>(static_cast<uint32_t>(e) & kSlotMask); }

struct TimingRec {
  cudaEvent_t ev[3];  // before the partial kernel, between partial and merge, after the merge
};

}  // namespace

struct mkv_pool {
  mkv_pool_config cfg{};
  bool host_only = false;
  uint8_t* fp8_slab = nullptr;
  uint8_t* tq3_slab = nullptr;
  int32_t* d_tables = nullptr;
  int32_t* d_status = nullptr;
  int64_t fp8_slot_bytes = 0, tq3_slot_bytes = 0;
  int sm_count = 148;
  int decode_sms = 0;  // SMs decode plans for (0: all of the device's)
  std::vector<Seq> seqs;
  Allocator alloc[2];
  int64_t launches = 0;
  int64_t fail_after = -1;  // test hook: device operations that still succeed before one fails
  int decode_kernels = MKV_DECODE_AUTO;  // per-format grids, one fused grid, or chosen per call
  int page_fmt = MKV_FMT_FP8;  // format of written pages: FP8, or BF16 in a control pool
  bool timing = false;
  std::vector<TimingRec> timing_recs;
  std::vector<cudaEvent_t> spare_events;
};

namespace {

bool valid_pool(mkv_pool_t p) { return p != nullptr; }

// Relative time of one page of each format in a CTA (measured with device timestamps on the
// long-context workload: 0.45 us per TQ3 page and 0.48-0.53 us per FP8 page per CTA).  Units are
// balanced by time, not bytes: an FP8 page carries 2.3x the bytes of a TQ3 page but costs less
// arithmetic per byte.
constexpr int64_t kFp8PageCost = 11;
constexpr int64_t kTq3PageCost = 10;
// Automatic choice of partial kernels: one fused grid when FP8 pages carry more than this share
// of the call's planned time.  Measured on the long-context workload: at 4% FP8 pages the
// per-format grids are faster (150.8 against 156.3 us), at 25% the fused grid (170.0 against
// 198.8 us): FP8 CTAs need more shared memory than TQ3 CTAs, so beyond one FP8 CTA per SM the
// per-format grids no longer fit one wave.  (The FP8 grid gets CTAs in proportion to its cost,
// so below this share it holds fewer CTAs than there are SMs.)
constexpr double kFusedAboveFp8Share = 0.15;

// SMs a decode call's cut is planned for: the device's, or fewer when the caller asked so.
int plan_sms(const mkv_pool* p) {
  return p->decode_sms > 0 && p->decode_sms < p->sm_count ? p->decode_sms : p->sm_count;
}

// Decode kernels of a call over these sequences with NC query columns per KV head
// (kDecodeSplit, kDecodeFused or kDecodeBf16).
int decode_mode(const mkv_pool* p, const int32_t* seq_ids, int32_t n, int32_t NC) {
  if (p->page_fmt == MKV_FMT_BF16) return kDecodeBf16;
  if (p->decode_kernels != MKV_DECODE_AUTO)
    return p->decode_kernels == MKV_DECODE_FUSED ? kDecodeFused : kDecodeSplit;
  int64_t c8 = 0, c3 = 0;
  for (int32_t i = 0; i < n; ++i) {
    const Seq& s = p->seqs[seq_ids[i]];
    c8 += static_cast<int64_t>(s.fp8_pages.size()) * kFp8PageCost;
    c3 += static_cast<int64_t>(s.n3) * kTq3PageCost;
  }
  // the fused grid keeps as many CTAs per SM as the TQ3 grid (D 64 and 128): one grid is enough
  const int D = p->cfg.head_dim;
  if (partial_ctas_per_sm(D, NC, kDecodeFused) >= partial_ctas_per_sm(D, NC, kDecodeSplit))
    return kDecodeFused;
  return c8 > kFusedAboveFp8Share * static_cast<double>(c8 + c3) ? kDecodeFused : kDecodeSplit;
}

int64_t page_head_bytes(const mkv_pool_config& c) {
  return (c.flags & MKV_POOL_BF16_CONTROL) ? bf16_head_bytes(c.head_dim) : fp8_head_bytes(c.head_dim);
}

int check_seq(mkv_pool_t p, int32_t s) {
  if (s < 0 || s >= p->cfg.max_seqs)
    return fail(MKV_ERR_BAD_SEQ, "sequence %d outside [0, %d)", s, p->cfg.max_seqs);
  return MKV_OK;
}

// Sequence-list checks shared by the calls that take one, in the documented order: every id in
// range (BAD_SEQ) before any other argument error (INVALID_ARG: an id listed twice, a negative
// count).  `counts` may be NULL.
int check_seq_list(mkv_pool_t p, const int32_t* seq_ids, int32_t n, const int32_t* counts) {
  for (int32_t i = 0; i < n; ++i)
    if (int e = check_seq(p, seq_ids[i])) return e;
  std::vector<uint8_t> seen(p->cfg.max_seqs, 0);
  for (int32_t i = 0; i < n; ++i) {
    if (seen[seq_ids[i]]) return fail(MKV_ERR_INVALID_ARG, "sequence %d listed twice", seq_ids[i]);
    seen[seq_ids[i]] = 1;
    if (counts && counts[i] < 0) return fail(MKV_ERR_INVALID_ARG, "negative token count");
  }
  return MKV_OK;
}

int validate_config(const mkv_pool_config* c) {
  if (!c) return fail(MKV_ERR_INVALID_ARG, "config is NULL");
  if (c->num_kv_heads < 1) return fail(MKV_ERR_INVALID_ARG, "num_kv_heads must be >= 1");
  if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256)
    return fail(MKV_ERR_UNSUPPORTED, "head_dim %d not built (64, 128, 256)", c->head_dim);
  if (c->page_size != kPageTokens) return fail(MKV_ERR_INVALID_ARG, "page_size must be 16");
  if (c->max_seqs < 1 || c->max_pages_per_seq < 1)
    return fail(MKV_ERR_INVALID_ARG, "max_seqs and max_pages_per_seq must be >= 1");
  if (c->fp8_slots < 1 || c->tq3_slots < 0 || c->fp8_slots > static_cast<int32_t>(kSlotMask) ||
      c->tq3_slots > static_cast<int32_t>(kSlotMask))
    return fail(MKV_ERR_INVALID_ARG, "slot counts out of range");
  if (c->sink_pages < 0) return fail(MKV_ERR_INVALID_ARG, "sink_pages must be >= 0");
  if (c->flags & ~(MKV_POOL_HOST_ONLY | MKV_POOL_BF16_CONTROL))
    return fail(MKV_ERR_INVALID_ARG, "unknown flags");
  if (static_cast<int64_t>(c->max_seqs) * c->max_pages_per_seq > (1LL << 31) - 1)
    return fail(MKV_ERR_INVALID_ARG, "table too large");
  if (c->max_pages_per_seq > INT32_MAX / kPageTokens)
    return fail(MKV_ERR_INVALID_ARG, "max_pages_per_seq too large: token counts are int32");
  return MKV_OK;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Device status buffer: the status word (padded to 256 bytes).
size_t status_bytes(const mkv_pool_config&) { return 256; }

struct LaunchDesc {
  int32_t s0 = 0, s1 = 0;   // call positions [s0, s1)
  int32_t u0 = 0, u1 = 0;   // units [u0, u1) of DecodePlan::unit, CTA by CTA
  int32_t n_ctas = 0;       // CTAs per KV head
  int32_t n_fp8 = 0;        // of which FP8 CTAs (per-format grids), the first ones
};

struct DecodePlan {
  int32_t NC = 0, g = 0;
  int mode = kDecodeSplit;         // partial kernels of the call
  std::vector<SeqDesc> seq;        // per call position
  std::vector<UnitDesc> unit;      // launch by launch, CTA by CTA
  std::vector<int32_t> pos;        // call position of each unit's sequence
  std::vector<int32_t> cta;        // CTA of each unit within its launch
  std::vector<int64_t> cost;       // relative time of each unit (per KV head)
  std::vector<LaunchDesc> launch;
  int64_t parts = 0;
  size_t off_ml = 0, off_acc = 0, bytes = 0;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Work-unit cut shared by both decode entry points (no allocation).  A launch runs one grid per
// page format (or one fused grid) of CTAs x KV heads, sized for a single wave: at most
// SMs x resident CTAs per SM.  A unit is one format's pages inside a logical page range of one
// sequence and yields one partial state.  cut_launch picks one of two cuts: per group (below) or
// the line cut, where a grid's pages -- every sequence's pages of its format, in call order --
// form one line, cut into CTAs of equal cost; a CTA takes a unit for each sequence its share of
// the line touches, so the longest CTA, which ends the wave, is within a few pages of the
// average however unequal the sequences are.  For the line cut:
//   - Pages are weighted by measured time per CTA (FP8 11, TQ3 10), not by bytes, and every
//     run of pages that starts a unit adds kUnitCost (the unit's scan, Q set-up, ring refill
//     and combine), so a CTA that starts several units takes fewer pages.
//   - A sequence's FP8 pages are split into runs at gaps of more than kFp8RunGap pages (the
//     sink pages and the recent window are far apart): a unit's kernel scans its whole logical
//     range for pages of its format, and one run keeps that range short.
//   - Cut points that would leave a unit of fewer than a few pages move to the run's edge; a
//     unit holds at most kMaxPagesPerUnit pages.
constexpr int kMinTq3PagesPerUnit = 8;
constexpr int kMinFp8PagesPerUnit = 4;
constexpr int64_t kUnitCost = 60;
constexpr int32_t kFp8RunGap = 2048;

// Pages of format slot f (0: FP8 or BF16, 1: TQ3) of a sequence.
inline int64_t group_pages(const Seq& s, int f) {
  return f == 0 ? static_cast<int64_t>(s.fp8_pages.size()) : static_cast<int64_t>(s.n3);
}

// End of the run of format slot f that starts at page number a (of n) of the sequence.
inline int64_t run_end(const Seq& s, int f, int64_t a, int64_t n) {
  if (f == 1) return n;
  const std::vector<int32_t>& f8 = s.fp8_pages;
  int64_t e = a + 1;
  while (e < n && f8[e] - f8[e - 1] <= kFp8RunGap) ++e;
  return e;
}

// Cut one line -- the pages of the format slots in `fmts` (bit f) of call positions [s0, s1),
// in order -- into at most k CTAs of equal cost, numbered from *n_ctas on.  emit(unit, cost,
// pos, cta) is called CTA by CTA; n_parts[pos] counts each sequence's units (their part
// indices).  Returns false as soon as emit does.
template <class Emit>
bool cut_line(const mkv_pool* p, const int32_t* seq_ids, int32_t s0, int32_t s1, unsigned fmts,
              int64_t k, int32_t* n_parts, int32_t* n_ctas, Emit&& emit) {
  const int64_t b[2] = {kFp8PageCost, kTq3PageCost};
  const int64_t m[2] = {kMinFp8PagesPerUnit, kMinTq3PagesPerUnit};
  int64_t T = 0, pages = 0;
  for (int32_t i = s0; i < s1; ++i)
    for (int f = 0; f < 2; ++f)
      if (fmts >> f & 1) {
        const Seq& s = p->seqs[seq_ids[i]];
        const int64_t n = group_pages(s, f);
        for (int64_t a = 0; a < n; a = run_end(s, f, a, n)) T += kUnitCost;
        T += n * b[f];
        pages += n;
      }
  if (T == 0 || k <= 0) return true;
  // pieces of at least a few pages each
  k = std::max<int64_t>(1, std::min<int64_t>(k, pages / ((fmts & 2) ? m[1] : m[0])));
  int64_t j = 0;        // current piece
  int64_t owner = -1;   // the piece that last took a CTA number
  int64_t R0 = 0;       // line position of the current run (its unit cost, then its pages)
  for (int32_t i = s0; i < s1; ++i) {
    const Seq& s = p->seqs[seq_ids[i]];
    const std::vector<int32_t>& f8 = s.fp8_pages;
    const int64_t n8 = static_cast<int64_t>(f8.size());
    const int32_t table = static_cast<int32_t>(s.table.size());
    for (int f = 0; f < 2; ++f) {
      if (!(fmts >> f & 1)) continue;
      const int64_t n = group_pages(s, f);
      int64_t c8 = 0;  // FP8 pages before the current TQ3 page (logical = TQ3 number + c8)
      auto logical = [&](int64_t t) {  // logical page of TQ3 page number t (t < n)
        while (c8 < n8 && f8[c8] <= t + c8) ++c8;
        return static_cast<int32_t>(t + c8);
      };
      auto put = [&](int64_t a, int64_t e) -> bool {  // pages [a, e) of this group, piece j
        if (owner != j) {
          owner = j;
          ++*n_ctas;
        }
        const int64_t parts = (e - a + kMaxPagesPerUnit - 1) / kMaxPagesPerUnit;
        for (int64_t q = 0; q < parts; ++q) {
          const int64_t u0 = a + q * (e - a) / parts, u1 = a + (q + 1) * (e - a) / parts;
          UnitDesc u{};
          if (f == 0) {
            u.first = f8[u0];
            u.last = f8[u1 - 1] + 1;
            u.fmt = static_cast<uint8_t>(p->page_fmt);
          } else {
            // TQ3 ranges tile the table: the first starts at page 0, the last ends at its end,
            // each other one at the logical page of its first TQ3 page
            u.first = u0 == 0 ? 0 : logical(u0);
            u.last = u1 == n ? table : logical(u1);
            u.fmt = 1;
          }
          u.part = static_cast<uint16_t>(std::min<int32_t>(n_parts[i], 65535));
          ++n_parts[i];
          if (!emit(u, (u1 - u0) * b[f], i, *n_ctas - 1)) return false;
        }
        return true;
      };
      for (int64_t ra = 0; ra < n;) {
        const int64_t rb = run_end(s, f, ra, n);
        const int64_t P0 = R0 + kUnitCost, R1 = P0 + (rb - ra) * b[f];
        int64_t a = ra;
        while (a < rb) {
          const int64_t x = j + 1 < k ? T * (j + 1) / k : T;  // where piece j ends on the line
          if (x >= R1) {  // piece j takes the rest of the run
            if (!put(a, rb)) return false;
            a = rb;
            break;
          }
          // piece j ends inside the run: nearest page boundary, moved so that no unit of the
          // run is shorter than m pages where the run allows
          int64_t e = x <= P0 ? ra : ra + (x - P0 + b[f] / 2) / b[f];
          e = std::max(a, std::min(e, rb));
          if (e > a && e - a < m[f]) e = a == ra ? ra : std::min(rb, a + m[f]);
          if (e < rb && rb - e < m[f]) e = rb;
          if (e > a && !put(a, e)) return false;
          a = e;
          ++j;
        }
        R0 = R1;
        ra = rb;
      }
    }
  }
  return true;
}

// Units of one launch (call positions [s0, s1)), one of two cuts:
//   - per group (the default): every (sequence, format) group is split into equal parts, one
//     CTA each, the unit cost chosen by bisection as the smallest whose cut fits the wave
//     (or, when the groups alone outnumber the wave, one unit per group and 512 pages, the
//     hardware scheduler then balancing the waves); units go largest first, FP8 units first
//     for the per-format grids.  Every CTA starts one unit.
//   - the line cut (cut_line) when the per-group cut fits one wave but its longest unit is
//     more than 1 / kLineCutBelow times the wave's average: many unequal sequences (32 of 2K to
//     32K tokens left it 38% above).  A few CTAs then start two or more units, which costs more
//     than their unit cost accounts for where the per-group cut is already balanced (the
//     long-context workload: 157 against 151 us).
// Returns false when emit does.
constexpr double kLineCutBelow = 0.85;

template <class Emit>
bool cut_launch(const mkv_pool* p, const int32_t* seq_ids, int32_t s0, int32_t s1, int32_t NC,
                int mode, int32_t* n_parts, LaunchDesc* ld, Emit&& emit) {
  const int Hkv = p->cfg.num_kv_heads;
  const int64_t slots =
      static_cast<int64_t>(plan_sms(p)) * partial_ctas_per_sm(p->cfg.head_dim, NC, mode);
  // CTAs of the wave per KV head; a launch holds at most kDecodeMaxUnits units
  int64_t U = std::max<int64_t>(1, std::min<int64_t>(slots / Hkv, kDecodeMaxUnits - 2));
  ld->s0 = s0;
  ld->s1 = s1;
  ld->n_ctas = 0;
  ld->n_fp8 = 0;

  // ---- per-group cut
  const int64_t b[2] = {kFp8PageCost, kTq3PageCost};
  const int mins[2] = {kMinFp8PagesPerUnit, kMinTq3PagesPerUnit};
  int64_t total = 0;
  for (int32_t i = s0; i < s1; ++i)
    for (int f = 0; f < 2; ++f) total += group_pages(p->seqs[seq_ids[i]], f) * b[f];
  // units of a group at unit cost c: as many as its cost needs, clamped to the page limits
  auto units_at = [](double c, int64_t cost, int64_t pages, int min_pages) -> int64_t {
    const int64_t lo = (pages + kMaxPagesPerUnit - 1) / kMaxPagesPerUnit;
    const int64_t hi = std::max<int64_t>(lo, std::max<int64_t>(1, pages / min_pages));
    const int64_t u = static_cast<int64_t>(std::ceil(static_cast<double>(cost) / c - 1e-9));
    return std::max(lo, std::min(std::max<int64_t>(u, 1), hi));
  };
  auto count_at = [&](double c) -> int64_t {
    int64_t sum = 0;
    for (int32_t i = s0; i < s1; ++i)
      for (int f = 0; f < 2; ++f) {
        const int64_t n = group_pages(p->seqs[seq_ids[i]], f);
        if (n > 0) sum += units_at(c, n * b[f], n, mins[f]);
      }
    return sum;
  };
  // smallest unit cost whose cut needs at most U units (the largest unit bounds the wave)
  double lo_c = std::max(1.0, static_cast<double>(total) / U), hi_c = lo_c;
  while (count_at(hi_c) > U && hi_c < 4.0 * total) hi_c *= 2.0;
  for (int it = 0; it < 40 && hi_c - lo_c > 0.5; ++it) {
    const double mid = 0.5 * (lo_c + hi_c);
    (count_at(mid) <= U ? hi_c : lo_c) = mid;
  }
  const double unit_cost = hi_c;
  const bool fits = count_at(unit_cost) <= U;
  // groups in launch order: per-format grids take the FP8 groups first; largest units first
  int32_t order[2 * kDecodeMaxSeqs];
  int64_t ucost[2 * kDecodeMaxSeqs];
  int32_t ng = 0;
  int64_t longest = 0;
  for (int32_t i = s0; i < s1; ++i)
    for (int f = 0; f < 2; ++f) {
      const int64_t n = group_pages(p->seqs[seq_ids[i]], f);
      if (n == 0) continue;
      const int64_t u = units_at(unit_cost, n * b[f], n, mins[f]);
      ucost[ng] = (n + u - 1) / u * b[f];
      longest = std::max(longest, ucost[ng]);
      order[ng++] = 2 * (i - s0) + f;
    }
  const bool line = fits && static_cast<double>(total) / static_cast<double>(U) <
                                kLineCutBelow * static_cast<double>(longest);
  if (!line) {
    int32_t idx[2 * kDecodeMaxSeqs];
    for (int32_t g = 0; g < ng; ++g) idx[g] = g;
    std::sort(idx, idx + ng, [&](int32_t x, int32_t y) {
      const int fx = order[x] & 1, fy = order[y] & 1;
      if (mode == kDecodeSplit && fx != fy) return fx < fy;  // FP8 (0) first
      return ucost[x] != ucost[y] ? ucost[x] > ucost[y] : x < y;
    });
    for (int32_t g = 0; g < ng; ++g) {
      const int32_t i = s0 + order[idx[g]] / 2;
      const int f = order[idx[g]] & 1;
      if (mode == kDecodeSplit && f == 1 && ld->n_fp8 == 0) ld->n_fp8 = ld->n_ctas;
      const Seq& s = p->seqs[seq_ids[i]];
      const std::vector<int32_t>& f8 = s.fp8_pages;
      const int64_t n8 = static_cast<int64_t>(f8.size());
      const int64_t n = group_pages(s, f);
      const int64_t u = units_at(unit_cost, n * b[f], n, mins[f]);
      // unit k takes pages number [k n / u, (k+1) n / u) of the group.  TQ3 ranges tile the
      // table: each starts at the logical page of its first TQ3 page (the first at page 0) and
      // ends where the next one starts (the last at the end of the table); every page is FP8
      // or TQ3, so TQ3 page number j sits at logical page j + c, c the FP8 pages before it
      const int32_t table = static_cast<int32_t>(s.table.size());
      int64_t c = 0;
      int32_t start = 0;
      for (int64_t k = 0; k < u; ++k) {
        const int64_t j0 = k * n / u, j1 = (k + 1) * n / u;
        UnitDesc d{};
        if (f == 0) {
          if (j1 <= j0) continue;
          d.first = f8[j0];
          d.last = f8[j1 - 1] + 1;
          d.fmt = static_cast<uint8_t>(p->page_fmt);
        } else {
          int32_t end = table;
          if (k + 1 < u) {
            while (c < n8 && f8[c] <= j1 + c) ++c;
            end = static_cast<int32_t>(j1 + c);
          }
          d.first = start;
          d.last = end;
          d.fmt = 1;
          start = end;
          if (j1 <= j0) continue;
        }
        d.part = static_cast<uint16_t>(std::min<int32_t>(n_parts[i], 65535));
        ++n_parts[i];
        if (!emit(d, (j1 - j0) * b[f], i, ld->n_ctas)) return false;
        ++ld->n_ctas;
      }
    }
    if (mode == kDecodeSplit && ld->n_fp8 == 0) {  // no TQ3 group: every CTA is an FP8 one
      bool any3 = false;
      for (int32_t g = 0; g < ng; ++g) any3 |= (order[g] & 1) == 1;
      if (!any3) ld->n_fp8 = ld->n_ctas;
    }
    return true;
  }

  // ---- line cut
  int64_t c8 = 0, c3 = 0, bound = 0, runs8 = 0;
  for (int32_t i = s0; i < s1; ++i) {
    const Seq& s = p->seqs[seq_ids[i]];
    for (int f = 0; f < 2; ++f) {
      const int64_t n = group_pages(s, f);
      int64_t runs = 0;
      for (int64_t a = 0; a < n; a = run_end(s, f, a, n)) ++runs;
      (f == 0 ? c8 : c3) += n * b[f] + runs * kUnitCost;
      if (f == 0) runs8 += runs;
      // units beyond one per CTA: one more per run a cut crosses, and the 512-page splits
      bound += runs + n / kMaxPagesPerUnit;
    }
  }
  // the launch's units fit the parameter block: units <= CTAs + bound
  U = std::max<int64_t>(1, std::min<int64_t>(U, kDecodeMaxUnits - 2 - bound));
  if (mode == kDecodeSplit) {
    int64_t k8 = 0, k3 = 0;
    if (c8 > 0 && c3 > 0) {
      k8 = std::llround(static_cast<double>(U) * c8 / static_cast<double>(c8 + c3));
      // an FP8 CTA starts at most a few units (each a ring refill from memory)
      k8 = std::max<int64_t>((runs8 + 3) / 4, k8);
      k8 = std::max<int64_t>(1, std::min<int64_t>(k8, U - 1));  // both grids get a CTA
      k3 = std::max<int64_t>(1, U - k8);
    } else {
      (c8 > 0 ? k8 : k3) = U;
    }
    if (!cut_line(p, seq_ids, s0, s1, 1u, k8, n_parts, &ld->n_ctas, emit)) return false;
    ld->n_fp8 = ld->n_ctas;
    return cut_line(p, seq_ids, s0, s1, 2u, k3, n_parts, &ld->n_ctas, emit);
  }
  return cut_line(p, seq_ids, s0, s1, 3u, U, n_parts, &ld->n_ctas, emit);
}

int plan_decode(mkv_pool_t p, const int32_t* seq_ids, int32_t n, int32_t q_len, int32_t Hq,
                DecodePlan* plan) {
  if (n < 0 || (n > 0 && !seq_ids)) return fail(MKV_ERR_INVALID_ARG, "bad sequence list");
  if (n > p->cfg.max_seqs)
    return fail(MKV_ERR_INVALID_ARG, "at most max_seqs (%d) sequences per decode call", p->cfg.max_seqs);
  if (q_len < 1) return fail(MKV_ERR_INVALID_ARG, "q_len must be >= 1");
  const int Hkv = p->cfg.num_kv_heads, D = p->cfg.head_dim;
  if (Hq < Hkv || Hq % Hkv) return fail(MKV_ERR_INVALID_ARG, "num_q_heads %d not a multiple of Hkv %d", Hq, Hkv);
  plan->g = Hq / Hkv;
  plan->NC = q_len * plan->g;
  if (!partial_supported(D, plan->NC))
    return fail(MKV_ERR_UNSUPPORTED, "q_len * num_q_heads / Hkv = %d > 32 is not built", plan->NC);
  for (int32_t i = 0; i < n; ++i) {
    if (int e = check_seq(p, seq_ids[i])) return e;
    const Seq& s = p->seqs[seq_ids[i]];
    if (s.ctx < q_len || s.ctx == 0)
      return fail(MKV_ERR_EMPTY_CONTEXT, "sequence %d has %d tokens < q_len %d", seq_ids[i], s.ctx, q_len);
    if (group_pages(s, 0) > static_cast<int64_t>(kMaxPagesPerUnit) * kDecodeMaxUnits ||
        group_pages(s, 1) > static_cast<int64_t>(kMaxPagesPerUnit) * kDecodeMaxUnits)
      return fail(MKV_ERR_UNSUPPORTED, "sequence %d has more than %d pages of one format",
                  seq_ids[i], kMaxPagesPerUnit * kDecodeMaxUnits);
  }
  plan->seq.resize(n);
  plan->unit.clear();
  plan->pos.clear();
  plan->cta.clear();
  plan->cost.clear();
  plan->launch.clear();
  std::vector<int32_t> np(n, 0);
  plan->mode = decode_mode(p, seq_ids, n, plan->NC);
  // launches over groups of whole sequences, each cut for one wave: at most kDecodeMaxSeqs
  // sequences, and no more 512-page units than a launch holds (the per-group cut needs one per
  // group and 512 pages when the groups outnumber the wave; the line cut sizes itself)
  for (int32_t s0 = 0, s1 = 0; s0 < n; s0 = s1) {
    int64_t need = 0;
    for (s1 = s0; s1 < n && s1 - s0 < kDecodeMaxSeqs; ++s1) {
      const Seq& s = p->seqs[seq_ids[s1]];
      int64_t add = 0;
      for (int f = 0; f < 2; ++f)
        add += (group_pages(s, f) + kMaxPagesPerUnit - 1) / kMaxPagesPerUnit;
      if (s1 > s0 && need + add > kDecodeMaxUnits) break;
      need += add;
    }
    LaunchDesc ld;
    ld.u0 = static_cast<int32_t>(plan->unit.size());
    cut_launch(p, seq_ids, s0, s1, plan->NC, plan->mode,
               np.data(), &ld, [&](const UnitDesc& u, int64_t cost, int32_t i, int32_t cta) {
      plan->unit.push_back(u);
      plan->pos.push_back(i);
      plan->cta.push_back(cta);
      plan->cost.push_back(cost);
      return true;
    });
    ld.u1 = static_cast<int32_t>(plan->unit.size());
    if (ld.u1 - ld.u0 > kDecodeMaxUnits)
      return fail(MKV_ERR_UNSUPPORTED, "a launch needs %d work units; one holds %d",
                  ld.u1 - ld.u0, kDecodeMaxUnits);
    plan->launch.push_back(ld);
  }
  int64_t parts = 0;
  for (int32_t i = 0; i < n; ++i) {
    SeqDesc& d = plan->seq[i];
    d.row = seq_ids[i];
    d.ctx = p->seqs[seq_ids[i]].ctx;
    d.out_row = i;
    d.part0 = static_cast<int32_t>(parts);
    d.n_parts = np[i];
    d.pad = 0;
    parts += np[i];
  }
  if (parts > INT32_MAX / 2) return fail(MKV_ERR_INVALID_ARG, "call too large");
  plan->parts = parts;
  const size_t cols = static_cast<size_t>(parts) * Hkv * plan->NC;
  plan->off_ml = 0;
  plan->off_acc = align256(cols * 2 * 4);
  plan->bytes = std::max<size_t>(256, plan->off_acc + align256(cols * D * 4));
  return MKV_OK;
}

// Fill a launch's CTA table from the CTA number of each of its units (units come CTA by CTA).
// Returns false when the units are not in CTA order or a CTA has none.
bool fill_cta_table(DecodeParams* prm, const int32_t* cta, int32_t nu, int32_t n_ctas) {
  if (n_ctas < 0 || n_ctas > kDecodeMaxUnits || nu > kDecodeMaxUnits) return false;
  int32_t c = -1;
  for (int32_t k = 0; k < nu; ++k) {
    if (cta[k] == c) continue;
    if (cta[k] != c + 1) return false;
    c = cta[k];
    prm->cta_unit0[c] = static_cast<uint16_t>(k);
  }
  if (c + 1 != n_ctas) return false;
  prm->cta_unit0[n_ctas] = static_cast<uint16_t>(nu);
  prm->n_units = nu;
  prm->n_ctas = n_ctas;
  return true;
}

// Every device operation of a state-changing call (kernel launch or memset) goes through here:
// the test hook can make it fail, host-only pools skip it, and launches are counted.  The calls
// stage their host-state changes and commit them only after all their device operations were
// issued, so a failure here leaves the pool's host state as it was before the call.
template <class F>
int device_op(mkv_pool_t p, const char* what, F&& f) {
  if (p->fail_after == 0) {
    p->fail_after = -1;
    return fail(MKV_ERR_CUDA, "%s: launch failure injected by mkv_test_fail_launch", what);
  }
  if (p->fail_after > 0) --p->fail_after;
  if (p->host_only) return MKV_OK;
  ++p->launches;
  const cudaError_t e = f();
  return e == cudaSuccess ? MKV_OK : cuda_fail(e, what);
}

cudaEvent_t get_event(mkv_pool_t p) {
  if (!p->spare_events.empty()) {
    cudaEvent_t e = p->spare_events.back();
    p->spare_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* mkv_last_error(void) { return g_last_error.c_str(); }

int mkv_pool_required_bytes(const mkv_pool_config* cfg, size_t* fp8_slab, size_t* tq3_slab,
                            size_t* tables, size_t* status) {
  if (int e = validate_config(cfg)) return e;
  const size_t Hkv = cfg->num_kv_heads, D = cfg->head_dim;
  if (fp8_slab) *fp8_slab = static_cast<size_t>(cfg->fp8_slots) * Hkv * page_head_bytes(*cfg);
  if (tq3_slab) *tq3_slab = static_cast<size_t>(cfg->tq3_slots) * Hkv * tq3_head_bytes(D);
  if (tables) *tables = static_cast<size_t>(cfg->max_seqs) * cfg->max_pages_per_seq * 4;
  if (status) *status = status_bytes(*cfg);
  return ok();
}

int mkv_pool_create(const mkv_pool_config* cfg, void* fp8_slab, void* tq3_slab,
                    int32_t* d_tables, int32_t* d_status, mkv_pool_t* out) {
  if (int e = validate_config(cfg)) return e;
  if (!out) return fail(MKV_ERR_INVALID_ARG, "out is NULL");
  const bool host_only = (cfg->flags & MKV_POOL_HOST_ONLY) != 0;
  if (host_only) {
    if (fp8_slab || tq3_slab || d_tables || d_status)
      return fail(MKV_ERR_INVALID_ARG, "host-only pools take no device buffers");
  } else {
    if (!fp8_slab || (!tq3_slab && cfg->tq3_slots > 0) || !d_tables || !d_status)
      return fail(MKV_ERR_INVALID_ARG, "device buffers must not be NULL");
    const uintptr_t a = reinterpret_cast<uintptr_t>(fp8_slab) | reinterpret_cast<uintptr_t>(tq3_slab) |
                        reinterpret_cast<uintptr_t>(d_tables) | reinterpret_cast<uintptr_t>(d_status);
    if (a & 255) return fail(MKV_ERR_INVALID_ARG, "device buffers must be 256-byte aligned");
  }
  mkv_pool* p = new mkv_pool();
  p->cfg = *cfg;
  p->host_only = host_only;
  p->fp8_slab = static_cast<uint8_t*>(fp8_slab);
  p->tq3_slab = static_cast<uint8_t*>(tq3_slab);
  p->d_tables = d_tables;
  p->d_status = d_status;
  p->fp8_slot_bytes = static_cast<int64_t>(cfg->num_kv_heads) * page_head_bytes(*cfg);
  p->page_fmt = (cfg->flags & MKV_POOL_BF16_CONTROL) ? MKV_FMT_BF16 : MKV_FMT_FP8;
  p->tq3_slot_bytes = static_cast<int64_t>(cfg->num_kv_heads) * tq3_head_bytes(cfg->head_dim);
  p->seqs.resize(cfg->max_seqs);
  p->alloc[0].init(cfg->fp8_slots);
  p->alloc[1].init(cfg->tq3_slots);
  if (!host_only) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaMemsetAsync(d_tables, 0xFF, static_cast<size_t>(cfg->max_seqs) * cfg->max_pages_per_seq * 4, 0);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_status, 0, status_bytes(*cfg), 0);
    if (e == cudaSuccess) e = cudaStreamSynchronize(0);
    if (e != cudaSuccess) {
      delete p;
      return cuda_fail(e, "pool init");
    }
  }
  *out = p;
  return ok();
}

void mkv_pool_destroy(mkv_pool_t p) {
  if (!p) return;
  for (auto& r : p->timing_recs)
    for (auto e : r.ev) cudaEventDestroy(e);
  for (auto e : p->spare_events) cudaEventDestroy(e);
  delete p;
}

int mkv_pool_set_slot_order(mkv_pool_t p, int32_t fmt, const int32_t* order, int32_t n) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (fmt != MKV_FMT_FP8 && fmt != MKV_FMT_TQ3 && fmt != MKV_FMT_BF16)
    return fail(MKV_ERR_INVALID_ARG, "bad format");
  Allocator& a = p->alloc[slab_of(fmt)];
  if (n != a.n || (n > 0 && !order)) return fail(MKV_ERR_INVALID_ARG, "order must list all %d slots", a.n);
  std::vector<uint8_t> seen(n, 0);
  for (int32_t i = 0; i < n; ++i) {
    if (order[i] < 0 || order[i] >= n || seen[order[i]])
      return fail(MKV_ERR_INVALID_ARG, "order is not a permutation");
    seen[order[i]] = 1;
  }
  for (int32_t i = 0; i < n; ++i) a.rank[order[i]] = i;
  a.rebuild();
  return ok();
}

int mkv_append_kv(mkv_pool_t p, const int32_t* seq_ids, const int32_t* n_new, int32_t n_seqs,
                  const void* k_bf16, const void* v_bf16, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (n_seqs < 0 || (n_seqs > 0 && (!seq_ids || !n_new)))
    return fail(MKV_ERR_INVALID_ARG, "bad sequence list");
  const int32_t MP = p->cfg.max_pages_per_seq;
  int64_t need = 0, rows = 0;
  if (int e = check_seq_list(p, seq_ids, n_seqs, n_new)) return e;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq& s = p->seqs[seq_ids[i]];
    const int64_t pages_after = (static_cast<int64_t>(s.ctx) + n_new[i] + kPageTokens - 1) / kPageTokens;
    if (pages_after > MP)
      return fail(MKV_ERR_OUT_OF_PAGES, "sequence %d would need %lld pages > %d", seq_ids[i],
                  static_cast<long long>(pages_after), MP);
    need += pages_after - static_cast<int64_t>(s.table.size());
    rows += n_new[i];
  }
  if (need > p->alloc[0].n_free)
    return fail(MKV_ERR_OUT_OF_PAGES, "FP8 slab has %d free slots, %lld needed", p->alloc[0].n_free,
                static_cast<long long>(need));
  if (rows > 0 && !p->host_only && (!k_bf16 || !v_bf16))
    return fail(MKV_ERR_INVALID_ARG, "k/v are NULL");
  if (rows > INT32_MAX) return fail(MKV_ERR_INVALID_ARG, "too many tokens");

  // ---- stage: new FP8 slots and the page writes, against the tables as they will be
  std::vector<int32_t> taken;      // new slots, sequences in order, pages ascending
  std::vector<size_t> first_new(n_seqs);
  std::vector<AppendDesc> descs;
  int32_t row = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq& s = p->seqs[seq_ids[i]];
    const int32_t L0 = s.ctx, n = n_new[i], before = static_cast<int32_t>(s.table.size());
    const int32_t pages_after = (L0 + n + kPageTokens - 1) / kPageTokens;
    first_new[i] = taken.size();
    for (int32_t pg = before; pg < pages_after; ++pg) taken.push_back(p->alloc[0].take());
    for (int32_t t = 0; t < n;) {
      const int32_t pos = L0 + t, page = pos / kPageTokens, off = pos % kPageTokens;
      const int32_t cnt = std::min(kPageTokens - off, n - t);
      AppendDesc d;
      d.slot = page < before ? slot_of(s.table[page]) : taken[first_new[i] + (page - before)];
      d.table_index = seq_ids[i] * MP + page;
      d.first_row = row + t;
      d.n_old = static_cast<int16_t>(off);
      d.n_new = static_cast<int16_t>(cnt);
      descs.push_back(d);
      t += cnt;
    }
    row += n;
  }
  // ---- launch
  int rc = MKV_OK;
  if (!descs.empty()) {
    AppendParams* prm = new AppendParams;
    prm->fp8_slab = p->fp8_slab;
    prm->tables = p->d_tables;
    prm->status = p->d_status;
    prm->k = static_cast<const uint16_t*>(k_bf16);
    prm->v = static_cast<const uint16_t*>(v_bf16);
    prm->slot_bytes = p->fp8_slot_bytes;
    prm->Hkv = p->cfg.num_kv_heads;
    prm->D = p->cfg.head_dim;
    prm->bf16 = p->page_fmt == MKV_FMT_BF16 ? 1 : 0;
    for (size_t b = 0; b < descs.size() && rc == MKV_OK; b += kAppendMaxDesc) {
      const size_t m = std::min<size_t>(kAppendMaxDesc, descs.size() - b);
      prm->n_desc = static_cast<int32_t>(m);
      std::memcpy(prm->desc, descs.data() + b, m * sizeof(AppendDesc));
      rc = device_op(p, "append launch", [&] { return launch_append(*prm, as_stream(stream)); });
    }
    delete prm;
  }
  if (rc != MKV_OK) {
    for (auto it = taken.rbegin(); it != taken.rend(); ++it) p->alloc[0].give(*it);
    return rc;
  }
  // ---- commit
  for (int32_t i = 0; i < n_seqs; ++i) {
    Seq& s = p->seqs[seq_ids[i]];
    const int32_t pages_after = (s.ctx + n_new[i] + kPageTokens - 1) / kPageTokens;
    if (s.prot.size() < static_cast<size_t>(pages_after)) s.prot.resize(pages_after, 0);
    for (size_t k = first_new[i]; static_cast<int32_t>(s.table.size()) < pages_after; ++k) {
      s.fp8_pages.push_back(static_cast<int32_t>(s.table.size()));
      s.table.push_back(entry_of(p->page_fmt, taken[k]));
    }
    s.ctx += n_new[i];
  }
  return ok();
}

int mkv_set_protected(mkv_pool_t p, int32_t seq, int32_t page, int32_t flag) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (int e = check_seq(p, seq)) return e;
  Seq& s = p->seqs[seq];
  if (page < 0 || page >= static_cast<int32_t>(s.table.size()))
    return fail(MKV_ERR_INVALID_ARG, "page %d of sequence %d is not mapped", page, seq);
  s.prot[page] = flag ? 1 : 0;
  return ok();
}

int mkv_demote_pages(mkv_pool_t p, const int32_t* seq_ids, int32_t n_seqs, int32_t window,
                     int32_t* n_demoted, void* stream) {
  if (n_demoted) *n_demoted = 0;
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (n_seqs < 0 || (n_seqs > 0 && !seq_ids)) return fail(MKV_ERR_INVALID_ARG, "bad sequence list");
  if (int e = check_seq_list(p, seq_ids, n_seqs, nullptr)) return e;
  if (window < 0) return fail(MKV_ERR_INVALID_ARG, "window must be >= 0");
  struct Work { int32_t seq, page; };
  std::vector<Work> work;
  for (int32_t i = 0; i < n_seqs && p->page_fmt == MKV_FMT_FP8; ++i) {  // control: never
    const Seq& s = p->seqs[seq_ids[i]];
    const int64_t L = s.ctx;
    for (int32_t pg : s.fp8_pages) {
      const bool full = static_cast<int64_t>(kPageTokens) * (pg + 1) <= L;
      const bool anchor = pg < p->cfg.sink_pages ||
                          static_cast<int64_t>(kPageTokens) * pg + kPageTokens > L - window ||
                          s.prot[pg];
      if (full && !anchor) work.push_back({seq_ids[i], pg});
    }
  }
  if (static_cast<int64_t>(work.size()) > p->alloc[1].n_free)
    return fail(MKV_ERR_OUT_OF_PAGES, "TQ3 slab has %d free slots, %zu needed", p->alloc[1].n_free, work.size());
  // ---- stage: a TQ3 slot per page, in (sequence, page) order
  std::vector<DemoteDesc> descs;
  descs.reserve(work.size());
  for (const Work& w : work) {
    const Seq& s = p->seqs[w.seq];
    descs.push_back({slot_of(s.table[w.page]), p->alloc[1].take(),
                     w.seq * p->cfg.max_pages_per_seq + w.page});
  }
  // ---- launch: one launch writes the pages and publishes their table entries; a call that
  // needs several launches publishes no entry until every page is written (retag launches
  // last), so a failed launch never leaves a device entry naming an unwritten page
  int rc = MKV_OK;
  if (!descs.empty()) {
    const bool single = descs.size() <= static_cast<size_t>(kDemoteMaxDesc);
    DemoteParams* prm = new DemoteParams;
    prm->fp8_slab = p->fp8_slab;
    prm->tq3_slab = p->tq3_slab;
    prm->tables = p->d_tables;
    prm->fp8_slot_bytes = p->fp8_slot_bytes;
    prm->tq3_slot_bytes = p->tq3_slot_bytes;
    prm->Hkv = p->cfg.num_kv_heads;
    prm->D = p->cfg.head_dim;
    prm->publish = single ? 1 : 0;
    for (size_t b = 0; b < descs.size() && rc == MKV_OK; b += kDemoteMaxDesc) {
      const size_t m = std::min<size_t>(kDemoteMaxDesc, descs.size() - b);
      prm->n_desc = static_cast<int32_t>(m);
      std::memcpy(prm->desc, descs.data() + b, m * sizeof(DemoteDesc));
      rc = device_op(p, "demote launch", [&] { return launch_demote(*prm, as_stream(stream)); });
    }
    delete prm;
    if (!single && rc == MKV_OK) {
      RetagParams* rp = new RetagParams;
      rp->tables = p->d_tables;
      for (size_t b = 0; b < descs.size() && rc == MKV_OK; b += kRetagMax) {
        const size_t m = std::min<size_t>(kRetagMax, descs.size() - b);
        rp->n = static_cast<int32_t>(m);
        for (size_t k = 0; k < m; ++k) {
          rp->index[k] = descs[b + k].table_index;
          rp->entry[k] = entry_of(MKV_FMT_TQ3, descs[b + k].dst_slot);
        }
        rc = device_op(p, "retag launch", [&] { return launch_retag(*rp, as_stream(stream)); });
      }
      delete rp;
    }
  }
  if (rc != MKV_OK) {
    for (auto it = descs.rbegin(); it != descs.rend(); ++it) p->alloc[1].give(it->dst_slot);
    return rc;
  }
  // ---- commit: retag, then free the FP8 slots (reusable by later calls in stream order)
  for (size_t k = 0; k < work.size(); ++k) {
    Seq& s = p->seqs[work[k].seq];
    s.table[work[k].page] = entry_of(MKV_FMT_TQ3, descs[k].dst_slot);
    s.n3 += 1;
  }
  for (int32_t i = 0; i < n_seqs; ++i) {
    Seq& s = p->seqs[seq_ids[i]];
    s.fp8_pages.erase(std::remove_if(s.fp8_pages.begin(), s.fp8_pages.end(),
                                     [&](int32_t pg) { return fmt_of(s.table[pg]) != p->page_fmt; }),
                      s.fp8_pages.end());
  }
  for (const DemoteDesc& d : descs) p->alloc[0].give(d.src_slot);
  if (n_demoted) *n_demoted = static_cast<int32_t>(descs.size());
  return ok();
}

int mkv_decode_workspace_bytes(mkv_pool_t p, const int32_t* seq_ids, int32_t n_seqs,
                               int32_t q_len, int32_t Hq, size_t* bytes) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (!bytes) return fail(MKV_ERR_INVALID_ARG, "bytes is NULL");
  DecodePlan plan;
  if (int e = plan_decode(p, seq_ids, n_seqs, q_len, Hq, &plan)) return e;
  *bytes = plan.bytes;
  return ok();
}

int mkv_decode_plan(mkv_pool_t p, const int32_t* seq_ids, int32_t n_seqs, int32_t q_len,
                    int32_t Hq, int32_t* units_out, int32_t cap, int32_t* n_units,
                    int32_t* ctas_per_wave) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (!n_units || cap < 0) return fail(MKV_ERR_INVALID_ARG, "n_units is NULL or cap < 0");
  DecodePlan plan;
  if (int e = plan_decode(p, seq_ids, n_seqs, q_len, Hq, &plan)) return e;
  const int64_t nu = static_cast<int64_t>(plan.unit.size());
  *n_units = static_cast<int32_t>(nu);
  if (ctas_per_wave)
    *ctas_per_wave = plan_sms(p) * partial_ctas_per_sm(p->cfg.head_dim, plan.NC, plan.mode);
  if (!units_out) return ok();  // count query
  if (nu > cap) return fail(MKV_ERR_INVALID_ARG, "%lld units do not fit in %d", (long long)nu, cap);
  int32_t cta0 = 0;
  for (const LaunchDesc& ld : plan.launch) {
    for (int32_t k = ld.u0; k < ld.u1; ++k) {
      const UnitDesc& u = plan.unit[k];
      int32_t* o = units_out + 6 * k;
      o[0] = plan.pos[k];
      o[1] = u.fmt;
      o[2] = u.first;
      o[3] = u.last;
      o[4] = static_cast<int32_t>(plan.cost[k] / (u.fmt == 1 ? kTq3PageCost : kFp8PageCost));
      o[5] = cta0 + plan.cta[k];
    }
    cta0 += ld.n_ctas;
  }
  return ok();
}

int mkv_decode_attention(mkv_pool_t p, const int32_t* seq_ids, int32_t n_seqs, int32_t q_len,
                         const void* q_bf16, int32_t Hq, float sm_scale, float* out,
                         void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return fail(MKV_ERR_INVALID_ARG, "host-only pool cannot decode");
  DecodePlan plan;
  if (int e = plan_decode(p, seq_ids, n_seqs, q_len, Hq, &plan)) return e;
  if (!std::isfinite(sm_scale)) return fail(MKV_ERR_INVALID_ARG, "sm_scale is not finite");
  if (n_seqs == 0) return ok();
  if (!q_bf16 || !out || !workspace) return fail(MKV_ERR_INVALID_ARG, "q/out/workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(MKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < plan.bytes)
    return fail(MKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes, plan.bytes);
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams* prm = new DecodeParams;
  prm->fp8_slab = p->fp8_slab;
  prm->tq3_slab = p->tq3_slab;
  prm->tables = p->d_tables;
  prm->status = p->d_status;
  prm->q = static_cast<const uint16_t*>(q_bf16);
  prm->out = out;
  prm->part_ml = reinterpret_cast<float*>(ws + plan.off_ml);
  prm->part_acc = reinterpret_cast<float*>(ws + plan.off_acc);
  prm->fp8_slot_bytes = p->fp8_slot_bytes;
  prm->tq3_slot_bytes = p->tq3_slot_bytes;
  prm->Hkv = p->cfg.num_kv_heads;
  prm->D = p->cfg.head_dim;
  prm->g = plan.g;
  prm->q_len = q_len;
  prm->NC = plan.NC;
  prm->Hq = Hq;
  prm->max_pages = p->cfg.max_pages_per_seq;
  prm->fp8_slots = p->cfg.fp8_slots;
  prm->tq3_slots = p->cfg.tq3_slots;
  prm->logit_scale = sm_scale * 1.4426950408889634f;
  TimingRec rec{};
  bool timed = p->timing;
  if (timed)
    for (auto& e : rec.ev)
      if (!(e = get_event(p))) timed = false;
  cudaError_t err = timed ? cudaEventRecord(rec.ev[0], st) : cudaSuccess;
  // one launch (partial grids + merge) per group of whole sequences
  for (size_t li = 0; li < plan.launch.size() && err == cudaSuccess; ++li) {
    const LaunchDesc& ld = plan.launch[li];
    for (int32_t i = ld.s0; i < ld.s1; ++i) prm->seq[i - ld.s0] = plan.seq[i];
    const int32_t nu = ld.u1 - ld.u0;
    for (int32_t k = 0; k < nu; ++k) {
      prm->unit[k] = plan.unit[ld.u0 + k];
      prm->unit[k].seq = static_cast<uint8_t>(plan.pos[ld.u0 + k] - ld.s0);
    }
    if (!fill_cta_table(prm, plan.cta.data() + ld.u0, nu, ld.n_ctas)) {
      err = cudaErrorInvalidValue;
      break;
    }
    prm->n_fp8 = plan.mode == kDecodeSplit ? ld.n_fp8 : 0;
    prm->n_seqs = ld.s1 - ld.s0;
    prm->fused = plan.mode == kDecodeFused ? 1 : 0;
    prm->page_fmt = p->page_fmt;
    const bool last = li + 1 == plan.launch.size();
    err = launch_partial(*prm, st);
    ++p->launches;
    if (timed && last && err == cudaSuccess) err = cudaEventRecord(rec.ev[1], st);
    if (err == cudaSuccess) err = launch_merge(*prm, st), ++p->launches;
  }
  if (timed && err == cudaSuccess) err = cudaEventRecord(rec.ev[2], st);
  delete prm;
  if (timed) {
    if (err == cudaSuccess) p->timing_recs.push_back(rec);
    else for (auto e : rec.ev) p->spare_events.push_back(e);
  }
  if (err != cudaSuccess) return cuda_fail(err, "decode launch");
  return ok();
}

// Decode with the library's static partial-state scratch instead of a caller workspace.  Same
// units, order and kernels as mkv_decode_attention (so the same results), planned into a
// parameter block on the stack: no device allocation and, on success, no host allocation.
int mkv_decode_attention_noalloc(mkv_pool_t p, const int32_t* seq_ids, int32_t n_seqs,
                                 int32_t q_len, const void* q_bf16, int32_t Hq, float sm_scale,
                                 float* out, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return fail(MKV_ERR_INVALID_ARG, "host-only pool cannot decode");
  if (n_seqs < 0 || (n_seqs > 0 && !seq_ids)) return fail(MKV_ERR_INVALID_ARG, "bad sequence list");
  if (n_seqs > p->cfg.max_seqs)
    return fail(MKV_ERR_INVALID_ARG, "at most max_seqs (%d) sequences per decode call", p->cfg.max_seqs);
  if (n_seqs > kDecodeMaxSeqs)
    return fail(MKV_ERR_UNSUPPORTED, "the no-allocation decode takes at most %d sequences per call", kDecodeMaxSeqs);
  if (q_len < 1) return fail(MKV_ERR_INVALID_ARG, "q_len must be >= 1");
  if (!std::isfinite(sm_scale)) return fail(MKV_ERR_INVALID_ARG, "sm_scale is not finite");
  const int Hkv = p->cfg.num_kv_heads, D = p->cfg.head_dim;
  if (Hq < Hkv || Hq % Hkv) return fail(MKV_ERR_INVALID_ARG, "num_q_heads %d not a multiple of Hkv %d", Hq, Hkv);
  const int32_t g = Hq / Hkv, NC = q_len * g;
  if (!partial_supported(D, NC))
    return fail(MKV_ERR_UNSUPPORTED, "q_len * num_q_heads / Hkv = %d > 32 is not built", NC);
  for (int32_t i = 0; i < n_seqs; ++i) {
    if (int e = check_seq(p, seq_ids[i])) return e;
    const Seq& s = p->seqs[seq_ids[i]];
    if (s.ctx < q_len || s.ctx == 0)
      return fail(MKV_ERR_EMPTY_CONTEXT, "sequence %d has %d tokens < q_len %d", seq_ids[i], s.ctx, q_len);
  }
  if (n_seqs == 0) return ok();
  if (!q_bf16 || !out) return fail(MKV_ERR_INVALID_ARG, "q/out is NULL");
  DecodeParams prm;  // about 28 KB of stack (the cut adds about 8 KB)
  int32_t np[kDecodeMaxSeqs] = {};
  int32_t nu = 0, last_cta = -1;
  auto keep = [&](const UnitDesc& u, int64_t, int32_t i, int32_t cta) {
    if (nu >= kDecodeMaxUnits || cta < last_cta || cta > last_cta + 1) return false;
    if (cta != last_cta) prm.cta_unit0[cta] = static_cast<uint16_t>(nu);
    last_cta = cta;
    prm.unit[nu] = u;
    prm.unit[nu].seq = static_cast<uint8_t>(i);  // n_seqs <= kDecodeMaxSeqs: one launch
    ++nu;
    return true;
  };
  const int mode = decode_mode(p, seq_ids, n_seqs, NC);
  LaunchDesc ld;
  if (!cut_launch(p, seq_ids, 0, n_seqs, NC, mode, np, &ld, keep) || last_cta + 1 != ld.n_ctas)
    return fail(MKV_ERR_UNSUPPORTED, "the no-allocation decode takes at most %d work units per call", kDecodeMaxUnits);
  prm.cta_unit0[ld.n_ctas] = static_cast<uint16_t>(nu);
  prm.n_ctas = ld.n_ctas;
  prm.n_fp8 = mode == kDecodeSplit ? ld.n_fp8 : 0;
  int32_t parts = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    SeqDesc& d = prm.seq[i];
    d.row = seq_ids[i];
    d.ctx = p->seqs[seq_ids[i]].ctx;
    d.out_row = i;
    d.part0 = parts;
    d.n_parts = np[i];
    d.pad = 0;
    parts += np[i];
  }
  const size_t cols = static_cast<size_t>(parts) * Hkv * NC;
  const size_t off_acc = align256(cols * 2 * 4);
  const size_t bytes = off_acc + align256(cols * D * 4);
  void* scratch = nullptr;
  size_t cap = 0;
  cudaError_t err = static_decode_scratch(&scratch, &cap);
  if (err != cudaSuccess) return cuda_fail(err, "static scratch address");
  if (bytes > cap)
    return fail(MKV_ERR_WORKSPACE_TOO_SMALL,
                "call needs %zu bytes of partial-state scratch; the static scratch holds %zu", bytes, cap);
  prm.fused = mode == kDecodeFused ? 1 : 0;
  prm.page_fmt = p->page_fmt;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  prm.fp8_slab = p->fp8_slab;
  prm.tq3_slab = p->tq3_slab;
  prm.tables = p->d_tables;
  prm.status = p->d_status;
  prm.q = static_cast<const uint16_t*>(q_bf16);
  prm.out = out;
  prm.part_ml = reinterpret_cast<float*>(ws);
  prm.part_acc = reinterpret_cast<float*>(ws + off_acc);
  prm.fp8_slot_bytes = p->fp8_slot_bytes;
  prm.tq3_slot_bytes = p->tq3_slot_bytes;
  prm.Hkv = Hkv;
  prm.D = D;
  prm.g = g;
  prm.q_len = q_len;
  prm.NC = NC;
  prm.Hq = Hq;
  prm.max_pages = p->cfg.max_pages_per_seq;
  prm.fp8_slots = p->cfg.fp8_slots;
  prm.tq3_slots = p->cfg.tq3_slots;
  prm.logit_scale = sm_scale * 1.4426950408889634f;
  prm.n_seqs = n_seqs;
  prm.n_units = nu;
  cudaStream_t st = as_stream(stream);
  err = launch_partial(prm, st);
  ++p->launches;
  if (err == cudaSuccess) err = launch_merge(prm, st), ++p->launches;
  if (err != cudaSuccess) return cuda_fail(err, "decode launch");
  return ok();
}

int mkv_seq_reset(mkv_pool_t p, int32_t seq, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (int e = check_seq(p, seq)) return e;
  Seq& s = p->seqs[seq];
  const size_t n = s.table.size();
  if (n > 0) {
    const int rc = device_op(p, "reset", [&] {
      return cudaMemsetAsync(p->d_tables + static_cast<int64_t>(seq) * p->cfg.max_pages_per_seq,
                             0xFF, n * 4, as_stream(stream));
    });
    if (rc != MKV_OK) return rc;
  }
  for (int32_t e : s.table) p->alloc[slab_of(fmt_of(e))].give(slot_of(e));
  s = Seq();
  return ok();
}

int mkv_selftest_wait(mkv_pool_t p, int64_t limit_ns, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return fail(MKV_ERR_INVALID_ARG, "host-only pool has no device");
  if (limit_ns < 0 || limit_ns > 2000000000LL)
    return fail(MKV_ERR_INVALID_ARG, "limit must be in [0, 2 s]");
  cudaError_t e = launch_wait_selftest(p->d_status, static_cast<uint64_t>(limit_ns), as_stream(stream));
  ++p->launches;
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ok();
}

int mkv_selftest_tc_logits(mkv_pool_t p, const void* a_f16, const void* q_f16, float* d_out,
                           void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return fail(MKV_ERR_INVALID_ARG, "host-only pool has no device");
  if (!a_f16 || !q_f16 || !d_out) return fail(MKV_ERR_INVALID_ARG, "a/q/d is NULL");
  cudaError_t e = launch_tc_logits_selftest(a_f16, q_f16, d_out, p->d_status, as_stream(stream));
  ++p->launches;
  if (e != cudaSuccess) return cuda_fail(e, "tensor-memory self-test launch");
  return ok();
}

int mkv_prefill_kv(mkv_pool_t p, const int32_t* seq_ids, const int32_t* n_tokens, int32_t n_seqs,
                   const void* k_bf16, const void* v_bf16, int32_t anchor_window_tokens,
                   void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (n_seqs < 0 || (n_seqs > 0 && (!seq_ids || !n_tokens)))
    return fail(MKV_ERR_INVALID_ARG, "bad sequence list");
  if (int e = check_seq_list(p, seq_ids, n_seqs, n_tokens)) return e;
  if (anchor_window_tokens < 0) return fail(MKV_ERR_INVALID_ARG, "negative anchor window");
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq& s = p->seqs[seq_ids[i]];
    if (s.ctx || !s.table.empty())
      return fail(MKV_ERR_INVALID_ARG, "prefill needs an empty sequence (%d is not)", seq_ids[i]);
  }
  const int32_t MP = p->cfg.max_pages_per_seq, sink = p->cfg.sink_pages;
  // page p of a prefill of n tokens is packed to TQ3 at once iff the anchor policy would demote
  // it: p >= sink and 16p + 16 <= n - W (new pages carry no protection)
  auto direct = [&](int64_t pg, int64_t n) {  // (a control pool writes every page as BF16)
    return p->page_fmt == MKV_FMT_FP8 && pg >= sink &&
           kPageTokens * pg + kPageTokens <= n - anchor_window_tokens;
  };
  int64_t need[2] = {0, 0}, rows = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int64_t pages = (static_cast<int64_t>(n_tokens[i]) + kPageTokens - 1) / kPageTokens;
    if (pages > MP)
      return fail(MKV_ERR_OUT_OF_PAGES, "sequence %d would need %lld pages > %d", seq_ids[i],
                  static_cast<long long>(pages), MP);
    for (int64_t pg = 0; pg < pages; ++pg) ++need[direct(pg, n_tokens[i]) ? 1 : 0];
    rows += n_tokens[i];
  }
  for (int f = 0; f < 2; ++f)
    if (need[f] > p->alloc[f].n_free)
      return fail(MKV_ERR_OUT_OF_PAGES, "%s slab has %d free slots, %lld needed", f ? "TQ3" : "FP8",
                  p->alloc[f].n_free, static_cast<long long>(need[f]));
  if (rows > 0 && !p->host_only && (!k_bf16 || !v_bf16))
    return fail(MKV_ERR_INVALID_ARG, "k/v are NULL");
  if (rows > INT32_MAX) return fail(MKV_ERR_INVALID_ARG, "too many tokens");

  // ---- stage: pages ascending, each taking a slot of its own format
  std::vector<int32_t> taken[2];   // slots per format, in the order taken
  std::vector<AppendDesc> fp8_descs;
  std::vector<PackDesc> tq3_descs;
  int32_t row = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int32_t n = n_tokens[i], pages = (n + kPageTokens - 1) / kPageTokens;
    for (int32_t pg = 0; pg < pages; ++pg) {
      const int32_t first_row = row + kPageTokens * pg;
      const int32_t table_index = seq_ids[i] * MP + pg;
      const int f = direct(pg, n) ? 1 : 0;
      const int32_t slot = p->alloc[f].take();
      taken[f].push_back(slot);
      if (f == 1) {
        tq3_descs.push_back({slot, table_index, first_row});
      } else {
        AppendDesc d;
        d.slot = slot;
        d.table_index = table_index;
        d.first_row = first_row;
        d.n_old = 0;
        d.n_new = static_cast<int16_t>(std::min(kPageTokens, n - kPageTokens * pg));
        fp8_descs.push_back(d);
      }
    }
    row += n;
  }
  // ---- launch (new pages only: their table entries were unmapped, so entries published by an
  // earlier launch of a failed call are ignored and later overwritten)
  cudaStream_t st = as_stream(stream);
  int rc = MKV_OK;
  if (!fp8_descs.empty()) {
    AppendParams* ap = new AppendParams;
    ap->fp8_slab = p->fp8_slab;
    ap->tables = p->d_tables;
    ap->status = p->d_status;
    ap->k = static_cast<const uint16_t*>(k_bf16);
    ap->v = static_cast<const uint16_t*>(v_bf16);
    ap->slot_bytes = p->fp8_slot_bytes;
    ap->Hkv = p->cfg.num_kv_heads;
    ap->D = p->cfg.head_dim;
    ap->bf16 = p->page_fmt == MKV_FMT_BF16 ? 1 : 0;
    for (size_t b = 0; b < fp8_descs.size() && rc == MKV_OK; b += kAppendMaxDesc) {
      const size_t m = std::min<size_t>(kAppendMaxDesc, fp8_descs.size() - b);
      ap->n_desc = static_cast<int32_t>(m);
      std::memcpy(ap->desc, fp8_descs.data() + b, m * sizeof(AppendDesc));
      rc = device_op(p, "prefill launch", [&] { return launch_append(*ap, st); });
    }
    delete ap;
  }
  if (!tq3_descs.empty() && rc == MKV_OK) {
    PackParams* pp = new PackParams;
    pp->k = static_cast<const uint16_t*>(k_bf16);
    pp->v = static_cast<const uint16_t*>(v_bf16);
    pp->tq3_slab = p->tq3_slab;
    pp->tables = p->d_tables;
    pp->tq3_slot_bytes = p->tq3_slot_bytes;
    pp->Hkv = p->cfg.num_kv_heads;
    pp->D = p->cfg.head_dim;
    pp->vec16 = ((reinterpret_cast<uintptr_t>(k_bf16) | reinterpret_cast<uintptr_t>(v_bf16)) & 15) ? 0 : 1;
    for (size_t b = 0; b < tq3_descs.size() && rc == MKV_OK; b += kPackMaxDesc) {
      const size_t m = std::min<size_t>(kPackMaxDesc, tq3_descs.size() - b);
      pp->n_desc = static_cast<int32_t>(m);
      std::memcpy(pp->desc, tq3_descs.data() + b, m * sizeof(PackDesc));
      rc = device_op(p, "prefill launch", [&] { return launch_pack(*pp, st); });
    }
    delete pp;
  }
  if (rc != MKV_OK) {
    for (int f = 0; f < 2; ++f)
      for (auto it = taken[f].rbegin(); it != taken[f].rend(); ++it) p->alloc[f].give(*it);
    return rc;
  }
  // ---- commit
  size_t next[2] = {0, 0};
  for (int32_t i = 0; i < n_seqs; ++i) {
    Seq& s = p->seqs[seq_ids[i]];
    const int32_t n = n_tokens[i], pages = (n + kPageTokens - 1) / kPageTokens;
    s.prot.assign(pages, 0);
    for (int32_t pg = 0; pg < pages; ++pg) {
      const int f = direct(pg, n) ? 1 : 0;
      s.table.push_back(entry_of(f == 1 ? MKV_FMT_TQ3 : p->page_fmt, taken[f][next[f]++]));
      if (f == 1) ++s.n3;
      else s.fp8_pages.push_back(pg);
    }
    s.ctx = n;
  }
  return ok();
}

int mkv_materialise_kv(mkv_pool_t p, int32_t seq, float* k_out, float* v_out,
                       int64_t max_tokens, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return fail(MKV_ERR_INVALID_ARG, "host-only pool has no device pages");
  if (int e = check_seq(p, seq)) return e;
  const Seq& s = p->seqs[seq];
  if (s.ctx == 0) return ok();
  if (!k_out || !v_out) return fail(MKV_ERR_INVALID_ARG, "output is NULL");
  if (max_tokens < s.ctx)
    return fail(MKV_ERR_INVALID_ARG, "outputs hold %lld tokens < context %d",
                static_cast<long long>(max_tokens), s.ctx);
  MaterialiseParams prm{};
  prm.fp8_slab = p->fp8_slab;
  prm.tq3_slab = p->tq3_slab;
  prm.table = p->d_tables + static_cast<int64_t>(seq) * p->cfg.max_pages_per_seq;
  prm.status = p->d_status;
  prm.k_out = k_out;
  prm.v_out = v_out;
  prm.fp8_slot_bytes = p->fp8_slot_bytes;
  prm.tq3_slot_bytes = p->tq3_slot_bytes;
  prm.Hkv = p->cfg.num_kv_heads;
  prm.D = p->cfg.head_dim;
  prm.ctx = s.ctx;
  prm.fp8_slots = p->cfg.fp8_slots;
  prm.tq3_slots = p->cfg.tq3_slots;
  prm.page_fmt = p->page_fmt;
  cudaError_t e = launch_materialise(prm, as_stream(stream));
  ++p->launches;
  if (e != cudaSuccess) return cuda_fail(e, "materialise launch");
  return ok();
}

int mkv_seq_copy(mkv_pool_t p, int32_t src, int32_t dst, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (int e = check_seq(p, src)) return e;
  if (int e = check_seq(p, dst)) return e;
  if (src == dst || !p->seqs[dst].table.empty() || p->seqs[dst].ctx)
    return fail(MKV_ERR_INVALID_ARG, "destination must be a different, empty sequence");
  const Seq& s = p->seqs[src];
  int64_t need[2] = {0, 0};
  for (int32_t e : s.table) need[slab_of(fmt_of(e))]++;
  for (int f = 0; f < 2; ++f)
    if (need[f] > p->alloc[f].n_free) return fail(MKV_ERR_OUT_OF_PAGES, "slab %d exhausted", f);
  // ---- stage: a slot of the same format per page, pages ascending
  Seq d;
  d.ctx = s.ctx;
  d.prot = s.prot;
  d.n3 = s.n3;
  d.fp8_pages = s.fp8_pages;
  std::vector<CopyDesc> descs;
  for (size_t pg = 0; pg < s.table.size(); ++pg) {
    const int f = fmt_of(s.table[pg]);
    const int32_t ns = p->alloc[slab_of(f)].take();
    d.table.push_back(entry_of(f, ns));
    descs.push_back({slot_of(s.table[pg]), ns, f, dst * p->cfg.max_pages_per_seq + static_cast<int32_t>(pg)});
  }
  // ---- launch (the destination was empty: entries published before a failure are ignored)
  int rc = MKV_OK;
  if (!descs.empty()) {
    CopyParams* prm = new CopyParams;
    prm->fp8_slab = p->fp8_slab;
    prm->tq3_slab = p->tq3_slab;
    prm->tables = p->d_tables;
    prm->fp8_slot_bytes = p->fp8_slot_bytes;
    prm->tq3_slot_bytes = p->tq3_slot_bytes;
    for (size_t b = 0; b < descs.size() && rc == MKV_OK; b += kCopyMaxDesc) {
      const size_t m = std::min<size_t>(kCopyMaxDesc, descs.size() - b);
      prm->n_desc = static_cast<int32_t>(m);
      std::memcpy(prm->desc, descs.data() + b, m * sizeof(CopyDesc));
      rc = device_op(p, "copy launch", [&] { return launch_copy(*prm, as_stream(stream)); });
    }
    delete prm;
  }
  if (rc != MKV_OK) {
    for (auto it = descs.rbegin(); it != descs.rend(); ++it)
      p->alloc[slab_of(it->fmt)].give(it->dst_slot);
    return rc;
  }
  p->seqs[dst] = std::move(d);
  return ok();
}

int mkv_get_block_table(mkv_pool_t p, int32_t seq, int32_t* host_out, int32_t cap,
                        int32_t* n_pages, int32_t* ctx_len) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (int e = check_seq(p, seq)) return e;
  const Seq& s = p->seqs[seq];
  if (cap < 0 || (cap > 0 && !host_out)) return fail(MKV_ERR_INVALID_ARG, "bad output buffer");
  const int32_t n = static_cast<int32_t>(s.table.size());
  for (int32_t i = 0; i < std::min(cap, n); ++i) host_out[i] = s.table[i];
  if (n_pages) *n_pages = n;
  if (ctx_len) *ctx_len = s.ctx;
  return ok();
}

int mkv_slot_bytes(mkv_pool_t p, int32_t fmt, size_t* bytes) {
  if (!valid_pool(p) || !bytes) return fail(MKV_ERR_INVALID_ARG, "NULL argument");
  if (fmt == p->page_fmt) *bytes = p->fp8_slot_bytes;
  else if (fmt == MKV_FMT_TQ3) *bytes = p->tq3_slot_bytes;
  else return fail(MKV_ERR_INVALID_ARG, "bad format");
  return ok();
}

int mkv_read_slot(mkv_pool_t p, int32_t entry, void* host_out, size_t cap, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return fail(MKV_ERR_INVALID_ARG, "host-only pool has no slabs");
  if (entry == MKV_ENTRY_UNMAPPED) return fail(MKV_ERR_INVALID_ARG, "unmapped entry");
  const int f = fmt_of(entry);
  const int32_t slot = slot_of(entry);
  if ((f != MKV_FMT_TQ3 && f != p->page_fmt) || slot >= (f == MKV_FMT_TQ3 ? p->cfg.tq3_slots : p->cfg.fp8_slots))
    return fail(MKV_ERR_INVALID_ARG, "entry 0x%x names no slot", entry);
  const int64_t b = f == MKV_FMT_TQ3 ? p->tq3_slot_bytes : p->fp8_slot_bytes;
  if (!host_out || cap < static_cast<size_t>(b)) return fail(MKV_ERR_INVALID_ARG, "output buffer too small");
  const uint8_t* src = (f == MKV_FMT_TQ3 ? p->tq3_slab : p->fp8_slab) + slot * b;
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaMemcpyAsync(host_out, src, b, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "read slot");
  return ok();
}

int mkv_pool_stats(mkv_pool_t p, int64_t* live, int32_t* n8, int32_t* n3, double* bpt) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  int64_t tokens = 0, c8 = 0, c3 = 0;
  for (const Seq& s : p->seqs) {
    tokens += s.ctx;
    c8 += static_cast<int64_t>(s.fp8_pages.size());
    c3 += s.n3;
  }
  if (live) *live = tokens;
  if (n8) *n8 = static_cast<int32_t>(c8);
  if (n3) *n3 = static_cast<int32_t>(c3);
  if (bpt) *bpt = tokens ? static_cast<double>(c8 * p->fp8_slot_bytes + c3 * p->tq3_slot_bytes) / tokens : 0.0;
  return ok();
}

int mkv_get_device_status(mkv_pool_t p, void* stream) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (p->host_only) return ok();
  cudaStream_t st = as_stream(stream);
  int32_t h = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&h, p->d_status, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, 4);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (h & kStatusTimeout) return fail(MKV_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait ran out (status 0x%x)", h);
  if (h & kStatusCheck) return fail(MKV_ERR_DEVICE_CHECK, "a kernel found an invalid entry or input (status 0x%x)", h);
  return ok();
}

int mkv_timing_enable(mkv_pool_t p, int32_t enable) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  p->timing = enable != 0;
  return ok();
}

int mkv_timing_read(mkv_pool_t p, double* ms_partial, double* ms_merge, int64_t* calls) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  double a = 0, b = 0;
  cudaError_t err = cudaSuccess;
  for (auto& r : p->timing_recs) {
    float t0 = 0, t1 = 0;
    if (err == cudaSuccess) err = cudaEventSynchronize(r.ev[2]);
    if (err == cudaSuccess) err = cudaEventElapsedTime(&t0, r.ev[0], r.ev[1]);
    if (err == cudaSuccess) err = cudaEventElapsedTime(&t1, r.ev[1], r.ev[2]);
    a += t0;
    b += t1;
  }
  const int64_t n = static_cast<int64_t>(p->timing_recs.size());
  for (auto& r : p->timing_recs)
    for (auto e : r.ev) p->spare_events.push_back(e);
  p->timing_recs.clear();
  if (err != cudaSuccess) return cuda_fail(err, "timing read");
  if (ms_partial) *ms_partial = a;
  if (ms_merge) *ms_merge = b;
  if (calls) *calls = n;
  return ok();
}

int mkv_set_decode_kernels(mkv_pool_t p, int32_t mode) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (mode != MKV_DECODE_SPLIT && mode != MKV_DECODE_FUSED && mode != MKV_DECODE_AUTO)
    return fail(MKV_ERR_INVALID_ARG, "unknown decode kernel mode %d", mode);
  p->decode_kernels = mode;
  return ok();
}

int mkv_set_decode_sms(mkv_pool_t p, int32_t sms) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (sms < 0) return fail(MKV_ERR_INVALID_ARG, "sms must be >= 0");
  p->decode_sms = sms;
  return ok();
}

int mkv_test_fail_launch(mkv_pool_t p, int32_t after) {
  if (!valid_pool(p)) return fail(MKV_ERR_INVALID_ARG, "pool is NULL");
  if (after < -1) return fail(MKV_ERR_INVALID_ARG, "after must be >= -1");
  p->fail_after = after;
  return ok();
}

int mkv_launch_count(mkv_pool_t p, int64_t* launches) {
  if (!valid_pool(p) || !launches) return fail(MKV_ERR_INVALID_ARG, "NULL argument");
  *launches = p->launches;
  return ok();
}

}  // extern "C"
