/*
 * mkv.h -- C ABI of the mixed-format paged KV cache and its decode attention (sm_100a).
 *
 * The method ("Minima-KV: Retention-Preserving KV Cache Compression with Mixed-Format Paged
 * Attention", as summarised on brainszone.ai, pt and fr pages):
 *   - the KV cache is a hierarchy of pages stored in different numeric formats
 *     (section "O que os autores propõem");
 *   - recently used pages and pages marked protected ("anchor") stay in FP8, older
 *     non-anchor pages are converted to a denser packed format, "packed TQ3"; every page of
 *     a live request stays directly addressable (section "Âncoras em FP8, arquivo em TQ3");
 *   - a separate kernel per format computes partial attention states and a globally
 *     normalised online-softmax merge combines them, so decode runs directly over the
 *     heterogeneous cache with no dense single-format shadow copy
 *     (section "Como os resultados parciais são combinados");
 *   - the figure of merit is KV bytes per live token (section "Memória e compressão").
 *
 * Formats (the pages fix no bit layout; these are the library's):
 *   FP8  OCP E4M3 codes, one fp32 scale per (page, KV head, K-or-V).  Writes quantise with
 *        scale = fp32(amax/448) over the tokens being written; when a later write to the same
 *        page needs a larger scale the page's existing codes are re-encoded to it
 *        (rescale-on-grow).  Codes are nearest-even, saturating; scale 0 means codes 0.
 *   TQ3  3-bit codes q in 0..7 dequantised as (q - 3.5) * s, one fp16 scale s per 32
 *        channels per token per KV head (s = fp16(fp32(amax/3.5)), absmax); the 32 codes of a
 *        group are packed into 12 bytes, code j in bits 3j..3j+2 of the little-endian 96-bit
 *        integer.  A TQ3 page is computed from the full FP8 page it replaces.
 *
 * Slot layouts (one slot = one 16-token page for all KV heads; bytes per KV head h, heads in
 * order; mkv_read_slot returns exactly these bytes):
 *   FP8 slot, per head (32*D + 16 bytes):
 *       K codes [16 tokens][D]  |  V codes [16][D]  |  K scale f32  |  V scale f32  |  8 zero bytes
 *       rows of tokens not yet written are zero.
 *   TQ3 slot, per head (14*D bytes), G = D/32:
 *       K records [G][16 tokens][12 B] | K scales [G][16] f16 | V records [G][16][12 B] | V scales [G][16] f16
 *
 * Block-table entry (int32): -1 = unmapped, else (format << 30) | slot, format 0 = FP8,
 * 1 = TQ3, 2 = BF16 (control pools only; such an entry is negative as an int32, so test for
 * -1, not for the sign).  Sequence ids are rows of the table; a multi-layer cache uses one row
 * per (layer, sequence).
 *
 * Ownership: every device buffer is allocated and owned by the caller (e.g. by PyTorch) and
 * must outlive the pool; the pool owns only host state (allocators, the host copy of the
 * tables, protection flags).  All device work is asynchronous on the caller's stream
 * (a cudaStream_t passed as void*; NULL = legacy default stream); inputs must stay valid until
 * the stream reaches the call.  Calls on one pool must come from one host thread at a time and
 * be ordered on one stream (or ordered by the caller): slots freed by a call are reused by
 * later calls in stream order.
 *
 * Errors: every int-returning call returns MKV_OK or a negative MKV_ERR_* code and sets a
 * thread-local message readable with mkv_last_error().  Host validation runs before any
 * launch; a call that fails validation leaves the pool unchanged.  A call whose launch fails
 * (MKV_ERR_CUDA) leaves the pool's host state -- tables, free slots, lengths, flags -- unchanged
 * too: state changes are staged and committed after the call's last launch.  On the device, a
 * call issued as one launch either ran or did not; a call so large that it is split into several
 * launches may, when a later one fails, have written pages into slots that stay free and, for
 * an append, have re-encoded existing partial pages (rescale-on-grow): reset the sequences of
 * such a call.  A split demotion publishes no table entry before all its pages are written.
 * When several arguments of a
 * call taking a sequence list are wrong, an out-of-range id (BAD_SEQ) is reported before any
 * other argument error (INVALID_ARG), and those before a capacity error (OUT_OF_PAGES).  Device-side checks (bad
 * table entries, bounded waits that ran out) are recorded in the caller's status word and
 * reported by mkv_get_device_status().
 */
#ifndef MKV_H_
#define MKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MKV_API __attribute__((visibility("default")))

enum {
  MKV_OK = 0,
  MKV_ERR_INVALID_ARG = -1,         /* bad pointer, size, shape or flag */
  MKV_ERR_BAD_SEQ = -2,             /* sequence id outside [0, max_seqs) */
  MKV_ERR_OUT_OF_PAGES = -3,        /* a slab or a sequence's table has no room */
  MKV_ERR_EMPTY_CONTEXT = -4,       /* decode of a sequence shorter than q_len (or empty) */
  MKV_ERR_PAGE_NOT_FULL = -5,       /* reserved: explicit demotion of a partial page */
  MKV_ERR_WORKSPACE_TOO_SMALL = -6, /* decode workspace below mkv_decode_workspace_bytes */
  MKV_ERR_CUDA = -7,                /* a CUDA runtime call or launch failed */
  MKV_ERR_DEVICE_CHECK = -8,        /* a kernel found an invalid table entry or input */
  MKV_ERR_DEVICE_TIMEOUT = -9,      /* a kernel's bounded wait ran out */
  MKV_ERR_UNSUPPORTED = -10         /* valid but not built (e.g. head_dim, GQA width) */
};

#define MKV_FMT_FP8 0
#define MKV_FMT_TQ3 1
#define MKV_FMT_BF16 2 /* pages of a BF16 control pool */
#define MKV_PAGE_TOKENS 16
#define MKV_ENTRY_UNMAPPED (-1)

/* Pool flags. */
#define MKV_POOL_HOST_ONLY 1 /* track tables on the host only: no device buffers, no launches */
/* A control pool, the comparator the pages measure the method against (sections "Memória e
 * compressão" and "Verificação canário"): every page holds its bf16 values as they are (format
 * MKV_FMT_BF16, in the first slab: per KV head K rows [16][D] then V rows [16][D], bf16, rows
 * not yet written zero; 64*D bytes per head), no page is ever demoted, and decode runs a BF16
 * partial kernel over them.  The TQ3 slab is unused (tq3_slots may be 0). */
#define MKV_POOL_BF16_CONTROL 2

typedef struct mkv_pool* mkv_pool_t;

typedef struct {
  int32_t num_kv_heads;      /* Hkv >= 1 */
  int32_t head_dim;          /* D: 64, 128 or 256 */
  int32_t page_size;         /* must be 16 */
  int32_t max_seqs;          /* rows of the block table */
  int32_t max_pages_per_seq; /* columns of the block table; 16 x it must fit int32 (token
                                counts), and max_seqs x it must too (table entries) */
  int32_t fp8_slots;         /* slots in the FP8 slab */
  int32_t tq3_slots;         /* slots in the TQ3 slab */
  int32_t sink_pages;        /* leading pages of every sequence that stay FP8 (page 0: 1) */
  int32_t flags;             /* MKV_POOL_* */
} mkv_pool_config;

/* Device bytes the caller must provide for a pool with this configuration:
 * FP8 slab, TQ3 slab, block table (int32 [max_seqs][max_pages_per_seq]) and the device
 * status word (256 bytes).  Any output pointer may be NULL.  Pure host computation. */
MKV_API int mkv_pool_required_bytes(const mkv_pool_config* cfg, size_t* fp8_slab_bytes,
                                    size_t* tq3_slab_bytes, size_t* table_bytes,
                                    size_t* status_bytes);

/* Create a pool over caller-owned device buffers (sizes from mkv_pool_required_bytes; each
 * 256-byte aligned).  The table is set to "unmapped" and the status word cleared on the
 * legacy default stream, which is synchronised before return.  With MKV_POOL_HOST_ONLY all
 * four pointers must be NULL and only host state is kept.  *out receives the handle. */
MKV_API int mkv_pool_create(const mkv_pool_config* cfg, void* fp8_slab, void* tq3_slab,
                            int32_t* d_tables, int32_t* d_status, mkv_pool_t* out);

/* Free the pool's host state.  Device buffers remain the caller's.  NULL is ignored. */
MKV_API void mkv_pool_destroy(mkv_pool_t pool);

/* Set the order in which free slots of a format are handed out: order[i] is the slot given
 * i-th when all are free; in general the free slot earliest in the order goes first.
 * order is a host array holding a permutation of [0, n_slots).  Host only. */
MKV_API int mkv_pool_set_slot_order(mkv_pool_t pool, int32_t fmt, const int32_t* order,
                                    int32_t n);

/* Append n_new[i] tokens to sequence seq_ids[i] (host arrays of n_seqs entries, sequences
 * distinct).  k_bf16 and v_bf16 are device arrays bf16 [sum(n_new)][Hkv][D], rows grouped by
 * sequence in seq_ids order.  New pages are FP8, taken lowest-order-first in seq_ids order,
 * pages ascending; tokens are quantised into their pages as described above (the "FP8 page
 * write").  Errors: BAD_SEQ, INVALID_ARG, OUT_OF_PAGES (nothing changed), CUDA. */
MKV_API int mkv_append_kv(mkv_pool_t pool, const int32_t* seq_ids, const int32_t* n_new,
                          int32_t n_seqs, const void* k_bf16, const void* v_bf16, void* stream);

/* Mark (flag != 0) or unmark a logical page of a sequence as protected: a protected page is
 * an anchor and is never demoted.  Marking a page that is already TQ3 changes nothing
 * about its format.  Host only.  Errors: BAD_SEQ, INVALID_ARG (page not mapped). */
MKV_API int mkv_set_protected(mkv_pool_t pool, int32_t seq, int32_t logical_page,
                              int32_t flag);

/* The anchor policy step.  For each listed sequence (length L) demote every full FP8 page p
 * that is not an anchor -- p >= sink_pages, 16p + 16 <= L - window_tokens, not protected --
 * to TQ3 (section "Âncoras em FP8, arquivo em TQ3").  TQ3 slots are taken lowest-order-first
 * in (seq_ids order, page ascending); the FP8 slots are freed at the end of the call (reusable
 * by later calls in stream order).  *n_demoted (host, may be NULL) receives the page count.
 * Errors: BAD_SEQ, INVALID_ARG, OUT_OF_PAGES (nothing changed), CUDA. */
MKV_API int mkv_demote_pages(mkv_pool_t pool, const int32_t* seq_ids, int32_t n_seqs,
                             int32_t window_tokens, int32_t* n_demoted, void* stream);

/* Workspace bytes mkv_decode_attention needs for this call (host computation). */
MKV_API int mkv_decode_workspace_bytes(mkv_pool_t pool, const int32_t* seq_ids,
                                       int32_t n_seqs, int32_t q_len, int32_t num_q_heads,
                                       size_t* bytes);

/* The work units mkv_decode_attention would cut for this call (host computation; also on
 * host-only pools), for inspection and tests.  A unit is the pages of one format (0 FP8, 1 TQ3,
 * 2 BF16) inside a logical page range of one sequence, and yields one partial state per query
 * column and KV head.  A call is split into launches of whole sequences (at most 256, and
 * fewer when their pages need more than 1536 units of 512 pages), each sized for one wave.
 * Within a launch each (sequence, format) group is cut into equal units, one CTA (of each KV
 * head) per unit; where that leaves the wave badly balanced, a grid's pages -- all sequences'
 * pages of its format, or of both for the fused grid, in call order -- are instead cut into
 * CTAs of equal cost, and a CTA takes the units of its share one after another, so it may
 * span sequences.  units_out (host int32 [cap][6]) receives, CTA by CTA: {call position of
 * the sequence, format, first logical page, end logical page (exclusive), pages of that format
 * in the range, CTA number (counted on across launches)}; with units_out NULL the call only
 * counts.  *n_units receives the unit count, also when it exceeds cap (then INVALID_ARG and
 * nothing is written); *ctas_per_wave (may be NULL) the CTA budget of one wave the cut aims at
 * (SMs x resident partial CTAs per SM; 148 x 1 where no device is visible).  Errors: as
 * mkv_decode_workspace_bytes, INVALID_ARG. */
MKV_API int mkv_decode_plan(mkv_pool_t pool, const int32_t* seq_ids, int32_t n_seqs,
                            int32_t q_len, int32_t num_q_heads, int32_t* units_out, int32_t cap,
                            int32_t* n_units, int32_t* ctas_per_wave);

/* Decode attention directly over the mixed-format cache (section "Como os resultados
 * parciais são combinados"): for sequence seq_ids[i] of length L, query j < q_len (the new
 * tokens are the last q_len positions), query head hq (KV head hq / (num_q_heads/Hkv)):
 *     out[i][j][hq][:] = sum_t softmax_t(sm_scale * q . K_t) V_t   over t <= L - q_len + j
 * with K, V the dequantised cache.  Per launch of whole sequences (see mkv_decode_plan), the
 * partial grids and a merge: every sequence is cut into units of one page format and a logical page range; each
 * format has its own partial-attention code producing (running max, denominator, unnormalised
 * accumulator) per query column of a unit; the merge kernel combines all partial states of a
 * (sequence, KV head, column) with global normalisation.  No dense copy of the cache is made;
 * the workspace holds only partial states.
 *   q_bf16    device bf16 [n_seqs][q_len][num_q_heads][D]
 *   out       device fp32 [n_seqs][q_len][num_q_heads][D]
 *   workspace device scratch of ws_bytes >= mkv_decode_workspace_bytes(...), 256-B aligned
 * Constraints: num_q_heads % Hkv == 0, q_len * (num_q_heads / Hkv) <= 32 (else UNSUPPORTED),
 * n_seqs <= max_seqs (rows may repeat), at most 1536 x 512 pages of one format per sequence
 * (else UNSUPPORTED: a launch holds 1536 work units of at most 512 pages; the call is split
 * into as many launches as its sequences need).
 * Errors: BAD_SEQ, EMPTY_CONTEXT, INVALID_ARG, UNSUPPORTED, WORKSPACE_TOO_SMALL, CUDA. */
MKV_API int mkv_decode_attention(mkv_pool_t pool, const int32_t* seq_ids, int32_t n_seqs,
                                 int32_t q_len, const void* q_bf16, int32_t num_q_heads,
                                 float sm_scale, float* out, void* workspace, size_t ws_bytes,
                                 void* stream);

/* Decode attention like mkv_decode_attention, for callers that cannot allocate device memory
 * (e.g. code running under stream capture where allocation is not allowed, or a host runtime
 * that owns the whole device-memory budget and hands out no scratch).  The partial states go
 * to a static device array inside this library instead of a caller workspace; nothing here has
 * a counterpart in the method's description.  The caller still passes q (device bf16
 * [n_seqs][q_len][num_q_heads][D]) and out (device fp32, same shape).
 *   - Limit: the static array holds 32 MiB; a call whose partial states need more returns
 *     MKV_ERR_WORKSPACE_TOO_SMALL.  At most 256 sequences and 1536 work units per call
 *     (MKV_ERR_UNSUPPORTED beyond).  Other errors as mkv_decode_attention.
 *   - The array is allocated when the library's device code is loaded and is held by every
 *     GPU that loads it until the process exits.
 *   - The first call on a device resolves the array's device address (cudaGetSymbolAddress
 *     with that device current) and keeps it for the life of the process; make that first call
 *     before any stream capture.  After cudaDeviceReset on that device the kept address is
 *     stale: do not call this entry point on that device again in the same process.
 *   - The call plans its launch in about 40 KB on the calling thread's stack: call it from
 *     threads with at least 64 KB of stack to spare.
 *   - All calls share the array and it keeps the last call's contents; nothing in it needs to
 *     start at zero.  Calls that overlap on the GPU (other streams, other pools on the same
 *     device) race on it: order them.
 *   - Allocates no device memory and, when it succeeds, no host memory.
 * Results are identical to mkv_decode_attention's for the same inputs. */
MKV_API int mkv_decode_attention_noalloc(mkv_pool_t pool, const int32_t* seq_ids, int32_t n_seqs,
                                         int32_t q_len, const void* q_bf16, int32_t num_q_heads,
                                         float sm_scale, float* out, void* stream);

/* Which partial-attention kernels decode uses (both compute the same partial states; results
 * agree within the attention tolerance, the work cut differing):
 *   MKV_DECODE_SPLIT -- a separate kernel per page format, as the pages describe (section "Como
 *     os resultados parciais são combinados"): the FP8 grid, then the TQ3 grid launched as its
 *     programmatic dependent, so both share one wave;
 *   MKV_DECODE_FUSED -- one grid whose CTAs branch on their unit's format;
 *   MKV_DECODE_AUTO (default) -- per call: FUSED when the fused grid keeps as many CTAs per SM
 *     as the TQ3 grid (head_dim 64 and 128) or when FP8 pages carry more than 15% of the call's
 *     planned time; else SPLIT (for head_dim 256, FP8 CTAs need more shared memory than TQ3
 *     CTAs, so many of them no longer fit one wave of per-format grids).
 * Host only; applies to later decode calls on this pool.  Errors: INVALID_ARG. */
#define MKV_DECODE_SPLIT 0
#define MKV_DECODE_FUSED 1
#define MKV_DECODE_AUTO 2
MKV_API int mkv_set_decode_kernels(mkv_pool_t pool, int32_t mode);

/* Plan later decode calls on this pool for at most `sms` SMs (0, the default: all of the
 * device's): the work cut then fills one wave of that many SMs, leaving room for work the
 * caller runs beside decode on other streams.  It sizes the grid only: the hardware may still
 * place CTAs on any SM.  Host only.  Errors: INVALID_ARG (sms < 0). */
MKV_API int mkv_set_decode_sms(mkv_pool_t pool, int32_t sms);

/* Free every page of a sequence and clear its table row and flags. */
MKV_API int mkv_seq_reset(mkv_pool_t pool, int32_t seq, void* stream);

/* Give the empty sequence dst its own copy of every page of src (formats, flags and length
 * kept; slots taken lowest-order-first, pages ascending).  Errors: BAD_SEQ, INVALID_ARG,
 * OUT_OF_PAGES (nothing changed), CUDA. */
MKV_API int mkv_seq_copy(mkv_pool_t pool, int32_t src, int32_t dst, void* stream);

/* Host copy of a sequence's block table: up to cap entries into host_out (may be NULL when
 * cap == 0); *n_pages and *ctx_len (may be NULL) receive the page count and length. */
MKV_API int mkv_get_block_table(mkv_pool_t pool, int32_t seq, int32_t* host_out, int32_t cap,
                                int32_t* n_pages, int32_t* ctx_len);

/* Bytes of one slot of a format (FP8: Hkv*(32D+16), TQ3: Hkv*14D). */
MKV_API int mkv_slot_bytes(mkv_pool_t pool, int32_t fmt, size_t* bytes);

/* Copy the raw bytes of the slot a table entry names into host_out (cap >= slot bytes);
 * stream-ordered and synchronous (returns after the copy).  For bit-exact inspection. */
MKV_API int mkv_read_slot(mkv_pool_t pool, int32_t entry, void* host_out, size_t cap,
                          void* stream);

/* Self-test of failure detection (no counterpart in the pages): launch one kernel that waits on
 * a device barrier nothing completes, with the library's bounded wait cut to limit_ns
 * (0 .. 2e9).  The wait gives up and records a timeout in the status word, so the next
 * mkv_get_device_status returns MKV_ERR_DEVICE_TIMEOUT; the context stays usable.  Errors:
 * INVALID_ARG (host-only pool, limit out of range), CUDA. */
MKV_API int mkv_selftest_wait(mkv_pool_t pool, int64_t limit_ns, void* stream);

/* Self-test of the Blackwell tensor-memory MMA path that a tcgen05 logits kernel would use
 * (no counterpart in the pages; decode does not use it yet): one CTA computes
 * d_out[128][8] (fp32) = a[128][256] . q[8][256]^T (f16, row-major device buffers).  Each
 * thread writes one row of a into tensor memory, q is read by the tensor core from shared
 * memory, one thread issues tcgen05.mma and the result is read back from tensor memory.  A
 * bounded wait records MKV_ERR_DEVICE_TIMEOUT in the status word.  Errors: INVALID_ARG, CUDA. */
MKV_API int mkv_selftest_tc_logits(mkv_pool_t pool, const void* a_f16, const void* q_f16,
                                   float* d_out, void* stream);

/* Prefill-time compression: write the first n_tokens[i] tokens of each listed sequence, which
 * must be empty (k, v as for mkv_append_kv).  Every full page that the anchor policy would
 * demote at once -- page p >= sink_pages with 16p + 16 <= n - anchor_window_tokens (new pages
 * are not protected) -- is packed to TQ3 straight from the bf16 values, with the same
 * per-group scale and thresholds as demotion (sections "Âncoras em FP8, arquivo em TQ3" /
 * "Des ancres en FP8, une archive en TQ3" describe TQ3 as the archive format of older pages);
 * every other page is written as a fresh FP8 page, as by mkv_append_kv.  Pages take slots of
 * their own format, ascending, sequences in list order.  Values differ from append-then-demote
 * only through the FP8 rounding that the direct path skips.  Errors: BAD_SEQ, INVALID_ARG
 * (non-empty or repeated sequence, negative count or window, NULL k/v), OUT_OF_PAGES (nothing
 * changed), CUDA. */
MKV_API int mkv_prefill_kv(mkv_pool_t pool, const int32_t* seq_ids, const int32_t* n_tokens,
                           int32_t n_seqs, const void* k_bf16, const void* v_bf16,
                           int32_t anchor_window_tokens, void* stream);

/* Materialising profile (pt page, section "Qualidade em contexto longo": the profile in which
 * the hybrid pages really are expanded into tensors).  A debugging and quality-control path,
 * never part of decode: writes the sequence's dequantised K and V as dense fp32
 * [ctx][Hkv][D] rows into the caller's device buffers k_out and v_out (each at least
 * ctx * Hkv * D floats; max_tokens states their capacity in tokens).  FP8 values are
 * fp32(dec(code) * page scale) (the fp32 product, rounded to nearest even); TQ3 values are
 * (q - 3.5) * s (exact).  Asynchronous on the stream.  Errors: BAD_SEQ, INVALID_ARG (NULL
 * output, capacity below the context), CUDA; a bad table entry is a device check. */
MKV_API int mkv_materialise_kv(mkv_pool_t pool, int32_t seq, float* k_out, float* v_out,
                               int64_t max_tokens, void* stream);

/* Footprint (section "Memória e compressão"): live tokens, pages per format and KV slab bytes
 * held by live pages per live token. */
MKV_API int mkv_pool_stats(mkv_pool_t pool, int64_t* live_tokens, int32_t* fp8_pages,
                           int32_t* tq3_pages, double* kv_bytes_per_token);

/* Synchronise the stream, read and clear the device status word: MKV_OK,
 * MKV_ERR_DEVICE_CHECK or MKV_ERR_DEVICE_TIMEOUT. */
MKV_API int mkv_get_device_status(mkv_pool_t pool, void* stream);

/* Kernel timing for measurement: while enabled, every decode call records CUDA events on its
 * stream before its partial-attention kernel, between it and the merge kernel, and after the
 * merge.  mkv_timing_read synchronises on the recorded events and returns the summed
 * milliseconds of each kernel and the number of decode calls timed; it then clears the record.
 * (Calls split into several launch groups record the span of all of them as partial time.) */
MKV_API int mkv_timing_enable(mkv_pool_t pool, int32_t enable);
MKV_API int mkv_timing_read(mkv_pool_t pool, double* ms_partial, double* ms_merge,
                            int64_t* calls);

/* Test hook for the error paths (no counterpart in the pages): after `after` more device
 * operations of the state-changing calls (append, prefill, demotion, copy, reset: each kernel
 * launch or memset they issue; on a host-only pool each one they would issue) succeed, the next
 * one reports MKV_ERR_CUDA without being issued, and the hook switches itself off.  -1 switches
 * it off.  Lets a test make a launch fail on the host, with no device fault, and check that the
 * failed call left the pool's host state unchanged.  Errors: INVALID_ARG. */
MKV_API int mkv_test_fail_launch(mkv_pool_t pool, int32_t after);

/* Number of kernels this pool has launched since creation. */
MKV_API int mkv_launch_count(mkv_pool_t pool, int64_t* launches);

/* Thread-local description of the last error ("" if none). */
MKV_API const char* mkv_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MKV_H_ */
