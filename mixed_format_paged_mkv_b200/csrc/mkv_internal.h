// Host <-> kernel parameter blocks of the mixed-format paged KV cache (not part of the ABI).
//
// Every kernel takes one parameter block by value (__grid_constant__), so a launch carries its
// own descriptors: no staging buffer, no host->device copy before the kernel can start.  The
// blocks stay below the 32 KiB kernel-parameter limit; larger requests are split into several
// launches by the host code.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace mkv {

constexpr int kPageTokens = 16;
constexpr int kFmtShift = 30;
constexpr uint32_t kSlotMask = (1u << kFmtShift) - 1u;

// Bits of the device status word.
constexpr int32_t kStatusCheck = 1;    // invalid table entry, slot or non-finite input
constexpr int32_t kStatusTimeout = 2;  // a bounded wait ran out

// Bytes of one KV head inside a slot.
inline int64_t fp8_head_bytes(int D) { return 32LL * D + 16; }
inline int64_t tq3_head_bytes(int D) { return 14LL * D; }
inline int64_t bf16_head_bytes(int D) { return 64LL * D; }

// ------------------------------------------------------------------ append (FP8 page write)
struct AppendDesc {
  int32_t slot;         // FP8 slot of the page
  int32_t table_index;  // row * max_pages + logical page (written when the page is new)
  int32_t first_row;    // input row of the first token written into this page
  int16_t n_old;        // tokens already in the page
  int16_t n_new;        // tokens written by this call
};
constexpr int kAppendMaxDesc = 1536;
struct AppendParams {
  uint8_t* fp8_slab;
  int32_t* tables;
  int32_t* status;
  const uint16_t* k;  // bf16 bits [rows][Hkv][D]
  const uint16_t* v;
  int64_t slot_bytes;
  int32_t Hkv, D;
  int32_t bf16;       // 1: a control pool's BF16 pages (values stored as they are)
  int32_t n_desc;
  AppendDesc desc[kAppendMaxDesc];
};

// ------------------------------------------------------------------ demote (FP8 -> TQ3)
struct DemoteDesc {
  int32_t src_slot;     // FP8 slot
  int32_t dst_slot;     // TQ3 slot
  int32_t table_index;  // entry retagged to TQ3
};
constexpr int kDemoteMaxDesc = 2560;
struct DemoteParams {
  const uint8_t* fp8_slab;
  uint8_t* tq3_slab;
  int32_t* tables;
  int64_t fp8_slot_bytes, tq3_slot_bytes;
  int32_t Hkv, D;
  int32_t publish;  // 1: also set each page's table entry to TQ3 (else a retag launch does)
  int32_t n_desc;
  DemoteDesc desc[kDemoteMaxDesc];
};

// ------------------------------------------------------------------ table retag
// tables[index[k]] = entry[k]: publishes the entries of a demotion split over several launches
// once every page is written.
constexpr int kRetagMax = 3800;
struct RetagParams {
  int32_t* tables;
  int32_t n;
  int32_t index[kRetagMax];
  int32_t entry[kRetagMax];
};

// ------------------------------------------------------------------ prefill (bf16 -> TQ3)
struct PackDesc {
  int32_t dst_slot;     // TQ3 slot
  int32_t table_index;  // entry set to TQ3
  int32_t first_row;    // input row of the page's first token
};
constexpr int kPackMaxDesc = 2560;
struct PackParams {
  const uint16_t* k;  // bf16 bits [rows][Hkv][D]
  const uint16_t* v;
  uint8_t* tq3_slab;
  int32_t* tables;
  int64_t tq3_slot_bytes;
  int32_t Hkv, D;
  int32_t vec16;  // 1: k and v are 16-byte aligned (vector loads), 0: element loads
  int32_t n_desc;
  PackDesc desc[kPackMaxDesc];
};

// ------------------------------------------------------------------ slot copy
struct CopyDesc {
  int32_t src_slot, dst_slot, fmt, table_index;
};
constexpr int kCopyMaxDesc = 1920;
struct CopyParams {
  uint8_t* fp8_slab;
  uint8_t* tq3_slab;
  int32_t* tables;
  int64_t fp8_slot_bytes, tq3_slot_bytes;
  int32_t n_desc;
  CopyDesc desc[kCopyMaxDesc];
};

// ------------------------------------------------------------------ materialise (debug / QC)
// Dense fp32 copy of one sequence's dequantised K and V; never used by decode.
struct MaterialiseParams {
  const uint8_t* fp8_slab;
  const uint8_t* tq3_slab;
  const int32_t* table;  // the sequence's block-table row
  int32_t* status;
  float* k_out;  // [ctx][Hkv][D]
  float* v_out;
  int64_t fp8_slot_bytes, tq3_slot_bytes;
  int32_t Hkv, D, ctx, fp8_slots, tq3_slots;
  int32_t page_fmt;  // format of the first slab's pages: 0 FP8, 2 BF16 (control pool)
};

// ------------------------------------------------------------------ decode
// Decode = partial kernel + merge kernel.  Work unit = (sequence, format, logical page range).
// A partial CTA takes a run of consecutive units for one KV head: for each it scans the
// block-table entries of the range, streams the pages of its format through a shared-memory
// ring and writes one partial state per query column.  The units of a CTA are cut from a line
// of all sequences' pages of its grid, so a CTA may finish one sequence and start the next.
// The merge kernel combines every partial state of a (sequence, KV head, column).
struct SeqDesc {
  int32_t row;      // table row (sequence id)
  int32_t ctx;      // context length L (includes the q_len new tokens)
  int32_t out_row;  // position of the sequence in the call (rows of q and out)
  int32_t part0;    // first partial-state index of this sequence
  int32_t n_parts;  // units of this sequence (partial states per KV head)
  int32_t pad;
};
struct UnitDesc {
  int32_t first;  // logical pages [first, last)
  int32_t last;
  uint8_t seq;    // index into DecodeParams::seq
  uint8_t fmt;    // 0 FP8, 1 TQ3, 2 BF16
  uint16_t part;  // index of this unit's partial state within its sequence
};
constexpr int kDecodeMaxSeqs = 256;
constexpr int kDecodeMaxUnits = 1536;
constexpr int kMaxPagesPerUnit = 512;  // pages of the unit's format inside its range
static_assert(kDecodeMaxSeqs <= 256 && kDecodeMaxUnits <= 65535, "UnitDesc field widths");
struct DecodeParams {
  const uint8_t* fp8_slab;
  const uint8_t* tq3_slab;
  const int32_t* tables;
  int32_t* status;    // status word
  const uint16_t* q;  // bf16 bits [n][q_len][Hq][D]
  float* out;         // fp32 [n][q_len][Hq][D]
  float* part_ml;     // [part][Hkv][NC][2]: running max (log2 units), denominator
  float* part_acc;    // [part][Hkv][NC][D]: unnormalised accumulator
  int64_t fp8_slot_bytes, tq3_slot_bytes;
  int32_t Hkv, D, g, q_len, NC, Hq;
  int32_t max_pages, fp8_slots, tq3_slots;
  float logit_scale;  // sm_scale * log2(e)
  int32_t n_seqs;     // sequences in this launch
  int32_t n_units;    // units in this launch, CTA by CTA
  int32_t n_ctas;     // CTAs per KV head: FP8 CTAs [0, n_fp8), then TQ3 CTAs (per-format
  int32_t n_fp8;      // grids); the fused and BF16 grids take all n_ctas x Hkv CTAs
  int32_t fused;      // 1: one grid branching per unit; 0: an FP8 grid, then a TQ3 grid
  int32_t page_fmt;   // format of written pages: 0 FP8 (mixed pools), 2 BF16 (control pools)
  SeqDesc seq[kDecodeMaxSeqs];
  UnitDesc unit[kDecodeMaxUnits];
  uint16_t cta_unit0[kDecodeMaxUnits + 1];  // CTA c takes units [cta_unit0[c], cta_unit0[c+1])
};

// Every parameter block fits the 32,764-byte kernel-parameter limit.
static_assert(sizeof(AppendParams) <= 32764 && sizeof(DemoteParams) <= 32764 &&
                  sizeof(RetagParams) <= 32764 && sizeof(PackParams) <= 32764 &&
                  sizeof(CopyParams) <= 32764 && sizeof(DecodeParams) <= 32764,
              "kernel parameter block too large");

cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_demote(const DemoteParams& p, cudaStream_t s);
cudaError_t launch_retag(const RetagParams& p, cudaStream_t s);
cudaError_t launch_copy(const CopyParams& p, cudaStream_t s);
cudaError_t launch_materialise(const MaterialiseParams& p, cudaStream_t s);
cudaError_t launch_pack(const PackParams& p, cudaStream_t s);
cudaError_t launch_partial(const DecodeParams& p, cudaStream_t s);
cudaError_t launch_merge(const DecodeParams& p, cudaStream_t s);
bool partial_supported(int D, int NC);
// CTAs of the partial kernel for (D, NC) that one SM keeps resident (queried once): the TQ3
// kernel's (per-format grids), the fused kernel's or the BF16 control kernel's.
constexpr int kDecodeSplit = 0, kDecodeFused = 1, kDecodeBf16 = 2;
int partial_ctas_per_sm(int D, int NC, int mode);
cudaError_t static_decode_scratch(void** ptr, size_t* bytes);

}  // namespace mkv
