// Partial-attention kernels: templates shared by the per-head-dim translation units
// (decode_d64.cu, decode_d128.cu, decode_d256.cu), each of which instantiates the kernels
// of one head dimension, so that they compile in parallel.  The design is described at the
// top of decode.cu.
#pragma once
#include <cfloat>

#include "device_util.cuh"
#include "mkv_internal.h"

namespace mkv {

namespace {

constexpr float kLazyRescale = 8.f;  // log2 units

// Partial-kernel kinds: one format per grid, both mixed formats (branching per CTA), or the
// BF16 control pages.
enum Kind { kKindFp8 = 0, kKindTq3 = 1, kKindFused = 2, kKindBf16 = 3 };
// Page formats (block-table tags).
enum Fmt { kFp8 = 0, kTq3 = 1, kBf16 = 2 };

template <int D, int NT, int K>
struct Cfg {
  // Team layout (more than 8 query columns, FP8/TQ3 pages): TW warps; each decodes the K of
  // one page of a batch of TW pages for all NT n-tiles and shares its probabilities through
  // shared memory, then every warp multiplies the whole batch by the V of its own GW channel
  // groups.  Otherwise (one n-tile, or the BF16 control) warp nt of group pw takes n-tile nt of
  // the group's pages.
  static constexpr bool TEAM = NT > 1 && K != kKindBf16;
  static constexpr int TW = D == 64 ? 2 : 4;
  static constexpr int PW = TEAM ? 1 : (NT == 1 ? 4 : (NT == 2 ? 2 : 1));  // page-parallel groups
  static constexpr int WARPS = TEAM ? TW : NT * PW;  // warp nt of group pw: nt + NT*pw
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int FP8_STAGE = 32 * D + 16;
  static constexpr int TQ3_STAGE = 14 * D;
  // BF16 control page: its 32 rows (16 K, 16 V) copied one by one into rows padded by 16
  // bytes, so the 8 rows an ldmatrix reads fall on distinct banks
  static constexpr int BF16_ROW = 2 * D + 16;
  static constexpr int BF16_STAGE = 32 * BF16_ROW;
  // Stage s only ever holds pages i with i % NST == s, and they belong to warp group i % PW:
  // with NST a multiple of PW each stage has a fixed owner, which refills it when done.
  static constexpr int FP8_NST = 8;
  static constexpr int TQ3_NST = TEAM ? 2 * TW : 8;
  static constexpr int BF16_NST = 8;
  static_assert(FP8_NST % PW == 0 && TQ3_NST % PW == 0 && BF16_NST % PW == 0, "stage ownership");
  static_assert(FP8_NST <= 8 && TQ3_NST <= 8 && BF16_NST <= 8, "stage barriers (kRingBarriers)");
  static constexpr int RING_FP8 = (K == kKindFp8 || K == kKindFused) ? FP8_NST * FP8_STAGE : 0;
  static constexpr int RING_TQ3 = (K == kKindTq3 || K == kKindFused) ? TQ3_NST * TQ3_STAGE
                                  : (K == kKindBf16 ? BF16_NST * BF16_STAGE : 0);
  // end-of-unit combine: (m, l) and acc of every warp (team: of every n-tile, then the warps'
  // denominators)
  static constexpr int COMBINE = TEAM ? NT * 8 * (D + 2) * 4 + TW * NT * 8 * 4
                                      : PW * NT * 8 * (D + 2) * 4;
  // team exchange, two batches: P fragments [batch][page][n-tile][lane] (uint2), then the
  // page references and sums [batch][page][n-tile][column] (float2)
  static constexpr int XCH_P = TEAM ? 2 * TW * NT * 32 * 8 : 0;
  static constexpr int XCH = TEAM ? XCH_P + 2 * TW * NT * 8 * 4 : 0;

  static constexpr int RING = RING_FP8 > RING_TQ3 ? (RING_FP8 > COMBINE ? RING_FP8 : COMBINE)
                                                  : (RING_TQ3 > COMBINE ? RING_TQ3 : COMBINE);
  // header: full[16] mbarriers | release counters | fills issued | misc | page list |
  //         Q fragments | TQ3 K corrections | ring
  static constexpr int OFF_CNT = 128;
  static constexpr int OFF_FILLS = OFF_CNT + 64;
  static constexpr int OFF_MISC = OFF_FILLS + 64;
  static constexpr int OFF_LIST = OFF_MISC + 64;
  static constexpr int OFF_QF = (OFF_LIST + kMaxPagesPerUnit * 8 + 127) / 128 * 128;
  static constexpr int QF = NT * D * 16;
  static constexpr int OFF_CORR = OFF_QF + QF;
  static constexpr int OFF_XCH = (OFF_CORR + NT * (D / 32) * 32 + 127) / 128 * 128;
  static constexpr int OFF_RING = (OFF_XCH + XCH + 127) / 128 * 128;
  static constexpr int SMEM = OFF_RING + RING;
  // CTAs per SM the launch bounds aim at (registers: 65536 / (THREADS * that))
  // (an FP8 CTA fits beside three TQ3 CTAs: both kernels at 4 for D 256)
  static constexpr int MINB = TEAM ? (D == 64 ? 8 : (D == 256 ? 3 : 4))
                             : K == kKindBf16 ? 1 : D == 256 ? (K == kKindFused ? 3 : 4)
                                                             : (D == 128 ? 5 : 6);
  // table entries per lane in flight while scanning a unit's range: deep for the kernels that
  // take FP8 units (whose ranges can be long and sparse) where the launch bounds leave more
  // than 128 registers, or 128 to a one-tile kernel (the others spill); TQ3 ranges are dense
  static constexpr int REG_BUDGET = 65536 / (THREADS * MINB);
  static constexpr int SCAN =
      K != kKindTq3 && (REG_BUDGET > 128 || (REG_BUDGET == 128 && NT == 1)) ? 32 : 8;
};

// Stage barriers every unit initialises, whatever its format's ring length (at most 8), so
// that a CTA's next unit can invalidate and initialise them again.
constexpr int kRingBarriers = 8;

struct Smem {
  uint64_t* full;   // [stage]: the stage's page landed (arrive + bulk-copy bytes)
  int32_t* cnt;     // [stage]: warps done with the stage's page (several n-tiles per page);
                    // team layout: then [2][TW] flags of pages that raised a reference
  int32_t* fills;   // [stage]: copies issued into the stage
  int32_t* misc;    // [0] page count, [1] abort flag, [4..7] logit scales per n-tile
  int2* list;       // {slot, logical page} of the unit's pages
  uint4* qf;        // Q fragments [NT][D/32][32 lanes]
  float2* corr;     // TQ3 K corrections [NT][D/32][4 column pairs]
  uint8_t* xch;     // team exchange (P fragments, page references and sums)
  uint8_t* ring;
};

template <int D, int NT, int K>
__device__ __forceinline__ Smem carve(uint8_t* base) {
  using C = Cfg<D, NT, K>;
  Smem s;
  s.full = reinterpret_cast<uint64_t*>(base);
  s.cnt = reinterpret_cast<int32_t*>(base + C::OFF_CNT);
  s.fills = reinterpret_cast<int32_t*>(base + C::OFF_FILLS);
  s.misc = reinterpret_cast<int32_t*>(base + C::OFF_MISC);
  s.list = reinterpret_cast<int2*>(base + C::OFF_LIST);
  s.qf = reinterpret_cast<uint4*>(base + C::OFF_QF);
  s.corr = reinterpret_cast<float2*>(base + C::OFF_CORR);
  s.xch = base + C::OFF_XCH;
  s.ring = base + C::OFF_RING;
  return s;
}

__device__ __forceinline__ uint32_t f16x2_const(float lo, float hi) { return pack_f16x2(lo, hi); }

// K-warp softmax state for the thread's two columns (2c, 2c+1): reference maximum (log2 units)
// and this thread's share of the denominator.
struct KState {
  float m[2];
  float l[2];
};

// V-warp accumulator: acc[mt][0..3] = (channel row r, col 2c), (r, 2c+1), (r+8, 2c),
// (r+8, 2c+1) of channel tile mt; tile 2G+j row r holds channel 32G+4r+2j, row r+8 channel
// 32G+4r+2j+1.
template <int D>
struct VState {
  float acc[D / 16][4];
};

// Logits -> probabilities for one page (thread holds logits x[0..3] for tokens (r, r+8) x
// columns (2c, 2c+1), in log2 units).  Gives the probabilities pr (same positions) and the
// factors (a0, a1) by which earlier accumulations of the two columns must be rescaled (1 when
// the reference maximum did not move).  P^T as B fragments (tokens 0-7, 8-15) is the movmatrix
// transpose of the packed pairs (pr0, pr1) and (pr2, pr3).
__device__ __forceinline__ void softmax_k(KState& st, float (&x)[4], float (&pr)[4], float& a0,
                                          float& a1) {
  float mx0 = fmaxf(x[0], x[2]);
  float mx1 = fmaxf(x[1], x[3]);
  a0 = a1 = 1.f;
  const bool need = (mx0 > st.m[0] + kLazyRescale) || (mx1 > st.m[1] + kLazyRescale);
  if (__any_sync(0xffffffffu, need)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float n0 = fmaxf(st.m[0], mx0), n1 = fmaxf(st.m[1], mx1);
    a0 = (n0 == -INFINITY) ? 1.f : fast_exp2(st.m[0] - n0);
    a1 = (n1 == -INFINITY) ? 1.f : fast_exp2(st.m[1] - n1);
    st.l[0] *= a0;
    st.l[1] *= a1;
    st.m[0] = n0;
    st.m[1] = n1;
  }
  const float r0 = st.m[0] == -INFINITY ? 0.f : st.m[0];
  const float r1 = st.m[1] == -INFINITY ? 0.f : st.m[1];
  pr[0] = fast_exp2(x[0] - r0);
  pr[1] = fast_exp2(x[1] - r1);
  pr[2] = fast_exp2(x[2] - r0);
  pr[3] = fast_exp2(x[3] - r1);
  st.l[0] += pr[0] + pr[2];
  st.l[1] += pr[1] + pr[3];
}

__device__ __forceinline__ void mask_page(float (&x)[4], int tok0, int r, int lim0, int lim1) {
  if (tok0 + r > lim0) x[0] = -INFINITY;
  if (tok0 + r > lim1) x[1] = -INFINITY;
  if (tok0 + r + 8 > lim0) x[2] = -INFINITY;
  if (tok0 + r + 8 > lim1) x[3] = -INFINITY;
}

// ------------------------------------------------------------------ TQ3 page
// K records (group G, token t) at 12*(16G + t); V records after K records + K scales.
// Channel order inside the MMAs (free: the K reduction is order independent, V channels are
// un-permuted when stored): TQ3 K, group G, lane quad column c: MMA k 2c,2c+1 <- channels
// 8c+0, 8c+4 (k-block 0), 8c+1, 8c+5 (k-block 0, upper k), 8c+2, 8c+6 / 8c+3, 8c+7 (k-block 1).
template <int D>
__device__ __forceinline__ void tq3_logits(const uint8_t* pg, const uint4* qf, const float2* corr,
                                           int lane, int kw, int ks, float (&x)[4]) {
  constexpr int G = D / 32;
  const int r = lane >> 2, c = lane & 3;
  const uint8_t* krec = pg;
  const __half* kscale = reinterpret_cast<const __half*>(pg + G * 16 * 12);
  // K images: the window puts code j of the lane's 8-code chunk at bit 7 + 3j, so code k of a
  // pair lands in mantissa bits 7-9 of the low half (value 8 + c) and code k+4 in bits 3-5 of
  // the high half (value 128 + c) after a right shift by 3k; both exact.  The offsets 11.5 and
  // 131.5 (base + 3.5) times the query sums are the group's starting accumulator (corr).
  uint32_t kMask = 0x00380380u, kMagic = 0x58004800u;
  opaque(kMask, kMagic);
  x[0] = x[1] = x[2] = x[3] = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t* ra = reinterpret_cast<const uint32_t*>(krec + 12 * (16 * g + r));
    const uint32_t* rb = ra + 24;  // token r + 8
    const uint32_t xa = __funnelshift_r(ra[kw], ra[kw + 1], ks);  // code j at bit 3j+7
    const uint32_t xb = __funnelshift_r(rb[kw], rb[kw + 1], ks);
    const uint32_t a0 = and_or(xa, kMask, kMagic), b0 = and_or(xb, kMask, kMagic);
    const uint32_t a1 = and_or(xa >> 3, kMask, kMagic), b1 = and_or(xb >> 3, kMask, kMagic);
    const uint32_t a2 = and_or(xa >> 6, kMask, kMagic), b2 = and_or(xb >> 6, kMask, kMagic);
    const uint32_t a3 = and_or(xa >> 9, kMask, kMagic), b3 = and_or(xb >> 9, kMask, kMagic);
    const uint4 qb = qf[32 * g + lane];
    const float2 cr = corr[4 * g + c];
    float cg[4];
    mma_f16_16816(cg, a0, b0, a1, b1, qb.x, qb.y, {cr.x, cr.y, cr.x, cr.y});
    mma_f16_16816(cg, a2, b2, a3, b3, qb.z, qb.w, cg);
    const float sa = __half2float(kscale[16 * g + r]);
    const float sb = __half2float(kscale[16 * g + r + 8]);
    x[0] = fmaf(sa, cg[0], x[0]);
    x[1] = fmaf(sa, cg[1], x[1]);
    x[2] = fmaf(sb, cg[2], x[2]);
    x[3] = fmaf(sb, cg[3], x[3]);
  }
}

// Largest V scale of a TQ3 page (f16 bits; scales are never negative), the same on every lane:
// each lane folds G bytes of the page's [G][16] f16 V scales, then one warp reduction.
template <int D>
__device__ __forceinline__ uint32_t tq3_v_scale_max(const uint8_t* pg, int lane) {
  constexpr int G = D / 32;
  const uint8_t* vs = pg + G * 16 * 14 + G * 16 * 12;
  uint32_t w;
  if constexpr (G == 8) {
    const uint2 x = reinterpret_cast<const uint2*>(vs)[lane];
    w = hmax2_u32(x.x, x.y);
  } else if constexpr (G == 4) {
    w = reinterpret_cast<const uint32_t*>(vs)[lane];
  } else {
    w = reinterpret_cast<const uint16_t*>(vs)[lane];
  }
  return __reduce_max_sync(0xffffffffu, max(w & 0xffffu, w >> 16));
}

// A page's V scales all lie at or below 2^7 and the largest at or above 2^-6 (f16 bits): then
// P * s, with P <= 2^8 under the lazy softmax reference, is at most 2^15 and, for the page's
// largest scales, a normal f16 down to P = 2^-8, so the plain f16 product keeps full precision.
constexpr uint32_t kVScaleLo = 0x2400u;  // 2^-6
constexpr uint32_t kVScaleHi = 0x5800u;  // 2^7

// V: A = V^T tile (channels x tokens); lane row r holds channels 32G+4r+{0,1} (tile 2G) and
// 32G+4r+{2,3} (tile 2G+1) for tokens (2c, 2c+1) and (2c+8, 2c+9); codes -> exact (c - 3.5);
// the per-(token, group) scale multiplies P in f16.
//
// WIDE is the path for pages whose scale maximum is outside [2^-6, 2^7]: each group's 16 token
// scales are first divided by a power of two 2^(e-16) taken from the group's largest scale on
// the page (quad reduction; e its biased f16 exponent, at least 1), so the scaled values are
// below 4 and P * s / 2^(e-16) < 2^10 cannot overflow, while the group's largest products stay
// normal f16 down to P = 2^-16; the group's P.V tiles are computed from zero and added to the
// accumulator times 2^(e-16) in fp32, exactly undoing the division.
template <int D, bool WIDE>
__device__ __forceinline__ void tq3_pv(VState<D>& st, const uint8_t* pg, int lane, int vw,
                                       int vs1, uint32_t pb0, uint32_t pb1) {
  constexpr int G = D / 32;
  const int c = lane & 3;
  const uint8_t* vrec = pg + G * 16 * 14;
  const __half* vscale = reinterpret_cast<const __half*>(vrec + G * 16 * 12);
  uint32_t m0 = 0x000E000Eu, g0 = 0x60006000u, m1 = 0x00700070u, g1 = 0x54005400u;
  uint32_t m2 = 0x03800380u, g2 = 0x48004800u;
  opaque(m0, g0, m1, g1, m2, g2);
  const uint32_t s0 = f16x2_const(515.5f, 515.5f), s1 = f16x2_const(67.5f, 67.5f);
  const uint32_t s2 = f16x2_const(11.5f, 11.5f);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t* rc = reinterpret_cast<const uint32_t*>(vrec + 12 * (16 * g + 2 * c));
    const uint32_t f0 = __funnelshift_r(rc[vw], rc[vw + 1], vs1);        // token 2c
    const uint32_t f1 = __funnelshift_r(rc[vw + 3], rc[vw + 4], vs1);    // token 2c+1
    const uint32_t f8 = __funnelshift_r(rc[vw + 24], rc[vw + 25], vs1);  // token 2c+8
    const uint32_t f9 = __funnelshift_r(rc[vw + 27], rc[vw + 28], vs1);  // token 2c+9
    const uint32_t z01 = __byte_perm(f0, f1, 0x5410);
    const uint32_t z89 = __byte_perm(f8, f9, 0x5410);
    const uint32_t a0 = hsub2_u32(and_or(z01, m0, g0), s0), b0 = hsub2_u32(and_or(z89, m0, g0), s0);
    const uint32_t a1 = hsub2_u32(and_or(z01, m1, g1), s1), b1 = hsub2_u32(and_or(z89, m1, g1), s1);
    const uint32_t a2 = hsub2_u32(and_or(z01, m2, g2), s2), b2 = hsub2_u32(and_or(z89, m2, g2), s2);
    const uint32_t a3 = hsub2_u32(and_or(z01 >> 3, m2, g2), s2);
    const uint32_t b3 = hsub2_u32(and_or(z89 >> 3, m2, g2), s2);
    uint32_t sv0 = *reinterpret_cast<const uint32_t*>(vscale + 16 * g + 2 * c);
    uint32_t sv8 = *reinterpret_cast<const uint32_t*>(vscale + 16 * g + 2 * c + 8);
    if constexpr (!WIDE) {
      const uint32_t q0 = hmul2_u32(pb0, sv0), q1 = hmul2_u32(pb1, sv8);
      mma_f16_16816(st.acc[2 * g], a0, a1, b0, b1, q0, q1, st.acc[2 * g]);
      mma_f16_16816(st.acc[2 * g + 1], a2, a3, b2, b3, q0, q1, st.acc[2 * g + 1]);
    } else {
      uint32_t m = hmax2_u32(sv0, sv8);  // tokens 2c, 2c+1, 2c+8, 2c+9; the quad holds all 16
      m = hmax2_u32(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = hmax2_u32(m, __shfl_xor_sync(0xffffffffu, m, 2));
      const int e = max(static_cast<int>(max(m & 0xffffu, m >> 16) >> 10), 1);
      const uint32_t down = static_cast<uint32_t>(31 - e) * 0x04000400u;  // f16x2 2^(16-e)
      const float up = __int_as_float((e + 111) << 23);                   // fp32 2^(e-16)
      sv0 = hmul2_u32(sv0, down);
      sv8 = hmul2_u32(sv8, down);
      const uint32_t q0 = hmul2_u32(pb0, sv0), q1 = hmul2_u32(pb1, sv8);
      float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
      mma_f16_16816(t0, a0, a1, b0, b1, q0, q1, t0);
      mma_f16_16816(t1, a2, a3, b2, b3, q0, q1, t1);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        st.acc[2 * g][j] = fmaf(up, t0[j], st.acc[2 * g][j]);
        st.acc[2 * g + 1][j] = fmaf(up, t1[j], st.acc[2 * g + 1][j]);
      }
    }
  }
}

// ------------------------------------------------------------------ FP8 page
// K rows at t*D, V rows at 16*D + t*D, then sK, sV (fp32).
// K channel order: k-block kb = 4j + i, lane quad column c: k 2c,2c+1 <- channels
// 64j+16c+4i+{0,1}, k 2c+8,2c+9 <- 64j+16c+4i+{2,3}.
template <int D>
__device__ __forceinline__ void fp8_logits(const uint8_t* pg, const uint4* qf, int lane,
                                           float (&x)[4]) {
  const int r = lane >> 2, c = lane & 3;
  const float sk = *reinterpret_cast<const float*>(pg + 32 * D);
  float cg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < D / 64; ++j) {
    const uint4 wa = *reinterpret_cast<const uint4*>(pg + r * D + 64 * j + 16 * c);
    const uint4 wb = *reinterpret_cast<const uint4*>(pg + (r + 8) * D + 64 * j + 16 * c);
    const uint32_t va[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t vb[4] = {wb.x, wb.y, wb.z, wb.w};
    const uint4 q01 = qf[32 * (2 * j) + lane], q23 = qf[32 * (2 * j + 1) + lane];
    const uint32_t qq[8] = {q01.x, q01.y, q01.z, q01.w, q23.x, q23.y, q23.z, q23.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mma_f16_16816(cg, e4m3x2_to_f16x2(va[i]), e4m3x2_to_f16x2(vb[i]),
                    e4m3x2_to_f16x2(va[i] >> 16), e4m3x2_to_f16x2(vb[i] >> 16),
                    qq[2 * i], qq[2 * i + 1], cg);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = cg[j] * sk;
}

// V channel order as for TQ3 (lane row r: channels 32g+4r+{0..3}); the page's V scale
// multiplies the page's P.V result per channel tile.
template <int D>
__device__ __forceinline__ void fp8_pv(VState<D>& st, const uint8_t* pg, int lane, uint32_t pb0,
                                       uint32_t pb1) {
  const int r = lane >> 2, c = lane & 3;
  const float sv = *reinterpret_cast<const float*>(pg + 32 * D + 4);
  const uint8_t* vrows = pg + 16 * D;
#pragma unroll
  for (int g = 0; g < D / 32; ++g) {
    const int off = 32 * g + 4 * r;
    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c) * D + off);
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c + 1) * D + off);
    const uint32_t w8 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c + 8) * D + off);
    const uint32_t w9 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c + 9) * D + off);
    const uint32_t lo01 = __byte_perm(w0, w1, 0x5140), hi01 = __byte_perm(w0, w1, 0x7362);
    const uint32_t lo89 = __byte_perm(w8, w9, 0x5140), hi89 = __byte_perm(w8, w9, 0x7362);
    float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
    mma_f16_16816(t0, e4m3x2_to_f16x2(lo01), e4m3x2_to_f16x2(lo01 >> 16),
                  e4m3x2_to_f16x2(lo89), e4m3x2_to_f16x2(lo89 >> 16), pb0, pb1, t0);
    mma_f16_16816(t1, e4m3x2_to_f16x2(hi01), e4m3x2_to_f16x2(hi01 >> 16),
                  e4m3x2_to_f16x2(hi89), e4m3x2_to_f16x2(hi89 >> 16), pb0, pb1, t1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      st.acc[2 * g][e] = fmaf(sv, t0[e], st.acc[2 * g][e]);
      st.acc[2 * g + 1][e] = fmaf(sv, t1[e], st.acc[2 * g + 1][e]);
    }
  }
}

// ------------------------------------------------------------------ team kernels: NT n-tiles
// The same page arithmetic with the codes of a page decoded once for all NT n-tiles of the KV
// head (more than 8 query columns).  Q fragments and TQ3 corrections of n-tile nt sit at
// qf + nt*(D/32)*32 and corr + nt*(D/32)*4.
template <int D, int NT>
__device__ __forceinline__ void tq3_logits_nt(const uint8_t* pg, const uint4* qf,
                                              const float2* corr, int lane, int kw, int ks,
                                              float (&x)[NT][4]) {
  constexpr int G = D / 32;
  const int r = lane >> 2, c = lane & 3;
  const uint8_t* krec = pg;
  const __half* kscale = reinterpret_cast<const __half*>(pg + G * 16 * 12);
  uint32_t kMask = 0x00380380u, kMagic = 0x58004800u;
  opaque(kMask, kMagic);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) x[nt][0] = x[nt][1] = x[nt][2] = x[nt][3] = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t* ra = reinterpret_cast<const uint32_t*>(krec + 12 * (16 * g + r));
    const uint32_t* rb = ra + 24;  // token r + 8
    const uint32_t xa = __funnelshift_r(ra[kw], ra[kw + 1], ks);
    const uint32_t xb = __funnelshift_r(rb[kw], rb[kw + 1], ks);
    const uint32_t a0 = and_or(xa, kMask, kMagic), b0 = and_or(xb, kMask, kMagic);
    const uint32_t a1 = and_or(xa >> 3, kMask, kMagic), b1 = and_or(xb >> 3, kMask, kMagic);
    const uint32_t a2 = and_or(xa >> 6, kMask, kMagic), b2 = and_or(xb >> 6, kMask, kMagic);
    const uint32_t a3 = and_or(xa >> 9, kMask, kMagic), b3 = and_or(xb >> 9, kMask, kMagic);
    const float sa = __half2float(kscale[16 * g + r]);
    const float sb = __half2float(kscale[16 * g + r + 8]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4 qb = qf[nt * G * 32 + 32 * g + lane];
      const float2 cr = corr[nt * G * 4 + 4 * g + c];
      float cg[4];
      mma_f16_16816(cg, a0, b0, a1, b1, qb.x, qb.y, {cr.x, cr.y, cr.x, cr.y});
      mma_f16_16816(cg, a2, b2, a3, b3, qb.z, qb.w, cg);
      x[nt][0] = fmaf(sa, cg[0], x[nt][0]);
      x[nt][1] = fmaf(sa, cg[1], x[nt][1]);
      x[nt][2] = fmaf(sb, cg[2], x[nt][2]);
      x[nt][3] = fmaf(sb, cg[3], x[nt][3]);
    }
  }
}

template <int D, int NT>
__device__ __forceinline__ void fp8_logits_nt(const uint8_t* pg, const uint4* qf, int lane,
                                              float (&x)[NT][4]) {
  const int r = lane >> 2, c = lane & 3;
  const float sk = *reinterpret_cast<const float*>(pg + 32 * D);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) x[nt][0] = x[nt][1] = x[nt][2] = x[nt][3] = 0.f;
#pragma unroll
  for (int j = 0; j < D / 64; ++j) {
    const uint4 wa = *reinterpret_cast<const uint4*>(pg + r * D + 64 * j + 16 * c);
    const uint4 wb = *reinterpret_cast<const uint4*>(pg + (r + 8) * D + 64 * j + 16 * c);
    const uint32_t va[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t vb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a0 = e4m3x2_to_f16x2(va[i]), a1 = e4m3x2_to_f16x2(vb[i]);
      const uint32_t a2 = e4m3x2_to_f16x2(va[i] >> 16), a3 = e4m3x2_to_f16x2(vb[i] >> 16);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint4 q = qf[nt * (D / 32) * 32 + 32 * (2 * j + (i >> 1)) + lane];
        mma_f16_16816(x[nt], a0, a1, a2, a3, (i & 1) ? q.z : q.x, (i & 1) ? q.w : q.y, x[nt]);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) x[nt][e] *= sk;
}

// P.V of the channel groups [g0, g0 + GW) for all n-tiles: acc[2 lg + j][nt] is channel tile
// 2 (g0 + lg) + j (channel order as for one n-tile); pb[nt] the n-tile's P^T fragments.
template <int D, int NT, int GW, bool WIDE>
__device__ __forceinline__ void tq3_pv_nt(float (&acc)[2 * GW][NT][4], const uint8_t* pg,
                                          int lane, int vw, int vs1, int g0,
                                          const uint2 (&pb)[NT]) {
  constexpr int G = D / 32;
  const int c = lane & 3;
  const uint8_t* vrec = pg + G * 16 * 14;
  const __half* vscale = reinterpret_cast<const __half*>(vrec + G * 16 * 12);
  uint32_t m0 = 0x000E000Eu, g0m = 0x60006000u, m1 = 0x00700070u, g1 = 0x54005400u;
  uint32_t m2 = 0x03800380u, g2 = 0x48004800u;
  opaque(m0, g0m, m1, g1, m2, g2);
  const uint32_t s0 = f16x2_const(515.5f, 515.5f), s1 = f16x2_const(67.5f, 67.5f);
  const uint32_t s2 = f16x2_const(11.5f, 11.5f);
#pragma unroll
  for (int lg = 0; lg < GW; ++lg) {
    const int g = g0 + lg;
    const uint32_t* rc = reinterpret_cast<const uint32_t*>(vrec + 12 * (16 * g + 2 * c));
    const uint32_t f0 = __funnelshift_r(rc[vw], rc[vw + 1], vs1);        // token 2c
    const uint32_t f1 = __funnelshift_r(rc[vw + 3], rc[vw + 4], vs1);    // token 2c+1
    const uint32_t f8 = __funnelshift_r(rc[vw + 24], rc[vw + 25], vs1);  // token 2c+8
    const uint32_t f9 = __funnelshift_r(rc[vw + 27], rc[vw + 28], vs1);  // token 2c+9
    const uint32_t z01 = __byte_perm(f0, f1, 0x5410);
    const uint32_t z89 = __byte_perm(f8, f9, 0x5410);
    const uint32_t a0 = hsub2_u32(and_or(z01, m0, g0m), s0), b0 = hsub2_u32(and_or(z89, m0, g0m), s0);
    const uint32_t a1 = hsub2_u32(and_or(z01, m1, g1), s1), b1 = hsub2_u32(and_or(z89, m1, g1), s1);
    const uint32_t a2 = hsub2_u32(and_or(z01, m2, g2), s2), b2 = hsub2_u32(and_or(z89, m2, g2), s2);
    const uint32_t a3 = hsub2_u32(and_or(z01 >> 3, m2, g2), s2);
    const uint32_t b3 = hsub2_u32(and_or(z89 >> 3, m2, g2), s2);
    uint32_t sv0 = *reinterpret_cast<const uint32_t*>(vscale + 16 * g + 2 * c);
    uint32_t sv8 = *reinterpret_cast<const uint32_t*>(vscale + 16 * g + 2 * c + 8);
    if constexpr (!WIDE) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t q0 = hmul2_u32(pb[nt].x, sv0), q1 = hmul2_u32(pb[nt].y, sv8);
        mma_f16_16816(acc[2 * lg][nt], a0, a1, b0, b1, q0, q1, acc[2 * lg][nt]);
        mma_f16_16816(acc[2 * lg + 1][nt], a2, a3, b2, b3, q0, q1, acc[2 * lg + 1][nt]);
      }
    } else {
      uint32_t m = hmax2_u32(sv0, sv8);
      m = hmax2_u32(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = hmax2_u32(m, __shfl_xor_sync(0xffffffffu, m, 2));
      const int e = max(static_cast<int>(max(m & 0xffffu, m >> 16) >> 10), 1);
      const uint32_t down = static_cast<uint32_t>(31 - e) * 0x04000400u;  // f16x2 2^(16-e)
      const float up = __int_as_float((e + 111) << 23);                   // fp32 2^(e-16)
      sv0 = hmul2_u32(sv0, down);
      sv8 = hmul2_u32(sv8, down);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t q0 = hmul2_u32(pb[nt].x, sv0), q1 = hmul2_u32(pb[nt].y, sv8);
        float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
        mma_f16_16816(t0, a0, a1, b0, b1, q0, q1, t0);
        mma_f16_16816(t1, a2, a3, b2, b3, q0, q1, t1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * lg][nt][j] = fmaf(up, t0[j], acc[2 * lg][nt][j]);
          acc[2 * lg + 1][nt][j] = fmaf(up, t1[j], acc[2 * lg + 1][nt][j]);
        }
      }
    }
  }
}

template <int D, int NT, int GW>
__device__ __forceinline__ void fp8_pv_nt(float (&acc)[2 * GW][NT][4], const uint8_t* pg,
                                          int lane, int g0, const uint2 (&pb)[NT]) {
  const int r = lane >> 2, c = lane & 3;
  const float sv = *reinterpret_cast<const float*>(pg + 32 * D + 4);
  const uint8_t* vrows = pg + 16 * D;
#pragma unroll
  for (int lg = 0; lg < GW; ++lg) {
    const int off = 32 * (g0 + lg) + 4 * r;
    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c) * D + off);
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c + 1) * D + off);
    const uint32_t w8 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c + 8) * D + off);
    const uint32_t w9 = *reinterpret_cast<const uint32_t*>(vrows + (2 * c + 9) * D + off);
    const uint32_t lo01 = __byte_perm(w0, w1, 0x5140), hi01 = __byte_perm(w0, w1, 0x7362);
    const uint32_t lo89 = __byte_perm(w8, w9, 0x5140), hi89 = __byte_perm(w8, w9, 0x7362);
    const uint32_t a0 = e4m3x2_to_f16x2(lo01), a1 = e4m3x2_to_f16x2(lo01 >> 16);
    const uint32_t a2 = e4m3x2_to_f16x2(lo89), a3 = e4m3x2_to_f16x2(lo89 >> 16);
    const uint32_t b0 = e4m3x2_to_f16x2(hi01), b1 = e4m3x2_to_f16x2(hi01 >> 16);
    const uint32_t b2 = e4m3x2_to_f16x2(hi89), b3 = e4m3x2_to_f16x2(hi89 >> 16);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
      mma_f16_16816(t0, a0, a1, a2, a3, pb[nt].x, pb[nt].y, t0);
      mma_f16_16816(t1, b0, b1, b2, b3, pb[nt].x, pb[nt].y, t1);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * lg][nt][e] = fmaf(sv, t0[e], acc[2 * lg][nt][e]);
        acc[2 * lg + 1][nt][e] = fmaf(sv, t1[e], acc[2 * lg + 1][nt][e]);
      }
    }
  }
}

// ------------------------------------------------------------------ BF16 control page
// Stage rows (ROW = 2D + 16 bytes): K token t at t*ROW, V token t at (16 + t)*ROW.  The values
// are the stored bf16, so both contractions use bf16 MMAs on them directly; Q is bf16 too.
// Logits: A = K (16 tokens x 16 channels per k-step) by ldmatrix, B = Q fragments
// [D/32][32 lanes] {k-step 2w: b0, b1 | k-step 2w+1: b0, b1}.
template <int D>
__device__ __forceinline__ void bf16_logits(const uint8_t* pg, const uint4* qf, int lane,
                                            float (&x)[4]) {
  constexpr int ROW = 2 * D + 16;
  const int m = lane >> 3;
  const uint8_t* base = pg + ((m & 1) * 8 + (lane & 7)) * ROW + (m >> 1) * 16;
  float cg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < D / 32; ++w) {
    const uint4 qb = qf[32 * w + lane];
    uint32_t a[4];
    ldmatrix_x4(a, base + 64 * w);
    mma_bf16_16816(cg, a[0], a[1], a[2], a[3], qb.x, qb.y, cg);
    ldmatrix_x4(a, base + 64 * w + 32);
    mma_bf16_16816(cg, a[0], a[1], a[2], a[3], qb.z, qb.w, cg);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = cg[j];
}

// P.V: A = V^T tile mt (channels 16mt.., tokens) by transposing ldmatrix of the V rows; P is
// split into bf16 hi + lo parts (about 16 significant bits) and both are multiplied in.
// acc[mt]: rows r, r+8 = channels 16mt + r, 16mt + 8 + r.
template <int D>
__device__ __forceinline__ void bf16_pv(VState<D>& st, const uint8_t* pg, int lane,
                                        const float (&pr)[4]) {
  constexpr int ROW = 2 * D + 16;
  const uint32_t h01 = pack_bf16x2(pr[0], pr[1]), h23 = pack_bf16x2(pr[2], pr[3]);
  const uint32_t l01 = pack_bf16x2(pr[0] - bf16_lo(h01), pr[1] - bf16_hi(h01));
  const uint32_t l23 = pack_bf16x2(pr[2] - bf16_lo(h23), pr[3] - bf16_hi(h23));
  const uint32_t ph0 = movmatrix_trans(h01), ph1 = movmatrix_trans(h23);
  const uint32_t pl0 = movmatrix_trans(l01), pl1 = movmatrix_trans(l23);
  const uint8_t* base =
      pg + (16 + (lane & 7) + 8 * (lane >> 4)) * ROW + 16 * ((lane >> 3) & 1);
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    uint32_t a[4];
    ldmatrix_x4_trans(a, base + 32 * mt);
    mma_bf16_16816(st.acc[mt], a[0], a[1], a[2], a[3], ph0, ph1, st.acc[mt]);
    mma_bf16_16816(st.acc[mt], a[0], a[1], a[2], a[3], pl0, pl1, st.acc[mt]);
  }
}

// bf16 Q fragments of n-tile nt in natural channel order (exact; no scaling, no correction).
template <int D>
__device__ __forceinline__ float build_q_bf16(const DecodeParams& p, const SeqDesc& sd, int h,
                                              int nt, int lane, uint4* qf);

// Query column n of this CTA's KV head -> its bf16 row, or nullptr for padding columns.
__device__ __forceinline__ const uint16_t* q_row(const DecodeParams& p, const SeqDesc& sd,
                                                 int h, int n) {
  if (n >= p.NC) return nullptr;
  const int qi = n / p.g, hq = h * p.g + (n % p.g);
  return p.q + ((static_cast<int64_t>(sd.out_row) * p.q_len + qi) * p.Hq + hq) * p.D;
}

// Build the f16 Q fragments of n-tile nt (columns 8nt..8nt+7) in this format's channel order
// into shared memory, scaled by a power of two that brings the tile's largest |q| into
// [2^13, 2^14) (f16 images of the bf16 queries keep their precision); returns the logit scale
// with the power of two undone.
template <int D, bool FP8>
__device__ __forceinline__ float build_q(const DecodeParams& p, const SeqDesc& sd, int h, int nt,
                                         int lane, uint4* qf, float* corr) {
  const int r = lane >> 2, c = lane & 3;
  const uint16_t* qr = q_row(p, sd, h, 8 * nt + r);
  float qv[D / 4];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < D / 4; ++i) {
    // FP8 order: channels 64j+16c+e (j = i/16, e = i%16); TQ3 order: 32g+8c+e (g = i/8)
    const int ch = FP8 ? 64 * (i / 16) + 16 * c + (i % 16) : 32 * (i / 8) + 8 * c + (i % 8);
    const float v = qr ? bf16_bits_to_float(qr[ch]) : 0.f;
    qv[i] = v;
    amax = fmaxf(amax, fabsf(v));
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int e = 0;
  if (amax > 0.f && isfinite(amax)) {
    frexpf(amax, &e);  // amax in [2^(e-1), 2^e)
    e = max(-100, min(100, 14 - e));
  }
  const float qs = ldexpf(1.f, e);
#pragma unroll
  for (int w = 0; w < D / 32; ++w) {
    uint4 f;
    if constexpr (FP8) {
      // two k-blocks (4j+i, 4j+i+1) per uint4: channels +0,+1 | +2,+3 of each
      const float* v = qv + 8 * w;
      f.x = pack_f16x2(v[0] * qs, v[1] * qs);
      f.y = pack_f16x2(v[2] * qs, v[3] * qs);
      f.z = pack_f16x2(v[4] * qs, v[5] * qs);
      f.w = pack_f16x2(v[6] * qs, v[7] * qs);
    } else {
      // k-block pairs (8c+0, 8c+4), (8c+1, 8c+5), (8c+2, 8c+6), (8c+3, 8c+7) of group w
      const float* v = qv + 8 * w;
      f.x = pack_f16x2(v[0] * qs, v[4] * qs);
      f.y = pack_f16x2(v[1] * qs, v[5] * qs);
      f.z = pack_f16x2(v[2] * qs, v[6] * qs);
      f.w = pack_f16x2(v[3] * qs, v[7] * qs);
      // correction of this column and group: -(11.5 * sum of the f16 q that meet codes 0-3
      // of a chunk + 131.5 * sum of those that meet codes 4-7), over the 4 chunks
      float lo = 0.f, hi = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo += __half2float(__float2half_rn(v[e] * qs));
        hi += __half2float(__float2half_rn(v[e + 4] * qs));
      }
      float part = -(11.5f * lo + 131.5f * hi);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (c == 0) corr[8 * w + r] = part;  // [group][column pair][2]: column r = 2(r/2) + r%2
    }
    qf[32 * w + lane] = f;
  }
  return p.logit_scale * ldexpf(1.f, -e);
}

template <int D>
__device__ __forceinline__ float build_q_bf16(const DecodeParams& p, const SeqDesc& sd, int h,
                                              int nt, int lane, uint4* qf) {
  const int r = lane >> 2, c = lane & 3;
  const uint16_t* qr = q_row(p, sd, h, 8 * nt + r);
  auto pair = [&](int ch) -> uint32_t {
    return qr ? static_cast<uint32_t>(qr[ch]) | (static_cast<uint32_t>(qr[ch + 1]) << 16) : 0u;
  };
#pragma unroll
  for (int w = 0; w < D / 32; ++w)
    qf[32 * w + lane] = make_uint4(pair(32 * w + 2 * c), pair(32 * w + 8 + 2 * c),
                                   pair(32 * w + 16 + 2 * c), pair(32 * w + 24 + 2 * c));
  return p.logit_scale;
}

// Scanner warp: collect the unit's pages of format fmt from table entries [first, last).  A
// round reads 32 x DEPTH entries (DEPTH loads per lane in flight), so a sparse range of a few
// thousand pages costs a few memory latencies.  Kernels with registers to spare take 32.
template <int DEPTH>
__device__ __forceinline__ int scan_range(const DecodeParams& p, const int32_t* row, int first,
                                          int last, int fmt, int lane, int2* list) {
  const int nslots = fmt == 1 ? p.tq3_slots : p.fp8_slots;
  const unsigned lt = (1u << lane) - 1u;
  int count = 0;
  bool bad = false;
  for (int base = first; base < last; base += 32 * DEPTH) {
    int32_t e[DEPTH];
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) {
      const int idx = base + 32 * j + lane;
      e[j] = idx < last ? row[idx] : -1;
    }
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) {
      const int idx = base + 32 * j + lane;
      const uint32_t f = static_cast<uint32_t>(e[j]) >> kFmtShift;
      const int slot = static_cast<int>(static_cast<uint32_t>(e[j]) & kSlotMask);
      const bool mapped = e[j] != -1;  // a BF16 entry (format 2) has the sign bit set
      const bool known = f == 1 || static_cast<int>(f) == p.page_fmt;
      bad |= (idx < last) && (!mapped || !known || slot >= (f == 1 ? p.tq3_slots : p.fp8_slots));
      const bool take = mapped && static_cast<int>(f) == fmt && slot < nslots;
      const unsigned b = __ballot_sync(0xffffffffu, take);
      const int pos = count + __popc(b & lt);
      if (take && pos < kMaxPagesPerUnit) list[pos] = make_int2(slot, idx);
      count += __popc(b);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) flag_status(p.status, kStatusCheck);
  if (count > kMaxPagesPerUnit) {
    if (lane == 0) flag_status(p.status, kStatusCheck);
    count = kMaxPagesPerUnit;
  }
  return count;
}

// Page geometry of a format inside a partial kernel of kind K.
template <int D, int NT, int K, int F>
struct Page {
  using C = Cfg<D, NT, K>;
  static constexpr int STAGE = F == kFp8 ? C::FP8_STAGE : (F == kTq3 ? C::TQ3_STAGE : C::BF16_STAGE);
  static constexpr int NST = F == kFp8 ? C::FP8_NST : (F == kTq3 ? C::TQ3_NST : C::BF16_NST);
  // bytes of one KV head in a slot of the format
  static constexpr int HEAD = F == kFp8 ? 32 * D + 16 : (F == kTq3 ? 14 * D : 64 * D);
};

// One thread: (re)initialise the stage barriers and counters for a unit.  For a CTA's second
// and later units the barriers are invalidated first: the previous unit waited for every copy
// it issued and the CTA synchronised since, so none of them is in use.
__device__ __forceinline__ void init_ring(const Smem& sm, bool again) {
  for (int s = 0; s < kRingBarriers; ++s) {
    if (again) mbar_inval(&sm.full[s]);
    mbar_init(&sm.full[s], 1);
    sm.cnt[s] = 0;
    sm.fills[s] = 0;
  }
  sm.misc[1] = 0;
  mbar_fence_init();
}

// Warp-collective: start the bulk copy of page i of the unit (list entry i) into its ring
// stage.  FP8 and TQ3 pages are one contiguous copy issued by lane 0; a BF16 page is 32 row
// copies, one per lane, into padded stage rows.
template <class PG, int F>
__device__ __forceinline__ void fill_stage(const Smem& sm, const uint8_t* slab, int64_t slot_bytes,
                                           int h, int i, int lane) {
  const int s = i % PG::NST;
  const int2 e = sm.list[i];
  const uint8_t* src = slab + static_cast<int64_t>(e.x) * slot_bytes +
                       static_cast<int64_t>(h) * PG::HEAD;
  if (lane == 0) {
    sm.fills[s] += 1;
    mbar_arrive_expect_tx(&sm.full[s], PG::HEAD);
  }
  if constexpr (F == kBf16) {
    constexpr int ROWB = PG::HEAD / 32;  // 2D bytes
    __syncwarp();
    bulk_g2s(sm.ring + s * PG::STAGE + lane * (ROWB + 16), src + lane * ROWB, ROWB, &sm.full[s]);
  } else {
    if (lane == 0) bulk_g2s(sm.ring + s * PG::STAGE, src, PG::STAGE, &sm.full[s]);
  }
}

template <int D, int NT, int K, int F>
__device__ void run_unit(const DecodeParams& p, const SeqDesc& sd, const UnitDesc& u, int h,
                         Smem sm, bool again) {
  using C = Cfg<D, NT, K>;
  using PG = Page<D, NT, K, F>;
  constexpr int STAGE = PG::STAGE;
  constexpr int NST = PG::NST;
  constexpr int SCANNER = C::WARPS - 1;  // the warp that scans the range and starts the copies
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
  const int nt = warp % NT, pw = warp / NT;

  const uint8_t* slab = F == kTq3 ? p.tq3_slab : p.fp8_slab;
  const int64_t slot_bytes = F == kTq3 ? p.tq3_slot_bytes : p.fp8_slot_bytes;
  if (warp == SCANNER) {
    // the first fills are in flight while the other warps build their Q fragments
    if (lane == 0) init_ring(sm, again);
    __syncwarp();
    const int32_t* row = p.tables + static_cast<int64_t>(sd.row) * p.max_pages;
    const int n = scan_range<C::SCAN>(p, row, u.first, u.last, F, lane, sm.list);
    __syncwarp();
    if (lane == 0) sm.misc[0] = n;
    for (int i = 0; i < min(n, NST); ++i) fill_stage<PG, F>(sm, slab, slot_bytes, h, i, lane);
  }
  if (pw == 0) {
    uint4* qf = sm.qf + nt * (D / 32) * 32;
    float ls;
    if constexpr (F == kBf16)
      ls = build_q_bf16<D>(p, sd, h, nt, lane, qf);
    else
      ls = build_q<D, F == kFp8>(p, sd, h, nt, lane, qf,
                                 reinterpret_cast<float*>(sm.corr + nt * (D / 32) * 4));
    if (lane == 0) reinterpret_cast<float*>(sm.misc)[4 + nt] = ls;
  }
  __syncthreads();
  const int count = sm.misc[0];

  KState ks;
  VState<D> vs;
  ks.m[0] = ks.m[1] = -INFINITY;
  ks.l[0] = ks.l[1] = 0.f;
  {
    const int n0 = 8 * nt + 2 * c, n1 = n0 + 1;
    const int lim0 = n0 < p.NC ? sd.ctx - p.q_len + n0 / p.g : sd.ctx - 1;
    const int lim1 = n1 < p.NC ? sd.ctx - p.q_len + n1 / p.g : sd.ctx - 1;
    const int min_lim = sd.ctx - p.q_len;
    const float ls = reinterpret_cast<const float*>(sm.misc)[4 + nt];
    const uint4* qf = sm.qf + nt * (D / 32) * 32;
    const float2* corr = sm.corr + nt * (D / 32) * 4;
    // TQ3 K chunk c of a record starts at bit 24c; read from bit 24c-7 (codes at 7+3k).
    // TQ3 V field of row r starts at bit 12r; read from bit 12r-1 (codes at 1+3k).
    const int kbit = 24 * c - 7, vbit = 12 * r - 1;
    const int kw = kbit >= 0 ? kbit >> 5 : -1, ks5 = kbit & 31;
    const int vw = vbit >= 0 ? vbit >> 5 : -1, vs1 = vbit & 31;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) vs.acc[mt][e] = 0.f;

    bool aborted = false;
    for (int i = pw; i < count; i += C::PW) {
      const int s = i % NST;
      if (!mbar_wait_warp(&sm.full[s], (i / NST) & 1)) {
        if (lane == 0) {
          flag_status(p.status, kStatusTimeout);
          atomicExch(&sm.misc[1], 1);
        }
        aborted = true;
        break;
      }
      const int tok0 = 16 * sm.list[i].y;
      const uint8_t* pg = sm.ring + s * STAGE;
      float x[4];
      if constexpr (F == kFp8)
        fp8_logits<D>(pg, qf, lane, x);
      else if constexpr (F == kTq3)
        tq3_logits<D>(pg, qf, corr, lane, kw, ks5, x);
      else
        bf16_logits<D>(pg, qf, lane, x);
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] *= ls;
      if (tok0 + 15 > min_lim) mask_page(x, tok0, r, lim0, lim1);
      float pr[4];
      float a0, a1;
      softmax_k(ks, x, pr, a0, a1);
      if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          vs.acc[mt][0] *= a0;
          vs.acc[mt][2] *= a0;
          vs.acc[mt][1] *= a1;
          vs.acc[mt][3] *= a1;
        }
      }
      if constexpr (F == kBf16) {
        bf16_pv<D>(vs, pg, lane, pr);
      } else {
        const uint32_t pb0 = movmatrix_trans(pack_f16x2(pr[0], pr[1]));
        const uint32_t pb1 = movmatrix_trans(pack_f16x2(pr[2], pr[3]));
        if constexpr (F == kFp8) {
          fp8_pv<D>(vs, pg, lane, pb0, pb1);
        } else {
          const uint32_t vmax = tq3_v_scale_max<D>(pg, lane);
          if (vmax >= kVScaleLo && vmax <= kVScaleHi)
            tq3_pv<D, false>(vs, pg, lane, vw, vs1, pb0, pb1);
          else
            tq3_pv<D, true>(vs, pg, lane, vw, vs1, pb0, pb1);
        }
      }
      // release the stage: its owner refills it with the page one ring-length ahead.  Every
      // lane's reads of the stage are ordered before the async-proxy overwrite.
      if (i + NST < count) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        bool last = true;
        if constexpr (NT > 1) {  // the n-tile warps of this page: the last one done refills
          if (lane == 0) {
            __threadfence_block();
            last = atomicAdd(&sm.cnt[s], 1) == NT - 1;
            if (last) sm.cnt[s] = 0;
            __threadfence_block();
          }
          last = __shfl_sync(0xffffffffu, last, 0);
        }
        if (last) fill_stage<PG, F>(sm, slab, slot_bytes, h, i + NST, lane);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      ks.l[0] += __shfl_xor_sync(0xffffffffu, ks.l[0], o);
      ks.l[1] += __shfl_xor_sync(0xffffffffu, ks.l[1], o);
    }
    if (aborted && lane == 0) {
      // drain: wait (bounded) for the last copy issued into each of this group's stages, so
      // none is in flight when the CTA's shared memory is released
      for (int s = pw; s < NST; s += C::PW) {
        const int f = *reinterpret_cast<volatile int32_t*>(&sm.fills[s]);
        if (f > 0) mbar_wait(&sm.full[s], (f - 1) & 1, 100000000ull);
      }
    }
  }
  __syncthreads();  // ring no longer needed: reuse it for the cross-warp combine

  // every page-parallel warp stores its state; then all of them combine a share of the
  // columns' channels: M = max m, l = sum l 2^(m-M), acc = sum acc 2^(m-M)
  float* cmb = reinterpret_cast<float*>(sm.ring);
  constexpr int REGION = 8 * (D + 2);  // per (warp, n-tile): (m, l) of 8 columns, then acc [8][D]
  {
    float* reg = cmb + (pw * NT + nt) * REGION;
    if (r == 0) {
      reg[2 * (2 * c)] = ks.m[0];
      reg[2 * (2 * c) + 1] = ks.l[0];
      reg[2 * (2 * c + 1)] = ks.m[1];
      reg[2 * (2 * c + 1) + 1] = ks.l[1];
    }
    float* ra = reg + 16;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      // channels of accumulator rows r and r + 8 of tile mt
      const int ch0 = F == kBf16 ? 16 * mt + r : 32 * (mt >> 1) + 4 * r + 2 * (mt & 1);
      const int ch1 = F == kBf16 ? ch0 + 8 : ch0 + 1;
      ra[(2 * c) * D + ch0] = vs.acc[mt][0];
      ra[(2 * c + 1) * D + ch0] = vs.acc[mt][1];
      ra[(2 * c) * D + ch1] = vs.acc[mt][2];
      ra[(2 * c + 1) * D + ch1] = vs.acc[mt][3];
    }
  }
  __syncthreads();
  {
    const int part = sd.part0 + u.part;
    const float* regs = cmb + nt * REGION;  // warp w's region: regs + w * NT * REGION
    for (int q = pw * 32 + lane; q < 8 * (D / 4); q += 32 * C::PW) {
      const int col = q / (D / 4), ch = 4 * (q % (D / 4));
      const int n = 8 * nt + col;
      if (n >= p.NC) continue;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::PW; ++w) M = fmaxf(M, regs[w * NT * REGION + 2 * col]);
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < C::PW; ++w) {
          const float* rw = regs + w * NT * REGION;
          const float mw = rw[2 * col];
          if (mw == -INFINITY) continue;
          const float a = exp2f(mw - M);
          L += rw[2 * col + 1] * a;
          const float4 v = *reinterpret_cast<const float4*>(rw + 16 + col * D + ch);
          acc.x += a * v.x;
          acc.y += a * v.y;
          acc.z += a * v.z;
          acc.w += a * v.w;
        }
      }
      const int64_t base = (static_cast<int64_t>(part) * p.Hkv + h) * p.NC + n;
      if (ch == 0) {
        p.part_ml[2 * base] = M;
        p.part_ml[2 * base + 1] = L;
      }
      *reinterpret_cast<float4*>(p.part_acc + base * D + ch) = acc;
    }
  }
}

// Team layout (more than 8 query columns; FP8 or TQ3 pages).  The unit's pages are taken in
// batches of TW: warp w decodes the K of page b + w once for all NT n-tiles, computes the
// page's logits and probabilities against the common reference of each column (identical on
// every warp), and publishes their P^T fragments; after one team barrier every warp multiplies
// the whole batch by the V of its own channel groups.  Every page's codes are decoded once.
// The reference is raised lazily, as on the one-tile path: a page whose column exceeds it by
// more than 8 uses its own reference (the column maximum, so the dominant token's probability
// is exactly 1) and flags the batch; after the barrier every warp raises the common reference
// to the batch's largest and rescales that batch's P and its own accumulators.  Probabilities
// fed to the MMAs stay <= 2^8.  Each warp sums the denominators of its own K pages; the sums meet
// in the combine.
template <int D, int NT, int K, int F>
__device__ void run_unit_team(const DecodeParams& p, const SeqDesc& sd, const UnitDesc& u, int h,
                              Smem sm, bool again) {
  using C = Cfg<D, NT, K>;
  using PG = Page<D, NT, K, F>;
  constexpr int TW = C::TW, NST = PG::NST, STAGE = PG::STAGE;
  constexpr int GW = (D / 32) / TW;  // channel groups of 32 per warp
  static_assert(NST % TW == 0 && NST >= 2 * TW, "two batches in flight");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
  const uint8_t* slab = F == kTq3 ? p.tq3_slab : p.fp8_slab;
  const int64_t slot_bytes = F == kTq3 ? p.tq3_slot_bytes : p.fp8_slot_bytes;

  if (warp == TW - 1) {
    if (lane == 0) init_ring(sm, again);
    __syncwarp();
    const int32_t* row = p.tables + static_cast<int64_t>(sd.row) * p.max_pages;
    const int n = scan_range<C::SCAN>(p, row, u.first, u.last, F, lane, sm.list);
    __syncwarp();
    if (lane == 0) sm.misc[0] = n;
    for (int i = 0; i < min(n, NST); ++i) fill_stage<PG, F>(sm, slab, slot_bytes, h, i, lane);
  }
  for (int nt = warp; nt < NT; nt += TW) {
    const float ls = build_q<D, F == kFp8>(p, sd, h, nt, lane, sm.qf + nt * (D / 32) * 32,
                                           reinterpret_cast<float*>(sm.corr + nt * (D / 32) * 4));
    if (lane == 0) reinterpret_cast<float*>(sm.misc)[4 + nt] = ls;
  }
  __syncthreads();
  const int count = sm.misc[0];

  const float* lsc = reinterpret_cast<const float*>(sm.misc) + 4;  // logit scale per n-tile
  const int min_lim = sd.ctx - p.q_len;
  const int kbit = 24 * c - 7, vbit = 12 * r - 1;
  const int kw = kbit >= 0 ? kbit >> 5 : -1, ks5 = kbit & 31;
  const int vw = vbit >= 0 ? vbit >> 5 : -1, vs1 = vbit & 31;
  const int g0 = warp * GW;
  uint2* xp = reinterpret_cast<uint2*>(sm.xch);              // [2][TW][NT][32] P^T fragments
  float* xr = reinterpret_cast<float*>(sm.xch + C::XCH_P);   // [2][TW][NT][8] page references
  int32_t* xf = sm.cnt;  // [2][TW] per page: bit 0 raised a reference, bit 1 V scales out of range

  float acc[2 * GW][NT][4];
#pragma unroll
  for (int j = 0; j < 2 * GW; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[j][nt][0] = acc[j][nt][1] = acc[j][nt][2] = acc[j][nt][3] = 0.f;
  // common references (log2 units, integers once set) of columns 2c, 2c+1 and r of every
  // n-tile; this lane's share of the denominators of its K pages (columns 2c, 2c+1)
  float mc[NT][2], mr[NT], lk[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mc[nt][0] = mc[nt][1] = mr[nt] = -INFINITY;
    lk[nt][0] = lk[nt][1] = 0.f;
  }

  for (int b = 0; b < count; b += TW) {
    const int par = (b / TW) & 1;
    const int nb = min(TW, count - b);
    // K: this warp's page of the batch
    bool ok = true, raised = false, wide = false;
    float lp[NT][2];  // the page's denominator shares, relative to its references
    float rf[NT][2];  // the page's references of columns 2c, 2c+1
    const int ik = b + warp;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      lp[nt][0] = lp[nt][1] = 0.f;
      rf[nt][0] = mc[nt][0];
      rf[nt][1] = mc[nt][1];
    }
    if (ik < count) {
      const int s = ik % NST;
      ok = mbar_wait_warp(&sm.full[s], (ik / NST) & 1);
      if (ok) {
        const uint8_t* pg = sm.ring + s * STAGE;
        float x[NT][4];
        if constexpr (F == kFp8)
          fp8_logits_nt<D, NT>(pg, sm.qf, lane, x);
        else
          tq3_logits_nt<D, NT>(pg, sm.qf, sm.corr, lane, kw, ks5, x);
        const int tok0 = 16 * sm.list[ik].y;
        const bool edge = tok0 + 15 > min_lim;
        if constexpr (F == kTq3) {
          // the V range check, once per page for the whole team
          const uint32_t vmax = tq3_v_scale_max<D>(pg, lane);
          wide = !(vmax >= kVScaleLo && vmax <= kVScaleHi);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float ls = lsc[nt];
#pragma unroll
          for (int j = 0; j < 4; ++j) x[nt][j] *= ls;
          if (edge) {
            // causal limits of columns 2c, 2c+1 (padding columns see the whole context)
            const int n0 = 8 * nt + 2 * c, n1 = n0 + 1;
            mask_page(x[nt], tok0, r, n0 < p.NC ? min_lim + n0 / p.g : sd.ctx - 1,
                      n1 < p.NC ? min_lim + n1 / p.g : sd.ctx - 1);
          }
          float m0 = fmaxf(x[nt][0], x[nt][2]), m1 = fmaxf(x[nt][1], x[nt][3]);
          const bool need = m0 > mc[nt][0] + kLazyRescale || m1 > mc[nt][1] + kLazyRescale;
          if (__any_sync(0xffffffffu, need)) {
            // this page raises: its own references (the column maxima) where needed
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
              m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
              m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
            }
            if (m0 > mc[nt][0] + kLazyRescale) rf[nt][0] = m0;
            if (m1 > mc[nt][1] + kLazyRescale) rf[nt][1] = m1;
            raised = true;
          }
          const float r0 = rf[nt][0] == -INFINITY ? 0.f : rf[nt][0];
          const float r1 = rf[nt][1] == -INFINITY ? 0.f : rf[nt][1];
          float pr[4];
          pr[0] = fast_exp2(x[nt][0] - r0);
          pr[1] = fast_exp2(x[nt][1] - r1);
          pr[2] = fast_exp2(x[nt][2] - r0);
          pr[3] = fast_exp2(x[nt][3] - r1);
          lp[nt][0] = pr[0] + pr[2];
          lp[nt][1] = pr[1] + pr[3];
          xp[((par * TW + warp) * NT + nt) * 32 + lane] =
              make_uint2(movmatrix_trans(pack_f16x2(pr[0], pr[1])),
                         movmatrix_trans(pack_f16x2(pr[2], pr[3])));
        }
        if (raised) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            if (r == 0) {
              xr[((par * TW + warp) * NT + nt) * 8 + 2 * c] = rf[nt][0];
              xr[((par * TW + warp) * NT + nt) * 8 + 2 * c + 1] = rf[nt][1];
            }
        }
      }
    }
    if (lane == 0) xf[par * TW + warp] = (raised ? 1 : 0) | (wide ? 2 : 0);
    // the batch's probabilities are published; every warp of the team stops together on a
    // failed wait
    if (!barrier_and(1, 32 * TW, ok)) {
      if (lane == 0) {
        flag_status(p.status, kStatusTimeout);
        atomicExch(&sm.misc[1], 1);
      }
      break;
    }
    // the previous batch's stages: every warp fenced its reads of them before this barrier, so
    // warp w refills the stage of page b - TW + w with the page NST ahead
    if (b >= TW && b - TW + warp + NST < count)
      fill_stage<PG, F>(sm, slab, slot_bytes, h, b - TW + warp + NST, lane);
    // the batch's page flags, two bits per page
    int fl = 0;
#pragma unroll
    for (int q = 0; q < TW; ++q) fl |= (q < nb ? xf[par * TW + q] : 0) << (2 * q);
    const bool any_raised = (fl & 0x5555) != 0;
    // column r's reference before this batch: the P scale of a page that did not raise
    float mr_old[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mr_old[nt] = mr[nt];
    if (any_raised) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float n0 = mc[nt][0], n1 = mc[nt][1], nr = mr[nt];
        for (int q = 0; q < nb; ++q) {
          if (!(xf[par * TW + q] & 1)) continue;
          const float* rq = xr + ((par * TW + q) * NT + nt) * 8;
          n0 = fmaxf(n0, rq[2 * c]);
          n1 = fmaxf(n1, rq[2 * c + 1]);
          nr = fmaxf(nr, rq[r]);
        }
        const float a0 = fast_exp2(mc[nt][0] - n0), a1 = fast_exp2(mc[nt][1] - n1);  // 0 from -inf
        lk[nt][0] *= a0;
        lk[nt][1] *= a1;
#pragma unroll
        for (int j = 0; j < 2 * GW; ++j) {
          acc[j][nt][0] *= a0;
          acc[j][nt][2] *= a0;
          acc[j][nt][1] *= a1;
          acc[j][nt][3] *= a1;
        }
        // this warp's page: its sums move to the new references
        lk[nt][0] = fmaf(lp[nt][0], rf[nt][0] == -INFINITY ? 0.f : fast_exp2(rf[nt][0] - n0), lk[nt][0]);
        lk[nt][1] = fmaf(lp[nt][1], rf[nt][1] == -INFINITY ? 0.f : fast_exp2(rf[nt][1] - n1), lk[nt][1]);
        mc[nt][0] = n0;
        mc[nt][1] = n1;
        mr[nt] = nr;
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        lk[nt][0] += lp[nt][0];
        lk[nt][1] += lp[nt][1];
      }
    }
    // V: every page of the batch, this warp's channel groups
    // No wait here: the page's K warp observed its copy complete (mbarrier acquire) before the
    // team barrier, whose memory ordering carries that to every warp of the team.
    auto v_page = [&](int q) {
      const int s = (b + q) % NST;
      {
        const uint8_t* pg = sm.ring + s * STAGE;
        uint2 pb[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) pb[nt] = xp[((par * TW + q) * NT + nt) * 32 + lane];
        const int fq = fl >> (2 * q);
        if (any_raised) {
          // column r: 2^(page reference - common reference), the page's own reference if it
          // raised, else the one before this batch
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float rq = (fq & 1) ? xr[((par * TW + q) * NT + nt) * 8 + r] : mr_old[nt];
            const float f = rq == -INFINITY ? 0.f : fast_exp2(rq - mr[nt]);
            const uint32_t f2 = pack_f16x2(f, f);  // <= 1 (0 for a column the page does not see)
            pb[nt].x = hmul2_u32(pb[nt].x, f2);
            pb[nt].y = hmul2_u32(pb[nt].y, f2);
          }
        }
        if constexpr (F == kFp8) {
          fp8_pv_nt<D, NT, GW>(acc, pg, lane, g0, pb);
        } else {
          if (!(fq & 2))
            tq3_pv_nt<D, NT, GW, false>(acc, pg, lane, vw, vs1, g0, pb);
          else
            tq3_pv_nt<D, NT, GW, true>(acc, pg, lane, vw, vs1, g0, pb);
        }
      }
    };
    if constexpr (K == kKindFused) {
      for (int q = 0; q < nb; ++q) v_page(q);
    } else {
      // unrolled over the batch (per-format grids: measured 4% faster; the fused grid, with
      // both formats' code in one kernel, runs slower unrolled)
#pragma unroll
      for (int q = 0; q < TW; ++q) {
        if (q >= nb) break;
        v_page(q);
      }
    }
    // this warp's reads of the batch's stages come before the async-proxy refills that follow
    // the next barrier
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  // drain (bounded) after a failed wait: the last copy issued into every stage lands before the
  // ring is reused
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      const int f = *reinterpret_cast<volatile int32_t*>(&sm.fills[s]);
      if (f > 0) mbar_wait(&sm.full[s], (f - 1) & 1, 100000000ull);
    }
  }
  __syncthreads();

  // combine: per n-tile, (m, l) of its 8 columns and acc [8][D] (every warp its channels); the
  // denominators are summed over the lanes of a column and then over the warps
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lk[nt][0] += __shfl_xor_sync(0xffffffffu, lk[nt][0], o);
      lk[nt][1] += __shfl_xor_sync(0xffffffffu, lk[nt][1], o);
    }
  float* cmb = reinterpret_cast<float*>(sm.ring);
  constexpr int REGION = 8 * (D + 2);
  float* lsum = cmb + NT * REGION;  // [TW][NT][8]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float* reg = cmb + nt * REGION;
    if (r == 0) {
      lsum[(warp * NT + nt) * 8 + 2 * c] = lk[nt][0];
      lsum[(warp * NT + nt) * 8 + 2 * c + 1] = lk[nt][1];
      if (warp == 0) {
        reg[2 * (2 * c)] = mc[nt][0];
        reg[2 * (2 * c + 1)] = mc[nt][1];
      }
    }
    float* ra = reg + 16;
#pragma unroll
    for (int j = 0; j < 2 * GW; ++j) {
      const int mt = 2 * g0 + j;
      const int ch0 = 32 * (mt >> 1) + 4 * r + 2 * (mt & 1), ch1 = ch0 + 1;
      ra[(2 * c) * D + ch0] = acc[j][nt][0];
      ra[(2 * c + 1) * D + ch0] = acc[j][nt][1];
      ra[(2 * c) * D + ch1] = acc[j][nt][2];
      ra[(2 * c + 1) * D + ch1] = acc[j][nt][3];
    }
  }
  __syncthreads();
  const int part = sd.part0 + u.part;
  for (int q = threadIdx.x; q < NT * 8 * (D / 4); q += C::THREADS) {
    const int nt = q / (8 * (D / 4)), rem = q % (8 * (D / 4));
    const int col = rem / (D / 4), ch = 4 * (rem % (D / 4));
    const int n = 8 * nt + col;
    if (n >= p.NC) continue;
    const float* reg = cmb + nt * REGION;
    const int64_t base = (static_cast<int64_t>(part) * p.Hkv + h) * p.NC + n;
    if (ch == 0) {
      float L = 0.f;
      for (int w = 0; w < TW; ++w) L += lsum[(w * NT + nt) * 8 + col];
      p.part_ml[2 * base] = reg[2 * col];
      p.part_ml[2 * base + 1] = L;
    }
    *reinterpret_cast<float4*>(p.part_acc + base * D + ch) =
        *reinterpret_cast<const float4*>(reg + 16 + col * D + ch);
  }
}

// Partial-attention kernel of one kind.  Grid = CTAs x KV heads: CTA c of KV head h takes
// units [cta_unit0[c], cta_unit0[c+1]) one after another.  The FP8 grid covers CTAs
// [0, n_fp8), the TQ3 grid [n_fp8, n_ctas), the fused and BF16 grids all of them.
template <int D, int NT, int K>
__device__ __forceinline__ void run_one(const DecodeParams& p, const UnitDesc& u, int h,
                                        const Smem& sm, bool again) {
  const SeqDesc& sd = p.seq[u.seq];
  if constexpr (Cfg<D, NT, K>::TEAM) {
    if constexpr (K == kKindFp8) {
      run_unit_team<D, NT, K, kFp8>(p, sd, u, h, sm, again);
    } else if constexpr (K == kKindTq3) {
      run_unit_team<D, NT, K, kTq3>(p, sd, u, h, sm, again);
    } else {
      if (u.fmt == kFp8)
        run_unit_team<D, NT, K, kFp8>(p, sd, u, h, sm, again);
      else
        run_unit_team<D, NT, K, kTq3>(p, sd, u, h, sm, again);
    }
  } else if constexpr (K == kKindFp8) {
    run_unit<D, NT, K, kFp8>(p, sd, u, h, sm, again);
  } else if constexpr (K == kKindTq3) {
    run_unit<D, NT, K, kTq3>(p, sd, u, h, sm, again);
  } else if constexpr (K == kKindBf16) {
    run_unit<D, NT, K, kBf16>(p, sd, u, h, sm, again);
  } else {
    if (u.fmt == kFp8)
      run_unit<D, NT, K, kFp8>(p, sd, u, h, sm, again);
    else
      run_unit<D, NT, K, kTq3>(p, sd, u, h, sm, again);
  }
}

// MULTI: some CTA of the grid takes more than one unit (the line cut); a grid whose CTAs take
// one unit each runs the variant without the unit loop.
template <int D, int NT, int K, bool MULTI>
__global__ void __launch_bounds__(Cfg<D, NT, K>::THREADS, Cfg<D, NT, K>::MINB)
    partial_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // let the next kernel of the call (the TQ3 grid or the merge) start once every CTA of this
  // grid is resident: it reads nothing this grid writes before its griddepcontrol.wait
  pdl_launch_dependents();
  const Smem sm = carve<D, NT, K>(smem_raw);
  const int h = blockIdx.x % p.Hkv;
  const int cta = (K == kKindTq3 ? p.n_fp8 : 0) + blockIdx.x / p.Hkv;
  const int k0 = p.cta_unit0[cta], k1 = p.cta_unit0[cta + 1];
  if constexpr (!MULTI) {
    run_one<D, NT, K>(p, p.unit[k0], h, sm, false);
  } else {
    for (int k = k0; k < k1; ++k) {
      run_one<D, NT, K>(p, p.unit[k], h, sm, k > k0);
      // every warp is done with the unit's combine (which reuses the ring) before the next
      // unit refills the ring; a bounded wait that ran out (status flagged) skips the rest
      __syncthreads();
      if (sm.misc[1]) break;
    }
  }
  // the TQ3 grid, a programmatic dependent of the FP8 grid, ends only after it: the merge, a
  // dependent of this grid, then sees both grids' partial states
  if constexpr (K == kKindTq3) pdl_wait();
}

// Per-instantiation launch set-up, done once: the dynamic shared-memory opt-in and the number of
// CTAs the SM keeps resident (the planner sizes work units from it).
template <int D, int NT, int K>
struct KernelInfo {
  cudaError_t err = cudaSuccess;
  int ctas_per_sm = 1;
  KernelInfo() {
    using C = Cfg<D, NT, K>;
    err = cudaFuncSetAttribute(partial_kernel<D, NT, K, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(partial_kernel<D, NT, K, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    int n = 0, m = 0;
    if (err == cudaSuccess)
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, partial_kernel<D, NT, K, false>,
                                                          C::THREADS, C::SMEM);
    if (err == cudaSuccess)
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, partial_kernel<D, NT, K, true>,
                                                          C::THREADS, C::SMEM);
    // the planner sizes one wave for either variant
    ctas_per_sm = n > 0 && m > 0 ? (n < m ? n : m) : 1;
  }
  static const KernelInfo& get() {
    static const KernelInfo info;
    return info;
  }
};

// Launch with or without the programmatic-dependent attribute (overlap with the previous
// kernel of the stream, which then has to be one that only triggers it).
template <class... Args>
cudaError_t launch_ex(void (*kernel)(Args...), dim3 grid, int threads, int smem, bool dependent,
                      cudaStream_t s, const DecodeParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Grid of CTAs [c0, c1) x KV heads, the unit-loop variant only where a CTA takes several units.
template <int D, int NT, int K>
cudaError_t launch_t(const DecodeParams& p, int c0, int c1, bool dependent, cudaStream_t s) {
  using C = Cfg<D, NT, K>;
  const KernelInfo<D, NT, K>& info = KernelInfo<D, NT, K>::get();
  if (info.err != cudaSuccess) return info.err;
  const bool multi = p.cta_unit0[c1] - p.cta_unit0[c0] > c1 - c0;
  return launch_ex(multi ? partial_kernel<D, NT, K, true> : partial_kernel<D, NT, K, false>,
                   dim3((c1 - c0) * p.Hkv), C::THREADS, C::SMEM, dependent, s, p);
}

template <int D, int K>
int ctas_per_sm_d(int nt) {
  switch (nt) {
    case 1: return KernelInfo<D, 1, K>::get().ctas_per_sm;
    case 2: return KernelInfo<D, 2, K>::get().ctas_per_sm;
    case 3: return KernelInfo<D, 3, K>::get().ctas_per_sm;
    default: return KernelInfo<D, 4, K>::get().ctas_per_sm;
  }
}

template <int D, int K>
cudaError_t launch_d(const DecodeParams& p, int c0, int c1, bool dependent, cudaStream_t s) {
  switch ((p.NC + 7) / 8) {
    case 1: return launch_t<D, 1, K>(p, c0, c1, dependent, s);
    case 2: return launch_t<D, 2, K>(p, c0, c1, dependent, s);
    case 3: return launch_t<D, 3, K>(p, c0, c1, dependent, s);
    case 4: return launch_t<D, 4, K>(p, c0, c1, dependent, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Launch the partial grid of kind K over CTAs [c0, c1) (of the launch's CTA table) for head
// dimension D; the number of CTAs of kind K an SM keeps resident with NC query columns.
template <int D>
cudaError_t launch_partial_kind(int K, const DecodeParams& p, int c0, int c1, bool dependent,
                                cudaStream_t s) {
  if (c1 <= c0) return cudaSuccess;
  switch (K) {
    case kKindFp8: return launch_d<D, kKindFp8>(p, c0, c1, dependent, s);
    case kKindTq3: return launch_d<D, kKindTq3>(p, c0, c1, dependent, s);
    case kKindFused: return launch_d<D, kKindFused>(p, c0, c1, dependent, s);
    case kKindBf16: return launch_d<D, kKindBf16>(p, c0, c1, dependent, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
int partial_ctas_per_sm_kind(int K, int NC) {
  const int nt = (NC + 7) / 8;
  switch (K) {
    case kKindFp8: return ctas_per_sm_d<D, kKindFp8>(nt);
    case kKindFused: return ctas_per_sm_d<D, kKindFused>(nt);
    case kKindBf16: return ctas_per_sm_d<D, kKindBf16>(nt);
    default: return ctas_per_sm_d<D, kKindTq3>(nt);
  }
}

}  // namespace mkv
