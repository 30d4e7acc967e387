// Decode attention directly over the mixed-format paged cache.
//
// "Minima-KV ..." (brainszone.ai pt page, section "Como os resultados parciais são
// combinados"; fr "Comment les résultats partiels sont assemblés"): a separate kernel per page
// format computes partial attention states, and an online-softmax merge with global
// normalisation combines them -- no page is converted to a common format first and no dense
// copy of the cache is made (section "... sem a chamada sombra densa").
//
// Two launches per call.  The host cuts every sequence into work units -- (format, logical page
// range) -- and orders them largest first.  A CTA takes one (unit, KV head):
//   1. its producer warp scans the block-table entries of the range and keeps the pages of the
//      unit's format (FP8 units run fp8_page, TQ3 units tq3_page: separate per-format code and
//      separate partial states);
//   2. the producer streams those pages through a shared-memory ring with bulk async copies
//      completing on mbarriers;
//   3. consumer warps (pages round-robin) compute per page the logits, the online softmax
//      (running max m and denominator l per query column) and P.V;
//   4. the CTA combines its warps and writes its partial state (m, l, acc) per query column.
// A second kernel merges, per (sequence, KV head, query column), all partial states of both
// formats: M = max m, L = sum l 2^(m-M), O = sum acc 2^(m-M) / L.
//
// Tensor-core use: per page the logits are a 16-token x 8-column tile (tokens are the MMA M
// dimension, the q_len*g query columns of one KV head the N dimension) and P.V is a
// (16 channels x 16 tokens) x (16 tokens x 8 columns) tile, both mma.sync m16n8k16 with f16
// operands that are exact images of the stored codes.  Dequantisation happens in registers:
//   TQ3 K: codes -> exact f16 images (base + c); each group's MMA starts from the correction
//          -(base + 3.5) * (sum of the matching query values), so it yields sum q (c - 3.5);
//          the per-(token, group) scale multiplies the group's result (summed in fp32).
//   TQ3 V: codes -> (c - 3.5) exactly; the per-(token, group) scale multiplies P in f16.
//   FP8:   e4m3x2 -> f16x2 conversions; the per-page scales multiply logits / the page's P.V.
// Softmax runs in log2 units with a lazily raised reference maximum (raised only when a
// logit exceeds it by more than 8), so probabilities fed to the MMA are < 2^8.
#include <cfloat>

#include "device_util.cuh"
#include "mkv_internal.h"

namespace mkv {

namespace {

constexpr float kLazyRescale = 8.f;  // log2 units

template <int D, int NT>
struct Cfg {
  static constexpr int PW = NT == 1 ? 4 : (NT == 2 ? 2 : 1);  // page-parallel warps
  static constexpr int NWC = NT * PW;                          // consumer warps
  static constexpr int THREADS = 32 * (NWC + 1);               // + 1 producer warp
  static constexpr int PRODUCER = NWC;
  static constexpr int FP8_STAGE = 32 * D + 16;
  static constexpr int TQ3_STAGE = 14 * D;
  // Every stage must always be consumed by the same warp(s): a warp waits on a stage's fill f
  // with parity f & 1, which is only unambiguous if fill f-1 of that stage was its own (and so
  // already completed).  Hence ring depths are multiples of PW.
  static constexpr int FP8_NST = 8;
  static constexpr int TQ3_NST = 16;
  static_assert(FP8_NST % PW == 0 && TQ3_NST % PW == 0, "stage ownership");
  static constexpr int RING_FP8 = FP8_NST * FP8_STAGE;
  static constexpr int RING_TQ3 = TQ3_NST * TQ3_STAGE;
  // end-of-unit combine: (m, l) and acc of every consumer warp
  static constexpr int COMBINE = PW * NT * 8 * (D + 2) * 4;
  static constexpr int RING = RING_FP8 > RING_TQ3 ? (RING_FP8 > COMBINE ? RING_FP8 : COMBINE)
                                                  : (RING_TQ3 > COMBINE ? RING_TQ3 : COMBINE);
  // header: full[16] | empty[16] mbarriers | stage tags | misc | page list | Q fragments |
  //         TQ3 K corrections | ring
  static constexpr int OFF_TAG = 256;
  static constexpr int OFF_MISC = OFF_TAG + 64;
  static constexpr int OFF_LIST = OFF_MISC + 64;
  static constexpr int OFF_QF = (OFF_LIST + kMaxPagesPerUnit * 8 + 127) / 128 * 128;
  static constexpr int QF = NT * D * 16;
  static constexpr int OFF_CORR = OFF_QF + QF;
  static constexpr int OFF_RING = (OFF_CORR + NT * (D / 32) * 64 + 127) / 128 * 128;
  static constexpr int SMEM = OFF_RING + RING;
};

struct Smem {
  uint64_t* full;   // [stage]: page landed (producer arrive + bulk-copy bytes)
  uint64_t* empty;  // [stage]: the page's consumer warps are done with it
  int32_t* tag;     // logical page of each stage
  int32_t* misc;    // [0] page count, [1] abort flag, [4..7] logit scales per n-tile
  int2* list;       // {slot, logical page} of the unit's pages
  uint4* qf;        // Q fragments [NT][D/32][32 lanes]
  float4* corr;     // TQ3 K corrections [NT][D/32][4 column pairs] as {c0, c1, c0, c1}
  uint8_t* ring;
};

template <int D, int NT>
__device__ __forceinline__ Smem carve(uint8_t* base) {
  using C = Cfg<D, NT>;
  Smem s;
  s.full = reinterpret_cast<uint64_t*>(base);
  s.empty = s.full + 16;
  s.tag = reinterpret_cast<int32_t*>(base + C::OFF_TAG);
  s.misc = reinterpret_cast<int32_t*>(base + C::OFF_MISC);
  s.list = reinterpret_cast<int2*>(base + C::OFF_LIST);
  s.qf = reinterpret_cast<uint4*>(base + C::OFF_QF);
  s.corr = reinterpret_cast<float4*>(base + C::OFF_CORR);
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
// columns (2c, 2c+1), in log2 units).  Gives P^T as two B fragments (tokens 0-7, 8-15) and the
// factors (a0, a1) by which earlier accumulations of the two columns must be rescaled (1 when
// the reference maximum did not move).
__device__ __forceinline__ void softmax_k(KState& st, float (&x)[4], uint32_t& pb0,
                                          uint32_t& pb1, float& a0, float& a1) {
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
  const float p0 = fast_exp2(x[0] - r0), p1 = fast_exp2(x[1] - r1);
  const float p2 = fast_exp2(x[2] - r0), p3 = fast_exp2(x[3] - r1);
  st.l[0] += p0 + p2;
  st.l[1] += p1 + p3;
  pb0 = movmatrix_trans(pack_f16x2(p0, p1));
  pb1 = movmatrix_trans(pack_f16x2(p2, p3));
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
__device__ __forceinline__ void tq3_logits(const uint8_t* pg, const uint4* qf, const float4* corr,
                                           int lane, int kw, int ks5, float (&x)[4]) {
  constexpr int G = D / 32;
  const int r = lane >> 2, c = lane & 3;
  const uint8_t* krec = pg;
  const __half* kscale = reinterpret_cast<const __half*>(pg + G * 16 * 12);
  // K images: code k of a pair lands in mantissa bits 7-9 of the low half (value 8 + c) and
  // code k+4 in bits 3-5 of the high half (value 128 + c); both exact.  The offsets 11.5 and
  // 131.5 (base + 3.5) times the query sums are the group's starting accumulator (corr).
  uint32_t kMask = 0x00380380u, kMagic = 0x58004800u;
  opaque(kMask, kMagic);
  x[0] = x[1] = x[2] = x[3] = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t* ra = reinterpret_cast<const uint32_t*>(krec + 12 * (16 * g + r));
    const uint32_t* rb = ra + 24;  // token r + 8
    const uint32_t xa = __funnelshift_r(ra[kw], ra[kw + 1], ks5);  // code j at bit 3j+5
    const uint32_t xb = __funnelshift_r(rb[kw], rb[kw + 1], ks5);
    const uint32_t a0 = and_or(xa << 2, kMask, kMagic), b0 = and_or(xb << 2, kMask, kMagic);
    const uint32_t a1 = and_or(xa >> 1, kMask, kMagic), b1 = and_or(xb >> 1, kMask, kMagic);
    const uint32_t a2 = and_or(xa >> 4, kMask, kMagic), b2 = and_or(xb >> 4, kMask, kMagic);
    const uint32_t a3 = and_or(xa >> 7, kMask, kMagic), b3 = and_or(xb >> 7, kMask, kMagic);
    const uint4 qb = qf[32 * g + lane];
    const float4 cr = corr[4 * g + c];
    float cg[4] = {cr.x, cr.y, cr.z, cr.w};
    mma_f16_16816(cg, a0, b0, a1, b1, qb.x, qb.y, cg);
    mma_f16_16816(cg, a2, b2, a3, b3, qb.z, qb.w, cg);
    const float sa = __half2float(kscale[16 * g + r]);
    const float sb = __half2float(kscale[16 * g + r + 8]);
    x[0] = fmaf(sa, cg[0], x[0]);
    x[1] = fmaf(sa, cg[1], x[1]);
    x[2] = fmaf(sb, cg[2], x[2]);
    x[3] = fmaf(sb, cg[3], x[3]);
  }
}

// V: A = V^T tile (channels x tokens); lane row r holds channels 32G+4r+{0,1} (tile 2G) and
// 32G+4r+{2,3} (tile 2G+1) for tokens (2c, 2c+1) and (2c+8, 2c+9); codes -> exact (c - 3.5);
// the per-(token, group) scale multiplies P in f16.
template <int D>
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
    const uint32_t sv0 = *reinterpret_cast<const uint32_t*>(vscale + 16 * g + 2 * c);
    const uint32_t sv8 = *reinterpret_cast<const uint32_t*>(vscale + 16 * g + 2 * c + 8);
    const uint32_t q0 = hmul2_u32(pb0, sv0), q1 = hmul2_u32(pb1, sv8);
    mma_f16_16816(st.acc[2 * g], a0, a1, b0, b1, q0, q1, st.acc[2 * g]);
    mma_f16_16816(st.acc[2 * g + 1], a2, a3, b2, b3, q0, q1, st.acc[2 * g + 1]);
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
      if (c == 0) {  // stored twice per column pair: {col 2k, col 2k+1, col 2k, col 2k+1}
        float* c4 = corr + 16 * w + 4 * (r >> 1) + (r & 1);
        c4[0] = part;
        c4[2] = part;
      }
    }
    qf[32 * w + lane] = f;
  }
  return p.logit_scale * ldexpf(1.f, -e);
}

// Producer warp: collect the unit's pages of format fmt from table entries [first, last).
__device__ __forceinline__ int scan_range(const DecodeParams& p, const int32_t* row, int first,
                                          int last, int fmt, int lane, int2* list) {
  const int nslots = fmt == 0 ? p.fp8_slots : p.tq3_slots;
  const unsigned lt = (1u << lane) - 1u;
  int count = 0;
  bool bad = false;
  for (int base = first; base < last; base += 256) {
    int32_t e[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int idx = base + 32 * j + lane;
      e[j] = idx < last ? row[idx] : -2;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int idx = base + 32 * j + lane;
      const uint32_t f = static_cast<uint32_t>(e[j]) >> kFmtShift;
      const int slot = static_cast<int>(static_cast<uint32_t>(e[j]) & kSlotMask);
      const bool mapped = e[j] >= 0;
      bad |= (idx < last) && (!mapped || f > 1 || slot >= (f == 0 ? p.fp8_slots : p.tq3_slots));
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

template <int D, int NT, bool FP8>
__device__ void run_unit(const DecodeParams& p, const SeqDesc& sd, const UnitDesc& u, int h,
                         Smem sm) {
  using C = Cfg<D, NT>;
  constexpr int STAGE = FP8 ? C::FP8_STAGE : C::TQ3_STAGE;
  constexpr int NST = FP8 ? C::FP8_NST : C::TQ3_NST;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
  const int nt = warp % NT, pw = warp / NT;

  const uint8_t* slab = FP8 ? p.fp8_slab : p.tq3_slab;
  const int64_t slot_bytes = FP8 ? p.fp8_slot_bytes : p.tq3_slot_bytes;
  if (warp == C::PRODUCER) {
    // the producer owns the ring set-up, so its first fills (which need no free stage) are in
    // flight while the consumers build their Q fragments
    if (lane == 0) {
      for (int s = 0; s < NST; ++s) {
        mbar_init(&sm.full[s], 1);
        mbar_init(&sm.empty[s], NT);
      }
      sm.misc[1] = 0;
      mbar_fence_init();
    }
    const int32_t* row = p.tables + static_cast<int64_t>(sd.row) * p.max_pages;
    const int n = scan_range(p, row, u.first, u.last, FP8 ? 0 : 1, lane, sm.list);
    __syncwarp();
    if (lane == 0) {
      sm.misc[0] = n;
      for (int i = 0; i < min(n, NST); ++i) {
        const int2 e = sm.list[i];
        sm.tag[i] = e.y;
        mbar_arrive_expect_tx(&sm.full[i], STAGE);
        bulk_g2s(sm.ring + i * STAGE,
                 slab + static_cast<int64_t>(e.x) * slot_bytes + static_cast<int64_t>(h) * STAGE,
                 STAGE, &sm.full[i]);
      }
    }
  } else if (pw == 0) {
    const float ls = build_q<D, FP8>(p, sd, h, nt, lane, sm.qf + nt * (D / 32) * 32,
                                     reinterpret_cast<float*>(sm.corr + nt * (D / 32) * 4));
    if (lane == 0) reinterpret_cast<float*>(sm.misc)[4 + nt] = ls;
  }
  __syncthreads();
  const int count = sm.misc[0];

  KState ks;
  VState<D> vs;
  ks.m[0] = ks.m[1] = -INFINITY;
  ks.l[0] = ks.l[1] = 0.f;
  if (warp == C::PRODUCER) {
    // ---------------- producer: one lane streams the unit's pages into the ring
    if (lane == 0) {
      int issued = min(count, NST);
      for (int i = issued; i < count; ++i) {
        const int s = i % NST;
        if (i >= NST && !mbar_wait(&sm.empty[s], ((i / NST) - 1) & 1)) {
          flag_status(p.status, kStatusTimeout);
          atomicExch(&sm.misc[1], 1);
          break;
        }
        const int2 e = sm.list[i];
        sm.tag[s] = e.y;
        mbar_arrive_expect_tx(&sm.full[s], STAGE);
        bulk_g2s(sm.ring + s * STAGE,
                 slab + static_cast<int64_t>(e.x) * slot_bytes + static_cast<int64_t>(h) * STAGE,
                 STAGE, &sm.full[s]);
        issued = i + 1;
      }
      if (*reinterpret_cast<volatile int32_t*>(&sm.misc[1])) {
        // drain: wait (bounded) for the last fill of every stage so no copy is in flight
        for (int i = max(0, issued - NST); i < issued; ++i)
          mbar_wait(&sm.full[i % NST], (i / NST) & 1, 100000000ull);
      }
    }
  } else {
    // ---------------- consumers: logits, online softmax, P.V per page
    const int n0 = 8 * nt + 2 * c, n1 = n0 + 1;
    const int lim0 = n0 < p.NC ? sd.ctx - p.q_len + n0 / p.g : sd.ctx - 1;
    const int lim1 = n1 < p.NC ? sd.ctx - p.q_len + n1 / p.g : sd.ctx - 1;
    const int min_lim = sd.ctx - p.q_len;
    const float ls = reinterpret_cast<const float*>(sm.misc)[4 + nt];
    const uint4* qf = sm.qf + nt * (D / 32) * 32;
    const float4* corr = sm.corr + nt * (D / 32) * 4;
    // TQ3 K chunk c of a record starts at bit 24c; read from bit 24c-5 (codes at 5+3k).
    // TQ3 V field of row r starts at bit 12r; read from bit 12r-1 (codes at 1+3k).
    const int kbit = 24 * c - 5, vbit = 12 * r - 1;
    const int kw = kbit >= 0 ? kbit >> 5 : -1, ks5 = kbit & 31;
    const int vw = vbit >= 0 ? vbit >> 5 : -1, vs1 = vbit & 31;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) vs.acc[mt][e] = 0.f;

    for (int i = pw; i < count; i += C::PW) {
      const int s = i % NST;
      if (!mbar_wait_warp(&sm.full[s], (i / NST) & 1)) {
        if (lane == 0) {
          flag_status(p.status, kStatusTimeout);
          atomicExch(&sm.misc[1], 1);
        }
        break;
      }
      const int tok0 = 16 * sm.tag[s];
      const uint8_t* pg = sm.ring + s * STAGE;
      float x[4];
      if constexpr (FP8)
        fp8_logits<D>(pg, qf, lane, x);
      else
        tq3_logits<D>(pg, qf, corr, lane, kw, ks5, x);
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] *= ls;
      if (tok0 + 15 > min_lim) mask_page(x, tok0, r, lim0, lim1);
      uint32_t pb0, pb1;
      float a0, a1;
      softmax_k(ks, x, pb0, pb1, a0, a1);
      if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          vs.acc[mt][0] *= a0;
          vs.acc[mt][2] *= a0;
          vs.acc[mt][1] *= a1;
          vs.acc[mt][3] *= a1;
        }
      }
      if constexpr (FP8)
        fp8_pv<D>(vs, pg, lane, pb0, pb1);
      else
        tq3_pv<D>(vs, pg, lane, vw, vs1, pb0, pb1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      ks.l[0] += __shfl_xor_sync(0xffffffffu, ks.l[0], o);
      ks.l[1] += __shfl_xor_sync(0xffffffffu, ks.l[1], o);
    }
  }
  __syncthreads();  // ring no longer needed: reuse it for the cross-warp combine

  // every page-parallel warp stores its state; then all of them combine a share of the
  // columns' channels: M = max m, l = sum l 2^(m-M), acc = sum acc 2^(m-M)
  float* cmb = reinterpret_cast<float*>(sm.ring);
  constexpr int REGION = 8 * (D + 2);  // per (warp, n-tile): (m, l) of 8 columns, then acc [8][D]
  if (warp < C::NWC) {
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
      const int ch = 32 * (mt >> 1) + 4 * r + 2 * (mt & 1);
      ra[(2 * c) * D + ch] = vs.acc[mt][0];
      ra[(2 * c + 1) * D + ch] = vs.acc[mt][1];
      ra[(2 * c) * D + ch + 1] = vs.acc[mt][2];
      ra[(2 * c + 1) * D + ch + 1] = vs.acc[mt][3];
    }
  }
  __syncthreads();
  if (warp < C::NWC) {
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

// Merge of the partial states of one (sequence, KV head, query column): the globally
// normalised combination M = max m, L = sum l 2^(m-M), O = sum acc 2^(m-M) / L.  The maximum and
// the weights are computed once in shared memory; the accumulation over partials is then a
// branch-free sum of independent float4 loads, split over thread groups and reduced at the end.
constexpr int kMergeThreads = 256;
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ DecodeParams p) {
  __shared__ float w[kDecodeMaxUnits];
  __shared__ float red[kMergeThreads / 32];
  __shared__ float4 part[kMergeThreads];
  const int pair = blockIdx.x / p.NC, n = blockIdx.x % p.NC;
  const SeqDesc& sd = p.seq[pair / p.Hkv];
  const int h = pair % p.Hkv;
  const int S = sd.n_parts, D = p.D, tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int64_t base0 = (static_cast<int64_t>(sd.part0) * p.Hkv + h) * p.NC + n;
  const int64_t stride = static_cast<int64_t>(p.Hkv) * p.NC;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml);
  float mloc = -INFINITY;
  for (int j = tid; j < S; j += kMergeThreads) mloc = fmaxf(mloc, ml[base0 + j * stride].x);
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if (lane == 0) red[wp] = mloc;
  __syncthreads();
  float M = -INFINITY;
  for (int i = 0; i < kMergeThreads / 32; ++i) M = fmaxf(M, red[i]);
  __syncthreads();
  float lloc = 0.f;
  for (int j = tid; j < S; j += kMergeThreads) {
    const float2 v = ml[base0 + j * stride];
    const float wj = (v.x == -INFINITY || M == -INFINITY) ? 0.f : exp2f(v.x - M);
    w[j] = wj;
    lloc = fmaf(wj, v.y, lloc);
  }
  for (int o = 16; o > 0; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
  if (lane == 0) red[wp] = lloc;
  __syncthreads();
  float L = 0.f;
  for (int i = 0; i < kMergeThreads / 32; ++i) L += red[i];
  // accumulation: thread = (subset k of the partials, group c4 of 4 channels)
  const int groups = D / 4, nsub = kMergeThreads / groups;
  const int c4 = tid % groups, k = tid / groups;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* acc = reinterpret_cast<const float4*>(p.part_acc);
#pragma unroll 8
  for (int j = k; j < S; j += nsub) {
    const float4 a = acc[(base0 + j * stride) * groups + c4];
    const float wj = w[j];
    O.x = fmaf(wj, a.x, O.x);
    O.y = fmaf(wj, a.y, O.y);
    O.z = fmaf(wj, a.z, O.z);
    O.w = fmaf(wj, a.w, O.w);
  }
  part[tid] = O;
  __syncthreads();
  if (tid < groups) {
    float4 t = part[tid];
    for (int i = 1; i < nsub; ++i) {
      const float4 u = part[tid + i * groups];
      t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int qi = n / p.g, hq = h * p.g + n % p.g;
    float* out = p.out + ((static_cast<int64_t>(sd.out_row) * p.q_len + qi) * p.Hq + hq) * D;
    reinterpret_cast<float4*>(out)[tid] = make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
  }
}

template <int D, int NT>
__global__ void __launch_bounds__(Cfg<D, NT>::THREADS, D == 256 ? 3 : 4)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Smem sm = carve<D, NT>(smem_raw);
  const int h = blockIdx.x % p.Hkv;
  const UnitDesc& u = p.unit[blockIdx.x / p.Hkv];
  const SeqDesc& sd = p.seq[u.seq];
  if (u.fmt == 0)
    run_unit<D, NT, true>(p, sd, u, h, sm);
  else
    run_unit<D, NT, false>(p, sd, u, h, sm);
}

// Per-instantiation launch set-up, done once: the dynamic shared-memory opt-in and the number of
// CTAs the SM keeps resident (the planner sizes work units from it).
template <int D, int NT>
struct KernelInfo {
  cudaError_t err = cudaSuccess;
  int ctas_per_sm = 1;
  KernelInfo() {
    using C = Cfg<D, NT>;
    err = cudaFuncSetAttribute(decode_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM);
    int n = 0;
    if (err == cudaSuccess)
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<D, NT>, C::THREADS,
                                                          C::SMEM);
    ctas_per_sm = n > 0 ? n : 1;
  }
  static const KernelInfo& get() {
    static const KernelInfo info;
    return info;
  }
};

template <int D, int NT>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  using C = Cfg<D, NT>;
  const KernelInfo<D, NT>& info = KernelInfo<D, NT>::get();
  if (info.err != cudaSuccess) return info.err;
  decode_kernel<D, NT><<<p.n_units * p.Hkv, C::THREADS, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

template <int D>
int ctas_per_sm_d(int nt) {
  switch (nt) {
    case 1: return KernelInfo<D, 1>::get().ctas_per_sm;
    case 2: return KernelInfo<D, 2>::get().ctas_per_sm;
    case 3: return KernelInfo<D, 3>::get().ctas_per_sm;
    default: return KernelInfo<D, 4>::get().ctas_per_sm;
  }
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, cudaStream_t s) {
  switch ((p.NC + 7) / 8) {
    case 1: return launch_t<D, 1>(p, s);
    case 2: return launch_t<D, 2>(p, s);
    case 3: return launch_t<D, 3>(p, s);
    case 4: return launch_t<D, 4>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int partial_ctas_per_sm(int D, int NC) {
  const int nt = (NC + 7) / 8;
  switch (D) {
    case 64: return ctas_per_sm_d<64>(nt);
    case 128: return ctas_per_sm_d<128>(nt);
    default: return ctas_per_sm_d<256>(nt);
  }
}

bool partial_supported(int D, int NC) {
  return (D == 64 || D == 128 || D == 256) && NC >= 1 && NC <= 32;
}

cudaError_t launch_merge(const DecodeParams& p, cudaStream_t s) {
  if (p.n_seqs <= 0) return cudaSuccess;
  merge_kernel<<<p.n_seqs * p.Hkv * p.NC, kMergeThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_partial(const DecodeParams& p, cudaStream_t s) {
  if (p.n_units <= 0) return cudaSuccess;
  switch (p.D) {
    case 64: return launch_d<64>(p, s);
    case 128: return launch_d<128>(p, s);
    case 256: return launch_d<256>(p, s);
    default: return cudaErrorInvalidValue;
  }
}


// ------------------------------------------------------------------ static decode scratch
// Partial-state scratch for mkv_decode_attention_noalloc: a file-scope device array, so that
// callers that cannot allocate device memory can still decode.  Every device that loads the
// library holds it until exit; all calls share it.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device.  The first call on a device
// resolves it with cudaGetSymbolAddress (with that device current) and caches it; later calls
// only read the cache.
cudaError_t static_decode_scratch(void** ptr, size_t* bytes) {
  constexpr int kMaxDevices = 64;
  static void* cache[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = __atomic_load_n(&cache[dev], __ATOMIC_ACQUIRE);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    __atomic_store_n(&cache[dev], p, __ATOMIC_RELEASE);
  }
  *ptr = p;
  *bytes = kStaticScratchBytes;
  return cudaSuccess;
}

}  // namespace mkv
