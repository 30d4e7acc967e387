// Decode attention directly over the mixed-format paged cache.
//
// "Minima-KV ..." (brainszone.ai pt page, section "Como os resultados parciais são
// combinados"; fr "Comment les résultats partiels sont assemblés"): a separate kernel per page
// format computes partial attention states, and an online-softmax merge with global
// normalisation combines them -- no page is converted to a common format first and no dense
// copy of the cache is made (section "... sem a chamada sombra densa").
//
// Three launches per call:
//   plan_kernel     per sequence, compacts the block-table row into an FP8 page list and a TQ3
//                   page list ({slot, logical page}), in logical order.
//   partial_kernel  per (sequence, KV head, split of one format's list): streams the pages of
//                   the split through a shared-memory ring with bulk async copies and computes
//                   (m, l, acc) for the GQA group's query columns.  FP8 CTAs and TQ3 CTAs run
//                   different code (fp8_page / tq3_page) and write separate partial states;
//                   they share one grid so the small FP8 share does not run alone on a few SMs.
//   merge_kernel    per (sequence, query column): M = max m, L = sum l 2^(m-M),
//                   O = sum acc 2^(m-M) / L.
//
// Tensor-core use: per page the logits are a 16-token x 8-column tile (tokens are the MMA M
// dimension, the q_len*g query columns of one KV head the N dimension) and P.V is a
// (16 channels x 16 tokens) x (16 tokens x 8 columns) tile, both mma.sync m16n8k16 with f16
// operands that are exact images of the stored codes.  Dequantisation happens in registers:
//   TQ3 K: codes -> (c - 3.5) exactly; the per-(token, group) scale multiplies the group's
//          MMA result (logits are summed over groups in fp32).
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
constexpr int kMaxListPerCta = 256;

template <int D, int NT>
struct Cfg {
  static constexpr int G = D / 32;
  static constexpr int PW = NT == 1 ? 4 : (NT == 2 ? 2 : 1);  // page-parallel warps
  static constexpr int NWC = NT * PW;                          // consumer warps
  static constexpr int THREADS = 32 * (NWC + 1);               // + 1 producer warp
  static constexpr int FP8_STAGE = 32 * D + 16;
  static constexpr int TQ3_STAGE = 14 * D;
  static constexpr int FP8_NST = 8;
  static constexpr int TQ3_NST = 16;
  static constexpr int RING_FP8 = FP8_NST * FP8_STAGE;
  static constexpr int RING_TQ3 = TQ3_NST * TQ3_STAGE;
  static constexpr int COMBINE = (PW - 1) * NT * 8 * (D + 2) * 4;
  static constexpr int RING = RING_FP8 > RING_TQ3 ? (RING_FP8 > COMBINE ? RING_FP8 : COMBINE)
                                                  : (RING_TQ3 > COMBINE ? RING_TQ3 : COMBINE);
  // header: 2 x 16 mbarriers, 16 stage tags, abort flag, list buffer
  static constexpr int HDR = 256 + 64 + 16 + kMaxListPerCta * 8;
  static constexpr int SMEM = HDR + RING;
};

struct Smem {
  uint64_t* full;
  uint64_t* empty;
  int32_t* tag;    // logical page of each stage (-1: invalid entry)
  int32_t* abort;
  int2* list;
  uint8_t* ring;
};

__device__ __forceinline__ Smem carve(uint8_t* base) {
  Smem s;
  s.full = reinterpret_cast<uint64_t*>(base);
  s.empty = s.full + 16;
  s.tag = reinterpret_cast<int32_t*>(base + 256);
  s.abort = reinterpret_cast<int32_t*>(base + 256 + 64);
  s.list = reinterpret_cast<int2*>(base + 256 + 64 + 16);
  s.ring = base + 256 + 64 + 16 + kMaxListPerCta * 8;
  return s;
}

__device__ __forceinline__ uint32_t f16x2_const(float lo, float hi) { return pack_f16x2(lo, hi); }

// Per-warp online-softmax state for the thread's two columns (2c, 2c+1) and its share of the
// P.V accumulator: acc[mt][0..3] = (channel row r, col 2c), (r, 2c+1), (r+8, 2c), (r+8, 2c+1)
// of channel tile mt; tile 2G+j row r holds channel 32G + 4r + 2j, row r+8 channel 32G+4r+2j+1.
template <int D>
struct WarpState {
  float m[2];
  float l[2];
  float acc[D / 16][4];
};

// Logits -> probabilities for one page (thread holds logits x[0..3] for tokens (r, r+8) x
// columns (2c, 2c+1), in log2 units).  Returns P^T as two B fragments (tokens 0-7, 8-15).
template <int D>
__device__ __forceinline__ void softmax_page(WarpState<D>& st, float (&x)[4], uint32_t& pb0,
                                             uint32_t& pb1) {
  float mx0 = fmaxf(x[0], x[2]);
  float mx1 = fmaxf(x[1], x[3]);
  const bool need = (mx0 > st.m[0] + kLazyRescale) || (mx1 > st.m[1] + kLazyRescale);
  if (__any_sync(0xffffffffu, need)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float n0 = fmaxf(st.m[0], mx0), n1 = fmaxf(st.m[1], mx1);
    const float a0 = (n0 == -INFINITY) ? 1.f : exp2f(st.m[0] - n0);
    const float a1 = (n1 == -INFINITY) ? 1.f : exp2f(st.m[1] - n1);
    if (a0 != 1.f || a1 != 1.f) {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.acc[mt][0] *= a0;
        st.acc[mt][2] *= a0;
        st.acc[mt][1] *= a1;
        st.acc[mt][3] *= a1;
      }
      st.l[0] *= a0;
      st.l[1] *= a1;
    }
    st.m[0] = n0;
    st.m[1] = n1;
  }
  const float r0 = st.m[0] == -INFINITY ? 0.f : st.m[0];
  const float r1 = st.m[1] == -INFINITY ? 0.f : st.m[1];
  const float p0 = exp2f(x[0] - r0), p1 = exp2f(x[1] - r1);
  const float p2 = exp2f(x[2] - r0), p3 = exp2f(x[3] - r1);
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
__device__ __forceinline__ void tq3_page(WarpState<D>& st, const uint8_t* pg,
                                         const uint32_t (&qb)[D / 32][4], int lane,
                                         float ls, int tok0, bool masked, int lim0, int lim1,
                                         int kw, int ks5, int vw, int vs1) {
  constexpr int G = D / 32;
  const int r = lane >> 2, c = lane & 3;
  const uint8_t* krec = pg;
  const __half* kscale = reinterpret_cast<const __half*>(pg + G * 16 * 12);
  const uint8_t* vrec = pg + G * 16 * 14;
  const __half* vscale = reinterpret_cast<const __half*>(vrec + G * 16 * 12);
  const uint32_t kMask = 0x000E00E0u, kMagic = 0x60005000u;
  const uint32_t kSub = f16x2_const(35.5f, 515.5f);

  float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t* ra = reinterpret_cast<const uint32_t*>(krec + 12 * (16 * g + r));
    const uint32_t* rb = ra + 24;  // token r + 8
    const uint32_t xa = __funnelshift_r(ra[kw], ra[kw + 1], ks5);
    const uint32_t xb = __funnelshift_r(rb[kw], rb[kw + 1], ks5);
    uint32_t a[4], b[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a[j] = hsub2_u32(((xa >> (3 * j)) & kMask) | kMagic, kSub);
      b[j] = hsub2_u32(((xb >> (3 * j)) & kMask) | kMagic, kSub);
    }
    float cg[4] = {0.f, 0.f, 0.f, 0.f};
    mma_f16_16816(cg, a[0], b[0], a[1], b[1], qb[g][0], qb[g][1], cg);
    mma_f16_16816(cg, a[2], b[2], a[3], b[3], qb[g][2], qb[g][3], cg);
    const float sa = __half2float(kscale[16 * g + r]);
    const float sb = __half2float(kscale[16 * g + r + 8]);
    x[0] = fmaf(sa, cg[0], x[0]);
    x[1] = fmaf(sa, cg[1], x[1]);
    x[2] = fmaf(sb, cg[2], x[2]);
    x[3] = fmaf(sb, cg[3], x[3]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] *= ls;
  if (masked) mask_page(x, tok0, r, lim0, lim1);
  uint32_t pb0, pb1;
  softmax_page<D>(st, x, pb0, pb1);

  // V: A = V^T tile (channels x tokens); lane row r holds channels 32G+4r+{0,1} (tile 2G)
  // and 32G+4r+{2,3} (tile 2G+1) for tokens (2c, 2c+1) and (2c+8, 2c+9).
  const uint32_t m0 = 0x000E000Eu, g0 = 0x60006000u, s0 = f16x2_const(515.5f, 515.5f);
  const uint32_t m1 = 0x00700070u, g1 = 0x54005400u, s1 = f16x2_const(67.5f, 67.5f);
  const uint32_t m2 = 0x03800380u, g2 = 0x48004800u, s2 = f16x2_const(11.5f, 11.5f);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t* rc = reinterpret_cast<const uint32_t*>(vrec + 12 * (16 * g + 2 * c));
    const uint32_t f0 = __funnelshift_r(rc[vw], rc[vw + 1], vs1);        // token 2c
    const uint32_t f1 = __funnelshift_r(rc[vw + 3], rc[vw + 4], vs1);    // token 2c+1
    const uint32_t f8 = __funnelshift_r(rc[vw + 24], rc[vw + 25], vs1);  // token 2c+8
    const uint32_t f9 = __funnelshift_r(rc[vw + 27], rc[vw + 28], vs1);  // token 2c+9
    const uint32_t z01 = __byte_perm(f0, f1, 0x5410);
    const uint32_t z89 = __byte_perm(f8, f9, 0x5410);
    const uint32_t a0 = hsub2_u32((z01 & m0) | g0, s0), b0 = hsub2_u32((z89 & m0) | g0, s0);
    const uint32_t a1 = hsub2_u32((z01 & m1) | g1, s1), b1 = hsub2_u32((z89 & m1) | g1, s1);
    const uint32_t a2 = hsub2_u32((z01 & m2) | g2, s2), b2 = hsub2_u32((z89 & m2) | g2, s2);
    const uint32_t a3 = hsub2_u32(((z01 >> 3) & m2) | g2, s2);
    const uint32_t b3 = hsub2_u32(((z89 >> 3) & m2) | g2, s2);
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
__device__ __forceinline__ void fp8_page(WarpState<D>& st, const uint8_t* pg,
                                         const uint32_t (&qb)[D / 16][2], int lane, float ls,
                                         int tok0, bool masked, int lim0, int lim1) {
  const int r = lane >> 2, c = lane & 3;
  const float sk = *reinterpret_cast<const float*>(pg + 32 * D);
  const float sv = *reinterpret_cast<const float*>(pg + 32 * D + 4);
  float cg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < D / 64; ++j) {
    const uint4 wa = *reinterpret_cast<const uint4*>(pg + r * D + 64 * j + 16 * c);
    const uint4 wb = *reinterpret_cast<const uint4*>(pg + (r + 8) * D + 64 * j + 16 * c);
    const uint32_t va[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t vb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mma_f16_16816(cg, e4m3x2_to_f16x2(va[i]), e4m3x2_to_f16x2(vb[i]),
                    e4m3x2_to_f16x2(va[i] >> 16), e4m3x2_to_f16x2(vb[i] >> 16),
                    qb[4 * j + i][0], qb[4 * j + i][1], cg);
    }
  }
  float x[4];
  const float lsk = ls * sk;
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = cg[j] * lsk;
  if (masked) mask_page(x, tok0, r, lim0, lim1);
  uint32_t pb0, pb1;
  softmax_page<D>(st, x, pb0, pb1);

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

// Query column n of this CTA's KV head -> (query index, query head).  Returns a pointer to the
// bf16 row or nullptr for padding columns.
__device__ __forceinline__ const uint16_t* q_row(const DecodeParams& p, const SeqDesc& sd,
                                                 int h, int n) {
  if (n >= p.NC) return nullptr;
  const int qi = n / p.g, hq = h * p.g + (n % p.g);
  return p.q + ((static_cast<int64_t>(sd.out_row) * p.q_len + qi) * p.Hq + hq) * p.D;
}

__device__ __forceinline__ uint32_t q_pair(float a, float b, float scale) {
  return pack_f16x2(a * scale, b * scale);
}

// Power-of-two factor bringing the warp's largest |q| into [2^13, 2^14) so that the f16 images
// of the bf16 queries keep their precision; returns the factor, *inv its inverse.
__device__ __forceinline__ float q_prescale(float amax, float* inv) {
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int e = 0;
  if (amax > 0.f && isfinite(amax)) {
    frexpf(amax, &e);  // amax in [2^(e-1), 2^e)
    e = 14 - e;
    e = max(-100, min(100, e));
  }
  *inv = ldexpf(1.f, -e);
  return ldexpf(1.f, e);
}

template <int D, int NT, bool FP8>
__device__ void run_partial(const DecodeParams& p, const SeqDesc& sd, int h, int list_off,
                            int count, int part, Smem sm) {
  using C = Cfg<D, NT>;
  constexpr int STAGE = FP8 ? C::FP8_STAGE : C::TQ3_STAGE;
  constexpr int NST = FP8 ? C::FP8_NST : C::TQ3_NST;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], NT);
    }
    *sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == C::NWC) {
    const int2* lst = p.lists + list_off;
    for (int i = lane; i < count; i += 32) sm.list[i] = lst[i];
  }
  __syncthreads();

  WarpState<D> st;
  const int nt = warp % NT, pw = warp / NT;

  if (warp == C::NWC) {
    // ---------------- producer: one lane streams the split's pages into the ring
    if (lane == 0) {
      const uint8_t* slab = FP8 ? p.fp8_slab : p.tq3_slab;
      const int64_t slot_bytes = FP8 ? p.fp8_slot_bytes : p.tq3_slot_bytes;
      const int nslots = FP8 ? p.fp8_slots : p.tq3_slots;
      int issued = 0;
      for (int i = 0; i < count; ++i) {
        const int s = i % NST;
        if (i >= NST && !mbar_wait(&sm.empty[s], ((i / NST) - 1) & 1)) {
          flag_status(p.status, kStatusTimeout);
          atomicExch(sm.abort, 1);
          break;
        }
        const int2 e = sm.list[i];
        const bool ok = static_cast<unsigned>(e.x) < static_cast<unsigned>(nslots) && e.y >= 0;
        sm.tag[s] = ok ? e.y : -1;
        if (ok) {
          mbar_arrive_expect_tx(&sm.full[s], STAGE);
          bulk_g2s(sm.ring + s * STAGE,
                   slab + static_cast<int64_t>(e.x) * slot_bytes + static_cast<int64_t>(h) * STAGE,
                   STAGE, &sm.full[s]);
        } else {
          flag_status(p.status, kStatusCheck);
          mbar_arrive(&sm.full[s]);
        }
        issued = i + 1;
      }
      if (*reinterpret_cast<volatile int32_t*>(sm.abort)) {
        // drain: wait (bounded) for the last fill of every stage so no copy is in flight
        for (int i = max(0, issued - NST); i < issued; ++i)
          mbar_wait(&sm.full[i % NST], (i / NST) & 1, 100000000ull);
      }
    }
  } else {
    // ---------------- consumers
    const int n0 = 8 * nt + 2 * c, n1 = n0 + 1;
    const int lim0 = n0 < p.NC ? sd.ctx - p.q_len + n0 / p.g : sd.ctx - 1;
    const int lim1 = n1 < p.NC ? sd.ctx - p.q_len + n1 / p.g : sd.ctx - 1;
    const int min_lim = sd.ctx - p.q_len;
    // Q fragment of column 8nt + r, in this format's channel order
    const uint16_t* qr = q_row(p, sd, h, 8 * nt + r);
    constexpr int QW = FP8 ? D / 16 : D / 32;
    constexpr int QB = FP8 ? 2 : 4;
    uint32_t qb[QW][QB];
    float qv[D / 4];  // this lane's D/4 query values in fragment order
    float amax = 0.f;
    if constexpr (FP8) {
#pragma unroll
      for (int j = 0; j < D / 64; ++j) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float v = qr ? bf16_bits_to_float(qr[64 * j + 16 * c + e]) : 0.f;
          qv[16 * j + e] = v;
          amax = fmaxf(amax, fabsf(v));
        }
      }
    } else {
#pragma unroll
      for (int g = 0; g < D / 32; ++g) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = qr ? bf16_bits_to_float(qr[32 * g + 8 * c + e]) : 0.f;
          qv[8 * g + e] = v;
          amax = fmaxf(amax, fabsf(v));
        }
      }
    }
    float inv;
    const float qs = q_prescale(amax, &inv);
    if constexpr (FP8) {
#pragma unroll
      for (int kb = 0; kb < D / 16; ++kb) {
        const float* v = qv + 4 * kb;  // channels 64j+16c+4i+{0..3}, kb = 4j+i
        qb[kb][0] = q_pair(v[0], v[1], qs);
        qb[kb][1] = q_pair(v[2], v[3], qs);
      }
    } else {
#pragma unroll
      for (int g = 0; g < D / 32; ++g) {
        const float* v = qv + 8 * g;   // channels 32g+8c+{0..7}
#pragma unroll
        for (int j = 0; j < 4; ++j) qb[g][j % QB] = q_pair(v[j], v[j + 4], qs);
      }
    }
    const float ls = p.logit_scale * inv;
    // TQ3 lane constants: K chunk c of a record starts at bit 24c; we read bits from 24c-5
    // (codes land at 5+3k); V field of row r starts at bit 12r; we read from 12r-1.
    const int kbit = 24 * c - 5, vbit = 12 * r - 1;
    const int kw = kbit >= 0 ? kbit >> 5 : -1, ks5 = kbit & 31;
    const int vw = vbit >= 0 ? vbit >> 5 : -1, vs1 = vbit & 31;

    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[mt][e] = 0.f;

    for (int i = pw; i < count; i += C::PW) {
      const int s = i % NST;
      if (!mbar_wait(&sm.full[s], (i / NST) & 1)) {
        flag_status(p.status, kStatusTimeout);
        atomicExch(sm.abort, 1);
        break;
      }
      const int logical = sm.tag[s];
      if (logical >= 0) {
        const int tok0 = 16 * logical;
        const bool masked = tok0 + 15 > min_lim;
        const uint8_t* pg = sm.ring + s * STAGE;
        if constexpr (FP8)
          fp8_page<D>(st, pg, qb, lane, ls, tok0, masked, lim0, lim1);
        else
          tq3_page<D>(st, pg, qb, lane, ls, tok0, masked, lim0, lim1, kw, ks5, vw, vs1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      st.l[0] += __shfl_xor_sync(0xffffffffu, st.l[0], o);
      st.l[1] += __shfl_xor_sync(0xffffffffu, st.l[1], o);
    }
  }
  __syncthreads();  // ring no longer needed: reuse it for the cross-warp combine

  float* cmb = reinterpret_cast<float*>(sm.ring);
  constexpr int REGION = 8 * (D + 2);
  if (warp < C::NWC && pw > 0) {
    float* reg = cmb + ((pw - 1) * NT + nt) * REGION;
    if (r == 0) {
      reg[2 * (2 * c)] = st.m[0];
      reg[2 * (2 * c) + 1] = st.l[0];
      reg[2 * (2 * c + 1)] = st.m[1];
      reg[2 * (2 * c + 1) + 1] = st.l[1];
    }
    float* ra = reg + 16;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const int ch = 32 * (mt >> 1) + 4 * r + 2 * (mt & 1);
      ra[(2 * c) * D + ch] = st.acc[mt][0];
      ra[(2 * c + 1) * D + ch] = st.acc[mt][1];
      ra[(2 * c) * D + ch + 1] = st.acc[mt][2];
      ra[(2 * c + 1) * D + ch + 1] = st.acc[mt][3];
    }
  }
  __syncthreads();
  if (warp < C::NWC && pw == 0) {
    for (int o = 1; o < C::PW; ++o) {
      const float* reg = cmb + ((o - 1) * NT + nt) * REGION;
      const float* ra = reg + 16;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int col = 2 * c + k;
        const float mo = reg[2 * col], lo = reg[2 * col + 1];
        const float M = fmaxf(st.m[k], mo);
        if (M == -INFINITY) continue;
        const float as = st.m[k] == -INFINITY ? 0.f : exp2f(st.m[k] - M);
        const float ao = mo == -INFINITY ? 0.f : exp2f(mo - M);
        st.l[k] = st.l[k] * as + lo * ao;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int ch = 32 * (mt >> 1) + 4 * r + 2 * (mt & 1);
          st.acc[mt][k] = st.acc[mt][k] * as + ra[col * D + ch] * ao;
          st.acc[mt][k + 2] = st.acc[mt][k + 2] * as + ra[col * D + ch + 1] * ao;
        }
        st.m[k] = M;
      }
    }
    // write the partial state of columns 8nt + 2c + k
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int n = 8 * nt + 2 * c + k;
      if (n >= p.NC) continue;
      const int64_t base = (static_cast<int64_t>(part) * p.Hkv + h) * p.NC + n;
      if (r == 0) {
        p.part_ml[2 * base] = st.m[k];
        p.part_ml[2 * base + 1] = st.l[k];
      }
      float* dst = p.part_acc + base * D;
#pragma unroll
      for (int g = 0; g < D / 32; ++g) {
        const float4 v = make_float4(st.acc[2 * g][k], st.acc[2 * g][k + 2],
                                     st.acc[2 * g + 1][k], st.acc[2 * g + 1][k + 2]);
        *reinterpret_cast<float4*>(dst + 32 * g + 4 * r) = v;
      }
    }
  }
}

template <int D, int NT>
__global__ void __launch_bounds__(Cfg<D, NT>::THREADS, 2)
    partial_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const int x = blockIdx.x, h = blockIdx.y;
  // sequence of this CTA: last s with seq[s].cta0 <= x
  int lo = 0, hi = p.n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seq[mid].cta0 <= x) lo = mid; else hi = mid - 1;
  }
  const SeqDesc& sd = p.seq[lo];
  const int local = x - sd.cta0;
  const int part = sd.part0 + local;
  if (local < sd.split8) {
    const int first = local * p.P8;
    const int count = min(p.P8, sd.n8 - first);
    run_partial<D, NT, true>(p, sd, h, sd.list8 + first, count, part, sm);
  } else {
    const int first = (local - sd.split8) * p.P3;
    const int count = min(p.P3, sd.n3 - first);
    run_partial<D, NT, false>(p, sd, h, sd.list3 + first, count, part, sm);
  }
}

// ------------------------------------------------------------------ plan
__global__ void __launch_bounds__(256) plan_kernel(const __grid_constant__ DecodeParams p) {
  __shared__ int w8[8], w3[8];
  const SeqDesc& sd = p.seq[blockIdx.x];
  const int32_t* row = p.tables + static_cast<int64_t>(sd.row) * p.max_pages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int base8 = 0, base3 = 0;
  for (int b = 0; b < sd.n_pages; b += 256) {
    const int idx = b + threadIdx.x;
    const bool valid = idx < sd.n_pages;
    const int32_t e = valid ? row[idx] : -1;
    const uint32_t fmt = static_cast<uint32_t>(e) >> kFmtShift;
    const int slot = static_cast<int>(static_cast<uint32_t>(e) & kSlotMask);
    const bool good = valid && e >= 0 && fmt <= 1 &&
                      slot < (fmt == 0 ? p.fp8_slots : p.tq3_slots);
    if (valid && !good) flag_status(p.status, kStatusCheck);
    const bool is8 = good && fmt == 0, is3 = good && fmt == 1;
    const unsigned b8 = __ballot_sync(0xffffffffu, is8), b3 = __ballot_sync(0xffffffffu, is3);
    if (lane == 0) {
      w8[warp] = __popc(b8);
      w3[warp] = __popc(b3);
    }
    __syncthreads();
    int off8 = 0, off3 = 0, tot8 = 0, tot3 = 0;
    for (int w = 0; w < 8; ++w) {
      if (w < warp) {
        off8 += w8[w];
        off3 += w3[w];
      }
      tot8 += w8[w];
      tot3 += w3[w];
    }
    if (is8) {
      const int rank = base8 + off8 + __popc(b8 & lt);
      if (rank < sd.n8) p.lists[sd.list8 + rank] = make_int2(slot, idx);
      else flag_status(p.status, kStatusCheck);
    }
    if (is3) {
      const int rank = base3 + off3 + __popc(b3 & lt);
      if (rank < sd.n3) p.lists[sd.list3 + rank] = make_int2(slot, idx);
      else flag_status(p.status, kStatusCheck);
    }
    base8 += tot8;
    base3 += tot3;
    __syncthreads();
  }
  if (base8 != sd.n8 || base3 != sd.n3) {
    if (threadIdx.x == 0) flag_status(p.status, kStatusCheck);
    for (int i = base8 + threadIdx.x; i < sd.n8; i += 256) p.lists[sd.list8 + i] = make_int2(-1, -1);
    for (int i = base3 + threadIdx.x; i < sd.n3; i += 256) p.lists[sd.list3 + i] = make_int2(-1, -1);
  }
}

// ------------------------------------------------------------------ merge
// grid (sequence, KV head * NC); one thread per channel.
__global__ void __launch_bounds__(256) merge_kernel(const __grid_constant__ DecodeParams p) {
  const SeqDesc& sd = p.seq[blockIdx.x];
  const int h = blockIdx.y / p.NC, n = blockIdx.y % p.NC;
  const int S = sd.split8 + sd.split3;
  const int64_t stride = static_cast<int64_t>(p.Hkv) * p.NC;
  const int64_t first = (static_cast<int64_t>(sd.part0) * p.Hkv + h) * p.NC + n;
  float M = -INFINITY;
  for (int j = 0; j < S; ++j) M = fmaxf(M, p.part_ml[2 * (first + j * stride)]);
  const int qi = n / p.g, hq = h * p.g + n % p.g;
  float* out = p.out + ((static_cast<int64_t>(sd.out_row) * p.q_len + qi) * p.Hq + hq) * p.D;
  for (int d = threadIdx.x; d < p.D; d += blockDim.x) {
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int j = 0; j < S; ++j) {
        const int64_t b = first + j * stride;
        const float m = p.part_ml[2 * b];
        if (m == -INFINITY) continue;
        const float w = exp2f(m - M);
        L = fmaf(w, p.part_ml[2 * b + 1], L);
        O = fmaf(w, p.part_acc[b * p.D + d], O);
      }
    }
    out[d] = L > 0.f ? O / L : 0.f;
  }
}

template <int D, int NT>
cudaError_t launch_partial_t(const DecodeParams& p, cudaStream_t s) {
  using C = Cfg<D, NT>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(partial_kernel<D, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  partial_kernel<D, NT><<<dim3(p.total_ctas, p.Hkv), C::THREADS, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_partial_d(const DecodeParams& p, cudaStream_t s) {
  switch ((p.NC + 7) / 8) {
    case 1: return launch_partial_t<D, 1>(p, s);
    case 2: return launch_partial_t<D, 2>(p, s);
    case 3: return launch_partial_t<D, 3>(p, s);
    case 4: return launch_partial_t<D, 4>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool partial_supported(int D, int NC) {
  return (D == 64 || D == 128 || D == 256) && NC >= 1 && NC <= 32;
}

cudaError_t launch_plan(const DecodeParams& p, cudaStream_t s) {
  plan_kernel<<<p.n_seqs, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_partial(const DecodeParams& p, cudaStream_t s) {
  if (p.total_ctas <= 0) return cudaSuccess;
  switch (p.D) {
    case 64: return launch_partial_d<64>(p, s);
    case 128: return launch_partial_d<128>(p, s);
    case 256: return launch_partial_d<256>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_merge(const DecodeParams& p, cudaStream_t s) {
  merge_kernel<<<dim3(p.n_seqs, p.Hkv * p.NC), p.D < 256 ? p.D : 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mkv
