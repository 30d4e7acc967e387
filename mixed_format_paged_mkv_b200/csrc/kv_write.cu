// Page writers of the mixed-format cache: FP8 append (with rescale-on-grow), FP8 -> TQ3
// demotion, and slot copies.  ("Minima-KV ...", brainszone.ai pt page, section "Âncoras em
// FP8, arquivo em TQ3": recent/anchor pages FP8, older pages converted to packed TQ3.)
//
// Bit-exactness: every rounding step is an explicit IEEE operation (__fdiv_rn, __fmul_rn,
// round-to-nearest-even conversions), so the codes and scales are identical to a float64
// host computation that applies the same roundings.
#include "device_util.cuh"
#include "mkv_internal.h"
#include "selftest.h"

namespace mkv {

namespace {

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

// One block per (touched page, KV head, K-or-V).
//   a = max|x| over the new tokens; cand = fp32(a/448)
//   empty page: scale = cand; cand > old: re-encode existing codes to cand; else keep old
//   new codes = e4m3(fp32(x/scale)) (0 when scale == 0)
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  __shared__ float red[8];
  const AppendDesc d = p.desc[blockIdx.x];
  const int h = blockIdx.y, which = blockIdx.z, D = p.D;
  if (p.bf16) {
    // BF16 control page: the rows are stored as they are; a fresh page zeroes its other rows
    uint16_t* rows = reinterpret_cast<uint16_t*>(p.fp8_slab + static_cast<int64_t>(d.slot) * p.slot_bytes +
                                                 static_cast<int64_t>(h) * (64 * D)) +
                     which * kPageTokens * D;
    const uint16_t* src = (which ? p.v : p.k) + (static_cast<int64_t>(d.first_row) * p.Hkv + h) * D;
    const int64_t src_stride = static_cast<int64_t>(p.Hkv) * D;
    bool finite = true;
    for (int i = threadIdx.x; i < d.n_new * D; i += blockDim.x) {
      const uint16_t b = src[(i / D) * src_stride + (i % D)];
      finite &= (b & 0x7F80u) != 0x7F80u;
      rows[d.n_old * D + i] = b;
    }
    if (__syncthreads_or(!finite) && threadIdx.x == 0) flag_status(p.status, kStatusCheck);
    if (d.n_old == 0)
      for (int i = d.n_new * D + threadIdx.x; i < kPageTokens * D; i += blockDim.x) rows[i] = 0;
    if (threadIdx.x == 0 && d.n_old == 0 && h == 0 && which == 0)
      p.tables[d.table_index] = static_cast<int32_t>((2u << kFmtShift) | static_cast<uint32_t>(d.slot));
    return;
  }
  uint8_t* head = p.fp8_slab + static_cast<int64_t>(d.slot) * p.slot_bytes +
                  static_cast<int64_t>(h) * (32 * D + 16);
  uint8_t* rows = head + which * kPageTokens * D;
  float* scale_ptr = reinterpret_cast<float*>(head + 32 * D) + which;
  const uint16_t* src = (which ? p.v : p.k) + (static_cast<int64_t>(d.first_row) * p.Hkv + h) * D;
  const int64_t src_stride = static_cast<int64_t>(p.Hkv) * D;
  const int n_old = d.n_old, n_new = d.n_new;

  float a = 0.f;
  bool finite = true;
  for (int i = threadIdx.x; i < n_new * D; i += blockDim.x) {
    const float x = bf16_bits_to_float(src[(i / D) * src_stride + (i % D)]);
    finite &= isfinite(x);
    a = fmaxf(a, fabsf(x));
  }
  if (!finite) flag_status(p.status, kStatusCheck);
  a = block_max(a, red);
  const float old = n_old ? *scale_ptr : 0.f;
  const float cand = __fdiv_rn(a, 448.f);
  float scale = old;
  bool rescale = false;
  if (n_old == 0) {
    scale = cand;
  } else if (cand > old) {
    scale = cand;
    rescale = true;
  }
  __syncthreads();  // everyone has read the old scale
  if (rescale) {
    for (int i = threadIdx.x; i < n_old * D; i += blockDim.x) {
      const float prev = __fmul_rn(e4m3_to_float(rows[i]), old);
      rows[i] = float_to_e4m3(__fdiv_rn(prev, scale));
    }
  }
  for (int i = threadIdx.x; i < n_new * D; i += blockDim.x) {
    const float x = bf16_bits_to_float(src[(i / D) * src_stride + (i % D)]);
    rows[n_old * D + i] = scale == 0.f ? uint8_t(0) : float_to_e4m3(__fdiv_rn(x, scale));
  }
  if (n_old == 0) {
    for (int i = n_new * D + threadIdx.x; i < kPageTokens * D; i += blockDim.x) rows[i] = 0;
    if (which == 0 && threadIdx.x < 8) head[32 * D + 8 + threadIdx.x] = 0;
  }
  if (threadIdx.x == 0) {
    *scale_ptr = scale;
    if (n_old == 0 && h == 0 && which == 0) p.tables[d.table_index] = d.slot;  // FP8 tag = 0
  }
}

// TQ3 record of one (token, KV head, K-or-V, group of 32 channels), computed by one thread from
// its 32 values x (fp32) and their largest magnitude amax:
//   s = fp16(min(fp32(amax/3.5), 65504)); q_j = #{k in -3..3 : x_j >= k*s};
//   code j in bits 3j..3j+2 of the 96-bit record (w0, w1, w2), least significant first.
// The threshold count is exact and needs no division: for x >= 0 (-0 included) it is
// 4 + #{k in 1..3 : x >= k*s}, for x < 0 it is 3 - #{k in 1..3 : |x| > k*s}; comparing the
// fp32 bit patterns of |x| (less one for negative x, which turns > into >=) with those of k*s
// (exact products) decides both as integer compares.
__device__ __forceinline__ uint32_t tq3_code(float x, int t1, int t2, int t3) {
  const uint32_t xb = __float_as_uint(x);
  const int neg = xb > 0x80000000u ? 1 : 0;
  const int u = static_cast<int>(xb & 0x7fffffffu) - neg;
  const int cnt = (u >= t1) + (u >= t2) + (u >= t3);
  return static_cast<uint32_t>(neg ? 3 - cnt : 4 + cnt);
}

// Places code j (constant after unrolling) at bits 3j..3j+2 of the record words acc[0..2].
__device__ __forceinline__ void put_code(uint32_t (&acc)[3], int j, uint32_t q) {
  const int bit = 3 * j;
  acc[bit >> 5] |= q << (bit & 31);
  if ((bit & 31) > 29) acc[(bit >> 5) + 1] |= q >> (32 - (bit & 31));
}

// ------------------------------------------------------------------ codes in the source domain
// The same threshold counts, taken four FP8 values (or two bf16 values) per 32-bit operation:
// since x is a monotonic function of the stored value, "x >= theta" is "the stored magnitude is
// at least the smallest magnitude whose x reaches theta", and those magnitude thresholds are
// found once per record.  For a lane value (magnitude m in its low 7 or 15 bits, sign on top),
// with P_k the threshold of x >= k*s (x >= 0) and N_k that of |x| > k*s (x < 0):
//   count = #{k : m >= (negative ? N_k : P_k)}, q = negative ? 3 - count : 4 + count,
// where "negative" excludes -0.  Setting bit 7 (15) of the magnitude and subtracting the lane's
// threshold leaves bit 7 (15) set exactly when m >= threshold, with no borrow between lanes.
// Since P_1 <= P_2 <= P_3 (and N likewise), count's bits are (ge2, ge1 ^ ge2 ^ ge3), and the
// code's three bits are (not negative, ge2 ^ negative, ge1 ^ ge2 ^ ge3 ^ negative).

// Replicates the top bit of every byte over the byte (prmt sign-replicate selectors).
__device__ __forceinline__ uint32_t byte_sign_mask(uint32_t x) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(d) : "r"(x));
  return d;
}
// Replicates bit 15 (31) over the low (high) 16-bit half.
__device__ __forceinline__ uint32_t half_sign_mask(uint32_t x) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, 0xBB99;" : "=r"(d) : "r"(x));
  return d;
}

// Codes of four E4M3 values (byte i = value i) as bits 3i..3i+2 of the result.  p_k: P_k in
// every byte; d_k: P_k ^ N_k in every byte (all thresholds <= 127).
__device__ __forceinline__ uint32_t tq3_codes_e4m3x4(uint32_t w, uint32_t p1, uint32_t p2,
                                                     uint32_t p3, uint32_t d1, uint32_t d2,
                                                     uint32_t d3) {
  const uint32_t mag = w & 0x7F7F7F7Fu;
  const uint32_t negb = ((mag + 0x7F7F7F7Fu) & w) & 0x80808080u;  // sign set and m != 0
  const uint32_t negm = byte_sign_mask(negb);
  const uint32_t t = w | 0x80808080u;
  const uint32_t g1 = t - (p1 ^ (d1 & negm));
  const uint32_t g2 = t - (p2 ^ (d2 & negm));
  const uint32_t g3 = t - (p3 ^ (d3 & negm));
  const uint32_t b0 = (g1 ^ g2 ^ g3 ^ negb) & 0x80808080u;
  const uint32_t b1 = (g2 ^ negb) & 0x80808080u;
  const uint32_t b2 = ~negb & 0x80808080u;
  const uint32_t q = (b0 >> 7) | (b1 >> 6) | (b2 >> 5);  // code i in bits 8i..8i+2
  const uint32_t pairs = q | (q >> 5);                    // codes 0,1 in bits 0-5; 2,3 in 16-21
  return (pairs & 0x3Fu) | ((pairs >> 10) & 0xFC0u);
}

// Codes of two bf16 values (low half first) as bits 0..5; p_k, d_k replicated in both halves.
__device__ __forceinline__ uint32_t tq3_codes_bf16x2(uint32_t w, uint32_t p1, uint32_t p2,
                                                     uint32_t p3, uint32_t d1, uint32_t d2,
                                                     uint32_t d3) {
  const uint32_t mag = w & 0x7FFF7FFFu;
  const uint32_t negb = ((mag + 0x7FFF7FFFu) & w) & 0x80008000u;
  const uint32_t negm = half_sign_mask(negb);
  const uint32_t t = w | 0x80008000u;
  const uint32_t g1 = t - (p1 ^ (d1 & negm));
  const uint32_t g2 = t - (p2 ^ (d2 & negm));
  const uint32_t g3 = t - (p3 ^ (d3 & negm));
  const uint32_t b0 = (g1 ^ g2 ^ g3 ^ negb) & 0x80008000u;
  const uint32_t b1 = (g2 ^ negb) & 0x80008000u;
  const uint32_t b2 = ~negb & 0x80008000u;
  const uint32_t q = (b0 >> 15) | (b1 >> 14) | (b2 >> 13);  // code i in bits 16i..16i+2
  return (q & 7u) | ((q >> 13) & 0x38u);
}

// 96-bit record from eight 12-bit chunks (chunk c = codes 4c..4c+3).
__device__ __forceinline__ void record_from_chunks12(const uint32_t (&c)[8], uint32_t& w0,
                                                     uint32_t& w1, uint32_t& w2) {
  w0 = c[0] | (c[1] << 12) | (c[2] << 24);
  w1 = (c[2] >> 8) | (c[3] << 4) | (c[4] << 16) | (c[5] << 28);
  w2 = (c[5] >> 4) | (c[6] << 8) | (c[7] << 20);
}

// Smallest E4M3 magnitude code m (0..126) with fp32(dec(m) * scale) >= theta, or 127 when none
// reaches it.  Exact for 2^-100 <= scale < 2^100 (every product of a nonzero code is then a
// normal float, and consecutive codes differ by more than 1/16 in value, far above the fp32
// rounding): with m* the largest code whose value is at most theta/scale, the answer is m* or
// m* + 1, and the code nearest to (an approximation of) theta/scale is m* or m* + 1, so checking
// it and the code below decides.
__device__ __forceinline__ uint32_t e4m3_threshold(float theta, float scale, float rscale) {
  const uint32_t m0 = float_to_e4m3(theta * rscale) & 0x7Fu;  // theta >= 0: RN, at most 126
  const uint32_t lo = m0 > 0 ? m0 - 1 : 0;
  const uint32_t h = e4m3x2_to_f16x2(lo | (m0 << 8));
  const __half2 hh = *reinterpret_cast<const __half2*>(&h);
  const float flo = __fmul_rn(__low2float(hh), scale), fm0 = __fmul_rn(__high2float(hh), scale);
  if (m0 > 0 && flo >= theta) return lo;
  if (fm0 >= theta) return m0;
  return m0 + 1;
}

// Stores one record and its scale into a TQ3 page-head area ([G][16] records, then [G][16]
// scales) for (group grp, token t).
__device__ __forceinline__ void store_record(uint8_t* area, int G, int grp, int t, uint32_t w0,
                                             uint32_t w1, uint32_t w2, __half sh) {
  uint32_t* rec = reinterpret_cast<uint32_t*>(area + 12 * (grp * kPageTokens + t));
  rec[0] = w0;
  rec[1] = w1;
  rec[2] = w2;
  reinterpret_cast<__half*>(area + G * kPageTokens * 12)[grp * kPageTokens + t] = sh;
}

// One CTA per (page, KV head) with 32 * G threads; thread = (K-or-V, group, token), tokens
// fastest, so the records and scales a warp writes are contiguous.  The thread reads its 32 FP8
// codes with two 16-byte loads; x = fp32(dec(code) * page scale), and since that rounding is
// monotonic, amax = fp32(max |dec| * page scale).
__global__ void __launch_bounds__(256) demote_kernel(const __grid_constant__ DemoteParams p) {
  const DemoteDesc d = p.desc[blockIdx.x];
  const int h = blockIdx.y, D = p.D, G = D / 32;
  const int t = threadIdx.x & 15, grp = (threadIdx.x >> 4) % G, which = threadIdx.x / (16 * G);
  const uint8_t* src = p.fp8_slab + static_cast<int64_t>(d.src_slot) * p.fp8_slot_bytes +
                       static_cast<int64_t>(h) * (32 * D + 16);
  uint8_t* dst = p.tq3_slab + static_cast<int64_t>(d.dst_slot) * p.tq3_slot_bytes +
                 static_cast<int64_t>(h) * (14 * D);
  const float scale = reinterpret_cast<const float*>(src + 32 * D)[which];
  const uint4* c4 = reinterpret_cast<const uint4*>(src + which * kPageTokens * D + t * D + 32 * grp);
  const uint4 ca = c4[0], cb = c4[1];
  const uint32_t cw[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
  uint32_t mx = 0;  // f16x2 of the largest |dec| (max.f16x2 skips NaN codes, like fmaxf)
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t lo = e4m3x2_to_f16x2(cw[k]), hi = e4m3x2_to_f16x2(cw[k] >> 16);
    mx = hmax2_u32(mx, hmax2_u32(lo & 0x7fff7fffu, hi & 0x7fff7fffu));
  }
  const __half2 m2 = *reinterpret_cast<const __half2*>(&mx);
  const float amax = __fmul_rn(fmaxf(__low2float(m2), __high2float(m2)), scale);
  uint32_t w0, w1, w2;
  __half sh;
  if (scale >= 0x1p-100f && scale < 0x1p100f) {
    // code domain: the thresholds of x >= k*s and |x| > k*s as E4M3 magnitudes
    sh = __float2half_rn(fminf(__fdiv_rn(amax, 3.5f), 65504.f));
    const float s = __half2float(sh), rscale = 1.f / scale;
    uint32_t pk[3], dk[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const float tk = static_cast<float>(k + 1) * s;  // exact
      const uint32_t pt = e4m3_threshold(tk, scale, rscale);
      const uint32_t nt = e4m3_threshold(__uint_as_float(__float_as_uint(tk) + 1u), scale, rscale);
      pk[k] = pt * 0x01010101u;
      dk[k] = (pt ^ nt) * 0x01010101u;
    }
    uint32_t ch[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      ch[k] = tq3_codes_e4m3x4(cw[k], pk[0], pk[1], pk[2], dk[0], dk[1], dk[2]);
    record_from_chunks12(ch, w0, w1, w2);
  } else {
    // extreme page scales: the fp32 values themselves, x = fp32(dec * scale), with the
    // record's thresholds t_k = bits(k*s)
    sh = __float2half_rn(fminf(__fdiv_rn(amax, 3.5f), 65504.f));
    const float s = __half2float(sh);
    const int t1 = __float_as_int(s), t2 = __float_as_int(2.f * s), t3 = __float_as_int(3.f * s);
    uint32_t acc[3] = {0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t lo = e4m3x2_to_f16x2(cw[k]), hi = e4m3x2_to_f16x2(cw[k] >> 16);
      const __half2 hl = *reinterpret_cast<const __half2*>(&lo);
      const __half2 hh = *reinterpret_cast<const __half2*>(&hi);
      put_code(acc, 4 * k + 0, tq3_code(__fmul_rn(__low2float(hl), scale), t1, t2, t3));
      put_code(acc, 4 * k + 1, tq3_code(__fmul_rn(__high2float(hl), scale), t1, t2, t3));
      put_code(acc, 4 * k + 2, tq3_code(__fmul_rn(__low2float(hh), scale), t1, t2, t3));
      put_code(acc, 4 * k + 3, tq3_code(__fmul_rn(__high2float(hh), scale), t1, t2, t3));
    }
    w0 = acc[0];
    w1 = acc[1];
    w2 = acc[2];
  }
  store_record(dst + which * (G * kPageTokens * 14), G, grp, t, w0, w1, w2, sh);
  if (p.publish && h == 0 && threadIdx.x == 0)
    p.tables[d.table_index] = static_cast<int32_t>((1u << kFmtShift) | static_cast<uint32_t>(d.dst_slot));
}

__global__ void __launch_bounds__(256) retag_kernel(const __grid_constant__ RetagParams p) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < p.n; k += gridDim.x * blockDim.x)
    p.tables[p.index[k]] = p.entry[k];
}

// Prefill: a full page packed to TQ3 straight from the bf16 input rows (the values are exact in
// fp32), with the same per-record packing as demotion.  One CTA per (page, KV head) with 32 * G
// threads, thread = (K-or-V, group, token); four 16-byte loads bring a record's 32 values.
__global__ void __launch_bounds__(256) pack_kernel(const __grid_constant__ PackParams p) {
  const PackDesc d = p.desc[blockIdx.x];
  const int h = blockIdx.y, D = p.D, G = D / 32;
  const int t = threadIdx.x & 15, grp = (threadIdx.x >> 4) % G, which = threadIdx.x / (16 * G);
  uint8_t* dst = p.tq3_slab + static_cast<int64_t>(d.dst_slot) * p.tq3_slot_bytes +
                 static_cast<int64_t>(h) * (14 * D);
  const uint16_t* src = (which ? p.v : p.k) +
                        (static_cast<int64_t>(d.first_row + t) * p.Hkv + h) * D + 32 * grp;
  uint32_t w[16];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (p.vec16) {  // both input arrays 16-byte aligned (checked on the host)
      const uint4 v = reinterpret_cast<const uint4*>(src)[k];
      w[4 * k] = v.x, w[4 * k + 1] = v.y, w[4 * k + 2] = v.z, w[4 * k + 3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[4 * k + e] = static_cast<uint32_t>(src[8 * k + 2 * e]) |
                       (static_cast<uint32_t>(src[8 * k + 2 * e + 1]) << 16);
    }
  }
  // largest magnitude, two bf16 values per operation (|x| by clearing the sign bits)
  uint32_t mx = 0u;
#pragma unroll
  for (int e = 0; e < 16; ++e) mx = bmax2_u32(mx, w[e] & 0x7fff7fffu);
  const float amax = fmaxf(bf16_lo(mx), bf16_hi(mx));
  // codes in the bf16 domain: x >= k*s is m >= ceil(t_k / 2^16) and |x| > k*s is
  // m >= floor(t_k / 2^16) + 1, with m the bf16 magnitude bits and t_k the fp32 bits of k*s
  uint32_t w0, w1, w2;
  const __half sh = __float2half_rn(fminf(__fdiv_rn(amax, 3.5f), 65504.f));
  const float s = __half2float(sh);
  uint32_t pk[3], dk[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const uint32_t tk = __float_as_uint(static_cast<float>(k + 1) * s);  // exact
    const uint32_t pt = (tk + 0xFFFFu) >> 16, nt = (tk >> 16) + 1u;
    pk[k] = pt * 0x00010001u;
    dk[k] = (pt ^ nt) * 0x00010001u;
  }
  uint32_t ch[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    ch[k] = tq3_codes_bf16x2(w[2 * k], pk[0], pk[1], pk[2], dk[0], dk[1], dk[2]) |
            (tq3_codes_bf16x2(w[2 * k + 1], pk[0], pk[1], pk[2], dk[0], dk[1], dk[2]) << 6);
  record_from_chunks12(ch, w0, w1, w2);
  store_record(dst + which * (G * kPageTokens * 14), G, grp, t, w0, w1, w2, sh);
  if (h == 0 && threadIdx.x == 0)
    p.tables[d.table_index] = static_cast<int32_t>((1u << kFmtShift) | static_cast<uint32_t>(d.dst_slot));
}

// One block per slot: copy all bytes, then publish the table entry.
__global__ void __launch_bounds__(256) copy_kernel(const __grid_constant__ CopyParams p) {
  const CopyDesc d = p.desc[blockIdx.x];
  const int64_t bytes = d.fmt == 0 ? p.fp8_slot_bytes : p.tq3_slot_bytes;
  uint8_t* slab = d.fmt == 0 ? p.fp8_slab : p.tq3_slab;
  const uint4* s = reinterpret_cast<const uint4*>(slab + d.src_slot * bytes);
  uint4* t = reinterpret_cast<uint4*>(slab + d.dst_slot * bytes);
  for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) t[i] = s[i];
  if (threadIdx.x == 0)
    p.tables[d.table_index] =
        static_cast<int32_t>((static_cast<uint32_t>(d.fmt) << kFmtShift) | static_cast<uint32_t>(d.dst_slot));
}

// Materialising profile ("Minima-KV ..." pt page, section "Qualidade em contexto longo": the
// profile in which the hybrid pages really are expanded into tensors).  A debugging and
// quality-control path: one CTA per (page, KV head, K/V) writes the page's dequantised values
// as dense fp32 rows -- FP8: fp32(dec(code) * scale); TQ3: (q - 3.5) * s, exact.  Decode never
// calls it.
__global__ void __launch_bounds__(256) materialise_kernel(const __grid_constant__ MaterialiseParams p) {
  const int page = blockIdx.x, h = blockIdx.y, kv = blockIdx.z;
  const int D = p.D, n = min(kPageTokens, p.ctx - kPageTokens * page);
  const int32_t e = p.table[page];
  const int fmt = static_cast<int>(static_cast<uint32_t>(e) >> kFmtShift);
  const int64_t slot = static_cast<int64_t>(static_cast<uint32_t>(e) & kSlotMask);
  if (e == -1 || (fmt != 1 && fmt != p.page_fmt) || slot >= (fmt == 1 ? p.tq3_slots : p.fp8_slots)) {
    if (threadIdx.x == 0) flag_status(p.status, kStatusCheck);
    return;
  }
  float* out = (kv ? p.v_out : p.k_out) + (static_cast<int64_t>(kPageTokens) * page * p.Hkv + h) * D;
  const int64_t row_stride = static_cast<int64_t>(p.Hkv) * D;
  if (fmt == 2) {
    const uint16_t* rows = reinterpret_cast<const uint16_t*>(p.fp8_slab + slot * p.fp8_slot_bytes +
                                                             h * (64LL * D)) + kv * kPageTokens * D;
    for (int i = threadIdx.x; i < n * D; i += blockDim.x)
      out[(i / D) * row_stride + i % D] = bf16_bits_to_float(rows[i]);
  } else if (fmt == 0) {
    const uint8_t* base = p.fp8_slab + slot * p.fp8_slot_bytes + h * (32LL * D + 16);
    const uint8_t* codes = base + kv * kPageTokens * D;
    const float scale = reinterpret_cast<const float*>(base + 2 * kPageTokens * D)[kv];
    for (int i = threadIdx.x; i < n * D; i += blockDim.x)
      out[(i / D) * row_stride + i % D] = e4m3_to_float(codes[i]) * scale;
  } else {
    const int G = D / 32;
    const uint8_t* base = p.tq3_slab + slot * p.tq3_slot_bytes + h * (14LL * D) + kv * (7LL * D);
    const __half* scales = reinterpret_cast<const __half*>(base + G * kPageTokens * 12);
    for (int i = threadIdx.x; i < n * D; i += blockDim.x) {
      const int t = i / D, d = i % D, g = d / 32, j = d % 32;
      const uint8_t* rec = base + 12 * (kPageTokens * g + t);
      const int bit = 3 * j;  // LSB-first stream bit of code j
      const uint32_t two = rec[bit >> 3] | (static_cast<uint32_t>(rec[min((bit >> 3) + 1, 11)]) << 8);
      const float q = static_cast<float>((two >> (bit & 7)) & 7u);
      out[t * row_stride + d] = (q - 3.5f) * __half2float(scales[kPageTokens * g + t]);
    }
  }
}

// Self-test of the bounded waits: one thread waits on a barrier that nothing completes, gives
// up after limit_ns and records a timeout in the status word, as every wait of the library
// does; the context stays usable.
__global__ void wait_selftest_kernel(int32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    if (!mbar_wait(&bar, 0, limit_ns)) flag_status(status, kStatusTimeout);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_pack(const PackParams& p, cudaStream_t s) {
  if (p.n_desc <= 0) return cudaSuccess;
  pack_kernel<<<dim3(p.n_desc, p.Hkv), p.D, 0, s>>>(p);  // 32 * (D / 32) threads
  return cudaGetLastError();
}

cudaError_t launch_materialise(const MaterialiseParams& p, cudaStream_t s) {
  if (p.ctx <= 0) return cudaSuccess;
  const int pages = (p.ctx + kPageTokens - 1) / kPageTokens;
  materialise_kernel<<<dim3(pages, p.Hkv, 2), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  if (p.n_desc <= 0) return cudaSuccess;
  append_kernel<<<dim3(p.n_desc, p.Hkv, 2), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_demote(const DemoteParams& p, cudaStream_t s) {
  if (p.n_desc <= 0) return cudaSuccess;
  demote_kernel<<<dim3(p.n_desc, p.Hkv), p.D, 0, s>>>(p);  // 32 * (D / 32) threads
  return cudaGetLastError();
}

cudaError_t launch_retag(const RetagParams& p, cudaStream_t s) {
  if (p.n <= 0) return cudaSuccess;
  retag_kernel<<<(p.n + 255) / 256, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_copy(const CopyParams& p, cudaStream_t s) {
  if (p.n_desc <= 0) return cudaSuccess;
  copy_kernel<<<p.n_desc, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mkv
