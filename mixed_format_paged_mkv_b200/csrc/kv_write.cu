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

// TQ3 record of one (token, KV head, K-or-V, group of 32 channels), one channel per lane:
// s = fp16(min(fp32(amax/3.5), 65504)); q = #{k in -3..3 : x >= k*s}; the 32 codes packed
// LSB-first into the 12-byte record, the scale into the area's scale array.
__device__ __forceinline__ void pack_group(float x, int lane, uint8_t* area, int G, int grp, int t) {
  float amax = fabsf(x);
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half sh = __float2half_rn(fminf(__fdiv_rn(amax, 3.5f), 65504.f));
  const float s = __half2float(sh);
  uint32_t q = 0;
#pragma unroll
  for (int k = -3; k <= 3; ++k) q += (x >= __fmul_rn(static_cast<float>(k), s)) ? 1u : 0u;
  // bit 3*lane + i of the 96-bit record holds bit i of q
  const int bit = 3 * lane;
  uint32_t w0 = 0, w1 = 0, w2 = 0;
  if (bit < 32) w0 = q << bit;
  if (bit + 2 >= 32 && bit < 64) w1 = (bit >= 32) ? (q << (bit - 32)) : (q >> (32 - bit));
  if (bit + 2 >= 64) w2 = (bit >= 64) ? (q << (bit - 64)) : (q >> (64 - bit));
  w0 = __reduce_or_sync(0xffffffffu, w0);
  w1 = __reduce_or_sync(0xffffffffu, w1);
  w2 = __reduce_or_sync(0xffffffffu, w2);
  uint32_t* rec = reinterpret_cast<uint32_t*>(area + 12 * (grp * kPageTokens + t));
  if (lane == 0) rec[0] = w0;
  if (lane == 1) rec[1] = w1;
  if (lane == 2) rec[2] = w2;
  if (lane == 3) {
    __half* sc = reinterpret_cast<__half*>(area + G * kPageTokens * 12);
    sc[grp * kPageTokens + t] = sh;
  }
}

// One block per (page, KV head); one warp per (K-or-V, group of 32 channels, token), lane =
// channel.  x = fp32(dec(code) * page scale), packed by pack_group.
__global__ void __launch_bounds__(256) demote_kernel(const __grid_constant__ DemoteParams p) {
  const DemoteDesc d = p.desc[blockIdx.x];
  const int h = blockIdx.y, D = p.D, G = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t* src = p.fp8_slab + static_cast<int64_t>(d.src_slot) * p.fp8_slot_bytes +
                       static_cast<int64_t>(h) * (32 * D + 16);
  uint8_t* dst = p.tq3_slab + static_cast<int64_t>(d.dst_slot) * p.tq3_slot_bytes +
                 static_cast<int64_t>(h) * (14 * D);
  const float* scales = reinterpret_cast<const float*>(src + 32 * D);
  const int units = 2 * G * kPageTokens;
  for (int u = warp; u < units; u += blockDim.x >> 5) {
    const int which = u / (G * kPageTokens);
    const int grp = (u / kPageTokens) % G;
    const int t = u % kPageTokens;
    const uint8_t code = src[which * kPageTokens * D + t * D + grp * 32 + lane];
    const float x = __fmul_rn(e4m3_to_float(code), scales[which]);
    pack_group(x, lane, dst + which * (G * kPageTokens * 14), G, grp, t);
  }
  if (p.publish && h == 0 && threadIdx.x == 0)
    p.tables[d.table_index] = static_cast<int32_t>((1u << kFmtShift) | static_cast<uint32_t>(d.dst_slot));
}

__global__ void __launch_bounds__(256) retag_kernel(const __grid_constant__ RetagParams p) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < p.n; k += gridDim.x * blockDim.x)
    p.tables[p.index[k]] = p.entry[k];
}

// Prefill: a full page packed to TQ3 straight from the bf16 input rows (the values are exact in
// fp32), with the same per-group packing as demotion.  One block per (page, KV head).
__global__ void __launch_bounds__(256) pack_kernel(const __grid_constant__ PackParams p) {
  const PackDesc d = p.desc[blockIdx.x];
  const int h = blockIdx.y, D = p.D, G = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* dst = p.tq3_slab + static_cast<int64_t>(d.dst_slot) * p.tq3_slot_bytes +
                 static_cast<int64_t>(h) * (14 * D);
  const int units = 2 * G * kPageTokens;
  for (int u = warp; u < units; u += blockDim.x >> 5) {
    const int which = u / (G * kPageTokens);
    const int grp = (u / kPageTokens) % G;
    const int t = u % kPageTokens;
    const uint16_t* src = which ? p.v : p.k;
    const float x = bf16_bits_to_float(
        src[(static_cast<int64_t>(d.first_row + t) * p.Hkv + h) * D + grp * 32 + lane]);
    pack_group(x, lane, dst + which * (G * kPageTokens * 14), G, grp, t);
  }
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
  if (e < 0 || fmt > 1 || slot >= (fmt == 0 ? p.fp8_slots : p.tq3_slots)) {
    if (threadIdx.x == 0) flag_status(p.status, kStatusCheck);
    return;
  }
  float* out = (kv ? p.v_out : p.k_out) + (static_cast<int64_t>(kPageTokens) * page * p.Hkv + h) * D;
  const int64_t row_stride = static_cast<int64_t>(p.Hkv) * D;
  if (fmt == 0) {
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
  pack_kernel<<<dim3(p.n_desc, p.Hkv), 256, 0, s>>>(p);
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
  demote_kernel<<<dim3(p.n_desc, p.Hkv), 256, 0, s>>>(p);
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
