// Decode attention directly over the mixed-format paged cache.
//
// "Minima-KV ..." (brainszone.ai pt page, section "Como os resultados parciais são
// combinados"; fr "Comment les résultats partiels sont assemblés"): a separate kernel per page
// format computes partial attention states, and an online-softmax merge with global
// normalisation combines them -- no page is converted to a common format first and no dense
// copy of the cache is made (section "... sem a chamada sombra densa").
//
// The host cuts every sequence into work units -- (format, logical page range) -- and gives
// each CTA one unit or, when that balances the wave badly, a run of units of several sequences.
// Three launches per call (per launch group): the FP8 partial kernel over the FP8 CTAs, the
// TQ3 partial kernel over the TQ3 CTAs and the merge kernel.  The TQ3 and merge kernels are
// programmatic dependents of the kernel before them: the TQ3 CTAs fill the SM room the FP8
// CTAs leave (one wave of both formats), and the merge CTAs wait for the partial states with
// griddepcontrol.wait.  A fused variant runs both formats in one grid, branching per unit; the
// host picks it per call where it keeps the same occupancy or where FP8 pages carry much of the
// work.  The partial kernels are templates (decode_partial.cuh) compiled per head dimension
// (decode_d64.cu, decode_d128.cu, decode_d256.cu); this file holds the merge and the launches.
//
// A partial CTA with at most 8 query columns per KV head takes each of its units in turn:
//   1. one warp scans the block-table entries of the range, keeps the pages of the unit's format
//      and starts the first bulk async copies of those pages into a shared-memory ring;
//   2. the warps take pages round-robin; each ring stage always belongs to the same warp(s),
//      which refill it with the page one ring-length ahead as soon as they are done with it (no
//      producer warp: the stage's copy completes on its mbarrier);
//   3. per page the logits, the online softmax (running max m and denominator l per query
//      column) and P.V;
//   4. the CTA combines its warps and writes its partial state (m, l, acc) per query column.
// With more query columns a CTA is a team of warps that decodes each page once for all
// n-tiles (run_unit_team).
// The merge kernel combines, per (sequence, KV head, query column), all partial states of both
// formats: M = max m, L = sum l 2^(m-M), O = sum acc 2^(m-M) / L.
//
// Tensor-core use: per page the logits are a 16-token x 8-column tile (tokens are the MMA M
// dimension, the q_len*g query columns of one KV head the N dimension) and P.V is a
// (16 channels x 16 tokens) x (16 tokens x 8 columns) tile, both mma.sync m16n8k16 with f16
// operands that are exact images of the stored codes.  Dequantisation happens in registers:
//   TQ3 K: codes -> exact f16 images (base + c); each group's MMA starts from the correction
//          -(base + 3.5) * (sum of the matching query values), so it yields sum q (c - 3.5);
//          the per-(token, group) scale multiplies the group's result (summed in fp32).
//   TQ3 V: codes -> (c - 3.5) exactly; the per-(token, group) scale multiplies P in f16, with a
//          per-group power of two taken out first on pages whose scales would leave the f16
//          range.
//   FP8:   e4m3x2 -> f16x2 conversions; the per-page scales multiply logits / the page's P.V.
// Softmax runs in log2 units with a lazily raised reference maximum (raised only when a
// logit exceeds it by more than 8), so probabilities fed to the MMA are < 2^8.
#include "device_util.cuh"
#include "mkv_internal.h"

namespace mkv {

// Partial grids per head dimension (decode_d64.cu, decode_d128.cu, decode_d256.cu).
cudaError_t launch_partial_d64(int K, const DecodeParams& p, int c0, int c1, bool dependent,
                               cudaStream_t s);
cudaError_t launch_partial_d128(int K, const DecodeParams& p, int c0, int c1, bool dependent,
                                cudaStream_t s);
cudaError_t launch_partial_d256(int K, const DecodeParams& p, int c0, int c1, bool dependent,
                                cudaStream_t s);
int partial_ctas_per_sm_d64(int K, int NC);
int partial_ctas_per_sm_d128(int K, int NC);
int partial_ctas_per_sm_d256(int K, int NC);

namespace {

// Partial-kernel kinds (as in decode_partial.cuh) and the BF16 page tag.
enum Kind { kKindFp8 = 0, kKindTq3 = 1, kKindFused = 2, kKindBf16 = 3 };
constexpr int kBf16 = 2;

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

// Merge of the partial states of one (sequence, KV head, query column): the globally
// normalised combination M = max m, L = sum l 2^(m-M), O = sum acc 2^(m-M) / L.  One pass: a
// thread owns 4 channels of a subset of the partials (every nsub-th one) and keeps a running
// (m, l, acc) over them, loading eight partials at a time so that their loads are in flight
// together; the subsets are combined in shared memory at the end.  Two dependent rounds of
// memory access in all (the partial states, then the output) for up to 8 x nsub partials.
constexpr int kMergeThreads = 512;
constexpr int kMergeBatch = 8;
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ DecodeParams p) {
  __shared__ float4 part_o[kMergeThreads];
  __shared__ float2 part_ml[kMergeThreads];
  // launched as a programmatic dependent of the partial kernels: resident early, it reads the
  // partial states only once they are complete and visible
  pdl_wait();
  const int pair = blockIdx.x / p.NC, n = blockIdx.x % p.NC;
  const SeqDesc& sd = p.seq[pair / p.Hkv];
  const int h = pair % p.Hkv;
  const int S = sd.n_parts, D = p.D, tid = threadIdx.x;
  const int groups = D / 4, nsub = static_cast<int>(blockDim.x) / groups;
  const int c4 = tid % groups, k = tid / groups;
  const int64_t base0 = (static_cast<int64_t>(sd.part0) * p.Hkv + h) * p.NC + n;
  const int64_t stride = static_cast<int64_t>(p.Hkv) * p.NC;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml);
  const float4* acc = reinterpret_cast<const float4*>(p.part_acc);
  float m = -INFINITY, l = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = k; j0 < S; j0 += kMergeBatch * nsub) {
    float2 v[kMergeBatch];
    float4 a[kMergeBatch];
#pragma unroll
    for (int i = 0; i < kMergeBatch; ++i) {
      const int j = j0 + i * nsub;
      v[i] = make_float2(-INFINITY, 0.f);
      a[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < S) {
        v[i] = ml[base0 + j * stride];
        a[i] = acc[(base0 + j * stride) * groups + c4];
      }
    }
    float mb = m;
#pragma unroll
    for (int i = 0; i < kMergeBatch; ++i) mb = fmaxf(mb, v[i].x);
    if (mb == -INFINITY) continue;  // nothing attended so far
    const float r = exp2f(m - mb);  // 0 while m is still -inf
    l *= r;
    o.x *= r; o.y *= r; o.z *= r; o.w *= r;
#pragma unroll
    for (int i = 0; i < kMergeBatch; ++i) {
      const float wi = exp2f(v[i].x - mb);  // 0 for an empty partial
      l = fmaf(wi, v[i].y, l);
      o.x = fmaf(wi, a[i].x, o.x);
      o.y = fmaf(wi, a[i].y, o.y);
      o.z = fmaf(wi, a[i].z, o.z);
      o.w = fmaf(wi, a[i].w, o.w);
    }
    m = mb;
  }
  part_o[tid] = o;
  if (c4 == 0) part_ml[k] = make_float2(m, l);
  __syncthreads();
  if (tid < groups) {
    float M = -INFINITY;
    for (int i = 0; i < nsub; ++i) M = fmaxf(M, part_ml[i].x);
    float L = 0.f;
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int i = 0; i < nsub; ++i) {
        const float2 q = part_ml[i];
        if (q.x == -INFINITY) continue;
        const float wi = exp2f(q.x - M);
        const float4 u = part_o[tid + i * groups];
        L = fmaf(wi, q.y, L);
        t.x = fmaf(wi, u.x, t.x);
        t.y = fmaf(wi, u.y, t.y);
        t.z = fmaf(wi, u.z, t.z);
        t.w = fmaf(wi, u.w, t.w);
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int qi = n / p.g, hq = h * p.g + n % p.g;
    float* out = p.out + ((static_cast<int64_t>(sd.out_row) * p.q_len + qi) * p.Hq + hq) * D;
    reinterpret_cast<float4*>(out)[tid] = make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
  }
}

// The kinds' launches and occupancies live in the per-head-dim translation units.
cudaError_t launch_kind_d(int K, const DecodeParams& p, int c0, int c1, bool dependent,
                          cudaStream_t s) {
  switch (p.D) {
    case 64: return launch_partial_d64(K, p, c0, c1, dependent, s);
    case 128: return launch_partial_d128(K, p, c0, c1, dependent, s);
    case 256: return launch_partial_d256(K, p, c0, c1, dependent, s);
    default: return cudaErrorInvalidValue;
  }
}

int ctas_per_sm_kind_d(int K, int D, int NC) {
  switch (D) {
    case 64: return partial_ctas_per_sm_d64(K, NC);
    case 128: return partial_ctas_per_sm_d128(K, NC);
    default: return partial_ctas_per_sm_d256(K, NC);
  }
}

}  // namespace

int partial_ctas_per_sm(int D, int NC, int mode) {
  switch (mode) {
    case kDecodeFused: return ctas_per_sm_kind_d(kKindFused, D, NC);
    case kDecodeBf16: return ctas_per_sm_kind_d(kKindBf16, D, NC);
    default: return ctas_per_sm_kind_d(kKindTq3, D, NC);
  }
}

bool partial_supported(int D, int NC) {
  return (D == 64 || D == 128 || D == 256) && NC >= 1 && NC <= 32;
}

// The merge follows the last partial grid of the call as its programmatic dependent.
cudaError_t launch_merge(const DecodeParams& p, cudaStream_t s) {
  if (p.n_seqs <= 0) return cudaSuccess;
  // D/4 threads per subset of partials; a thread keeps kMergeBatch partials in flight, so the
  // call's largest partial count needs ceil(max / kMergeBatch) subsets (a power of two, up to
  // the block limit; at least one warp)
  int max_parts = 1;
  for (int i = 0; i < p.n_seqs; ++i) max_parts = max(max_parts, p.seq[i].n_parts);
  const int groups = p.D / 4;
  const int want = (max_parts + kMergeBatch - 1) / kMergeBatch;
  int nsub = groups >= 32 ? 1 : 32 / groups;
  while (nsub < want && 2 * nsub * groups <= kMergeThreads) nsub *= 2;
  return launch_ex(merge_kernel, dim3(p.n_seqs * p.Hkv * p.NC), nsub * groups, 0,
                   p.n_ctas > 0, s, p);
}

// Split: the FP8 grid (CTAs [0, n_fp8)), then the TQ3 grid as its programmatic dependent, so
// the TQ3 CTAs fill the SM room the FP8 CTAs leave in the same wave.  Fused: one grid over all
// CTAs.  The first partial grid waits for everything before it.
cudaError_t launch_partial(const DecodeParams& p, cudaStream_t s) {
  if (p.n_ctas <= 0) return cudaSuccess;
  if (p.n_ctas > kDecodeMaxUnits || p.n_fp8 < 0 || p.n_fp8 > p.n_ctas ||
      p.cta_unit0[0] != 0 || p.cta_unit0[p.n_ctas] != p.n_units || p.n_units > kDecodeMaxUnits)
    return cudaErrorInvalidValue;
  for (int c = 0; c < p.n_ctas; ++c)
    if (p.cta_unit0[c + 1] <= p.cta_unit0[c]) return cudaErrorInvalidValue;
  if (p.page_fmt == kBf16) return launch_kind_d(kKindBf16, p, 0, p.n_ctas, false, s);
  if (p.fused) return launch_kind_d(kKindFused, p, 0, p.n_ctas, false, s);
  cudaError_t e = launch_kind_d(kKindFp8, p, 0, p.n_fp8, false, s);
  if (e == cudaSuccess) e = launch_kind_d(kKindTq3, p, p.n_fp8, p.n_ctas, p.n_fp8 > 0, s);
  return e;
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
