// tcgen05 building block for the TQ3 logits (not on the decode path yet): one CTA computes
// D[128 tokens][8 columns] = A[128][256 channels] . Q[8][256]^T with the fifth-generation tensor
// core.  Each thread of the warpgroup owns one token row and writes it into the A operand in
// tensor memory (TMEM lane = token, 32-bit column j = channels 2j, 2j+1) -- the layout a
// per-record dequantiser would produce; Q sits in shared memory in the K-major, unswizzled
// core-matrix layout (8 channels x 8 columns per 128-byte block); one thread issues sixteen
// K = 16 MMAs (M 128, N 8, f16 inputs, f32 accumulator in TMEM) and commits them to an mbarrier;
// every thread then reads its row of D back from TMEM.  The bounded wait records a timeout in
// the status word; TMEM is freed on every path.
#include <cuda_fp16.h>
#include <stdint.h>

#include "device_util.cuh"
#include "mkv_internal.h"
#include "selftest.h"

namespace mkv {
namespace {

constexpr int kTcM = 128, kTcK = 256, kTcN = 8;
constexpr int kTcACols = kTcK / 2;  // 32-bit TMEM columns holding A
constexpr int kTcCols = 256;        // allocation: A (128) + D (8), a power of two

__global__ void __launch_bounds__(128, 1)
    tc_logits_kernel(const __half* A, const __half* Q, float* D, int32_t* status) {
  __shared__ __align__(1024) uint8_t qsm[kTcK * kTcN * 2];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base_sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Q: channel block kb (channels 8kb..8kb+7) at kb*128 bytes, query column n at +16n
  for (int i = tid; i < kTcK * kTcN; i += blockDim.x) {
    const int n = i / kTcK, k = i % kTcK;
    reinterpret_cast<__half*>(qsm)[(k / 8) * 64 + n * 8 + (k % 8)] = Q[n * kTcK + k];
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&tmem_base_sm)), "r"(kTcCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // Q stores -> tensor core
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base_sm;

  // A: this thread's token row, eight 32-bit columns per store
  const uint32_t row_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  for (int j0 = 0; j0 < kTcACols; j0 += 8) {
    uint32_t r[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const __half2 h = __halves2half2(A[tid * kTcK + 2 * (j0 + q)], A[tid * kTcK + 2 * (j0 + q) + 1]);
      r[q] = *reinterpret_cast<const uint32_t*>(&h);
    }
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 ::"r"(row_base + j0), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]),
                   "r"(r[5]), "r"(r[6]), "r"(r[7]) : "memory");
  }
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

  if (tid == 0) {
    // instruction descriptor: D f32 (bits 4-5), A and B f16 and K-major, N >> 3 at bit 17,
    // M >> 4 at bit 24
    const uint32_t idesc = (1u << 4) | ((kTcN >> 3) << 17) | ((kTcM >> 4) << 24);
    for (int i = 0; i < kTcK / 16; ++i) {
      // shared-memory descriptor: start >> 4, leading-dimension offset (next 8 channels,
      // 128 B) >> 4 at bit 16, stride offset (next 8 columns; unused with N = 8) >> 4 at bit
      // 32, version 1 at bit 46, no swizzle
      const uint32_t saddr = smem_addr(qsm) + (2 * i) * 128;
      const uint64_t desc = static_cast<uint64_t>((saddr >> 4) & 0x3FFF) |
                            (static_cast<uint64_t>(128 >> 4) << 16) |
                            (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46);
      const uint32_t acc = i > 0 ? 1u : 0u;
      asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                   "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
                   ::"r"(tmem + kTcACols), "r"(tmem + 8 * i), "l"(desc), "r"(idesc), "r"(acc),
                     "r"(0u), "r"(0u), "r"(0u), "r"(0u) : "memory");
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(&bar)) : "memory");
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0, 100000000ull));
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (ok) {
    uint32_t v[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "r"(row_base + kTcACols) : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int n = 0; n < kTcN; ++n) D[tid * kTcN + n] = __uint_as_float(v[n]);
  } else if (lane == 0) {
    flag_status(status, kStatusTimeout);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols)
                 : "memory");
}

}  // namespace

cudaError_t launch_tc_logits_selftest(const void* a_f16, const void* q_f16, float* d,
                                      int32_t* status, cudaStream_t s) {
  tc_logits_kernel<<<1, 128, 0, s>>>(static_cast<const __half*>(a_f16),
                                     static_cast<const __half*>(q_f16), d, status);
  return cudaGetLastError();
}

}  // namespace mkv
