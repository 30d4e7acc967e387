// Launchers of the self-test kernels (failure detection, tensor-memory MMA building block).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace mkv {

// One thread waits on a barrier that nothing completes, gives up after limit_ns and records a
// timeout in *status.
cudaError_t launch_wait_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t s);

// D[128][8] (fp32) = A[128][256] . Q[8][256]^T (f16) through TMEM and tcgen05.mma.
cudaError_t launch_tc_logits_selftest(const void* a_f16, const void* q_f16, float* d,
                                      int32_t* status, cudaStream_t s);

}  // namespace mkv
